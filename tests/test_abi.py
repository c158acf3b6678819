"""The C-ABI libraries load without a GPU, export every symbol their headers declare, and
reject bad arguments before touching a device."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = {"pool": "msa_pool.h", "route": "msa_route.h", "gather": "msa_gather.h", "decode": "msa_decode.h",
           "prefill": "msa_prefill.h", "bank": "msa_bank.h"}


def _declared(header):
    text = open(os.path.join(ROOT, "include", header)).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(msa_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def msa():
    import top_kv_routing_b200 as m
    return m


@pytest.mark.parametrize("lib", sorted(HEADERS))
def test_library_exports_declared_symbols(msa, lib):
    path = os.path.join(msa.LIB_DIR, f"libmsa_{lib}.so")
    names = _declared(HEADERS[lib])
    assert names, lib
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if line.strip())
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    dll = ctypes.CDLL(path)
    for n in names:
        assert getattr(dll, n) is not None


def test_common_header_constants_match_binding(msa):
    text = open(os.path.join(ROOT, "include", "msa_common.h")).read()
    for name in ("MSA_DEVERR_CAPACITY", "MSA_DEVERR_BAD_DOC", "MSA_DEVERR_LOCAL_FULL", "MSA_DEVERR_BAD_OFFSETS",
                 "MSA_DEVERR_TIMEOUT", "MSA_DEVERR_UNCERTIFIED"):
        v = int(re.search(rf"#define {name} (\d+)u", text).group(1))
        assert getattr(msa, name) == v
    text = open(os.path.join(ROOT, "include", "msa_route.h")).read()
    for name in ("MSA_ROUTE_AUTO", "MSA_ROUTE_SCAN", "MSA_ROUTE_TENSOR", "MSA_ROUTE_TENSOR_F8", "MSA_ROUTE_LAYER_MEAN"):
        assert getattr(msa, name) == int(re.search(rf"#define {name} (\d+)", text).group(1))


def test_bank_header_constants_match_binding(msa):
    text = open(os.path.join(ROOT, "include", "msa_bank.h")).read()
    for name in ("MSA_BANK_KR", "MSA_BANK_KR_F8", "MSA_BANK_KV", "MSA_BANK_NORM"):
        assert getattr(msa, name) == int(re.search(rf"#define {name} (\d+)u", text).group(1))
    text = open(os.path.join(ROOT, "include", "msa_common.h")).read()
    assert msa.MSA_ERR_IO == int(re.search(r"MSA_ERR_IO = (\d+)", text).group(1))
    # the info struct as the header lays it out (4 int32, 2 int64, 1 uint32)
    import ctypes
    assert ctypes.sizeof(msa.MsaBankInfo) == 4 * 4 + 2 * 8 + 8


def test_count_chunks_host(msa):
    n, offs = msa.msa_count_chunks(np.array([0, 64, 65, 65, 200]), 64)
    assert n == 1 + 1 + 0 + 3 and offs.tolist() == [0, 1, 2, 2, 5]
    with pytest.raises(msa.MsaError):
        msa.msa_count_chunks(np.array([0, 5, 3]), 64)


def test_invalid_arguments_rejected_without_gpu(msa):
    with pytest.raises(msa.MsaError) as e:   # head_dim 64
        msa.msa_pool_blocks(None, None, np.zeros(8, np.float32), np.zeros(2, np.int64), np.zeros(2, np.int64), 1, 1,
                            8, 64, 64, 1e6, None, None, np.zeros(8, np.uint16), None, None, in_dtype=0, stream=0)
    assert e.value.status == msa.MSA_ERR_INVALID_ARG
    with pytest.raises(msa.MsaError) as e:   # top_k 65
        msa.msa_route_topk_workspace_size(1, 1, 1, 8, 10, 10, 65)
    assert e.value.status == msa.MSA_ERR_INVALID_ARG
    with pytest.raises(msa.MsaError) as e:   # E4M3 filter path without the E4M3 keys
        z = np.zeros(16, np.uint16)
        msa.msa_route_topk(z, [0, 1], z, np.zeros(2, np.int64), 1, 1, 1, 32, 8, 128, 4, np.zeros(4, np.int32),
                           np.zeros(4, np.float32), np.zeros(256, np.uint8), flags=msa.MSA_ROUTE_TENSOR_F8, stream=0)
    assert e.value.status == msa.MSA_ERR_INVALID_ARG
    with pytest.raises(msa.MsaError) as e:   # the layer-aggregated selection on the scan path
        z = np.zeros(16, np.uint16)
        msa.msa_route_topk(z, [0, 1], z, np.zeros(2, np.int64), 1, 1, 1, 32, 8, 128, 4, np.zeros(4, np.int32),
                           np.zeros(4, np.float32), np.zeros(256, np.uint8),
                           flags=msa.MSA_ROUTE_SCAN | msa.MSA_ROUTE_LAYER_MEAN, stream=0)
    assert e.value.status == msa.MSA_ERR_INVALID_ARG
    with pytest.raises(msa.MsaError) as e:   # head_dim 64
        msa.msa_route_filter_keys(np.zeros(16, np.uint16), 1, 1, 8, 64, np.zeros(16, np.uint8), stream=0)
    assert e.value.status == msa.MSA_ERR_INVALID_ARG
    with pytest.raises(msa.MsaError) as e:   # null ids
        msa.msa_gather_kv(np.zeros(16, np.uint16), 1, np.zeros(2, np.int64), None, 1, None, 1, 1, 1, 8, 128, 8,
                          np.zeros(16, np.uint16), np.zeros(1, np.int32), stream=0)
    assert e.value.status == msa.MSA_ERR_INVALID_ARG
    with pytest.raises(msa.MsaError) as e:   # 32 query heads over 5 key heads
        z = np.zeros(16, np.uint16)
        msa.msa_sparse_decode(z, z, z, 1, 1, 32, 5, 128, z, z, np.zeros(1, np.int32), 4, z, np.zeros(1, np.int32),
                              4, 16, 1e6, 0.1, z, z, stream=0)
    assert e.value.status == msa.MSA_ERR_INVALID_ARG
    z = np.zeros(16, np.uint16)
    for n_new, hq, h in ((4, 32, 5), (0, 32, 8), (4, 32, 2)):   # ratio 6.4; no tokens; ratio 16
        with pytest.raises(msa.MsaError) as e:
            msa.msa_sparse_prefill(z, z, z, n_new, 1, 1, hq, h, 128, z, z, np.zeros(1, np.int32), 8, z,
                                   np.zeros(1, np.int32), 4, 16, 1e6, 0.1, z, stream=0)
        assert e.value.status == msa.MSA_ERR_INVALID_ARG


def test_workspace_size_grows_with_bank(msa):
    a = msa.msa_route_topk_workspace_size(18, 1, 256, 8, 1000, 100, 16)
    b = msa.msa_route_topk_workspace_size(18, 1, 256, 8, 2000, 100, 16)
    assert b - a >= 18 * 1000 * 4 - 256


# ----------------------------------------------------------------------------- prototypes
_CTYPE = {"int32_t": ctypes.c_int32, "int64_t": ctypes.c_int64, "float": ctypes.c_float, "double": ctypes.c_double,
          "size_t": ctypes.c_size_t, "msa_dtype": ctypes.c_int32, "msa_stream_t": ctypes.c_void_p}


def _prototypes(header):
    """{name: [parameter C types]} of every function the header declares."""
    text = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", header)).read(), flags=re.S)
    out = {}
    for m in re.finditer(r"\b(msa_[a-z0-9_]+)\s*\(([^)]*)\)\s*;", text):
        params = [p.strip() for p in m.group(2).split(",")]
        params = [] if params == ["void"] or params == [""] else params
        # a parameter's type: the declaration without its trailing name
        out[m.group(1)] = [re.sub(r"\s*\b[A-Za-z_][A-Za-z_0-9]*$", "", p).strip() for p in params]
    return out


def _expected_ctype(c_type: str):
    t = c_type.replace("const ", "").strip()
    if "*" in t:
        return ctypes.c_void_p
    return _CTYPE[t]


@pytest.mark.parametrize("lib", sorted(HEADERS))
def test_binding_argtypes_follow_the_header_prototypes(msa, lib):
    # every entry point the binding declares takes the header's parameters in the header's
    # order and widths (pointers as c_void_p; char* and struct* count as pointers)
    import top_kv_routing_b200.abi as abi
    dll = getattr(abi, f"{lib}_lib")
    protos = _prototypes(HEADERS[lib])
    checked = 0
    for name, params in protos.items():
        fn = getattr(dll, name)
        if fn.argtypes is None:
            continue
        got = [a if a not in (ctypes.c_char_p,) else ctypes.c_void_p for a in fn.argtypes]
        want = [_expected_ctype(p) for p in params]
        assert len(got) == len(want), (name, len(got), len(want))
        for i, (g, w) in enumerate(zip(got, want)):
            ok = g == w or (w is ctypes.c_void_p and (g is ctypes.c_void_p or isinstance(g, type) and
                                                      issubclass(g, (ctypes._Pointer, ctypes.c_char_p))))
            assert ok, (name, i, params[i], g, w)
        checked += 1
    assert checked >= 1


def test_c_caller_compiled_against_the_headers(msa, tmp_path):
    # a C program built against include/*.h calls every entry point through the headers'
    # own prototypes with arguments the host checks must reject, and checks the statuses
    exe = tmp_path / "abi_check"
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), "-o",
                    str(exe), os.path.join(ROOT, "tests", "abi_check.c"), "-ldl"], check=True)
    out = subprocess.run([str(exe), msa.LIB_DIR], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout
