"""Thin ctypes binding over the six C-ABI libraries in ``lib/`` (see ``include/*.h``).

Argument marshalling only; every step runs in the libraries' CUDA kernels.  PyTorch is
used by callers for device memory and streams.  There is no CPU fallback: importing this
module fails if the libraries have not been built (``python top_kv_routing_b200/build.py``).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_DIR = os.path.join(_HERE, "lib")

MSA_OK, MSA_ERR_INVALID_ARG, MSA_ERR_UNSUPPORTED, MSA_ERR_CUDA, MSA_ERR_CAPACITY, MSA_ERR_TIMEOUT, MSA_ERR_IO = range(7)
MSA_F32, MSA_BF16 = 0, 1
MSA_ROUTE_AUTO, MSA_ROUTE_SCAN, MSA_ROUTE_TENSOR, MSA_ROUTE_TENSOR_F8 = 0, 1, 2, 3
MSA_ROUTE_LAYER_MEAN = 16  # OR-ed with a path: one selection for all layers
MSA_ROUTE_FILTER_SCORES = 32  # OR-ed with a tensor path: the filter's own top-k and scores
(MSA_DEVERR_CAPACITY, MSA_DEVERR_BAD_DOC, MSA_DEVERR_LOCAL_FULL, MSA_DEVERR_BAD_OFFSETS, MSA_DEVERR_TIMEOUT,
 MSA_DEVERR_UNCERTIFIED) = 1, 2, 4, 8, 16, 32

_STATUS = {1: "MSA_ERR_INVALID_ARG", 2: "MSA_ERR_UNSUPPORTED", 3: "MSA_ERR_CUDA", 4: "MSA_ERR_CAPACITY",
           5: "MSA_ERR_TIMEOUT", 6: "MSA_ERR_IO"}


class MsaError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        super().__init__(f"{where}: {_STATUS.get(status, status)}: {msg}")
        self.status = status


def _load(name: str) -> ctypes.CDLL:
    path = os.path.join(LIB_DIR, f"libmsa_{name}.so")
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build the CUDA libraries first "
                          "(python -m top_kv_routing_b200.build)")
    return ctypes.CDLL(path)


_p, _i32, _i64, _f32, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t

pool_lib = _load("pool")
route_lib = _load("route")
gather_lib = _load("gather")
decode_lib = _load("decode")
prefill_lib = _load("prefill")
bank_lib = _load("bank")

pool_lib.msa_count_chunks.argtypes = [_p, _i32, _i32, _p]
pool_lib.msa_count_chunks.restype = _i64
pool_lib.msa_pool_blocks.argtypes = [_p, _p, _p, _i32, _p, _p, _i32, _i64, _i32, _i32, _i32, _f32,
                                     _p, _p, _p, _p, _p, _p]
pool_lib.msa_pool_blocks.restype = _i32
pool_lib.msa_pool_last_error.restype = ctypes.c_char_p

route_lib.msa_route_topk_workspace_size.argtypes = [_i32, _i32, _i32, _i32, _i64, _i32, _i32,
                                                    ctypes.POINTER(_sz)]
route_lib.msa_route_topk_workspace_size.restype = _i32
route_lib.msa_route_topk.argtypes = [_p, _i32, _p, _i32, _p, _p, _p, _i32, _i64, _i32, _i32, _i32, _i32, _i32,
                                     _p, _p, _p, _sz, _i32, _p, _p]
route_lib.msa_route_topk_hidden.argtypes = [_p, _p, _i32, _p, _i32, _p, _p, _p, _i32, _i64, _i32, _i32, _i32, _i32,
                                            _i32, _p, _p, _p, _sz, _i32, _p, _p]
route_lib.msa_route_topk_hidden.restype = _i32
route_lib.msa_route_filter_keys.argtypes = [_p, _i32, _i64, _i32, _i32, _p, _p]
route_lib.msa_route_filter_keys.restype = _i32
route_lib.msa_route_topk.restype = _i32
route_lib.msa_route_last_launch_count.restype = _i32
route_lib.msa_route_last_error.restype = ctypes.c_char_p
route_lib.msa_route_wait_selftest.argtypes = [_i64, _i32, _p, _p]
route_lib.msa_route_wait_selftest.restype = _i32
route_lib.msa_route_set_pair_mode.argtypes = [_i32]
route_lib.msa_route_set_pair_mode.restype = _i32
route_lib.msa_route_set_profile_events.argtypes = [_p, _p]
route_lib.msa_route_set_profile_events.restype = _i32
route_lib.msa_route_set_query_profile_events.argtypes = [_p, _p]
route_lib.msa_route_set_query_profile_events.restype = _i32

gather_lib.msa_gather_kv.argtypes = [_p, _i64, _p, _p, _i32, _p, _i32, _i32, _i32, _i32, _i32, _i32, _p, _p,
                                     _p, _p]
gather_lib.msa_gather_kv.restype = _i32
gather_lib.msa_gather_last_error.restype = ctypes.c_char_p

decode_lib.msa_sparse_decode.argtypes = [_p, _p, _p, _i32, _i32, _i32, _i32, _i32, _p, _p, _p, _i32, _p, _p,
                                         _i32, _i32, _f32, _f32, _p, _p, _sz, _p, _p]
decode_lib.msa_sparse_decode_workspace_size.argtypes = [_i32, _i32, _i32, _i32, ctypes.POINTER(_sz)]
decode_lib.msa_sparse_decode_workspace_size.restype = _i32
decode_lib.msa_sparse_decode.restype = _i32
decode_lib.msa_decode_last_error.restype = ctypes.c_char_p
decode_lib.msa_sparse_decode_static.argtypes = [_p, _p, _p, _i32, _i32, _i32, _i32, _i32, _p, _p, _p, _i32, _p, _p,
                                                _i32, _i32, _f32, _f32, _p, _p, _p]
decode_lib.msa_sparse_decode_static.restype = _i32
MSA_DECODE_STATIC_SCRATCH_BYTES = 8 << 20

prefill_lib.msa_sparse_prefill.argtypes = [_p, _p, _p, _i32, _i32, _i32, _i32, _i32, _i32, _p, _p, _p, _i32, _p,
                                           _p, _i32, _i32, _f32, _f32, _p, _p, _p]
prefill_lib.msa_sparse_prefill.restype = _i32
prefill_lib.msa_prefill_last_error.restype = ctypes.c_char_p


class MsaBankInfo(ctypes.Structure):
    _fields_ = [("n_layers", _i32), ("n_heads", _i32), ("head_dim", _i32), ("block_tokens", _i32),
                ("n_docs", _i64), ("n_blocks", _i64), ("fields", ctypes.c_uint32)]


MSA_BANK_KR, MSA_BANK_KR_F8, MSA_BANK_KV, MSA_BANK_NORM = 1, 2, 4, 8
bank_lib.msa_bank_save.argtypes = [ctypes.c_char_p, ctypes.POINTER(MsaBankInfo), _p, _p, _p, _p, _p, _p, _sz, _p]
bank_lib.msa_bank_save.restype = _i32
bank_lib.msa_bank_read_info.argtypes = [ctypes.c_char_p, ctypes.POINTER(MsaBankInfo)]
bank_lib.msa_bank_read_info.restype = _i32
bank_lib.msa_bank_load.argtypes = [ctypes.c_char_p, _p, _p, _p, _p, _p, _p, _sz, _p]
bank_lib.msa_bank_load.restype = _i32
bank_lib.msa_bank_relayout.argtypes = [_p, _p, _i32, _i64, _i64, _i64, _p]
bank_lib.msa_bank_relayout.restype = _i32
bank_lib.msa_bank_append_offsets.argtypes = [_p, _i64, _p, _i64, _p]
bank_lib.msa_bank_append_offsets.restype = _i32
bank_lib.msa_bank_last_error.restype = ctypes.c_char_p

# Kernel launches enqueued by each entry point (the route count is read back per call).
LAUNCHES_POOL = 1
LAUNCHES_GATHER = 1
LAUNCHES_DECODE = 1
LAUNCHES_PREFILL = 3


def loaded_libraries() -> list[str]:
    return [os.path.join(LIB_DIR, f"libmsa_{n}.so") for n in ("pool", "route", "gather", "decode", "prefill", "bank")]


def _ptr(t) -> int | None:
    """Raw address of a torch tensor / numpy array (None stays NULL)."""
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


def _nbytes(t) -> int:
    if t is None:
        return 0
    if isinstance(t, np.ndarray):
        return t.nbytes
    return t.numel() * t.element_size()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _check(status: int, where: str, lib, err_fn: str):
    if status != MSA_OK:
        raise MsaError(status, where, (getattr(lib, err_fn)() or b"").decode())


# ----------------------------------------------------------------------------- step 1

def msa_count_chunks(doc_tok_offsets, chunk: int = 64):
    """Host: (block count, per-document block offsets int64 [n_docs+1])."""
    o = np.ascontiguousarray(doc_tok_offsets, dtype=np.int64)
    out = np.empty_like(o)
    n = pool_lib.msa_count_chunks(o.ctypes.data, len(o) - 1, chunk, out.ctypes.data)
    if n < 0:
        raise MsaError(MSA_ERR_INVALID_ARG, "msa_count_chunks", "bad offsets")
    return int(n), out


def msa_pool_blocks(k, v, kr, doc_tok_offsets, doc_chunk_offsets, n_docs: int, n_chunks: int, n_heads: int,
                    head_dim: int, chunk: int, rope_theta: float, k_bar=None, v_bar=None, kr_hat=None,
                    kr_norm=None, dev_err=None, in_dtype: int | None = None, stream=None):
    if in_dtype is None:
        x = next(t for t in (k, v, kr) if t is not None)
        in_dtype = MSA_BF16 if str(x.dtype) == "torch.bfloat16" else MSA_F32
    st = pool_lib.msa_pool_blocks(_ptr(k), _ptr(v), _ptr(kr), in_dtype, _ptr(doc_tok_offsets),
                                  _ptr(doc_chunk_offsets), n_docs, n_chunks, n_heads, head_dim, chunk,
                                  rope_theta, _ptr(k_bar), _ptr(v_bar), _ptr(kr_hat), _ptr(kr_norm),
                                  _ptr(dev_err), _stream(stream))
    _check(st, "msa_pool_blocks", pool_lib, "msa_pool_last_error")


# ----------------------------------------------------------------------------- step 2

def msa_route_topk_workspace_size(n_layers: int, n_queries: int, total_q_tokens: int, n_kv_heads: int,
                                  n_chunks: int, n_docs: int, top_k: int) -> int:
    out = _sz(0)
    st = route_lib.msa_route_topk_workspace_size(n_layers, n_queries, total_q_tokens, n_kv_heads, n_chunks,
                                                 n_docs, top_k, ctypes.byref(out))
    _check(st, "msa_route_topk_workspace_size", route_lib, "msa_route_last_error")
    return int(out.value)


def msa_route_topk(qr, q_offsets, kr_hat, doc_chunk_offsets, n_docs: int, n_chunks: int, n_layers: int,
                   n_q_heads: int, n_kv_heads: int, head_dim: int, top_k: int, out_ids, out_scores, workspace,
                   flags: int = MSA_ROUTE_AUTO, dev_err=None, q_dtype: int | None = None, stream=None,
                   kr_f8=None) -> int:
    """Returns the number of kernels the call enqueued.  kr_f8: the E4M3 keys written by
    msa_route_filter_keys (needed by MSA_ROUTE_TENSOR_F8, picked by MSA_ROUTE_AUTO)."""
    qo = np.ascontiguousarray(q_offsets, dtype=np.int32)
    if q_dtype is None:
        q_dtype = MSA_BF16 if str(qr.dtype) == "torch.bfloat16" else MSA_F32
    ws_bytes = _nbytes(workspace)
    st = route_lib.msa_route_topk(_ptr(qr), q_dtype, qo.ctypes.data, len(qo) - 1, _ptr(kr_hat), _ptr(kr_f8),
                                  _ptr(doc_chunk_offsets), n_docs, n_chunks, n_layers, n_q_heads, n_kv_heads,
                                  head_dim, top_k, _ptr(out_ids), _ptr(out_scores), _ptr(workspace), ws_bytes,
                                  flags, _ptr(dev_err), _stream(stream))
    _check(st, "msa_route_topk", route_lib, "msa_route_last_error")
    return int(route_lib.msa_route_last_launch_count())


def msa_route_topk_hidden(hidden, w_router_q, hidden_size: int, q_offsets, kr_hat, doc_chunk_offsets, n_docs: int,
                          n_chunks: int, n_layers: int, n_q_heads: int, n_kv_heads: int, head_dim: int, top_k: int,
                          out_ids, out_scores, workspace, flags: int = MSA_ROUTE_AUTO, dev_err=None, stream=None,
                          kr_f8=None) -> int:
    """msa_route_topk with the router query projection (hidden [T][hidden_size] bf16 times
    w_router_q [L][Hq*128][hidden_size] bf16) fused in; returns the launches enqueued."""
    qo = np.ascontiguousarray(q_offsets, dtype=np.int32)
    st = route_lib.msa_route_topk_hidden(_ptr(hidden), _ptr(w_router_q), hidden_size, qo.ctypes.data, len(qo) - 1,
                                         _ptr(kr_hat), _ptr(kr_f8), _ptr(doc_chunk_offsets), n_docs, n_chunks,
                                         n_layers, n_q_heads, n_kv_heads, head_dim, top_k, _ptr(out_ids),
                                         _ptr(out_scores), _ptr(workspace), _nbytes(workspace), flags, _ptr(dev_err),
                                         _stream(stream))
    _check(st, "msa_route_topk_hidden", route_lib, "msa_route_last_error")
    return int(route_lib.msa_route_last_launch_count())


def msa_route_filter_keys(kr_hat, n_layers: int, n_chunks: int, n_kv_heads: int, head_dim: int, kr_f8,
                          stream=None) -> None:
    """E4M3 filter copy of the unit routing keys (x 256, per-head renormalised) into kr_f8
    (uint8 tensor of kr_hat's shape)."""
    st = route_lib.msa_route_filter_keys(_ptr(kr_hat), n_layers, n_chunks, n_kv_heads, head_dim, _ptr(kr_f8),
                                         _stream(stream))
    _check(st, "msa_route_filter_keys", route_lib, "msa_route_last_error")


def msa_route_wait_selftest(wait_ns: int, release_first: bool, dev_err, stream=None) -> None:
    """The bounded-wait self test of the routing library (include/msa_route.h)."""
    st = route_lib.msa_route_wait_selftest(int(wait_ns), 1 if release_first else 0, _ptr(dev_err), _stream(stream))
    _check(st, "msa_route_wait_selftest", route_lib, "msa_route_last_error")


def msa_route_set_pair_mode(enabled: bool) -> None:
    """Tensor-core routing on SM pairs (M=256 tiles, the default) or one CTA per tile."""
    route_lib.msa_route_set_pair_mode(1 if enabled else 0)


def msa_route_set_profile_events(start_event=None, stop_event=None):
    """torch.cuda.Event pair (timing enabled) recorded around the score kernel of later
    msa_route_topk calls on this thread; None, None turns it off."""
    a = None if start_event is None else start_event.cuda_event
    b = None if stop_event is None else stop_event.cuda_event
    route_lib.msa_route_set_profile_events(a, b)


def msa_route_set_query_profile_events(start_event=None, stop_event=None):
    """The same around the query stage (preparation, or the fused projection)."""
    a = None if start_event is None else start_event.cuda_event
    b = None if stop_event is None else stop_event.cuda_event
    route_lib.msa_route_set_query_profile_events(a, b)


# ----------------------------------------------------------------------------- step 3

def msa_gather_kv(host_kv, n_store_chunks: int, doc_chunk_offsets, doc_store_offsets, n_docs: int, ids,
                  n_queries: int, n_layers: int, top_k: int, n_heads: int, head_dim: int, max_mem_chunks: int,
                  dev_kv, mem_len, dev_err=None, stream=None):
    st = gather_lib.msa_gather_kv(_ptr(host_kv), n_store_chunks, _ptr(doc_chunk_offsets), _ptr(doc_store_offsets),
                                  n_docs, _ptr(ids), n_queries, n_layers, top_k, n_heads, head_dim,
                                  max_mem_chunks, _ptr(dev_kv), _ptr(mem_len), _ptr(dev_err), _stream(stream))
    _check(st, "msa_gather_kv", gather_lib, "msa_gather_last_error")


# ----------------------------------------------------------------------------- step 4

def msa_sparse_decode_workspace_size(n_queries: int, n_layers: int, n_q_heads: int, n_kv_heads: int) -> int:
    out = _sz(0)
    st = decode_lib.msa_sparse_decode_workspace_size(n_queries, n_layers, n_q_heads, n_kv_heads, ctypes.byref(out))
    _check(st, "msa_sparse_decode_workspace_size", decode_lib, "msa_decode_last_error")
    return int(out.value)


def msa_sparse_decode(q, k_new, v_new, n_queries: int, n_layers: int, n_q_heads: int, n_kv_heads: int,
                      head_dim: int, local_k, local_v, local_len, local_cap: int, mem_kv, mem_len,
                      max_mem_chunks: int, rope_pos_offset: int, rope_theta: float, softmax_scale: float, out,
                      workspace, dev_err=None, stream=None):
    ws_bytes = _nbytes(workspace)
    st = decode_lib.msa_sparse_decode(_ptr(q), _ptr(k_new), _ptr(v_new), n_queries, n_layers, n_q_heads,
                                      n_kv_heads, head_dim, _ptr(local_k), _ptr(local_v), _ptr(local_len),
                                      local_cap, _ptr(mem_kv), _ptr(mem_len), max_mem_chunks, rope_pos_offset,
                                      rope_theta, softmax_scale, _ptr(out), _ptr(workspace), ws_bytes, _ptr(dev_err),
                                      _stream(stream))
    _check(st, "msa_sparse_decode", decode_lib, "msa_decode_last_error")


def msa_sparse_decode_static(q, k_new, v_new, n_queries: int, n_layers: int, n_q_heads: int, n_kv_heads: int,
                             head_dim: int, local_k, local_v, local_len, local_cap: int, mem_kv, mem_len,
                             max_mem_chunks: int, rope_pos_offset: int, rope_theta: float, softmax_scale: float,
                             out, dev_err=None, stream=None):
    """msa_sparse_decode with the library's built-in scratch instead of a caller workspace,
    for callers that cannot allocate device memory (see include/msa_decode.h)."""
    st = decode_lib.msa_sparse_decode_static(_ptr(q), _ptr(k_new), _ptr(v_new), n_queries, n_layers, n_q_heads,
                                             n_kv_heads, head_dim, _ptr(local_k), _ptr(local_v), _ptr(local_len),
                                             local_cap, _ptr(mem_kv), _ptr(mem_len), max_mem_chunks,
                                             rope_pos_offset, rope_theta, softmax_scale, _ptr(out), _ptr(dev_err),
                                             _stream(stream))
    _check(st, "msa_sparse_decode_static", decode_lib, "msa_decode_last_error")


# ----------------------------------------------------------------------------- prefill

def msa_sparse_prefill(q, k_new, v_new, n_new: int, n_queries: int, n_layers: int, n_q_heads: int, n_kv_heads: int,
                       head_dim: int, local_k, local_v, local_len, local_cap: int, mem_kv, mem_len,
                       max_mem_chunks: int, rope_pos_offset: int, rope_theta: float, softmax_scale: float, out,
                       dev_err=None, stream=None):
    """n_new tokens per query through sparse attention (include/msa_prefill.h)."""
    st = prefill_lib.msa_sparse_prefill(_ptr(q), _ptr(k_new), _ptr(v_new), n_new, n_queries, n_layers, n_q_heads,
                                        n_kv_heads, head_dim, _ptr(local_k), _ptr(local_v), _ptr(local_len),
                                        local_cap, _ptr(mem_kv), _ptr(mem_len), max_mem_chunks, rope_pos_offset,
                                        rope_theta, softmax_scale, _ptr(out), _ptr(dev_err), _stream(stream))
    _check(st, "msa_sparse_prefill", prefill_lib, "msa_prefill_last_error")


# ----------------------------------------------------------------------------- bank files

def _path(p) -> bytes:
    return os.fsencode(p)


def _bank_stream(stream):
    """The bank calls also serve host arrays on machines without a GPU (stream 0 there)."""
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else 0
    return _stream(stream)


def msa_bank_save(path, info: MsaBankInfo, doc_chunk_offsets, kr_hat=None, kr_f8=None, content_kv=None,
                  kr_norm=None, staging=None, stream=None):
    """Writes a bank file (include/msa_bank.h); doc_chunk_offsets is a host int64 array."""
    off = np.ascontiguousarray(doc_chunk_offsets, dtype=np.int64)
    st = bank_lib.msa_bank_save(_path(path), ctypes.byref(info), _ptr(off), _ptr(kr_hat), _ptr(kr_f8),
                                _ptr(content_kv), _ptr(kr_norm), _ptr(staging), _nbytes(staging) if staging is not None
                                else 0, _bank_stream(stream))
    _check(st, "msa_bank_save", bank_lib, "msa_bank_last_error")


def msa_bank_read_info(path) -> MsaBankInfo:
    info = MsaBankInfo()
    st = bank_lib.msa_bank_read_info(_path(path), ctypes.byref(info))
    _check(st, "msa_bank_read_info", bank_lib, "msa_bank_last_error")
    return info


def msa_bank_load(path, doc_chunk_offsets, kr_hat=None, kr_f8=None, content_kv=None, kr_norm=None, staging=None,
                  stream=None):
    """Reads a bank file into caller arrays; doc_chunk_offsets is a host int64 array [n_docs + 1]."""
    st = bank_lib.msa_bank_load(_path(path), _ptr(doc_chunk_offsets), _ptr(kr_hat), _ptr(kr_f8), _ptr(content_kv),
                                _ptr(kr_norm), _ptr(staging), _nbytes(staging) if staging is not None else 0,
                                _bank_stream(stream))
    _check(st, "msa_bank_load", bank_lib, "msa_bank_last_error")


def msa_bank_relayout(src, dst, n_layers: int, rows_old: int, rows_new: int, row_bytes: int, stream=None):
    st = bank_lib.msa_bank_relayout(_ptr(src), _ptr(dst), n_layers, rows_old, rows_new, row_bytes, _bank_stream(stream))
    _check(st, "msa_bank_relayout", bank_lib, "msa_bank_last_error")


def msa_bank_append_offsets(old_offsets, new_offsets) -> np.ndarray:
    a = np.ascontiguousarray(old_offsets, dtype=np.int64)
    b = np.ascontiguousarray(new_offsets, dtype=np.int64)
    out = np.empty(len(a) + len(b) - 1, dtype=np.int64)
    st = bank_lib.msa_bank_append_offsets(_ptr(a), len(a) - 1, _ptr(b), len(b) - 1, _ptr(out))
    _check(st, "msa_bank_append_offsets", bank_lib, "msa_bank_last_error")
    return out
