"""The allocation-free decode entry point.

Some callers of this library cannot allocate device memory (they only hold buffers handed
to them); msa_sparse_decode_static serves them with scratch built into the library.  This
file is collected last on purpose: it runs after every other test in the same process,
and must also pass on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

import msa_synth as syn
from tests.helpers import bf16_tensor, bf16_to_np

pytestmark = pytest.mark.gpu

H, HQ, D = 8, 32, 128


def _case(B, L, M_max, cap, seed):
    lens = [[(37 * b + 11 * l + seed) % (M_max + 1) for l in range(L)] for b in range(B)]
    mem_len = torch.tensor(lens, dtype=torch.int32, device="cuda")
    mem = bf16_tensor(syn.fill(seed, syn.STREAM_KBAR, 0, 0, 0, B * L * 2 * H * M_max, D, dtype="bf16")
                      ).reshape(B, L, 2, H, M_max, D)
    lk0 = bf16_tensor(syn.fill(seed, syn.STREAM_LOCAL_K, 0, 0, 0, B * L * H * cap, D, dtype="bf16")).reshape(
        B, L, H, cap, D)
    lv0 = bf16_tensor(syn.fill(seed, syn.STREAM_LOCAL_V, 0, 0, 0, B * L * H * cap, D, dtype="bf16")).reshape(
        B, L, H, cap, D)
    return mem, mem_len, lk0, lv0


def _step_inputs(seed, step, B, L):
    q = bf16_tensor(syn.fill(seed, syn.STREAM_DEC_Q, step, 0, 0, B * L * HQ, D, dtype="bf16")).reshape(B, L, HQ, D)
    kn = bf16_tensor(syn.fill(seed, syn.STREAM_DEC_K, step, 0, 0, B * L * H, D, dtype="bf16")).reshape(B, L, H, D)
    vn = bf16_tensor(syn.fill(seed, syn.STREAM_DEC_V, step, 0, 0, B * L * H, D, dtype="bf16")).reshape(B, L, H, D)
    return q, kn, vn


def test_static_scratch_decode_matches_workspace_decode_on_consecutive_calls():
    # The two entry points run the same kernel with the same key splits on the same inputs,
    # so their outputs and cache updates must agree bit for bit, call after call: first
    # two calls at one size, then a smaller size (its counters sit elsewhere in the shared
    # array, which still holds the earlier calls' bytes).  The static calls must not
    # allocate: neither torch's allocator nor the device's free memory moves across them
    # (after the first call, which may load the library's module and with it the array).
    import top_kv_routing_b200 as msa
    offset, cap = 16, 8
    plan = [(2, 3, 96, 21, 0), (2, 3, 96, 21, 1), (1, 2, 40, 22, 0)]
    states = {}
    for i, (B, L, M_max, seed, step) in enumerate(plan):
        if (B, L) not in states:
            mem, mem_len, lk0, lv0 = _case(B, L, M_max, cap, seed)
            states[(B, L)] = {"mem": mem, "mem_len": mem_len, "M_max": M_max,
                              "workspace": (lk0.clone(), lv0.clone(), torch.full((B,), 3, dtype=torch.int32,
                                                                                  device="cuda")),
                              "static": (lk0.clone(), lv0.clone(), torch.full((B,), 3, dtype=torch.int32,
                                                                               device="cuda")),
                              "ws": torch.zeros(msa.msa_sparse_decode_workspace_size(B, L, HQ, H), dtype=torch.uint8,
                                                device="cuda")}
        st = states[(B, L)]
        q, kn, vn = _step_inputs(seed, step, B, L)
        outs = {}
        for name in ("workspace", "static"):
            lk, lv, ln = st[name]
            out = torch.full((B, L, HQ, D), float("nan"), dtype=torch.bfloat16, device="cuda")
            err = torch.zeros(1, dtype=torch.int32, device="cuda")
            torch.cuda.synchronize()
            if name == "workspace":
                msa.msa_sparse_decode(q, kn, vn, B, L, HQ, H, D, lk, lv, ln, cap, st["mem"], st["mem_len"],
                                      st["M_max"], offset, 1e6, D ** -0.5, out, st["ws"], err)
            else:
                alloc0, free0 = torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0]
                msa.msa_sparse_decode_static(q, kn, vn, B, L, HQ, H, D, lk, lv, ln, cap, st["mem"], st["mem_len"],
                                             st["M_max"], offset, 1e6, D ** -0.5, out, err)
                torch.cuda.synchronize()
                assert torch.cuda.memory_allocated() == alloc0
                if i > 0:
                    assert torch.cuda.mem_get_info()[0] == free0
            torch.cuda.synchronize()
            assert int(err.item()) == 0
            outs[name] = bf16_to_np(out)
        a, b = outs["static"], outs["workspace"]
        assert np.isfinite(a).all()
        assert np.array_equal(a, b)
        for j in range(3):
            assert torch.equal(st["static"][j], st["workspace"][j])


def test_static_scratch_rejects_sizes_beyond_its_capacity():
    import top_kv_routing_b200 as msa
    B, L = 64, 512  # partial sums of these sizes need far more than the built-in scratch
    z = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(msa.MsaError) as e:
        msa.msa_sparse_decode_static(z, z, z, B, L, HQ, H, D, z, z, torch.zeros(B, dtype=torch.int32, device="cuda"),
                                     4, z, torch.zeros(1, dtype=torch.int32, device="cuda"), 4, 16, 1e6, 0.1, z)
    assert e.value.status == msa.MSA_ERR_CAPACITY
