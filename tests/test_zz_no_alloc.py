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
from tests.helpers import DEC_MAX_ABS, DEC_REL_L2, bf16_tensor, bf16_to_np, rel_l2

pytestmark = pytest.mark.gpu

H, HQ, D = 8, 32, 128


def test_static_scratch_decode_matches_workspace_decode_on_consecutive_calls():
    import top_kv_routing_b200 as msa
    B, L, M_max, cap, len0, offset = 2, 3, 96, 8, 3, 16
    mem_len = torch.tensor([[96, 17, 0], [5, 64, 1]], dtype=torch.int32, device="cuda")
    mem = bf16_tensor(syn.fill(21, syn.STREAM_KBAR, 0, 0, 0, B * L * 2 * H * M_max, D, dtype="bf16")
                      ).reshape(B, L, 2, H, M_max, D)
    lk0 = bf16_tensor(syn.fill(21, syn.STREAM_LOCAL_K, 0, 0, 0, B * L * H * cap, D, dtype="bf16")).reshape(
        B, L, H, cap, D)
    lv0 = bf16_tensor(syn.fill(21, syn.STREAM_LOCAL_V, 0, 0, 0, B * L * H * cap, D, dtype="bf16")).reshape(
        B, L, H, cap, D)
    # two independent copies of the decode state, one per entry point
    state = {name: (lk0.clone(), lv0.clone(), torch.full((B,), len0, dtype=torch.int32, device="cuda"))
             for name in ("workspace", "static")}
    ws = torch.zeros(msa.msa_sparse_decode_workspace_size(B, L, HQ, H), dtype=torch.uint8, device="cuda")
    for step in range(2):  # two calls in a row: the scratch keeps the previous call's bytes
        q = bf16_tensor(syn.fill(21, syn.STREAM_DEC_Q, step, 0, 0, B * L * HQ, D, dtype="bf16")).reshape(B, L, HQ, D)
        kn = bf16_tensor(syn.fill(21, syn.STREAM_DEC_K, step, 0, 0, B * L * H, D, dtype="bf16")).reshape(B, L, H, D)
        vn = bf16_tensor(syn.fill(21, syn.STREAM_DEC_V, step, 0, 0, B * L * H, D, dtype="bf16")).reshape(B, L, H, D)
        outs = {}
        for name, (lk, lv, ln) in state.items():
            out = torch.full((B, L, HQ, D), float("nan"), dtype=torch.bfloat16, device="cuda")
            err = torch.zeros(1, dtype=torch.int32, device="cuda")
            if name == "workspace":
                msa.msa_sparse_decode(q, kn, vn, B, L, HQ, H, D, lk, lv, ln, cap, mem, mem_len, M_max, offset, 1e6,
                                      D ** -0.5, out, ws, err)
            else:
                msa.msa_sparse_decode_static(q, kn, vn, B, L, HQ, H, D, lk, lv, ln, cap, mem, mem_len, M_max, offset,
                                             1e6, D ** -0.5, out, err)
            torch.cuda.synchronize()
            assert int(err.item()) == 0
            outs[name] = bf16_to_np(out)
        a, b = outs["static"], outs["workspace"]
        assert np.isfinite(a).all()
        assert np.abs(a - b).max() <= DEC_MAX_ABS and rel_l2(a, b) <= DEC_REL_L2
        for i in range(3):
            assert torch.equal(state["static"][i], state["workspace"][i])


def test_static_scratch_rejects_sizes_beyond_its_capacity():
    import top_kv_routing_b200 as msa
    B, L = 64, 512  # partial sums of these sizes need far more than the built-in scratch
    z = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(msa.MsaError) as e:
        msa.msa_sparse_decode_static(z, z, z, B, L, HQ, H, D, z, z, torch.zeros(B, dtype=torch.int32, device="cuda"),
                                     4, z, torch.zeros(1, dtype=torch.int32, device="cuda"), 4, 16, 1e6, 0.1, z)
    assert e.value.status == msa.MSA_ERR_CAPACITY
