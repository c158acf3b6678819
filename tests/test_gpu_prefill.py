"""GPU parity of msa_sparse_prefill (a block of new tokens per query through sparse
attention) against the oracle's prefill, which is the decode recurrence token by token:
ragged memory, a local prefix, blocks that span several CTAs with a ragged tail, every
group size, consecutive blocks, a decode step continuing from a prefilled cache, and the
full-cache and capacity edge cases."""
import numpy as np
import pytest
import torch

import msa_synth as syn
import oracle
from tests.helpers import DEC_MAX_ABS, DEC_REL_L2, POOL_TOL, bf16_tensor, bf16_to_np, rel_l2

pytestmark = pytest.mark.gpu

H, HQ, D = 8, 32, 128
THETA = 1e6


@pytest.fixture(scope="module")
def msa():
    import top_kv_routing_b200 as m
    return m


def _err():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def prefill_inputs(seed: int, block: int, B: int, L: int, T: int, hq: int, h: int):
    """bf16 bits of one block's q [B][L][T][hq][d], k_new and v_new [B][L][T][h][d] (the
    decode streams, sub-stream 1, layer slot = block index)."""
    q = syn.fill(seed, syn.STREAM_DEC_Q, block, 1, 0, B * L * T * hq, D, dtype="bf16").reshape(B, L, T, hq, D)
    k = syn.fill(seed, syn.STREAM_DEC_K, block, 1, 0, B * L * T * h, D, dtype="bf16").reshape(B, L, T, h, D)
    v = syn.fill(seed, syn.STREAM_DEC_V, block, 1, 0, B * L * T * h, D, dtype="bf16").reshape(B, L, T, h, D)
    return q, k, v


class Case:
    """Device state (memory, local cache, lengths) next to the oracle's copy of the cache."""

    def __init__(self, B, L, M_max, mem_len, len0, cap, seed=0, hq=HQ, h=H):
        self.B, self.L, self.M_max, self.cap, self.seed, self.hq, self.h = B, L, M_max, cap, seed, hq, h
        self.mem_len = mem_len
        self.mem_bits = syn.fill(seed, syn.STREAM_KBAR, 0, 0, 0, B * L * 2 * h * M_max, D,
                                 dtype="bf16").reshape(B, L, 2, h, M_max, D)
        lk = syn.fill(seed, syn.STREAM_LOCAL_K, 0, 0, 0, B * L * h * cap, D, dtype="bf16").reshape(B, L, h, cap, D)
        lv = syn.fill(seed, syn.STREAM_LOCAL_V, 0, 0, 0, B * L * h * cap, D, dtype="bf16").reshape(B, L, h, cap, D)
        self.d_mem = bf16_tensor(self.mem_bits)
        self.d_lk, self.d_lv = bf16_tensor(lk), bf16_tensor(lv)
        self.len = list(len0)
        self.d_len = torch.tensor(len0, dtype=torch.int32, device="cuda")
        self.d_mlen = torch.tensor(mem_len, dtype=torch.int32, device="cuda")
        self.o_lk = syn.bf16_bits_to_f32(lk).astype(np.float64).copy()
        self.o_lv = syn.bf16_bits_to_f32(lv).astype(np.float64).copy()
        self.err = _err()
        self.scale = D ** -0.5

    def prefill(self, msa, block, T, offset):
        B, L, hq, h = self.B, self.L, self.hq, self.h
        qb, kb, vb = prefill_inputs(self.seed, block, B, L, T, hq, h)
        out = torch.full((B, L, T, hq, D), float("nan"), dtype=torch.bfloat16, device="cuda")
        msa.msa_sparse_prefill(bf16_tensor(qb), bf16_tensor(kb), bf16_tensor(vb), T, B, L, hq, h, D, self.d_lk,
                               self.d_lv, self.d_len, self.cap, self.d_mem, self.d_mlen, self.M_max, offset, THETA,
                               self.scale, out, self.err)
        torch.cuda.synchronize()
        got = bf16_to_np(out)
        f = syn.bf16_bits_to_f32
        worst_abs, worst_rel = 0.0, 0.0
        for b in range(B):
            i0 = self.len[b]
            for l in range(L):
                m = min(self.mem_len[b][l], self.M_max)
                ref = oracle.prefill(f(qb[b, l]), f(kb[b, l]), f(vb[b, l]), f(self.mem_bits[b, l]), m,
                                     self.o_lk[b, l], self.o_lv[b, l], i0, offset + i0, THETA, self.scale)
                worst_abs = max(worst_abs, float(np.abs(got[b, l] - ref).max()))
                worst_rel = max(worst_rel, rel_l2(got[b, l], ref))
        # appended rows: rotated keys (bf16 rounding of the oracle's) and exact values
        lk, lv = bf16_to_np(self.d_lk), bf16_to_np(self.d_lv)
        for b in range(B):
            sl = slice(self.len[b], self.len[b] + T)
            assert np.abs(lk[b, :, :, sl] - self.o_lk[b, :, :, sl]).max() <= POOL_TOL
            assert np.array_equal(lv[b, :, :, sl], self.o_lv[b, :, :, sl].astype(np.float32))
        self.len = [x + T for x in self.len]
        assert self.d_len.cpu().tolist() == self.len
        return worst_abs, worst_rel


def _run(msa, case, blocks, offset=16):
    for s, T in enumerate(blocks):
        worst_abs, worst_rel = case.prefill(msa, s, T, offset)
        assert worst_abs <= DEC_MAX_ABS and worst_rel <= DEC_REL_L2, (s, T, worst_abs, worst_rel)
    assert int(case.err.item()) == 0


def test_prefill_ragged_memory_and_prefix(msa):
    # G = 4: 16 tokens per CTA, so 37 tokens take three CTAs (the last one ragged); then a
    # second block continues from the advanced lengths
    case = Case(B=2, L=2, M_max=300, mem_len=[[300, 17], [0, 5]], len0=[3, 0], cap=120)
    _run(msa, case, [37, 20])


def test_prefill_long_context(msa):
    case = Case(B=1, L=2, M_max=700, mem_len=[[700, 513]], len0=[250], cap=400, seed=3)
    _run(msa, case, [130])


def test_prefill_partly_filled_tiles(msa):
    # score tiles hold 128 keys: memory lengths 200 and 100 and local lengths 102..110 leave
    # 65..127 valid keys in a tile (both 64-key boxes loaded, the rest masked and its value
    # rows zeroed); 40 tokens at G = 4 span two units
    case = Case(B=1, L=2, M_max=200, mem_len=[[200, 100]], len0=[70], cap=110, seed=23)
    _run(msa, case, [40])


@pytest.mark.parametrize("hq,h,T", [(8, 8, 70), (16, 8, 33), (64, 8, 9)])
def test_prefill_group_sizes(msa, hq, h, T):
    # G = 1, 2, 8: 64, 32, 8 tokens per CTA, each with a ragged tail
    case = Case(B=1, L=1, M_max=40, mem_len=[[40]], len0=[2], cap=2 + T, seed=5, hq=hq, h=h)
    _run(msa, case, [T])


def test_prefill_single_token_and_empty_context(msa):
    # no memory, no prefix: the first token attends to itself alone (output = its value)
    case = Case(B=1, L=1, M_max=16, mem_len=[[0]], len0=[0], cap=8, seed=7)
    _run(msa, case, [1, 1, 5])


def test_decode_continues_from_prefilled_cache(msa):
    B, L, T = 2, 2, 21
    case = Case(B=B, L=L, M_max=64, mem_len=[[64, 1], [30, 0]], len0=[1, 4], cap=40, seed=11)
    _run(msa, case, [T])
    ws = torch.zeros(msa.msa_sparse_decode_workspace_size(B, L, HQ, H), dtype=torch.uint8, device="cuda")
    qb = syn.fill(11, syn.STREAM_DEC_Q, 0, 0, 0, B * L * HQ, D, dtype="bf16").reshape(B, L, HQ, D)
    kb = syn.fill(11, syn.STREAM_DEC_K, 0, 0, 0, B * L * H, D, dtype="bf16").reshape(B, L, H, D)
    vb = syn.fill(11, syn.STREAM_DEC_V, 0, 0, 0, B * L * H, D, dtype="bf16").reshape(B, L, H, D)
    out = torch.full((B, L, HQ, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    msa.msa_sparse_decode(bf16_tensor(qb), bf16_tensor(kb), bf16_tensor(vb), B, L, HQ, H, D, case.d_lk, case.d_lv,
                          case.d_len, case.cap, case.d_mem, case.d_mlen, case.M_max, 16, THETA, case.scale, out, ws,
                          case.err)
    torch.cuda.synchronize()
    got = bf16_to_np(out)
    f = syn.bf16_bits_to_f32
    for b in range(B):
        i = case.len[b]
        for l in range(L):
            ref = oracle.decode(f(qb[b, l]), f(kb[b, l]), f(vb[b, l]), f(case.mem_bits[b, l]), case.mem_len[b][l],
                                case.o_lk[b, l], case.o_lv[b, l], i, 16 + i, THETA, case.scale)
            assert np.abs(got[b, l] - ref).max() <= DEC_MAX_ABS and rel_l2(got[b, l], ref) <= DEC_REL_L2
    assert int(case.err.item()) == 0
    assert case.d_len.cpu().tolist() == [x + 1 for x in case.len]


def test_prefill_full_cache_sets_flag_and_skips(msa):
    # query 0's cache cannot hold the block: skipped whole; query 1 proceeds
    B, L, T, cap, M = 2, 1, 4, 6, 8
    case = Case(B=B, L=L, M_max=M, mem_len=[[M], [M]], len0=[3, 2], cap=cap, seed=13)
    lk0 = bf16_to_np(case.d_lk)
    qb, kb, vb = prefill_inputs(13, 0, B, L, T, HQ, H)
    out = torch.zeros((B, L, T, HQ, D), dtype=torch.bfloat16, device="cuda")
    msa.msa_sparse_prefill(bf16_tensor(qb), bf16_tensor(kb), bf16_tensor(vb), T, B, L, HQ, H, D, case.d_lk,
                           case.d_lv, case.d_len, cap, case.d_mem, case.d_mlen, M, 16, THETA, case.scale, out,
                           case.err)
    torch.cuda.synchronize()
    assert int(case.err.item()) & msa.MSA_DEVERR_LOCAL_FULL
    assert case.d_len.cpu().tolist() == [3, 6]
    got = bf16_to_np(out)
    assert float(np.abs(got[0]).sum()) == 0.0 and np.isfinite(got[1]).all() and float(np.abs(got[1]).sum()) > 0
    assert np.array_equal(bf16_to_np(case.d_lk)[0], lk0[0])
    f = syn.bf16_bits_to_f32
    ref = oracle.prefill(f(qb[1, 0]), f(kb[1, 0]), f(vb[1, 0]), f(case.mem_bits[1, 0]), M, case.o_lk[1, 0],
                         case.o_lv[1, 0], 2, 18, THETA, case.scale)
    assert np.abs(got[1, 0] - ref).max() <= DEC_MAX_ABS


def test_prefill_memory_length_clamped(msa):
    # mem_len above max_mem_chunks reads the first max_mem_chunks rows and flags it
    case = Case(B=1, L=1, M_max=20, mem_len=[[25]], len0=[0], cap=16, seed=17)
    worst_abs, worst_rel = case.prefill(msa, 0, 9, 16)
    assert worst_abs <= DEC_MAX_ABS and worst_rel <= DEC_REL_L2
    assert int(case.err.item()) == msa.MSA_DEVERR_CAPACITY


def test_prefill_bench_shape_sampled_layers(msa):
    # the benchmark's prefill: 256 tokens, 18 layers, GQA 32/8, 256 memory rows, empty
    # prefix; two layers checked in full against the oracle, every layer's output finite
    B, L, T, M = 1, 18, 256, 256
    case = Case(B=B, L=L, M_max=M, mem_len=[[M] * L], len0=[0], cap=T, seed=19)
    qb, kb, vb = prefill_inputs(19, 0, B, L, T, HQ, H)
    out = torch.full((B, L, T, HQ, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    msa.msa_sparse_prefill(bf16_tensor(qb), bf16_tensor(kb), bf16_tensor(vb), T, B, L, HQ, H, D, case.d_lk,
                           case.d_lv, case.d_len, T, case.d_mem, case.d_mlen, M, 16, THETA, case.scale, out, case.err)
    torch.cuda.synchronize()
    assert int(case.err.item()) == 0 and case.d_len.cpu().tolist() == [T]
    got = bf16_to_np(out)
    assert np.isfinite(got).all()
    f = syn.bf16_bits_to_f32
    for l in (0, 13):
        ref = oracle.prefill(f(qb[0, l]), f(kb[0, l]), f(vb[0, l]), f(case.mem_bits[0, l]), M, case.o_lk[0, l],
                             case.o_lv[0, l], 0, 16, THETA, case.scale)
        assert np.abs(got[0, l] - ref).max() <= DEC_MAX_ABS and rel_l2(got[0, l], ref) <= DEC_REL_L2, l
