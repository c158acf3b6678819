"""Per-step GPU parity: each C-ABI entry point against the CPU oracle on the same seeded
inputs (small sizes spanning several tiles and ragged tails, plus edge cases)."""
import numpy as np
import pytest
import torch

import msa_synth as syn
import oracle
from tests.helpers import (DEC_MAX_ABS, DEC_REL_L2, POOL_TOL, SCORE_TOL, bf16_tensor, bf16_to_np, check_topk,
                           rel_l2)

pytestmark = pytest.mark.gpu

H, HQ, D = 8, 32, 128


@pytest.fixture(scope="module")
def msa():
    import top_kv_routing_b200 as m
    return m


def _dev_i64(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int64)).cuda()


def _err():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


# ----------------------------------------------------------------------------- generator

def test_device_fill_matches_host():
    topic = syn.topics(3, 10)
    rows, rl = 333, 1024
    rt = (np.arange(rows) % 11) - 1
    host = syn.fill(3, syn.STREAM_KR, 2, 5, 100, rows, rl, sigma=0.5, topic=topic, row_topic=rt, dtype="bf16")
    dev = torch.empty(rows * rl, dtype=torch.bfloat16, device="cuda")
    syn.device_fill(dev, 3, syn.STREAM_KR, 2, 5, 100, rows, rl, 0.5, torch.from_numpy(topic).cuda(),
                    torch.from_numpy(rt.astype(np.int32)).cuda())
    assert np.array_equal(dev.view(torch.int16).cpu().numpy().view(np.uint16), host.reshape(-1))
    host32 = syn.fill(9, syn.STREAM_V, 0, 0, 7, 50, 256)
    dev32 = torch.empty(50 * 256, dtype=torch.float32, device="cuda")
    syn.device_fill(dev32, 9, syn.STREAM_V, 0, 0, 7, 50, 256)
    assert np.array_equal(dev32.cpu().numpy(), host32.reshape(-1))


# ----------------------------------------------------------------------------- step 1

def _pool_gpu(msa, k, v, kr, lens, chunk=64, theta=1e6, bf16_in=False):
    offs = syn.offsets(np.asarray(lens))
    C, coffs = msa.msa_count_chunks(offs, chunk)

    def dev(x):
        if x is None:
            return None
        if bf16_in:
            return bf16_tensor(x)
        return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()

    out = {n: torch.full((max(C, 1), H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
           for n in ("k_bar", "v_bar", "kr_hat")}
    kr_norm = torch.full((max(C, 1), H), float("nan"), device="cuda")
    err = _err()
    msa.msa_pool_blocks(dev(k), dev(v), dev(kr), _dev_i64(offs), _dev_i64(coffs), len(lens), C, H, D, chunk, theta,
                        out["k_bar"] if k is not None else None, out["v_bar"] if v is not None else None,
                        out["kr_hat"] if kr is not None else None, kr_norm if kr is not None else None, err,
                        in_dtype=msa.MSA_BF16 if bf16_in else msa.MSA_F32)
    torch.cuda.synchronize()
    res = {n: bf16_to_np(t)[:C] for n, t in out.items()}
    res["kr_norm"] = kr_norm.cpu().numpy()[:C]
    return res, int(err.item()), C


def _pool_compare(res, ref, which=("k_bar", "v_bar", "kr_hat")):
    for n in which:
        r = ref["kr_unit"] if n == "kr_hat" else ref[n]
        err = np.abs(res[n].astype(np.float64) - r).max()
        assert err <= POOL_TOL, (n, err)
    if "kr_hat" in which:
        np.testing.assert_allclose(res["kr_norm"], ref["kr_norm"], rtol=1e-4, atol=1e-6)


def test_pool_tiny_bank_fp32(msa):
    # 64 documents, lengths U[200, 1000], fp32 K, V, K_r (K_r with a per-document topic).
    bank = syn.make_bank(0, 64, syn.doc_lengths_uniform(0, 64, 200, 1000), 1)
    k = syn.raw_tokens(bank, 0, syn.STREAM_K, 0, bank.n_tokens)
    v = syn.raw_tokens(bank, 0, syn.STREAM_V, 0, bank.n_tokens)
    kr = syn.raw_tokens(bank, 0, syn.STREAM_KR, 0, bank.n_tokens)
    res, err, C = _pool_gpu(msa, k, v, kr, bank.lengths)
    assert err == 0 and C == bank.n_chunks
    ref = oracle.pool(k, v, kr, bank.doc_tok_offsets, H, D, 64, 1e6)
    _pool_compare(res, ref)


def test_pool_ragged_bf16_with_longest_document(msa):
    lens = np.array([1, 63, 64, 65, 127, 128, 129, 700, 8192, 3])
    offs = syn.offsets(lens)
    n = int(offs[-1])
    bank = syn.make_bank(4, len(lens), lens, 1)
    k = syn.raw_tokens(bank, 0, syn.STREAM_K, 0, n, dtype="bf16")
    v = syn.raw_tokens(bank, 0, syn.STREAM_V, 0, n, dtype="bf16")
    kr = syn.raw_tokens(bank, 0, syn.STREAM_KR, 0, n, dtype="bf16")
    res, err, C = _pool_gpu(msa, k, v, kr, lens, bf16_in=True)
    assert err == 0
    f = syn.bf16_bits_to_f32
    ref = oracle.pool(f(k), f(v), f(kr), offs, H, D, 64, 1e6)
    _pool_compare(res, ref)


def test_pool_passthrough_normalisation_chunk_1(msa):
    lens = np.array([3, 1, 7])
    rows = int(lens.sum())
    x = syn.fill(2, syn.STREAM_KRBAR, 0, 0, 0, rows, H * D, sigma=0.125, dtype="bf16").reshape(rows, H, D)
    x[4, 3] = 0  # a zero head stays zero
    res, err, C = _pool_gpu(msa, None, None, x, lens, chunk=1, theta=0.0, bf16_in=True)
    assert err == 0 and C == rows
    ref = oracle.pool(None, None, syn.bf16_bits_to_f32(x), syn.offsets(lens), H, D, 1, 1e6, rope_k=False)
    _pool_compare(res, ref, which=("kr_hat",))
    assert np.all(res["kr_hat"][4, 3] == 0)


def test_pool_rejects_bad_arguments(msa):
    with pytest.raises(msa.MsaError) as e:
        msa.msa_pool_blocks(None, torch.zeros(8, device="cuda"), None, _dev_i64([0, 1]), _dev_i64([0, 1]), 1, 1,
                            H, 64, 64, 1e6, None, None, None, None, None)
    assert e.value.status == msa.MSA_ERR_INVALID_ARG


# ----------------------------------------------------------------------------- step 2

def _route_bank(bank, layers):
    """Stored routing keys for each layer, bf16 bits [L][C][H][D]: pooled-level keys drawn
    by the generator, made unit-norm per head by the oracle (chunk = 1 pass-through) and
    rounded to bf16.  The same bits feed the GPU route and the oracle route."""
    C = bank.n_chunks
    out = []
    for l in range(layers):
        raw = syn.bf16_bits_to_f32(syn.pooled_router_keys(bank, l, 0, C))
        unit = oracle.pool(None, None, raw, np.arange(C + 1), H, D, 1, 1e6, rope_k=False)["kr_unit"]
        out.append(syn.f32_to_bf16_bits(unit.astype(np.float32)))
    bits = np.stack(out)
    return bits, bf16_tensor(bits), _dev_i64(bank.doc_chunk_offsets)


def _filter_keys(msa, kr_hat):
    L, C = kr_hat.shape[0], kr_hat.shape[1]
    kr_f8 = torch.empty(kr_hat.shape, dtype=torch.uint8, device="cuda")
    msa.msa_route_filter_keys(kr_hat, L, C, H, D, kr_f8)
    return kr_f8


def _route_gpu(msa, qr, q_offsets, kr_hat, coffs, n_docs, C, L, k, flags):
    B = len(q_offsets) - 1
    T = int(q_offsets[-1])
    ws = torch.empty(msa.msa_route_topk_workspace_size(L, B, T, H, C, n_docs, k), dtype=torch.uint8, device="cuda")
    ids = torch.full((B, L, k), -7, dtype=torch.int32, device="cuda")
    sc = torch.full((B, L, k), float("nan"), device="cuda")
    err = _err()
    kr_f8 = _filter_keys(msa, kr_hat) if flags == msa.MSA_ROUTE_TENSOR_F8 else None
    msa.msa_route_topk(torch.from_numpy(np.ascontiguousarray(qr, dtype=np.float32)).cuda(), q_offsets, kr_hat,
                       coffs, n_docs, C, L, HQ, H, D, k, ids, sc, ws, flags=flags, dev_err=err, kr_f8=kr_f8)
    torch.cuda.synchronize()
    return ids.cpu().numpy(), sc.cpu().numpy(), int(err.item())


def _route_case(msa, seed, lens, L, Ts, k, flags, n_targets=2):
    bank = syn.make_bank(seed, len(lens), lens, L)
    bits, kr_hat, coffs = _route_bank(bank, L)
    q_off = syn.offsets(np.asarray(Ts)).astype(np.int32)
    nonempty = [d for d in range(len(lens)) if lens[d] > 0]
    qr = np.zeros((L, int(q_off[-1]), HQ, D), dtype=np.float32)
    targets = {}
    for b, T in enumerate(Ts):
        tg = np.array([nonempty[i] for i in syn.pick_targets(seed, len(nonempty), min(n_targets, len(nonempty)), b)])
        targets[b] = tg
        for l in range(L):
            qr[l, q_off[b]:q_off[b + 1]] = syn.query_router(seed, l, b, T, HQ, D, bank.topic, tg)
    ids, sc, err = _route_gpu(msa, qr, q_off, kr_hat, coffs, len(lens), bank.n_chunks, L, k, flags)
    assert err == 0
    for b in range(len(Ts)):
        for l in range(L):
            keys = syn.bf16_bits_to_f32(bits[l])
            _, _, doc_scores, _ = oracle.route(qr[l, q_off[b]:q_off[b + 1]], keys, bank.doc_chunk_offsets, k,
                                               grouped=True)
            check_topk(ids[b, l], sc[b, l], doc_scores, k)
            planted = targets[b][:min(Ts[b], len(targets[b]))]   # token t carries target t mod n
            if k >= len(planted):
                assert set(planted.tolist()) <= set(ids[b, l].tolist())
    return ids, sc, err


@pytest.mark.parametrize("flags", [1, 2, 3])
def test_route_multi_query_multi_layer(msa, flags):
    lens = syn.doc_lengths_lognormal(1, 200)
    _route_case(msa, 1, lens, 2, [1, 5, 2], 16, flags)


@pytest.mark.parametrize("flags", [1, 2, 3])
def test_route_fewer_docs_than_k_and_empty_docs(msa, flags):
    lens = np.array([100, 0, 64, 0, 1, 300])
    ids, sc, _ = _route_case(msa, 2, lens, 1, [3], 8, flags)
    assert list(ids[0, 0, 6:]) == [-1, -1] and np.all(np.isneginf(sc[0, 0, 4:]))


@pytest.mark.parametrize("flags", [1, 2, 3])
def test_route_single_document(msa, flags):
    _route_case(msa, 3, np.array([65]), 1, [2], 4, flags, n_targets=1)


@pytest.mark.parametrize("flags", [2, 3])
@pytest.mark.parametrize("Ts", [[300, 40, 257], [64], [129], [33, 31, 1, 64]])
def test_route_tensor_long_queries_span_tiles(msa, Ts, flags):
    # several N tiles per block tile (queries crossing tile edges), ragged last M tile,
    # two layers (tiles at the layer boundary)
    lens = syn.doc_lengths_lognormal(7, 150)
    _route_case(msa, 7, lens, 2, Ts, 64, flags, n_targets=4)


@pytest.mark.parametrize("flags", [2, 3])
@pytest.mark.parametrize("pair", [True, False])
@pytest.mark.parametrize("Ts", [[256], [100, 156], [129]])
def test_route_tensor_pair_and_single_cta_tiles(msa, pair, Ts, flags):
    # N tiles of 128 / 256 run on SM pairs (M = 256) by default; both tilings must match the oracle
    lens = syn.doc_lengths_lognormal(11, 180)
    msa.msa_route_set_pair_mode(pair)
    try:
        _route_case(msa, 11, lens, 2, Ts, 32, flags, n_targets=4)
    finally:
        msa.msa_route_set_pair_mode(True)


@pytest.mark.parametrize("flags", [2, 3])
def test_route_tensor_selection_is_certified_for_planted_needles(msa, flags):
    # k = number of planted documents: the k-th exact score sits far above the filter's
    # margin over the best document left out, so the certification bit stays clear
    lens = syn.doc_lengths_lognormal(9, 400)
    _, _, err = _route_case(msa, 9, lens, 1, [64], 4, flags, n_targets=4)
    assert err == 0


def test_route_f8_layers_without_margin_fall_back_to_the_bf16_filter(msa):
    # router queries of pure noise: the top-k boundary sits inside the E4M3 error window,
    # so those layers cannot be certified from the E4M3 pass and are re-filtered in bf16;
    # the result must still be the exact top-k (and certified)
    lens = syn.doc_lengths_lognormal(14, 600)
    bank = syn.make_bank(14, len(lens), lens, 2)
    bits, kr_hat, coffs = _route_bank(bank, 2)
    T, k = 96, 16
    qr = syn.fill(14, syn.STREAM_QR, 0, 0, 0, 2 * T * HQ, D).reshape(2, T, HQ, D)
    ids, sc, err = _route_gpu(msa, qr, [0, T], kr_hat, coffs, len(lens), bank.n_chunks, 2, k, msa.MSA_ROUTE_TENSOR_F8)
    assert err == 0
    for l in range(2):
        _, _, doc_scores, _ = oracle.route(qr[l], syn.bf16_bits_to_f32(bits[l]), bank.doc_chunk_offsets, k,
                                           grouped=True)
        check_topk(ids[0, l], sc[0, l], doc_scores, k)


@pytest.mark.parametrize("flags", [1, 2, 3])
def test_route_many_equal_documents_take_the_lowest_ids(msa, flags):
    # 2,100 documents with identical blocks: every score ties, so the selection is the
    # lowest ids (more documents share the threshold score than the selection collects at
    # once, exercising the ordered fallback); ties cannot be certified by a filter, so the
    # tensor paths end in the exact scan, which takes the lowest ids too
    n_docs, per, k = 2100, 2, 16
    lens = np.full(n_docs, 64 * per)
    bank = syn.make_bank(15, n_docs, lens, 1)
    row = syn.fill(15, syn.STREAM_KRBAR, 0, 0, 0, 1, H * D).reshape(H, D).astype(np.float64)
    row /= np.linalg.norm(row, axis=1, keepdims=True)
    bits = np.broadcast_to(syn.f32_to_bf16_bits(row.astype(np.float32)), (1, bank.n_chunks, H, D)).copy()
    kr_hat = bf16_tensor(bits)
    coffs = _dev_i64(bank.doc_chunk_offsets)
    T = 1 if flags == 1 else 40
    qr = syn.fill(15, syn.STREAM_QR, 0, 0, 0, T * HQ, D).reshape(1, T, HQ, D)
    ids, sc, err = _route_gpu(msa, qr, [0, T], kr_hat, coffs, n_docs, bank.n_chunks, 1, k, flags)
    assert err == 0
    assert ids[0, 0].tolist() == list(range(k))
    assert np.all(sc[0, 0] == sc[0, 0, 0])


def _e4m3_decode(b):
    b = b.astype(np.int64)
    sign = np.where(b >> 7, -1.0, 1.0)
    e, m = (b >> 3) & 15, b & 7
    return sign * np.where(e == 0, m / 8.0 * 2.0 ** -6, (1 + m / 8.0) * 2.0 ** (e - 7.0))


def test_route_filter_keys_round_unit_heads_to_e4m3(msa):
    # every element is the E4M3 value nearest to 256 x the element of the unit head
    # (within half a unit in the last place of E4M3), a zero head stays zero
    L, C = 2, 77
    x = syn.fill(12, syn.STREAM_KRBAR, 0, 0, 0, L * C * H, D, sigma=0.3, dtype="bf16").reshape(L, C, H, D)
    x[1, 5, 2] = 0
    x[0, 0, 0, :4] = syn.f32_to_bf16_bits(np.array([3.0, -2.0, 1e-3, 0.0], dtype=np.float32))
    got = _e4m3_decode(_filter_keys(msa, bf16_tensor(x)).cpu().numpy())
    f = syn.bf16_bits_to_f32(x).astype(np.float64)
    ref = 256.0 * f / np.maximum(np.linalg.norm(f, axis=3, keepdims=True), 1e-8)
    a = np.abs(ref)
    ulp = np.where(a < 2.0 ** -6, 2.0 ** -9, 2.0 ** (np.floor(np.log2(np.maximum(a, 2.0 ** -6))) - 3))
    assert np.all(np.abs(got - ref) <= 0.5 * ulp * (1 + 1e-5) + 1e-9)
    assert np.all(got[1, 5, 2] == 0)
    assert np.abs(got).max() <= 256.0


def test_route_f8_and_bf16_filters_select_the_same_documents(msa):
    # both filters end in exact fp32 rescoring: on a planted bank the selections agree
    lens = syn.doc_lengths_lognormal(13, 500)
    a = _route_case(msa, 13, lens, 2, [256], 16, 2, n_targets=16)
    b = _route_case(msa, 13, lens, 2, [256], 16, 3, n_targets=16)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    assert a[2] == 0 and b[2] == 0


def test_route_auto_picks_tensor_for_long_query_and_scan_for_short(msa):
    lens = syn.doc_lengths_lognormal(8, 60)
    bank = syn.make_bank(8, 60, lens, 1)
    _, kr_hat, coffs = _route_bank(bank, 1)
    C = bank.n_chunks
    kr_f8 = _filter_keys(msa, kr_hat)
    # scan: qprep + scan + 2 top-k; tensor: prep + qprep + GEMM + top-k + rescore + final,
    # then the widened rescoring (top-k + rescore + final) over uncertified layers (60
    # documents: more than the 48 first candidates, fewer than the 1024 widened ones, so no
    # exact scan); E4M3: before the widened stage the bf16 pass over uncertified layers
    # (reset + GEMM + top-k + rescore + final)
    for T, f8, expect in ((4, None, 4), (40, None, 9), (4, kr_f8, 4), (40, kr_f8, 14)):
        ws = torch.empty(msa.msa_route_topk_workspace_size(1, 1, T, H, C, 60, 16), dtype=torch.uint8, device="cuda")
        ids = torch.empty((1, 1, 16), dtype=torch.int32, device="cuda")
        sc = torch.empty((1, 1, 16), device="cuda")
        n = msa.msa_route_topk(torch.randn((1, T, HQ, D), device="cuda"), [0, T], kr_hat, coffs, 60, C, 1, HQ, H, D,
                               16, ids, sc, ws, kr_f8=f8)
        assert n == expect


# ----------------------------------------------------------------------------- step 3

def test_gather_matches_oracle_bit_exact(msa):
    rng = np.random.default_rng(0)
    L, n_docs = 3, 40
    lens = syn.doc_lengths_lognormal(5, n_docs)
    bank = syn.make_bank(5, n_docs, lens, L)
    C = bank.n_chunks
    store = np.stack([syn.pooled_content(bank, l, 0, C) for l in range(L)])  # [L][C][2][H][D] bits
    host = torch.from_numpy(store.view(np.int16)).pin_memory()
    B, k, M_max = 2, 6, 768
    ids = rng.integers(-1, n_docs, size=(B, L, k)).astype(np.int32)
    ids[0, 0] = [3, 9, -1, 17, 0, 39]
    ref, ref_len = oracle.gather(store, bank.doc_chunk_offsets, np.maximum(ids, -1), M_max)
    dev_kv = torch.zeros((B, L, 2, H, M_max, D), dtype=torch.int16, device="cuda")
    mem_len = torch.full((B, L), -5, dtype=torch.int32, device="cuda")
    err = _err()
    msa.msa_gather_kv(host, C, _dev_i64(bank.doc_chunk_offsets), None, n_docs,
                      torch.from_numpy(ids).cuda(), B, L, k, H, D, M_max, dev_kv, mem_len, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert np.array_equal(mem_len.cpu().numpy(), ref_len)
    got = dev_kv.cpu().numpy().view(np.uint16)
    for b in range(B):
        for l in range(L):
            m = ref_len[b, l]
            assert np.array_equal(got[b, l, :, :, :m], ref[b, l, :, :, :m])


def test_gather_capacity_and_bad_id_flags(msa):
    L, n_docs = 1, 4
    lens = np.array([640, 640, 64, 64])
    bank = syn.make_bank(6, n_docs, lens, L)
    store = syn.pooled_content(bank, 0, 0, bank.n_chunks)[None]
    host = torch.from_numpy(store.view(np.int16)).pin_memory()
    ids = torch.tensor([[[0, 1, 7]]], dtype=torch.int32, device="cuda")
    dev_kv = torch.zeros((1, 1, 2, H, 12, D), dtype=torch.int16, device="cuda")
    mem_len = torch.zeros((1, 1), dtype=torch.int32, device="cuda")
    err = _err()
    msa.msa_gather_kv(host, bank.n_chunks, _dev_i64(bank.doc_chunk_offsets), None, n_docs, ids, 1, 1, 3, H, D, 12,
                      dev_kv, mem_len, err)
    torch.cuda.synchronize()
    e = int(err.item())
    assert e & msa.MSA_DEVERR_CAPACITY and e & msa.MSA_DEVERR_BAD_DOC
    assert int(mem_len.item()) == 12
    got = dev_kv.cpu().numpy().view(np.uint16)
    assert np.array_equal(got[0, 0, :, :, :10], np.transpose(store[0, :10], (1, 2, 0, 3)))


def test_gather_rejects_pageable_host_memory(msa):
    host = torch.zeros((1, 4, 2, H, D), dtype=torch.int16)
    with pytest.raises(msa.MsaError):
        msa.msa_gather_kv(host, 4, _dev_i64([0, 4]), None, 1, torch.zeros((1, 1, 1), dtype=torch.int32,
                          device="cuda"), 1, 1, 1, H, D, 8, torch.zeros((1, 1, 2, H, 8, D), dtype=torch.int16,
                          device="cuda"), torch.zeros((1, 1), dtype=torch.int32, device="cuda"))


# ----------------------------------------------------------------------------- step 4

def _decode_case(msa, B, L, M_max, mem_len, len0, cap, steps, offset, seed=0, hq=HQ, h=H):
    rng = np.random.default_rng(seed)
    g = hq // h
    mem_bits = syn.fill(seed, syn.STREAM_KBAR, 0, 0, 0, B * L * 2 * h * M_max, D, dtype="bf16")
    mem_bits = mem_bits.reshape(B, L, 2, h, M_max, D)
    loc_k = syn.fill(seed, syn.STREAM_LOCAL_K, 0, 0, 0, B * L * h * cap, D, dtype="bf16").reshape(B, L, h, cap, D)
    loc_v = syn.fill(seed, syn.STREAM_LOCAL_V, 0, 0, 0, B * L * h * cap, D, dtype="bf16").reshape(B, L, h, cap, D)
    d_mem = bf16_tensor(mem_bits)
    d_lk, d_lv = bf16_tensor(loc_k), bf16_tensor(loc_v)
    d_len = torch.tensor(len0, dtype=torch.int32, device="cuda")
    d_mlen = torch.tensor(mem_len, dtype=torch.int32, device="cuda")
    f = syn.bf16_bits_to_f32
    o_lk = f(loc_k).astype(np.float64).copy()
    o_lv = f(loc_v).astype(np.float64).copy()
    scale = D ** -0.5
    err = _err()
    worst_abs, worst_rel = 0.0, 0.0
    for s in range(steps):
        qb = syn.fill(seed, syn.STREAM_DEC_Q, s, 0, 0, B * L * hq, D, dtype="bf16").reshape(B, L, hq, D)
        kb = syn.fill(seed, syn.STREAM_DEC_K, s, 0, 0, B * L * h, D, dtype="bf16").reshape(B, L, h, D)
        vb = syn.fill(seed, syn.STREAM_DEC_V, s, 0, 0, B * L * h, D, dtype="bf16").reshape(B, L, h, D)
        out = torch.full((B, L, hq, D), float("nan"), dtype=torch.bfloat16, device="cuda")
        ws = torch.zeros(msa.msa_sparse_decode_workspace_size(B, L, hq, h), dtype=torch.uint8, device="cuda")
        msa.msa_sparse_decode(bf16_tensor(qb), bf16_tensor(kb), bf16_tensor(vb), B, L, hq, h, D, d_lk, d_lv, d_len, cap,
                              d_mem, d_mlen, M_max, offset, 1e6, scale, out, ws, err)
        torch.cuda.synchronize()
        got = bf16_to_np(out)
        for b in range(B):
            i = len0[b] + s
            for l in range(L):
                mk = f(mem_bits[b, l])
                ref = oracle.decode(f(qb[b, l]), f(kb[b, l]), f(vb[b, l]), mk, mem_len[b][l], o_lk[b, l], o_lv[b, l],
                                    i, offset + i, 1e6, scale)
                worst_abs = max(worst_abs, float(np.abs(got[b, l] - ref).max()))
                worst_rel = max(worst_rel, rel_l2(got[b, l], ref))
    assert int(err.item()) == 0
    assert worst_abs <= DEC_MAX_ABS and worst_rel <= DEC_REL_L2, (worst_abs, worst_rel)
    assert d_len.cpu().tolist() == [x + steps for x in len0]
    # appended rows: rotated keys (bf16 rounding of the oracle's) and exact values
    lk = bf16_to_np(d_lk)
    lv = bf16_to_np(d_lv)
    for b in range(B):
        sl = slice(len0[b], len0[b] + steps)
        assert np.abs(lk[b, :, :, sl] - o_lk[b, :, :, sl]).max() <= POOL_TOL
        assert np.array_equal(lv[b, :, :, sl], o_lv[b, :, :, sl].astype(np.float32))
    return worst_abs, worst_rel


def test_decode_matches_oracle_ragged_memory(msa):
    _decode_case(msa, B=2, L=3, M_max=300, mem_len=[[300, 17, 0], [5, 257, 1]], len0=[3, 0], cap=12, steps=4,
                 offset=16)


def test_decode_long_context_several_tiles(msa):
    _decode_case(msa, B=1, L=2, M_max=700, mem_len=[[700, 513]], len0=[250], cap=260, steps=3, offset=16, seed=3)


@pytest.mark.parametrize("hq,h", [(8, 8), (16, 8), (64, 8)])
def test_decode_group_sizes(msa, hq, h):
    _decode_case(msa, B=1, L=1, M_max=20, mem_len=[[20]], len0=[2], cap=6, steps=2, offset=4, seed=5, hq=hq, h=h)


def test_decode_full_cache_sets_flag_and_skips(msa):
    B, L, cap, M = 1, 1, 2, 4
    out = torch.zeros((B, L, HQ, D), dtype=torch.bfloat16, device="cuda")
    d_len = torch.tensor([cap], dtype=torch.int32, device="cuda")
    err = _err()
    z = lambda *s: torch.zeros(s, dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(msa.msa_sparse_decode_workspace_size(B, L, HQ, H), dtype=torch.uint8, device="cuda")
    msa.msa_sparse_decode(z(B, L, HQ, D), z(B, L, H, D), z(B, L, H, D), B, L, HQ, H, D, z(B, L, H, cap, D),
                          z(B, L, H, cap, D), d_len, cap, z(B, L, 2, H, M, D),
                          torch.tensor([[M]], dtype=torch.int32, device="cuda"), M, 4, 1e6, 0.1, out, ws, err)
    torch.cuda.synchronize()
    assert int(err.item()) & msa.MSA_DEVERR_LOCAL_FULL
    assert int(d_len.item()) == cap and float(out.float().abs().sum()) == 0.0
