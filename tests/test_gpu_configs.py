"""Parity at the configurations' own sizes, in the launch configuration the benchmark times
(E4M3 filter for long queries, SM-pair GEMM tiles, the scan for short ones).

Where the oracle cannot cover a whole bank in seconds, the checks use sampled outputs the
oracle computes one by one: the exact scores of the returned documents, of the planted
ones and of a hashed sample of the rest, which must satisfy the top-k rules at any size
(tests/fullsize.py).  Pooling at 10M tokens is checked on sampled documents regenerated on
the host; gather is byte-exact; decode is checked step by step on sampled layers.
"""
import numpy as np
import pytest
import torch

import msa_synth as syn
import oracle
from tests.fullsize import (D, DeviceBank, H, HQ, THETA, check_full_layer, check_sampled, decode_inputs, host_query,
                            host_store, oracle_doc_scores, oracle_gather_layer, random_docs)
from tests.helpers import DEC_MAX_ABS, DEC_REL_L2, POOL_TOL, bf16_tensor, bf16_to_np, check_topk, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msa():
    import top_kv_routing_b200 as m
    return m


def _free():
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _decode_and_check(msa, seed, mem, mem_len, M_max, L, steps, prefix_k, prefix_v, cap, k_off, ref_mem, layers,
                      sub=0):
    """steps decode tokens for one query on every layer (device), and the oracle's decode on
    `layers` with its own copy of the cache; ref_mem[l] = (mem [2][H][M_max][d], len)."""
    T0 = prefix_k.shape[2]
    lk = torch.zeros((1, L, H, cap, D), dtype=torch.bfloat16, device="cuda")
    lv = torch.zeros_like(lk)
    lk[0, :, :, :T0] = bf16_tensor(prefix_k)
    lv[0, :, :, :T0] = bf16_tensor(prefix_v)
    llen = torch.tensor([T0], dtype=torch.int32, device="cuda")
    ws = torch.zeros(msa.msa_sparse_decode_workspace_size(1, L, HQ, H), dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    f = syn.bf16_bits_to_f32
    o_lk = {l: np.zeros((H, cap, D)) for l in layers}
    o_lv = {l: np.zeros((H, cap, D)) for l in layers}
    for l in layers:
        o_lk[l][:, :T0] = f(prefix_k[l])
        o_lv[l][:, :T0] = f(prefix_v[l])
    scale = D ** -0.5
    worst_abs = worst_rel = 0.0
    for s in range(steps):
        qb, kb, vb = decode_inputs(seed, s, 1, L, sub)
        out = torch.full((1, L, HQ, D), float("nan"), dtype=torch.bfloat16, device="cuda")
        msa.msa_sparse_decode(bf16_tensor(qb), bf16_tensor(kb), bf16_tensor(vb), 1, L, HQ, H, D, lk, lv, llen, cap,
                              mem, mem_len, M_max, k_off, THETA, scale, out, ws, err)
        got = bf16_to_np(out)
        for l in layers:
            m, n = ref_mem[l]
            ref = oracle.decode(f(qb[0, l]), f(kb[0, l]), f(vb[0, l]), m, n, o_lk[l], o_lv[l], T0 + s, k_off + T0 + s,
                                THETA, scale)
            worst_abs = max(worst_abs, float(np.abs(got[0, l] - ref).max()))
            worst_rel = max(worst_rel, rel_l2(got[0, l], ref))
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert int(llen.item()) == T0 + steps
    assert worst_abs <= DEC_MAX_ABS and worst_rel <= DEC_REL_L2, (worst_abs, worst_rel)
    return worst_abs, worst_rel


# ----------------------------------------------------------------------------- config 0

def test_config0_tiny_bank_whole_chain_against_the_oracle_chain(msa):
    # 64 documents of U[200, 1000] tokens, fp32 K / V / K_r with topics, 1 layer; T = 16
    # with 2 planted documents, top-4; 8 decode tokens over a local KV of 16.  The device
    # and the oracle each run the whole chain on the same raw inputs.
    seed, n_docs, L, T, k, n_dec, T0 = 0, 64, 1, 16, 4, 8, 16
    lens = syn.doc_lengths_uniform(seed, n_docs, 200, 1000)
    bank = syn.make_bank(seed, n_docs, lens, L)
    n = bank.n_tokens
    kx = syn.raw_tokens(bank, 0, syn.STREAM_K, 0, n)
    vx = syn.raw_tokens(bank, 0, syn.STREAM_V, 0, n)
    krx = syn.raw_tokens(bank, 0, syn.STREAM_KR, 0, n)
    C, coffs = msa.msa_count_chunks(bank.doc_tok_offsets, 64)
    t = lambda a, dt=torch.float32: torch.from_numpy(np.ascontiguousarray(a)).to("cuda", dt)
    k_bar = torch.empty((C, H, D), dtype=torch.bfloat16, device="cuda")
    v_bar = torch.empty_like(k_bar)
    kr_hat = torch.empty((1, C, H, D), dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    d_coffs = t(coffs, torch.int64)
    msa.msa_pool_blocks(t(kx), t(vx), t(krx), t(bank.doc_tok_offsets, torch.int64), d_coffs, n_docs, C, H, D, 64,
                        THETA, k_bar, v_bar, kr_hat[0], None, err)
    kr_f8 = torch.empty((1, C, H, D), dtype=torch.uint8, device="cuda")
    msa.msa_route_filter_keys(kr_hat, 1, C, H, D, kr_f8)
    targets = syn.pick_targets(seed, n_docs, 2)
    qr = syn.query_router(seed, 0, 0, T, HQ, D, bank.topic, targets)
    ref = oracle.pool(kx, vx, krx, bank.doc_tok_offsets, H, D, 64, THETA)
    o_ids, _, o_doc, _ = oracle.route(qr, ref["kr_unit"], coffs, k)
    for flags in (msa.MSA_ROUTE_SCAN, msa.MSA_ROUTE_TENSOR, msa.MSA_ROUTE_TENSOR_F8):
        ws = torch.empty(msa.msa_route_topk_workspace_size(1, 1, T, H, C, n_docs, k), dtype=torch.uint8,
                         device="cuda")
        ids = torch.empty((1, 1, k), dtype=torch.int32, device="cuda")
        sc = torch.empty((1, 1, k), device="cuda")
        msa.msa_route_topk(t(qr[None]), [0, T], kr_hat, d_coffs, n_docs, C, 1, HQ, H, D, k, ids, sc, ws, flags=flags,
                           dev_err=err, kr_f8=kr_f8)
        torch.cuda.synchronize()
        g_ids, g_sc = ids.cpu().numpy()[0, 0], sc.cpu().numpy()[0, 0]
        check_topk(g_ids, g_sc, o_doc, k)
        assert set(targets.tolist()) <= set(g_ids.tolist())
        assert set(g_ids.tolist()) == set(o_ids.tolist())
    assert int(err.item()) == 0
    # gather from a host store of the device's pooled blocks, decode over it; the oracle
    # decodes over its own pooled blocks (bf16-rounded) for the same selection
    host_kv = torch.stack([k_bar, v_bar], dim=1)[None].cpu().pin_memory()
    M = k * int(np.diff(coffs).max())
    mem = torch.zeros((1, 1, 2, H, M, D), dtype=torch.bfloat16, device="cuda")
    mem_len = torch.zeros((1, 1), dtype=torch.int32, device="cuda")
    msa.msa_gather_kv(host_kv, C, d_coffs, None, n_docs, ids, 1, 1, k, H, D, M, mem, mem_len, err)
    bf = lambda x: syn.bf16_bits_to_f32(syn.f32_to_bf16_bits(np.asarray(x, dtype=np.float32)))
    rows = [c for d in o_ids if d >= 0 for c in range(coffs[d], coffs[d + 1])]
    ref_mem = np.zeros((2, H, M, D), dtype=np.float32)
    ref_mem[0, :, :len(rows)] = np.transpose(bf(ref["k_bar"][rows]), (1, 0, 2))
    ref_mem[1, :, :len(rows)] = np.transpose(bf(ref["v_bar"][rows]), (1, 0, 2))
    torch.cuda.synchronize()
    assert int(mem_len.item()) == len(rows)
    if list(g_ids) == list(o_ids):  # same order: the packed blocks line up
        got_mem = bf16_to_np(mem)[0, 0][:, :, :len(rows)]
        assert np.abs(got_mem - ref_mem[:, :, :len(rows)]).max() <= POOL_TOL
    pk = syn.fill(seed, syn.STREAM_LOCAL_K, 0, 0, 0, H * T0, D, dtype="bf16").reshape(1, H, T0, D)
    pv = syn.fill(seed, syn.STREAM_LOCAL_V, 0, 0, 0, H * T0, D, dtype="bf16").reshape(1, H, T0, D)
    _decode_and_check(msa, seed, mem, mem_len, M, 1, n_dec, pk, pv, T0 + n_dec, k, {0: (ref_mem, len(rows))}, [0])


# ----------------------------------------------------------------------------- config 1

def test_config1_1m_bank_route_gather_decode(msa):
    # 1,000 lognormal documents (~1M tokens), 18 layers; T = 64 with 16 planted documents,
    # top-16 (E4M3 filter, as benchmarked); gather from the full host store; 64 decode
    # tokens over a local KV of 64
    seed, n_docs, L, T, k, n_dec, T0 = 1, 1000, 18, 64, 16, 64, 64
    lens = syn.doc_lengths_lognormal(seed, n_docs)
    db = DeviceBank(msa, seed, lens, L)
    targets = syn.pick_targets(seed, n_docs, 16)
    qr = db.queries(1, T, lambda b: targets)
    ids, sc, err = db.route(qr, [0, T], k, msa.MSA_ROUTE_AUTO)
    assert err == 0
    extra = random_docs(seed, n_docs, 48)
    layers = [0, 9, 17]
    o_ids = {}
    for l in range(L):
        q = host_query(db.bank, l, 0, T, targets)
        if l in layers:  # the whole bank through the oracle: its own selection
            ds = check_full_layer(ids[0, l], sc[0, l], db.bank, l, q, k)
            o_ids[l] = oracle.topk(ds, k)[0]
            assert set(o_ids[l].tolist()) == set(ids[0, l].tolist()), l
        else:
            ref = oracle_doc_scores(db.bank, l, q, list(ids[0, l]) + list(targets) + list(extra))
            check_sampled(ids[0, l], sc[0, l], ref, k, planted=targets)

    store, store_np = host_store(seed, L, db.C)
    M = k * int(np.diff(db.coffs).max())
    mem = torch.zeros((1, L, 2, H, M, D), dtype=torch.bfloat16, device="cuda")
    mem_len = torch.zeros((1, L), dtype=torch.int32, device="cuda")
    d_err = torch.zeros(1, dtype=torch.int32, device="cuda")
    msa.msa_gather_kv(store, db.C, db.d_coffs, None, n_docs, torch.from_numpy(ids).cuda(), 1, L, k, H, D, M, mem,
                      mem_len, d_err)
    torch.cuda.synchronize()
    assert int(d_err.item()) == 0
    o_mem, o_len = oracle.gather(store_np, db.coffs, ids, M)
    assert np.array_equal(mem_len.cpu().numpy(), o_len)
    got = mem.view(torch.int16).cpu().numpy().view(np.uint16)
    for l in range(L):
        m = o_len[0, l]
        assert np.array_equal(got[0, l, :, :, :m], o_mem[0, l, :, :, :m])
    # decode, end to end on the oracle side: its memory is its own gather of its own
    # selection (attention does not depend on the order of the memory blocks)
    ref_mem = {}
    for l in layers:
        m, n = oracle_gather_layer(store_np, l, db.coffs, None, o_ids[l], M)
        ref_mem[l] = (m, n)
    pk = syn.fill(seed, syn.STREAM_LOCAL_K, 0, 0, 0, L * H * T0, D, dtype="bf16").reshape(L, H, T0, D)
    pv = syn.fill(seed, syn.STREAM_LOCAL_V, 0, 0, 0, L * H * T0, D, dtype="bf16").reshape(L, H, T0, D)
    _decode_and_check(msa, seed, mem, mem_len, M, L, n_dec, pk, pv, T0 + n_dec, k, ref_mem, layers)
    del db, store, mem
    _free()


# ----------------------------------------------------------------------------- config 2

@pytest.fixture(scope="module")
def bank10m(msa):
    lens = syn.doc_lengths_lognormal(2, 10_000)
    db = DeviceBank(msa, 2, lens, 18)
    yield db
    del db
    _free()


@pytest.mark.parametrize("T", [1, 8, 64, 256, 1024])
def test_config2_10m_bank_query_length_sweep(msa, bank10m, T):
    # ~163K blocks x 18 layers resident; the scan below 9 tokens, the tensor cores above
    # (E4M3 filter by default, the bf16 filter and the scan alongside where they apply)
    db, k = bank10m, 16
    targets = syn.pick_targets(2, db.n_docs, 16, sub=T)
    qr = db.queries(1, T, lambda b: targets, q_seed=20 + T)
    paths = [msa.MSA_ROUTE_AUTO]
    if T >= 64:
        paths.append(msa.MSA_ROUTE_TENSOR)
    if T == 64:
        paths.append(msa.MSA_ROUTE_SCAN)
    res = {p: db.route(qr, [0, T], k, p) for p in paths}
    planted = targets[:min(T, len(targets))]
    for p, (ids, sc, err) in res.items():
        assert err == 0, (p, err)
        for l in range(db.L):
            assert set(planted.tolist()) <= set(ids[0, l].tolist()), (p, l)
    extra = random_docs(2, db.n_docs, 64, sub=T)
    for l in (0, 17):
        q = host_query(db.bank, l, 0, T, targets, q_seed=20 + T)
        docs = set(planted.tolist()) | set(extra.tolist())
        for ids, _, _ in res.values():
            docs |= set(int(x) for x in ids[0, l])
        ref = oracle_doc_scores(db.bank, l, q, docs)
        for p, (ids, sc, _) in res.items():
            check_sampled(ids[0, l], sc[0, l], ref, k, planted=planted)


def test_config2_pool_10m_tokens_sampled_documents(msa):
    # one layer of raw bf16 K / V / K_r for the 10M-token bank pooled on the device; 20
    # sampled documents (the longest and shortest among them) regenerated on the host and
    # pooled by the oracle
    seed = 2
    lens = syn.doc_lengths_lognormal(seed, 10_000)
    bank = syn.make_bank(seed, len(lens), lens, 1)
    n, C = bank.n_tokens, bank.n_chunks
    toff, coffs = bank.doc_tok_offsets, bank.doc_chunk_offsets
    x = [torch.empty((n, H, D), dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    topic = torch.from_numpy(bank.topic).cuda()
    tok_docs = torch.from_numpy(syn.token_docs(toff)).cuda()
    for i, st in enumerate((syn.STREAM_K, syn.STREAM_V, syn.STREAM_KR)):
        syn.device_fill(x[i], seed, st, 0, 0, 0, n, H * D, 1.0, topic if i == 2 else None,
                        tok_docs if i == 2 else None)
    del tok_docs
    out = [torch.empty((C, H, D), dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    nr = torch.empty((C, H), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    msa.msa_pool_blocks(x[0], x[1], x[2], torch.from_numpy(toff).cuda(), torch.from_numpy(coffs).cuda(), len(lens), C,
                        H, D, 64, THETA, out[0], out[1], out[2], nr, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    del x
    docs = sorted(set(random_docs(seed, len(lens), 18).tolist()) | {int(np.argmax(lens)), int(np.argmin(lens))})
    for d in docs:
        t0, t1 = int(toff[d]), int(toff[d + 1])
        c0, c1 = int(coffs[d]), int(coffs[d + 1])
        raw = [syn.bf16_bits_to_f32(syn.raw_tokens(bank, 0, st, t0, t1 - t0, dtype="bf16"))
               for st in (syn.STREAM_K, syn.STREAM_V, syn.STREAM_KR)]
        ref = oracle.pool(raw[0], raw[1], raw[2], np.array([0, t1 - t0]), H, D, 64, THETA)
        for i, name in enumerate(("k_bar", "v_bar", "kr_unit")):
            got = bf16_to_np(out[i][c0:c1]).astype(np.float64)
            assert np.abs(got - ref[name]).max() <= POOL_TOL, (d, name)
        np.testing.assert_allclose(nr[c0:c1].cpu().numpy(), ref["kr_norm"], rtol=1e-4, atol=1e-6)
    del out, nr
    _free()


# ----------------------------------------------------------------------------- config 3

def test_config3_100m_bank_benchmark_path(msa):
    # the benchmarked workload: exactly 100M tokens / 1,562,500 blocks, 18 layers of bf16
    # unit keys plus the E4M3 copy in HBM, one T=256 query with 16 planted documents
    # (bf16 router vectors), top-16; gather from the 163,840-block pinned store the
    # benchmark uses; 128 decode tokens over a local KV of 256
    seed, n_docs, L, T, k, n_dec, T0, P = 3, 100_000, 18, 256, 16, 128, 256, 163_840
    lens = syn.doc_lengths_exact_total(seed, n_docs, 100_000_000)
    db = DeviceBank(msa, seed, lens, L)
    assert db.C == 1_562_500
    targets = syn.pick_targets(seed, n_docs, k, sub=0)
    qr = db.queries(1, T, lambda b: targets, dtype=torch.bfloat16)
    ids, sc, err = db.route(qr, [0, T], k, msa.MSA_ROUTE_AUTO)
    assert err == 0
    for l in range(L):
        assert set(targets.tolist()) <= set(ids[0, l].tolist()), l
    extra = random_docs(seed, n_docs, 200)
    for l in (0, 17):
        q = host_query(db.bank, l, 0, T, targets, dtype="bf16")
        ref = oracle_doc_scores(db.bank, l, q, list(ids[0, l]) + list(targets) + list(extra))
        check_sampled(ids[0, l], sc[0, l], ref, k, planted=targets)
    del qr
    db.kr_hat = db.kr_f8 = None  # the keys are no longer needed
    _free()

    store, store_np = host_store(seed, L, P)
    per_doc = np.diff(db.coffs)
    h = syn.hashes(syn.tensor_key(seed, syn.STREAM_TARGETS, 0, 99), np.arange(n_docs, dtype=np.uint64))
    store_off = (h % np.uint64(P - int(per_doc.max()))).astype(np.int64)
    M = k * int(per_doc.max())
    mem = torch.zeros((1, L, 2, H, M, D), dtype=torch.bfloat16, device="cuda")
    mem_len = torch.zeros((1, L), dtype=torch.int32, device="cuda")
    d_err = torch.zeros(1, dtype=torch.int32, device="cuda")
    msa.msa_gather_kv(store, P, db.d_coffs, torch.from_numpy(store_off).cuda(), n_docs, torch.from_numpy(ids).cuda(),
                      1, L, k, H, D, M, mem, mem_len, d_err)
    torch.cuda.synchronize()
    assert int(d_err.item()) == 0
    got = mem.view(torch.int16).cpu().numpy().view(np.uint16)
    got_len = mem_len.cpu().numpy()
    layers = [0, 17]
    ref_mem = {}
    for l in range(L):
        m, n = oracle_gather_layer(store_np, l, db.coffs, store_off, ids[0, l], M)
        assert got_len[0, l] == n
        assert np.array_equal(syn.bf16_bits_to_f32(got[0, l, :, :, :n]), m[:, :, :n]), l
        if l in layers:
            ref_mem[l] = (m, n)
    pk = syn.fill(seed, syn.STREAM_LOCAL_K, 0, 0, 0, L * H * T0, D, dtype="bf16").reshape(L, H, T0, D)
    pv = syn.fill(seed, syn.STREAM_LOCAL_V, 0, 0, 0, L * H * T0, D, dtype="bf16").reshape(L, H, T0, D)
    _decode_and_check(msa, seed, mem, mem_len, M, L, n_dec, pk, pv, T0 + n_dec, k, ref_mem, layers)
    del db, store, mem
    _free()


# ----------------------------------------------------------------------------- config 4

def test_config4_multi_round_interleave_batch_of_64(msa, bank10m):
    # the config-2 bank; 64 queries of 128 router tokens, each planted with a chain of three
    # documents A -> B -> C.  Round r routes over all of the query's tokens so far (128 +
    # 512 r), gathers, decodes 32 tokens; between rounds 512 synthetic local tokens are
    # appended whose router vectors carry the next document of the chain.  Every query
    # must recover its chain round by round; queries 0, 21, 42, 63 are checked against
    # the oracle on layers 0 and 17 (route), 0 and 63 also on decode.
    db, k, B, T0, A, R, DEC, qs = bank10m, 16, 64, 128, 512, 3, 32, 4
    L, C = db.L, db.C
    chains = [syn.pick_targets(qs, db.n_docs, 3, sub=b) for b in range(B)]
    cap = T0 + R * DEC + (R - 1) * A
    checked, dec_checked, layers = [0, 21, 42, 63], [0, 63], [0, 17]
    store, store_np = host_store(qs, L, C)
    M = k * int(np.diff(db.coffs).max())
    mem = torch.zeros((B, L, 2, H, M, D), dtype=torch.bfloat16, device="cuda")
    mem_len = torch.zeros((B, L), dtype=torch.int32, device="cuda")
    lk = torch.zeros((B, L, H, cap, D), dtype=torch.bfloat16, device="cuda")
    lv = torch.zeros_like(lk)
    llen = torch.zeros(B, dtype=torch.int32, device="cuda")
    d_err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws_dec = torch.zeros(msa.msa_sparse_decode_workspace_size(B, L, HQ, H), dtype=torch.uint8, device="cuda")
    seg = torch.empty((L * H * A, D), dtype=torch.bfloat16, device="cuda")
    f = syn.bf16_bits_to_f32
    o_lk = {(b, l): np.zeros((H, cap, D)) for b in dec_checked for l in layers}
    o_lv = {(b, l): np.zeros((H, cap, D)) for b in dec_checked for l in layers}

    def append_local(r, n):
        # segment r of every query's local K / V (n tokens) at its current length
        for b in range(B):
            pos = int(llen[b].item())
            for stream, cache, ocache in ((syn.STREAM_LOCAL_K, lk, o_lk), (syn.STREAM_LOCAL_V, lv, o_lv)):
                syn.device_fill(seg[:L * H * n], qs, stream, r, b, 0, L * H * n, D)
                cache[b, :, :, pos:pos + n] = seg[:L * H * n].view(L, H, n, D)
                if b in dec_checked:
                    for l in layers:
                        x = syn.fill(qs, stream, r, b, l * H * n, H * n, D, dtype="bf16").reshape(H, n, D)
                        ocache[(b, l)][:, pos:pos + n] = f(x)
            llen[b] += n

    append_local(0, T0)
    scale = D ** -0.5
    for r in range(R):
        T = T0 + r * A
        # route over every router token of each query so far
        qr = torch.empty((L, B * T, HQ, D), dtype=torch.bfloat16, device="cuda")
        for b in range(B):
            db.fill_segment(qr[:, b * T:b * T + T0], b, 0, chains[b][:1], qs)
            for rr in range(1, r + 1):
                t0 = T0 + (rr - 1) * A
                db.fill_segment(qr[:, b * T + t0:b * T + t0 + A], b, t0, chains[b][rr:rr + 1], qs)
        offs = [b * T for b in range(B + 1)]
        ids, sc, err = db.route(qr, offs, k, msa.MSA_ROUTE_AUTO)
        del qr
        assert err == 0, (r, err)
        for b in range(B):
            for l in range(L):
                assert set(chains[b][:r + 1].tolist()) <= set(ids[b, l].tolist()), (r, b, l)
        extra = random_docs(qs, db.n_docs, 32, sub=r)
        for b in checked:
            for l in layers:
                parts = [host_query(db.bank, l, b, T0, chains[b][:1], dtype="bf16", q_seed=qs)]
                for rr in range(1, r + 1):
                    t0 = T0 + (rr - 1) * A
                    parts.append(host_query(db.bank, l, b, A, chains[b][rr:rr + 1], dtype="bf16", q_seed=qs,
                                            tok0=t0))
                ref = oracle_doc_scores(db.bank, l, np.concatenate(parts),
                                        list(ids[b, l]) + list(chains[b]) + list(extra))
                check_sampled(ids[b, l], sc[b, l], ref, k, planted=chains[b][:r + 1])
        # gather this round's selections; byte-exact on the checked queries
        msa.msa_gather_kv(store, C, db.d_coffs, None, db.n_docs, torch.from_numpy(ids).cuda(), B, L, k, H, D, M,
                          mem, mem_len, d_err)
        torch.cuda.synchronize()
        assert int(d_err.item()) == 0
        got_len = mem_len.cpu().numpy()
        ref_mem = {}
        for b in checked:
            got = mem[b].view(torch.int16).cpu().numpy().view(np.uint16)
            for l in range(L):
                m, n = oracle_gather_layer(store_np, l, db.coffs, None, ids[b, l], M)
                assert got_len[b, l] == n and np.array_equal(f(got[l, :, :, :n]), m[:, :, :n]), (r, b, l)
                if b in dec_checked and l in layers:
                    ref_mem[(b, l)] = (m, n)
        # DEC decode tokens for all 64 queries
        worst_abs = worst_rel = 0.0
        for s in range(DEC):
            step = r * DEC + s
            dq = torch.empty((B, L, HQ, D), dtype=torch.bfloat16, device="cuda")
            dk = torch.empty((B, L, H, D), dtype=torch.bfloat16, device="cuda")
            dv = torch.empty_like(dk)
            syn.device_fill(dq, qs, syn.STREAM_DEC_Q, step, 0, 0, B * L * HQ, D)
            syn.device_fill(dk, qs, syn.STREAM_DEC_K, step, 0, 0, B * L * H, D)
            syn.device_fill(dv, qs, syn.STREAM_DEC_V, step, 0, 0, B * L * H, D)
            pos0 = llen.cpu().numpy()
            out = torch.full((B, L, HQ, D), float("nan"), dtype=torch.bfloat16, device="cuda")
            msa.msa_sparse_decode(dq, dk, dv, B, L, HQ, H, D, lk, lv, llen, cap, mem, mem_len, M, k, THETA, scale, out,
                                  ws_dec, d_err)
            got = bf16_to_np(out)
            for b in dec_checked:
                for l in layers:
                    row = b * L + l
                    qh = f(syn.fill(qs, syn.STREAM_DEC_Q, step, 0, row * HQ, HQ, D, dtype="bf16"))
                    kh = f(syn.fill(qs, syn.STREAM_DEC_K, step, 0, row * H, H, D, dtype="bf16"))
                    vh = f(syn.fill(qs, syn.STREAM_DEC_V, step, 0, row * H, H, D, dtype="bf16"))
                    m, n = ref_mem[(b, l)]
                    i = int(pos0[b])
                    ref = oracle.decode(qh, kh, vh, m, n, o_lk[(b, l)], o_lv[(b, l)], i, k + i, THETA, scale)
                    worst_abs = max(worst_abs, float(np.abs(got[b, l] - ref).max()))
                    worst_rel = max(worst_rel, rel_l2(got[b, l], ref))
        torch.cuda.synchronize()
        assert int(d_err.item()) == 0
        assert worst_abs <= DEC_MAX_ABS and worst_rel <= DEC_REL_L2, (r, worst_abs, worst_rel)
        if r + 1 < R:
            append_local(r + 1, A)
    assert llen.cpu().tolist() == [cap] * B
    del store, mem, lk, lv
    _free()
