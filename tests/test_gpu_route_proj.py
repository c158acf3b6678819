"""GPU parity of msa_route_topk_hidden (router query projection fused into routing)
against the oracle: Q_r = hidden . W^T per layer (oracle, fp64), then the oracle's
routing on those queries.  Several queries whose tokens span two 128-token tiles with a
ragged tail, every routing path, every group size the fused kernel takes, and planted
documents that the projected queries must find."""
import numpy as np
import pytest
import torch

import msa_synth as syn
import oracle
from tests.helpers import bf16_tensor, check_topk

pytestmark = pytest.mark.gpu

H, D = 8, 128


@pytest.fixture(scope="module")
def msa():
    import top_kv_routing_b200 as m
    return m


def _bank_keys(bank, L):
    """Stored unit routing keys (bf16 bits) [L][C][H][D], made unit by the oracle."""
    C = bank.n_chunks
    out = []
    for l in range(L):
        raw = syn.bf16_bits_to_f32(syn.pooled_router_keys(bank, l, 0, C))
        unit = oracle.pool(None, None, raw, np.arange(C + 1), H, D, 1, 1e6, rope_k=False)["kr_unit"]
        out.append(syn.f32_to_bf16_bits(unit.astype(np.float32)))
    return np.stack(out)


def _inputs(seed, bank, T, hidden, Hq, L, targets):
    """hidden [T][hidden] bf16 bits: the first 128 features carry the topic of the token's
    planted target plus noise; W [L][Hq*D][hidden] bf16 bits: near-identity on those 128
    features for every head, plus small noise (so each projected head points at the
    target's topic)."""
    tg = np.asarray(targets)[np.arange(T) % len(targets)]
    h = syn.fill(seed, syn.STREAM_QR, 90, 0, 0, T, hidden, sigma=1.0, dtype="f32")
    h[:, :D] = syn.fill(seed, syn.STREAM_QR, 91, 0, 0, T, D, sigma=0.5, topic=bank.topic, row_topic=tg, dtype="f32")
    h_bits = syn.f32_to_bf16_bits(h)
    w = syn.fill(seed, syn.STREAM_KBAR, 92, 0, 0, L * Hq * D, hidden, sigma=0.02, dtype="f32").reshape(L, Hq * D,
                                                                                                        hidden)
    for q in range(Hq):
        w[:, q * D + np.arange(D), np.arange(D)] += 1.0
    return h_bits, syn.f32_to_bf16_bits(w)


def _case(msa, seed, q_lens, hidden, Hq, flags, k=4, L=2, n_docs=40):
    lens = syn.doc_lengths_uniform(seed, n_docs, 64, 900)
    bank = syn.make_bank(seed, n_docs, lens, L)
    keys = _bank_keys(bank, L)
    C = bank.n_chunks
    q_off = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    T = int(q_off[-1])
    targets = [[(7 * b + 3) % n_docs, (11 * b + 5) % n_docs] for b in range(len(q_lens))]
    tok_targets = np.concatenate([np.asarray(targets[b])[np.arange(n) % 2] for b, n in enumerate(q_lens)])
    h_bits, w_bits = _inputs(seed, bank, T, hidden, Hq, L, tok_targets)
    B = len(q_lens)
    d_keys = bf16_tensor(keys)
    kr_f8 = None
    if flags in (msa.MSA_ROUTE_AUTO, msa.MSA_ROUTE_TENSOR_F8):
        kr_f8 = torch.empty(keys.shape, dtype=torch.uint8, device="cuda")
        msa.msa_route_filter_keys(d_keys, L, C, H, D, kr_f8)
    coffs = torch.from_numpy(bank.doc_chunk_offsets).cuda()
    ws = torch.empty(msa.msa_route_topk_workspace_size(L, B, T, H, C, n_docs, k), dtype=torch.uint8, device="cuda")
    ids = torch.full((B, L, k), -7, dtype=torch.int32, device="cuda")
    sc = torch.full((B, L, k), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    n = msa.msa_route_topk_hidden(bf16_tensor(h_bits), bf16_tensor(w_bits), hidden, q_off, d_keys, coffs, n_docs, C,
                                  L, Hq, H, D, k, ids, sc, ws, flags=flags, dev_err=err, kr_f8=kr_f8)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    gi, gs = ids.cpu().numpy(), sc.cpu().numpy()
    f = syn.bf16_bits_to_f32
    keys_f = f(keys)
    for l in range(L):
        q_all = oracle.router_project(f(h_bits), f(w_bits[l]), Hq)
        for b in range(B):
            q = q_all[q_off[b]:q_off[b + 1]]
            _, _, ds, _ = oracle.route(q, keys_f[l], bank.doc_chunk_offsets, k, grouped=True)
            check_topk(gi[b, l], gs[b, l], ds, k)
            assert set(targets[b]) <= set(gi[b, l].tolist()), (b, l, targets[b], gi[b, l])
    return n


@pytest.mark.parametrize("flags", [1, 2, 3])
def test_projected_routing_matches_oracle(msa, flags):
    # two queries (100 + 70 tokens: two 128-row tiles, the second ragged), hidden 256, GQA 32/8
    _case(msa, 3, [100, 70], 256, 32, flags)


@pytest.mark.parametrize("Hq", [16, 8])
def test_projected_routing_group_sizes(msa, Hq):
    _case(msa, 4, [40], 192, Hq, 2)


def test_projected_routing_short_query_takes_the_scan(msa):
    _case(msa, 5, [5], 128, 32, 0)


def test_projected_routing_launches_like_the_unfused_call(msa):
    # the projection replaces the query-preparation kernel one for one
    # (E4M3 path: prep, projection, GEMM, top-k, rescore, final, the five bf16-pass kernels
    # and the three of the widened rescoring, which return at once when every layer is
    # certified; the bank has more documents than the first candidates and fewer than the
    # widened ones, so no exact scan is enqueued)
    assert _case(msa, 6, [64], 128, 32, 3) == 14


def test_projected_routing_bench_shape_sampled_layers(msa):
    # the benchmark's projection shape: hidden 2560, 256 tokens, 18 layers, 32 heads; a
    # 300-document bank keeps the oracle's routing short; layers 0 and 11 checked
    L, T, hidden, Hq, k, n_docs = 18, 256, 2560, 32, 16, 300
    lens = syn.doc_lengths_uniform(8, n_docs, 64, 900)
    bank = syn.make_bank(8, n_docs, lens, L)
    keys = _bank_keys(bank, L)
    C = bank.n_chunks
    targets = syn.pick_targets(8, n_docs, 16, sub=3)
    tok_targets = np.asarray(targets)[np.arange(T) % 16]
    h_bits, _ = _inputs(8, bank, T, hidden, Hq, 1, tok_targets)  # (the hidden states only)
    # weights drawn on the device (377 MB); the host redraws the sampled layers' bits: noise
    # as bf16, plus the identity block, rounded to bf16 once (as the device add does)
    w_dev = torch.empty((L, Hq * D, hidden), dtype=torch.bfloat16, device="cuda")
    syn.device_fill(w_dev, 8, syn.STREAM_KBAR, 92, 0, 0, L * Hq * D, hidden, 0.02)
    w_dev.view(L, Hq, D, hidden)[..., :D] += torch.eye(D, dtype=torch.bfloat16, device="cuda")

    def host_w(l):
        noise = syn.fill(8, syn.STREAM_KBAR, 92, 0, l * Hq * D, Hq * D, hidden, sigma=0.02, dtype="bf16")
        x = syn.bf16_bits_to_f32(noise).reshape(Hq, D, hidden)
        x[:, np.arange(D), np.arange(D)] += 1.0
        return syn.bf16_bits_to_f32(syn.f32_to_bf16_bits(x)).reshape(Hq * D, hidden)
    d_keys = bf16_tensor(keys)
    kr_f8 = torch.empty(keys.shape, dtype=torch.uint8, device="cuda")
    msa.msa_route_filter_keys(d_keys, L, C, H, D, kr_f8)
    coffs = torch.from_numpy(bank.doc_chunk_offsets).cuda()
    ws = torch.empty(msa.msa_route_topk_workspace_size(L, 1, T, H, C, n_docs, k), dtype=torch.uint8, device="cuda")
    ids = torch.full((1, L, k), -7, dtype=torch.int32, device="cuda")
    sc = torch.full((1, L, k), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    msa.msa_route_topk_hidden(bf16_tensor(h_bits), w_dev, hidden, [0, T], d_keys, coffs, n_docs, C, L, Hq, H, D, k,
                              ids, sc, ws, flags=msa.MSA_ROUTE_TENSOR_F8, dev_err=err, kr_f8=kr_f8)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    gi, gs = ids.cpu().numpy(), sc.cpu().numpy()
    for l in range(L):
        assert set(np.asarray(targets).tolist()) == set(gi[0, l].tolist()), l  # the 16 planted documents
    f = syn.bf16_bits_to_f32
    for l in (0, 11):
        assert np.array_equal(w_dev[l].cpu().view(torch.int16).numpy().view(np.uint16),
                              syn.f32_to_bf16_bits(host_w(l)))
        q = oracle.router_project(f(h_bits), host_w(l), Hq)
        _, _, ds, _ = oracle.route(q, f(keys[l]), bank.doc_chunk_offsets, k, grouped=True)
        check_topk(gi[0, l], gs[0, l], ds, k)
