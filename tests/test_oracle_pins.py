"""Pins of the CPU oracle against what the pages and the mathematics fix (no GPU).

Each test checks the oracle against something other than itself: values the pages print,
hand-derived worked examples, closed forms, invariants, or a different library routine.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import msa_synth as syn
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------------------- RoPE

def test_rope_position_zero_is_identity():
    x = syn.fill(0, syn.STREAM_K, 0, 0, 0, 1, 128).astype(np.float64)[0]
    assert np.array_equal(oracle.rope(x, 0, 1e6), x)


@pytest.mark.parametrize("j", [0, 1, 17, 63])
def test_rope_rotate_half_pairing_and_frequency(j):
    # RoPE(e_j, p) = cos(p w_j) e_j + sin(p w_j) e_{j+64}, with w_j = theta^(-2j/128);
    # RoPE(e_{j+64}, p) = -sin(p w_j) e_j + cos(p w_j) e_{j+64}.
    d, theta, p = 128, 1e6, 37
    w = theta ** (-2.0 * j / d)
    e = np.zeros(d)
    e[j] = 1.0
    r = oracle.rope(e, p, theta)
    expect = np.zeros(d)
    expect[j] = math.cos(p * w)
    expect[j + 64] = math.sin(p * w)
    np.testing.assert_allclose(r, expect, atol=1e-15)
    e2 = np.zeros(d)
    e2[j + 64] = 1.0
    r2 = oracle.rope(e2, p, theta)
    expect2 = np.zeros(d)
    expect2[j] = -math.sin(p * w)
    expect2[j + 64] = math.cos(p * w)
    np.testing.assert_allclose(r2, expect2, atol=1e-15)


def test_rope_relative_position_and_norm():
    rng = np.random.default_rng(1)
    q, k = rng.standard_normal(128), rng.standard_normal(128)
    a = oracle.rope(q, 100, 1e6) @ oracle.rope(k, 90, 1e6)
    b = oracle.rope(q, 1010, 1e6) @ oracle.rope(k, 1000, 1e6)
    assert abs(a - b) < 1e-9
    assert abs(np.linalg.norm(oracle.rope(q, 777, 1e6)) - np.linalg.norm(q)) < 1e-12


# ----------------------------------------------------------------------------- blocks and bytes

@pytest.mark.parametrize("lens,expect", [([64], 1), ([65], 2), ([1], 1), ([0], 0), ([128, 1, 63], 4),
                                         ([8192], 128)])
def test_block_counts(lens, expect):
    total, offs = oracle.count_chunks(syn.offsets(np.array(lens)), 64)
    assert total == expect
    assert offs[-1] == expect


def test_100m_tokens_give_1_5625m_blocks():
    g = _golden("pages_figures.json")
    lens = syn.doc_lengths_exact_total(3, g["docs"]["value"], g["tokens"]["value"])
    total, _ = oracle.count_chunks(syn.offsets(lens), g["block_tokens"]["value"])
    assert total == 1_562_500
    assert abs(total - g["blocks_at_100M"]["value"]) / g["blocks_at_100M"]["value"] < 0.005


def test_byte_figures_match_pages():
    g = _golden("pages_figures.json")
    C = 1_562_500
    L, H, d = g["routing_layers"]["value"], g["kv_heads"]["value"], g["head_dim"]["value"]
    bf16 = 2
    kr_bytes = C * L * H * d * bf16
    content = 2 * kr_bytes
    assert kr_bytes == 57_600_000_000
    assert abs(kr_bytes - g["routing_key_bytes"]["value"]) / g["routing_key_bytes"]["value"] < 0.05
    assert abs(content - g["content_kv_bytes"]["value"]) / g["content_kv_bytes"]["value"] < 0.05
    assert abs(kr_bytes + content - g["total_cache_bytes"]["value"]) / g["total_cache_bytes"]["value"] < 0.05
    per_doc_blocks = g["tokens"]["value"] / g["docs"]["value"] / g["block_tokens"]["value"]
    per_query = g["top_k"]["value"] * per_doc_blocks * L * 2 * H * d * bf16
    assert abs(per_query - g["per_query_load_bytes"]["value"]) / g["per_query_load_bytes"]["value"] < 0.05


def test_group_ids_equal_csr_positions():
    # The deep dive's map_tensor_to_group_ids (section 5.3): a new 1-based group id
    # wherever the per-token doc id changes.  The CSR offsets must induce the same
    # grouping, and the document-local position restarts at 0 in each group.
    lens = np.array([3, 1, 5, 2])
    offs = syn.offsets(lens)
    doc_ids = syn.token_docs(offs) * 7 + 3  # arbitrary ids, constant inside a document
    change = np.concatenate([[0], (np.diff(doc_ids) != 0).astype(np.int64)])
    group = np.cumsum(change) + 1
    assert np.array_equal(group - 1, syn.token_docs(offs))
    pos = np.arange(offs[-1]) - offs[syn.token_docs(offs)]
    assert list(pos) == [0, 1, 2, 0, 0, 1, 2, 3, 4, 0, 1]


# ----------------------------------------------------------------------------- pooling

def _pool(k, v, kr, lens, H, d, theta=1e6):
    return oracle.pool(k, v, kr, syn.offsets(np.array(lens)), H, d, 64, theta)


def test_pool_constant_and_single_token_blocks():
    H, d = 2, 4
    n = 65
    v = np.full((n, H, d), 0.25, dtype=np.float32)
    kr = np.zeros((n, H, d), dtype=np.float32)
    kr[:, :, :] = np.arange(n, dtype=np.float32)[:, None, None]
    k = np.zeros((n, H, d), dtype=np.float32)
    k[:, :, 0] = 1.0
    out = _pool(k, v, kr, [n], H, d, theta=10000.0)
    assert out["v_bar"].shape == (2, H, d)
    assert np.all(out["v_bar"] == 0.25)                       # constant pools to itself
    assert np.all(out["kr_bar"][0] == 31.5)                   # mean of 0..63
    assert np.all(out["kr_bar"][1] == 64.0)                   # 1-token block is the token
    # K = e_0 rotated by angle p (w_0 = 1): (cos p, 0, sin p, 0).  Dirichlet sums give
    # the block mean in closed form.
    nn, x = 64, 1.0
    mean_cos = math.sin(nn * x / 2) * math.cos((nn - 1) * x / 2) / math.sin(x / 2) / nn
    mean_sin = math.sin(nn * x / 2) * math.sin((nn - 1) * x / 2) / math.sin(x / 2) / nn
    np.testing.assert_allclose(out["k_bar"][0, 0], [mean_cos, 0, mean_sin, 0], atol=1e-12)
    np.testing.assert_allclose(out["k_bar"][1, 1], [math.cos(64), 0, math.sin(64), 0], atol=1e-12)


def test_pool_partial_block_is_mean_of_real_tokens():
    H, d = 1, 8
    n = 100  # blocks of 64 and 36 tokens
    v = syn.fill(5, syn.STREAM_V, 0, 0, 0, n, H * d).reshape(n, H, d)
    out = _pool(None, v, None, [n], H, d)
    hand = v[64:].astype(np.float64).sum(axis=0) / 36.0
    np.testing.assert_allclose(out["v_bar"][1], hand, rtol=1e-14)
    hand0 = v[:64].astype(np.float64).sum(axis=0) / 64.0
    np.testing.assert_allclose(out["v_bar"][0], hand0, rtol=1e-14)


def test_pool_positions_restart_per_document():
    H, d = 1, 4
    k = np.zeros((6, H, d), dtype=np.float32)
    k[:, :, 1] = 1.0
    out = _pool(k, None, None, [3, 3], H, d)
    np.testing.assert_array_equal(out["k_bar"][0], out["k_bar"][1])
    # one document of six tokens would rotate the second half by positions 3..5
    one = _pool(k, None, None, [6], H, d)
    assert one["k_bar"].shape[0] == 1
    assert not np.allclose(one["k_bar"][0], out["k_bar"][0])


def test_pool_router_unit_keys_and_zero_vector():
    H, d = 2, 4
    kr = np.zeros((64, H, d), dtype=np.float32)
    kr[:, 0, :] = [3.0, 4.0, 0.0, 0.0]
    out = _pool(None, None, kr, [64], H, d)
    np.testing.assert_allclose(out["kr_norm"][0], [5.0, 0.0])
    np.testing.assert_allclose(out["kr_unit"][0, 0], [0.6, 0.8, 0, 0])
    assert np.all(out["kr_unit"][0, 1] == 0.0)                # zero vector stays zero


# ----------------------------------------------------------------------------- routing

def _worked():
    g = _golden("route_worked_example.json")
    q = np.array(g["query"], dtype=np.float32)
    kr = np.array(g["blocks"], dtype=np.float32)
    offs = np.array(g["doc_block_offsets"], dtype=np.int64)
    return g, q, kr, offs


@pytest.mark.parametrize("grouped", [False, True])
def test_route_worked_example(grouped):
    g, q, kr, offs = _worked()
    ids, sc, doc, blk = oracle.route(q, kr, offs, 2, grouped=grouped)
    np.testing.assert_allclose(blk, g["expected_block_scores"], atol=1e-12)
    np.testing.assert_allclose(doc, g["expected_doc_scores"], atol=1e-12)
    assert list(ids) == g["expected_top2"]["ids"]
    np.testing.assert_allclose(sc, g["expected_top2"]["scores"], atol=1e-12)
    ids4, sc4, _, _ = oracle.route(q, kr, offs, 4, grouped=grouped)
    assert list(ids4) == g["expected_top4"]["ids"]
    assert sc4[3] == -np.inf
    np.testing.assert_allclose(sc4[:3], g["expected_top4"]["scores"][:3], atol=1e-12)


def test_route_reduction_order_and_pairing_are_distinguished():
    # The fixture's values for the rejected orders differ from the accepted ones, so a
    # swap of the reductions or of the head pairing would fail the worked example.
    g, q, kr, offs = _worked()
    _, _, doc, _ = oracle.route(q, kr, offs, 2)
    assert abs(doc[2] - g["wrong_orders"]["max_over_tokens_then_mean_over_heads_doc2"]) > 0.1
    assert abs(doc[0] - g["wrong_orders"]["head_pairing_h_mod_H_block0_t0"]) > 0.1


def test_route_self_match_scores_one_and_scale_invariance():
    rng = np.random.default_rng(3)
    H, Hq, d = 8, 32, 128
    kr = rng.standard_normal((10, H, d)).astype(np.float32)
    q = np.repeat(kr[6][None, :, :], 4, axis=1).reshape(1, Hq, d)  # query head h = key head h//4
    offs = np.array([0, 4, 10])
    ids, sc, doc, _ = oracle.route(q, kr, offs, 2)
    assert ids[0] == 1 and abs(sc[0] - 1.0) < 1e-12
    _, _, doc2, _ = oracle.route(q * 3.5, kr * 0.01, offs, 2)
    np.testing.assert_allclose(doc2, doc, atol=1e-12)


def test_route_identical_heads_equal_single_head():
    rng = np.random.default_rng(4)
    d = 128
    k1 = rng.standard_normal((6, 1, d)).astype(np.float32)
    q1 = rng.standard_normal((3, 1, d)).astype(np.float32)
    offs = np.array([0, 2, 6])
    _, _, doc1, blk1 = oracle.route(q1, k1, offs, 2)
    k8 = np.repeat(k1, 8, axis=1)
    q32 = np.repeat(q1, 32, axis=1)
    _, _, doc8, blk8 = oracle.route(q32, k8, offs, 2)
    np.testing.assert_allclose(blk8, blk1, atol=1e-13)
    np.testing.assert_allclose(doc8, doc1, atol=1e-13)


def test_route_explicit_equals_grouped():
    rng = np.random.default_rng(5)
    q = rng.standard_normal((5, 32, 128)).astype(np.float32)
    kr = rng.standard_normal((40, 8, 128)).astype(np.float32)
    kr[3, 2] = 0.0  # zero key head: clamped norm
    offs = np.array([0, 3, 3, 20, 40])  # includes an empty document
    a = oracle.route(q, kr, offs, 3)
    b = oracle.route(q, kr, offs, 3, grouped=True)
    np.testing.assert_allclose(a[3], b[3], atol=1e-12)
    assert a[2][1] == -np.inf and b[2][1] == -np.inf
    assert list(a[0]) == list(b[0])


def test_query_sums_hand_worked():
    # 4 query heads, 2 key heads (G = 2): head 0 = (3, 4) -> (0.6, 0.8); head 1 = 2 e0 -> e0;
    # head 2 = -5 e1 -> -e1; head 3 = e3; a zero head 4 of a second token stays zero
    q = np.zeros((2, 4, 4), dtype=np.float32)
    q[0, 0, :2] = [3, 4]
    q[0, 1, 0] = 2
    q[0, 2, 1] = -5
    q[0, 3, 3] = 1
    q[1, 0, 2] = 7
    qt = oracle.query_sums(q, 2)
    np.testing.assert_allclose(qt[0, 0], [1.6 / 4, 0.8 / 4, 0, 0], atol=1e-15)
    np.testing.assert_allclose(qt[0, 1], [0, -0.25, 0, 0.25], atol=1e-15)
    np.testing.assert_allclose(qt[1, 0], [0, 0, 0.25, 0], atol=1e-15)
    np.testing.assert_allclose(qt[1, 1], 0, atol=0)


def test_query_sums_give_the_explicit_routing_scores():
    # sum_g <qt_g, k_g> / ||k_g|| is the explicit mean of the 32 cosines
    rng = np.random.default_rng(6)
    q = rng.standard_normal((3, 32, 128)).astype(np.float32)
    kr = rng.standard_normal((10, 8, 128)).astype(np.float32)
    _, _, _, blk = oracle.route(q, kr, np.array([0, 10]), 1)
    qt = oracle.query_sums(q, 8)
    k = kr.astype(np.float64)
    k /= np.linalg.norm(k, axis=2, keepdims=True)
    s = np.einsum("tgd,cgd->tc", qt, k)
    np.testing.assert_allclose(s.max(axis=0), blk, atol=1e-12)


def test_topk_matches_python_sorted_with_ties():
    s = np.array([0.5, 0.9, 0.5, -1.0, 0.9, 0.1, -np.inf])
    ids, sc = oracle.topk(s, 5)
    ref = sorted(range(len(s)), key=lambda i: (-s[i], i))[:5]
    assert list(ids) == ref == [1, 4, 0, 2, 5]
    ids9, sc9 = oracle.topk(s, 9)
    assert list(ids9[7:]) == [-1, -1] and np.all(sc9[7:] == -np.inf)


def test_route_recovers_planted_documents():
    # Tiny-bank recipe: 64 documents, K_r = N(0,1) + topic (norm 4); the query's tokens
    # carry the topics of two planted documents plus N(0, 0.5) noise.
    seed = 0
    lens = syn.doc_lengths_uniform(seed, 64, 200, 1000)
    bank = syn.make_bank(seed, 64, lens, 1)
    kr = syn.raw_tokens(bank, 0, syn.STREAM_KR, 0, bank.n_tokens)
    pooled = oracle.pool(None, None, kr, bank.doc_tok_offsets, 8, 128)
    targets = syn.pick_targets(seed, 64, 2)
    q = syn.query_router(seed, 0, 0, 16, 32, 128, bank.topic, targets)
    ids, sc, doc, _ = oracle.route(q, pooled["kr_bar"], bank.doc_chunk_offsets, 4)
    assert set(ids[:2].tolist()) == set(targets.tolist())
    assert sc[1] - sc[2] > 0.1


# ----------------------------------------------------------------------------- gather

def test_gather_matches_slicing_and_capacity():
    rng = np.random.default_rng(6)
    L, H, d = 2, 2, 8
    offs = np.array([0, 2, 5, 6, 10])
    C = offs[-1]
    host = rng.integers(0, 65535, size=(L, C, 2, H, d), dtype=np.uint16)
    ids = np.array([[[2, 0, -1], [3, 1, 0]]], dtype=np.int32)
    out, mem_len = oracle.gather(host, offs, ids, 12)
    assert mem_len.tolist() == [[3, 9]]
    for l in range(L):
        rows = [c for doc in ids[0, l] if doc >= 0 for c in range(offs[doc], offs[doc + 1])]
        ref = host[l, rows]                              # [m][2][H][d]
        got = out[0, l, :, :, :len(rows)]                # [2][H][m][d]
        assert np.array_equal(np.transpose(got, (2, 0, 1, 3)), ref)
        assert np.all(out[0, l, :, :, len(rows):] == 0)
    with pytest.raises(OverflowError):
        oracle.gather(host, offs, ids, 8)


# ----------------------------------------------------------------------------- decode

def _empty_local(H, cap, d):
    return np.zeros((H, cap, d)), np.zeros((H, cap, d))


def test_decode_single_key_returns_value():
    rng = np.random.default_rng(7)
    Hq, H, d = 8, 2, 16
    q = rng.standard_normal((Hq, d))
    kn, vn = rng.standard_normal((H, d)), rng.standard_normal((H, d))
    lk, lv = _empty_local(H, 4, d)
    out = oracle.decode(q, kn, vn, np.zeros((2, H, 1, d)), 0, lk, lv, 0, 5, 1e6, d ** -0.5)
    np.testing.assert_allclose(out, np.repeat(vn.astype(np.float32), Hq // H, axis=0), atol=1e-15)


def test_decode_zero_query_is_mean_of_values():
    rng = np.random.default_rng(8)
    Hq, H, d, M = 4, 1, 16, 5
    mem = rng.standard_normal((2, H, M + 3, d)).astype(np.float32)
    kn, vn = rng.standard_normal((H, d)), rng.standard_normal((H, d))
    lk, lv = _empty_local(H, 4, d)
    lv[0, :2] = rng.standard_normal((2, d))
    lk[0, :2] = rng.standard_normal((2, d))
    out = oracle.decode(np.zeros((Hq, d)), kn, vn, mem, M, lk, lv, 2, 7, 1e6, 0.1)
    vals = np.concatenate([mem[1, 0, :M], lv[0, :2], vn.astype(np.float32)])
    np.testing.assert_allclose(out, np.tile(vals.mean(axis=0), (Hq, 1)), atol=1e-13)


def test_decode_two_key_softmax_closed_form():
    d = 4
    q = np.array([[2.0, 0, 0, 0]])
    kn = np.zeros((1, d))
    vn = np.array([[0.0, 1.0, 0, 0]])
    mem = np.zeros((2, 1, 1, d), dtype=np.float32)
    mem[0, 0, 0] = [1.0, 0, 0, 0]
    mem[1, 0, 0] = [1.0, 0, 0, 0]
    lk, lv = _empty_local(1, 2, d)
    out = oracle.decode(q, kn, vn, mem, 1, lk, lv, 0, 0, 1e6, 0.5)  # pos 0: no rotation
    w = math.exp(1.0) / (math.exp(1.0) + 1.0)                         # logits 0.5*2 = 1 and 0
    np.testing.assert_allclose(out[0], [w, 1 - w, 0, 0], atol=1e-15)


def test_decode_without_memory_is_causal_gqa_attention():
    # With no memory the step is ordinary GQA attention of the newest token over the
    # rotated local keys: compare with torch's scaled_dot_product_attention in fp64.
    rng = np.random.default_rng(9)
    Hq, H, d, steps, off = 8, 2, 32, 6, 16
    lk, lv = _empty_local(H, steps, d)
    for i in range(steps):
        q = rng.standard_normal((Hq, d)).astype(np.float32)
        kn = rng.standard_normal((H, d)).astype(np.float32)
        vn = rng.standard_normal((H, d)).astype(np.float32)
        out = oracle.decode(q, kn, vn, np.zeros((2, H, 1, d), np.float32), 0, lk, lv, i, off + i, 1e6,
                            d ** -0.5)
        qr = np.stack([oracle.rope(q[h].astype(np.float64), off + i, 1e6) for h in range(Hq)])
        kk = torch.from_numpy(np.repeat(lk[:, :i + 1], Hq // H, axis=0))[None]
        vv = torch.from_numpy(np.repeat(lv[:, :i + 1], Hq // H, axis=0))[None]
        ref = torch.nn.functional.scaled_dot_product_attention(torch.from_numpy(qr)[None, :, None], kk, vv)
        np.testing.assert_allclose(out, ref[0, :, 0].numpy(), atol=1e-12)
        # the appended key is the rotated new key (position = offset + local index)
        np.testing.assert_allclose(lk[:, i], [oracle.rope(kn[h].astype(np.float64), off + i, 1e6)
                                              for h in range(H)], atol=0)
    assert np.all(lv[:, :steps] != 0)


def test_decode_depends_only_on_relative_positions_without_memory():
    rng = np.random.default_rng(10)
    Hq, H, d, steps = 4, 1, 16, 5
    data = [(rng.standard_normal((Hq, d)), rng.standard_normal((H, d)), rng.standard_normal((H, d)))
            for _ in range(steps)]
    outs = []
    for off in (0, 1000):
        lk, lv = _empty_local(H, steps, d)
        o = [oracle.decode(q, kn, vn, np.zeros((2, H, 1, d)), 0, lk, lv, i, off + i, 1e4, 0.25)
             for i, (q, kn, vn) in enumerate(data)]
        outs.append(np.array(o))
    np.testing.assert_allclose(outs[0], outs[1], atol=1e-9)


def test_decode_local_cache_full_is_an_error():
    lk, lv = _empty_local(1, 2, 4)
    with pytest.raises(OverflowError):
        oracle.decode(np.zeros((1, 4)), np.zeros((1, 4)), np.zeros((1, 4)), np.zeros((2, 1, 1, 4)), 0,
                      lk, lv, 2, 0, 1e6, 1.0)


def test_prefill_is_masked_gqa_attention_over_memory_prefix_and_causal_block():
    # Prefill of T new tokens with memory and an existing local prefix: token i attends
    # the memory, the prefix and the new tokens up to itself.  Compare with torch's
    # scaled_dot_product_attention (fp64) given the rotated queries and keys and that mask.
    rng = np.random.default_rng(21)
    Hq, H, d, T, M, pre, off = 8, 2, 32, 7, 5, 3, 4
    mem = rng.standard_normal((2, H, M + 2, d)).astype(np.float32)
    lk, lv = _empty_local(H, pre + T, d)
    pk = rng.standard_normal((H, pre, d))
    pv = rng.standard_normal((H, pre, d))
    lk[:, :pre], lv[:, :pre] = pk, pv
    q = rng.standard_normal((T, Hq, d)).astype(np.float32)
    kn = rng.standard_normal((T, H, d)).astype(np.float32)
    vn = rng.standard_normal((T, H, d)).astype(np.float32)
    out = oracle.prefill(q, kn, vn, mem, M, lk, lv, pre, off + pre, 1e6, d ** -0.5)
    qr = np.stack([[oracle.rope(q[i, h].astype(np.float64), off + pre + i, 1e6) for h in range(Hq)]
                   for i in range(T)])                                        # [T][Hq][d]
    kr = np.stack([[oracle.rope(kn[i, h].astype(np.float64), off + pre + i, 1e6) for h in range(H)]
                   for i in range(T)])                                        # [T][H][d]
    keys = np.concatenate([mem[0, :, :M].astype(np.float64), pk, np.transpose(kr, (1, 0, 2))], axis=1)
    vals = np.concatenate([mem[1, :, :M].astype(np.float64), pv, np.transpose(vn.astype(np.float64), (1, 0, 2))],
                          axis=1)                                             # [H][M+pre+T][d]
    n = M + pre + T
    mask = np.ones((T, n), dtype=bool)
    for i in range(T):
        mask[i, M + pre + i + 1:] = False
    kk = torch.from_numpy(np.repeat(keys, Hq // H, axis=0))[None]
    vv = torch.from_numpy(np.repeat(vals, Hq // H, axis=0))[None]
    qq = torch.from_numpy(np.transpose(qr, (1, 0, 2)))[None]                  # [1][Hq][T][d]
    ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, attn_mask=torch.from_numpy(mask))
    np.testing.assert_allclose(out, np.transpose(ref[0].numpy(), (1, 0, 2)), atol=1e-12)
    np.testing.assert_allclose(lk[:, pre:pre + T], np.transpose(kr, (1, 0, 2)), atol=0)


def test_prefill_zero_queries_average_the_visible_values():
    rng = np.random.default_rng(22)
    Hq, H, d, T, M = 4, 2, 16, 5, 3
    mem = rng.standard_normal((2, H, M, d)).astype(np.float32)
    lk, lv = _empty_local(H, T, d)
    vn = rng.standard_normal((T, H, d)).astype(np.float32)
    out = oracle.prefill(np.zeros((T, Hq, d), np.float32), rng.standard_normal((T, H, d)).astype(np.float32), vn,
                         mem, M, lk, lv, 0, 0, 1e6, 0.1)
    for i in range(T):
        for hq in range(Hq):
            h = hq // (Hq // H)
            vis = np.concatenate([mem[1, h].astype(np.float64), vn[:i + 1, h].astype(np.float64)])
            np.testing.assert_allclose(out[i, hq], vis.mean(axis=0), atol=1e-12)


def test_prefill_of_one_token_is_a_decode_step():
    rng = np.random.default_rng(23)
    Hq, H, d, M = 8, 2, 16, 4
    mem = rng.standard_normal((2, H, M, d)).astype(np.float32)
    q = rng.standard_normal((1, Hq, d)).astype(np.float32)
    kn = rng.standard_normal((1, H, d)).astype(np.float32)
    vn = rng.standard_normal((1, H, d)).astype(np.float32)
    a_k, a_v = _empty_local(H, 3, d)
    b_k, b_v = _empty_local(H, 3, d)
    a = oracle.prefill(q, kn, vn, mem, M, a_k, a_v, 2, 9, 1e6, 0.2)
    b = oracle.decode(q[0], kn[0], vn[0], mem, M, b_k, b_v, 2, 9, 1e6, 0.2)
    np.testing.assert_array_equal(a[0], b)


# ----------------------------------------------------------------------------- router projection

def test_router_projection_hand_example():
    # Q_r[t][j] = sum_k h[t][k] w[j][k] with w stored [features][hidden] (nn.Linear's
    # weight layout), features grouped into heads of d = 2: worked by hand.
    h = np.array([[1, 2], [3, -1]], np.float32)
    w = np.array([[3, 4], [0, 1], [1, 0], [2, 2], [-1, 5], [0, 0]], np.float32)
    q = oracle.router_project(h, w, 3)
    assert q.shape == (2, 3, 2)
    assert q.tolist() == [[[11, 2], [1, 6], [9, 0]], [[5, -1], [3, 4], [-8, 0]]]


def test_router_projection_one_hot_rows_select_hidden_features():
    rng = np.random.default_rng(31)
    T, hidden, Hq, d = 5, 24, 3, 8
    h = rng.standard_normal((T, hidden)).astype(np.float32)
    pick = rng.integers(0, hidden, size=Hq * d)
    w = np.zeros((Hq * d, hidden), np.float32)
    w[np.arange(Hq * d), pick] = 1.0
    q = oracle.router_project(h, w, Hq)
    np.testing.assert_array_equal(q.reshape(T, Hq * d), h[:, pick].astype(np.float64))


def test_routing_of_projected_queries_is_invariant_to_weight_scale():
    # the routing score is a cosine per head: scaling the projection weights by a
    # positive constant changes no score and no selection
    rng = np.random.default_rng(32)
    T, hidden, Hq, H, d, C = 4, 32, 4, 2, 8, 6
    h = rng.standard_normal((T, hidden)).astype(np.float32)
    w = rng.standard_normal((Hq * d, hidden)).astype(np.float32)
    kr = rng.standard_normal((C, H, d)).astype(np.float32)
    offs = np.array([0, 2, 3, 6])
    a = oracle.route(oracle.router_project(h, w, Hq), kr, offs, 2)
    b = oracle.route(oracle.router_project(h, 8 * w, Hq), kr, offs, 2)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_allclose(a[2], b[2], atol=1e-12)


# ----------------------------------------------------------------------------- layer-aggregated routing

def test_layer_mean_selection_hand_example():
    # per-layer document scores, worked by hand: means 0.5, 0.45, 0.5, -inf (doc 3 has no
    # block, so it ranks last at -inf); the tie between documents 0 and 2 goes to the
    # lower id; a fifth slot has no document (-1)
    ds = [[0.9, 0.1, 0.5, -np.inf], [0.1, 0.8, 0.5, -np.inf]]
    ids, sc, mean = oracle.layer_mean_topk(ds, 5)
    assert ids.tolist() == [0, 2, 1, 3, -1]
    assert np.isneginf(sc[4])
    assert sc[:3].tolist() == [0.5, 0.5, 0.45] and np.isneginf(sc[3])
    assert mean[:3].tolist() == [0.5, 0.45, 0.5]
    # each layer alone would pick differently: layer 0 -> 0, layer 1 -> 1
    assert oracle.layer_mean_topk(ds[:1], 1)[0].tolist() == [0]
    assert oracle.layer_mean_topk(ds[1:], 1)[0].tolist() == [1]


def test_layer_mean_routing_of_one_layer_or_equal_layers_is_the_per_layer_routing():
    rng = np.random.default_rng(41)
    T, Hq, H, d, k = 3, 4, 2, 8, 3
    offs = np.array([0, 2, 2, 5, 9, 10])
    kr = rng.standard_normal((10, H, d)).astype(np.float32)
    q = rng.standard_normal((T, Hq, d)).astype(np.float32)
    ref_ids, ref_sc, ref_ds, _ = oracle.route(q, kr, offs, k)
    for L in (1, 3):
        ids, sc, mean = oracle.route_layer_mean([q] * L, [kr] * L, offs, k)
        assert ids.tolist() == ref_ids.tolist()
        np.testing.assert_allclose(sc, ref_sc, rtol=1e-12)
        assert np.isneginf(mean[1])  # the empty document
