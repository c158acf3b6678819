"""The tensor-core routing filter and its certification on the GPU.

The filter scores (MSA_ROUTE_FILTER_SCORES) are checked against the oracle's exact document
scores within the error bound derived from the operands' rounding (worst-case form,
computed here from the oracle's query sums), including rows built so that a tensor core
that dropped low-order bits while accumulating would exceed it.  The banks of
tests/certify_banks.py, on which fixed error margins certify wrong selections or on which
near-ties outnumber every candidate list, must route to the oracle's exact top-k on every
path: E4M3 filter, bf16 filter, widened rescoring and the exact scan fallback."""
import numpy as np
import pytest
import torch

import msa_synth as syn
import oracle
from tests import certify_banks as cb
from tests.helpers import check_topk, e4m3

pytestmark = pytest.mark.gpu

H, HQ, D = 8, 32, 128
U_BF16, U_E4M3, KEY_DEV, ACC = 2.0 ** -8, 2.0 ** -4, 2.0 ** -8 + 2.0 ** -19, 2.0 ** -13


@pytest.fixture(scope="module")
def msa():
    import top_kv_routing_b200 as m
    return m


def _keys_dev(keys_layers):
    """[L][C][H][D] float32 values that are bf16-exact -> device bf16."""
    bits = syn.f32_to_bf16_bits(np.ascontiguousarray(keys_layers, dtype=np.float32))
    assert np.array_equal(syn.bf16_bits_to_f32(bits), np.asarray(keys_layers, dtype=np.float32))
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def _f8(msa, kr_hat):
    L, C = kr_hat.shape[:2]
    out = torch.empty(kr_hat.shape, dtype=torch.uint8, device="cuda")
    msa.msa_route_filter_keys(kr_hat, L, C, H, D, out)
    torch.cuda.synchronize()
    return out


def _e4m3_decode(b):
    b = b.astype(np.int64)
    sign = np.where(b >> 7, -1.0, 1.0)
    e, m = (b >> 3) & 15, b & 7
    return sign * np.where(e == 0, m / 8.0 * 2.0 ** -6, (1 + m / 8.0) * 2.0 ** (e - 7.0))


def _route(msa, q_layers, q_off, kr_hat, kr_f8, coffs, k, flags):
    """q_layers [L][T_total][Hq][D] float32 -> (ids, scores, dev_err) numpy."""
    L, C = kr_hat.shape[:2]
    n_docs = len(coffs) - 1
    B = len(q_off) - 1
    T = int(q_off[-1])
    ws = torch.empty(msa.msa_route_topk_workspace_size(L, B, T, H, C, n_docs, k), dtype=torch.uint8, device="cuda")
    ids = torch.full((B, L, k), -7, dtype=torch.int32, device="cuda")
    sc = torch.full((B, L, k), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    qr = torch.from_numpy(np.ascontiguousarray(q_layers, dtype=np.float32)).cuda()
    msa.msa_route_topk(qr, q_off, kr_hat, torch.from_numpy(np.asarray(coffs, np.int64)).cuda(), n_docs, C, L, HQ, H, D,
                       k, ids, sc, ws, flags=flags, dev_err=err, kr_f8=kr_f8)
    torch.cuda.synchronize()
    return ids.cpu().numpy(), sc.cpu().numpy(), int(err.item())


def worst_bound(q, kind):
    """Worst-case filter error bound of one query (all tokens) from the derivation, with the
    operand rounding of every element at its largest: q [T][Hq][D] -> float."""
    qt = oracle.query_sums(q, H)                       # [T][H][D]
    nq = np.linalg.norm(qt, axis=2)                     # [T][H]
    eta = 2.0 ** -10
    if kind == "bf16":
        per = U_BF16 * nq * (1 + KEY_DEV) + KEY_DEV * nq + ACC * (1 + KEY_DEV) * (1 + U_BF16) * nq
    else:
        n_da = U_E4M3 * nq + eta * np.sqrt(D) / 2048
        n_a = (1 + U_E4M3) * nq + eta * np.sqrt(D) / 2048
        per = ((n_da + U_E4M3 * n_a) * (1 + 2.0 ** -15) + 2.0 ** -18 * np.sqrt(D) * n_a + 2.0 ** -16 * nq
               + ACC * 1.07 * n_a)
    return float((per.sum(axis=1) * (1 + 2.0 ** -10) + 2.0 ** -20 * nq.sum(axis=1) + 2.0 ** -24).max())


# ----------------------------------------------------------------------------- filter error

def _filter_vs_oracle(msa, keys, coffs, q, k):
    """Filter scores of the returned documents against the oracle's exact scores; returns
    the largest error over the bound for each filter kind."""
    kr_hat = _keys_dev(keys[None])
    kr_f8 = _f8(msa, kr_hat)
    _, _, exact, _ = oracle.route(q, keys, coffs, k, grouped=True)
    out = {}
    for kind, flags in (("bf16", msa.MSA_ROUTE_TENSOR), ("e4m3", msa.MSA_ROUTE_TENSOR_F8)):
        ids, sc, err = _route(msa, q[None], [0, q.shape[0]], kr_hat, kr_f8, coffs, k,
                              flags | msa.MSA_ROUTE_FILTER_SCORES)
        assert err == 0
        bound = worst_bound(q, kind)
        worst = 0.0
        for d, f in zip(ids[0, 0], sc[0, 0]):
            if d < 0 or not np.isfinite(exact[d]):
                continue
            e = abs(float(f) - exact[d])
            assert e <= bound, (kind, int(d), float(f), exact[d], e, bound)
            worst = max(worst, e / bound)
        out[kind] = worst
    return out


@pytest.mark.parametrize("kind", ["planted", "noise", "concentrated"])
def test_filter_error_within_derived_bound(msa, kind):
    lens = syn.doc_lengths_lognormal(21, 64)
    bank = syn.make_bank(21, len(lens), lens, 1)
    keys = syn.bf16_bits_to_f32(syn.pooled_router_keys(bank, 0, 0, bank.n_chunks))
    keys = (keys / np.linalg.norm(keys.astype(np.float64), axis=2, keepdims=True)).astype(np.float32)
    keys = syn.bf16_bits_to_f32(syn.f32_to_bf16_bits(keys))
    T = 40
    if kind == "planted":
        q = syn.query_router(21, 0, 0, T, HQ, D, bank.topic, np.arange(8))
    elif kind == "noise":
        q = syn.fill(21, syn.STREAM_QR, 0, 0, 0, T * HQ, D).reshape(T, HQ, D)
    else:
        # every head of a token along one or two coordinates: no averaging over the elements
        q = np.zeros((T, HQ, D), dtype=np.float32)
        for t in range(T):
            q[t, :, t % D] = 1.0
            q[t, : HQ // 2, (7 * t + 3) % D] = 0.37
    res = _filter_vs_oracle(msa, keys, bank.doc_chunk_offsets, q, 64)
    assert all(v <= 1.0 for v in res.values()), res


@pytest.mark.parametrize("bank", ["e4m3_trap", "bf16_trap", "crowd"])
def test_filter_error_within_derived_bound_on_trap_banks(msa, bank):
    keys = {"e4m3_trap": cb.bank_e4m3_trap, "bf16_trap": cb.bank_bf16_trap,
            "crowd": lambda: cb.bank_crowd(40)}[bank]()
    res = _filter_vs_oracle(msa, keys, np.arange(len(keys) + 1), cb.e0_query(1), 56)
    assert all(v <= 1.0 for v in res.values()), res


def test_tensor_core_accumulation_keeps_small_products(msa):
    # Rows with one large product per key head and 63 products 2^-17 .. 2^-21 of it, all of
    # one sign: fp32 accumulation keeps them (to within 2^-24 of the running sum); an
    # accumulator that dropped them would be off by up to 4.8e-4 of the sum of |products|,
    # beyond the 2^-13 allowance of the bound.  The
    # query is exactly representable in both operand formats (entries +-1/8 on 64
    # coordinates: unit, so its sums are exact), and the test predicts each filter score from
    # the operands the kernels use (the E4M3 keys read back).
    rng = np.random.default_rng(5)
    n_docs = 48
    sgn = np.where(rng.standard_normal(64) > 0, 1.0, -1.0)
    q = np.zeros((1, HQ, D), dtype=np.float32)
    q[0, :, :64] = sgn / 8
    keys = np.zeros((n_docs, H, D), dtype=np.float32)
    for d in range(n_docs):
        for g in range(H):
            small = 2.0 ** -(17 + d % 5)
            row = np.zeros(D)
            row[0] = 1.0
            row[1:64] = small
            row[:64] *= sgn  # every product q_i k_i positive
            keys[d, g] = cb.bf16(row / np.linalg.norm(row))
    kr_hat = _keys_dev(keys[None])
    kr_f8 = _f8(msa, kr_hat)
    f8_keys = _e4m3_decode(kr_f8.cpu().numpy()[0])
    qt = np.float64(q[0, :4, :].sum(axis=0)) / HQ      # every group's query sum (exact): sgn/64
    coffs = np.arange(n_docs + 1)
    for kind, flags in (("bf16", msa.MSA_ROUTE_TENSOR), ("e4m3", msa.MSA_ROUTE_TENSOR_F8)):
        ids, sc, err = _route(msa, q[None], [0, 1], kr_hat, kr_f8, coffs, n_docs,
                              flags | msa.MSA_ROUTE_FILTER_SCORES)
        assert err == 0
        for d, f in zip(ids[0, 0], sc[0, 0]):
            if kind == "bf16":
                p = qt[None, :] * keys[d].astype(np.float64)
            else:
                p = e4m3(2048 * qt)[None, :] * f8_keys[d] / 2.0 ** 19
            want, mag = p.sum(), np.abs(p).sum()
            assert abs(float(f) - want) <= ACC * mag + 1e-12, (kind, int(d), float(f), want)


# ----------------------------------------------------------------------------- certification

def _trap(bank):
    return {"e4m3_trap": cb.bank_e4m3_trap, "bf16_trap": cb.bank_bf16_trap,
            "crowd_widened": lambda: cb.bank_crowd(100), "crowd_scan": lambda: cb.bank_crowd(1100)}[bank]()


@pytest.mark.parametrize("bank", ["e4m3_trap", "bf16_trap", "crowd_widened", "crowd_scan"])
@pytest.mark.parametrize("path", ["f8", "bf16", "scan", "auto"])
def test_trap_banks_route_to_the_exact_top_k(msa, bank, path):
    keys = _trap(bank)
    n_docs = len(keys)
    coffs = np.arange(n_docs + 1)
    kr_hat = _keys_dev(keys[None])
    kr_f8 = _f8(msa, kr_hat)
    T = 16 if path == "auto" else 1
    q = cb.e0_query(T)
    flags = {"f8": msa.MSA_ROUTE_TENSOR_F8, "bf16": msa.MSA_ROUTE_TENSOR, "scan": msa.MSA_ROUTE_SCAN,
             "auto": msa.MSA_ROUTE_AUTO}[path]
    ids, sc, err = _route(msa, q[None], [0, T], kr_hat, kr_f8 if path in ("f8", "auto") else None, coffs, 16, flags)
    assert err == 0
    _, _, exact, _ = oracle.route(q, keys, coffs, 16, grouped=True)
    check_topk(ids[0, 0], sc[0, 0], exact, 16)


@pytest.mark.parametrize("path", ["f8", "bf16"])
def test_trap_bank_batch_certifies_per_query(msa, path):
    # two queries in one call over the crowd bank, two layers: query 0 along coordinate 0
    # (no filter can certify it: the exact scan decides), query 1 along a tail coordinate
    # (spread scores, certified by the first filter); both exact
    keys = cb.bank_crowd(1100)
    L = 2
    kl = np.stack([keys, keys[::-1].copy()])
    n_docs = len(keys)
    coffs = np.arange(n_docs + 1)
    kr_hat = _keys_dev(kl)
    kr_f8 = _f8(msa, kr_hat)
    q0 = cb.e0_query(3)
    q1 = np.zeros((5, HQ, D), dtype=np.float32)
    q1[:, :, 3] = 1.0
    q1[:, :, 9] = 0.5
    ql = np.concatenate([q0, q1])[None].repeat(L, axis=0)
    flags = msa.MSA_ROUTE_TENSOR_F8 if path == "f8" else msa.MSA_ROUTE_TENSOR
    ids, sc, err = _route(msa, ql, [0, 3, 8], kr_hat, kr_f8, coffs, 16, flags)
    assert err == 0
    for b, (lo, hi) in enumerate(((0, 3), (3, 8))):
        for l in range(L):
            _, _, exact, _ = oracle.route(ql[l, lo:hi], kl[l], coffs, 16, grouped=True)
            check_topk(ids[b, l], sc[b, l], exact, 16)


@pytest.mark.parametrize("bank", ["e4m3_trap", "crowd_widened", "crowd_scan"])
@pytest.mark.parametrize("path", ["f8", "bf16"])
def test_trap_banks_layer_mean_selection(msa, bank, path):
    keys = _trap(bank)
    L = 2
    kl = np.stack([keys, keys])
    n_docs = len(keys)
    coffs = np.arange(n_docs + 1)
    kr_hat = _keys_dev(kl)
    kr_f8 = _f8(msa, kr_hat)
    q = cb.e0_query(2)
    ql = np.stack([q, q])
    flags = (msa.MSA_ROUTE_TENSOR_F8 if path == "f8" else msa.MSA_ROUTE_TENSOR) | msa.MSA_ROUTE_LAYER_MEAN
    ids, sc, err = _route(msa, ql, [0, 2], kr_hat, kr_f8, coffs, 16, flags)
    assert err == 0
    _, _, mean = oracle.route_layer_mean(ql, kl, coffs, 16)
    for l in range(L):
        check_topk(ids[0, l], sc[0, l], mean, 16)
    assert np.array_equal(ids[0, 0], ids[0, 1])
