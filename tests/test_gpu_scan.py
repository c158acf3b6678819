"""The streaming scan of few-token queries (MSA_ROUTE_SCAN, and MSA_ROUTE_AUTO while the
query's tokens fit the scan's registers) against the oracle's explicit routing: every key
head count the scan takes, 1 to 8 tokens split over up to four queries, several layers and
banks whose block counts leave ragged last units; the scan with more tokens than its
registers hold (the per-warp fallback kernel) on the same inputs."""
import numpy as np
import pytest
import torch

import msa_synth as syn
import oracle
from tests.helpers import check_topk

pytestmark = pytest.mark.gpu

HQ, D = 32, 128


@pytest.fixture(scope="module")
def msa():
    import top_kv_routing_b200 as m
    return m


def _bank(seed, n_docs, H, L, max_len=1400):
    lens = syn.doc_lengths_uniform(seed, n_docs, 1, max_len)
    offs = syn.offsets(lens)
    C, coffs = oracle.count_chunks(offs, 64)
    keys = []
    for l in range(L):
        raw = syn.fill(seed, syn.STREAM_KRBAR, l, 0, 0, C * H, D, sigma=1.0).reshape(C, H, D).astype(np.float64)
        raw[:, :, :8] += 3.0 * (np.arange(C) % 5)[:, None, None] / 5.0  # some structure shared by heads
        unit = raw / np.maximum(np.linalg.norm(raw, axis=2, keepdims=True), 1e-8)
        keys.append(syn.bf16_bits_to_f32(syn.f32_to_bf16_bits(unit.astype(np.float32))))
    return np.stack(keys), coffs, C


def _route(msa, keys, coffs, q, q_off, H, k, flags):
    L, C = keys.shape[:2]
    n_docs = len(coffs) - 1
    B = len(q_off) - 1
    T = int(q_off[-1])
    kr = torch.from_numpy(syn.f32_to_bf16_bits(keys).view(np.int16)).view(torch.bfloat16).cuda()
    ws = torch.empty(msa.msa_route_topk_workspace_size(L, B, T, H, C, n_docs, k), dtype=torch.uint8, device="cuda")
    ids = torch.full((B, L, k), -7, dtype=torch.int32, device="cuda")
    sc = torch.full((B, L, k), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    n = msa.msa_route_topk(torch.from_numpy(np.ascontiguousarray(q, dtype=np.float32)).cuda(), q_off, kr,
                           torch.from_numpy(coffs).cuda(), n_docs, C, L, HQ, H, D, k, ids, sc, ws, flags=flags,
                           dev_err=err)
    torch.cuda.synchronize()
    return ids.cpu().numpy(), sc.cpu().numpy(), int(err.item()), n


@pytest.mark.parametrize("H", [2, 4, 8, 16])
@pytest.mark.parametrize("Ts", [[1], [2], [1, 1], [3, 1], [2, 1, 1], [1, 2, 1, 4], [8]])
def test_scan_matches_the_oracle(msa, H, Ts):
    L, k, seed = 2, 16, 40 + H
    keys, coffs, C = _bank(seed, 173, H, L)
    q_off = syn.offsets(np.asarray(Ts)).astype(np.int32)
    T = int(q_off[-1])
    q = syn.fill(seed, syn.STREAM_QR, 0, 0, 0, L * T * HQ, D).reshape(L, T, HQ, D)
    ids, sc, err, _ = _route(msa, keys, coffs, q, q_off, H, k, msa.MSA_ROUTE_SCAN)
    assert err == 0
    for b in range(len(Ts)):
        for l in range(L):
            _, _, ds, _ = oracle.route(q[l, q_off[b]:q_off[b + 1]], keys[l], coffs, k)
            check_topk(ids[b, l], sc[b, l], ds, k)


def test_scan_on_a_bank_of_many_units(msa):
    # 3 layers x ~37,000 blocks: dozens of units per CTA, a ragged last unit in each layer
    H, L, k, seed = 8, 3, 16, 52
    keys, coffs, C = _bank(seed, 13_000, H, L, max_len=300)
    assert C % 14 != 0
    for Ts in ([1], [4], [2, 2]):
        q_off = syn.offsets(np.asarray(Ts)).astype(np.int32)
        T = int(q_off[-1])
        q = syn.fill(seed, syn.STREAM_QR, 1, 0, 0, L * T * HQ, D).reshape(L, T, HQ, D)
        ids, sc, err, n = _route(msa, keys, coffs, q, q_off, H, k, msa.MSA_ROUTE_AUTO)
        assert err == 0 and n == 4  # AUTO took the scan: query preparation, scan, two top-k kernels
        for b in range(len(Ts)):
            for l in (0, L - 1):
                _, _, ds, _ = oracle.route(q[l, q_off[b]:q_off[b + 1]], keys[l], coffs, k, grouped=True)
                check_topk(ids[b, l], sc[b, l], ds, k)
