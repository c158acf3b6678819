"""GPU parity of the layer-aggregated routing (MSA_ROUTE_LAYER_MEAN: one selection for
every layer, documents ranked by the mean over layers of their scores) against the
oracle's layer-mean routing, on the bf16 and E4M3 tensor paths, with planted queries, a
short query (which the flag keeps on the tensor path), and queries of pure noise (the
E4M3 selection then goes through the bf16 second pass)."""
import numpy as np
import pytest

import oracle
from tests.fullsize import DeviceBank, host_doc_keys, host_query, random_docs
from tests.helpers import check_topk

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msa():
    import top_kv_routing_b200 as m
    return m


def _check(msa, db, qr_targets, T, k, flags, q_seed=None):
    B = len(qr_targets)
    targets_of = lambda b: qr_targets[b]
    qr = db.queries(B, T, targets_of, q_seed=q_seed)
    ids, sc, err = db.route(qr, [T * b for b in range(B + 1)], k, flags | msa.MSA_ROUTE_LAYER_MEAN)
    assert err == 0
    n_docs = db.n_docs
    keys = [host_doc_keys(db.bank, l, range(n_docs)) for l in range(db.L)]
    for b in range(B):
        q_layers = [host_query(db.bank, l, b, T, targets_of(b), q_seed=q_seed) for l in range(db.L)]
        _, _, mean = oracle.route_layer_mean(q_layers, [kk for kk, _ in keys], keys[0][1], k)
        for l in range(db.L):
            assert np.array_equal(ids[b, l], ids[b, 0]) and np.array_equal(sc[b, l], sc[b, 0])
            check_topk(ids[b, l], sc[b, l], mean, k)
        want = [t for t in targets_of(b) if t >= 0]
        if want:
            assert set(want) <= set(ids[b, 0].tolist()), (b, want, ids[b, 0])
    return ids


@pytest.mark.parametrize("flags", [2, 3, 0])
def test_layer_mean_routing_matches_oracle(msa, flags):
    lens = np.full(300, 640)
    lens[::7] = 70
    db = DeviceBank(msa, 31, lens, 3)
    targets = [random_docs(31, 300, 4, sub=b).tolist() for b in range(2)]
    _check(msa, db, targets, 48, 8, flags)


def test_layer_mean_short_query_stays_on_the_tensor_path(msa):
    lens = np.full(120, 256)
    db = DeviceBank(msa, 32, lens, 2)
    ids = _check(msa, db, [random_docs(32, 120, 2).tolist()], 4, 4, 0)
    assert ids.shape == (1, 2, 4)


def test_layer_mean_noise_queries_take_the_second_pass(msa):
    # no planted topic: the E4M3 filter cannot certify the boundary, the call filters every
    # layer again with bf16 operands and the selection is still the exact one
    lens = np.full(200, 320)
    db = DeviceBank(msa, 33, lens, 2)
    _check(msa, db, [[-1], [-1]], 32, 6, 3, q_seed=99)
