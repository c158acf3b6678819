"""CPU checks of the certification test banks (tests/certify_banks.py) against the oracle:
each bank does what its GPU test relies on.  A fixed error margin (1e-3 for bf16 operands,
2^-6 for E4M3, the margins routing once certified with) certifies a selection that the
oracle's exact scores refute, while the bound derived from the operands' rounding does not
certify it; the crowd banks hold more near-ties inside the filter's error than the
candidate lists."""
import numpy as np

import oracle
from tests import certify_banks as cb

U_E4M3, KEY_DEV = 2.0 ** -4, 2.0 ** -8 + 2.0 ** -19


def _oracle_top(keys):
    ids, sc, ds, _ = oracle.route(cb.e0_query(1), keys, np.arange(len(keys) + 1), cb.K, grouped=True)
    return [int(i) for i in ids], sc, ds


def _unit_rounded(keys):
    # every head is the bf16 rounding of a unit vector: its norm is within 2^-8 of 1
    n = np.linalg.norm(keys.astype(np.float64), axis=2)
    assert np.all(np.abs(n - 1) <= KEY_DEV)


def test_model_scores_match_the_oracle():
    for keys in (cb.bank_e4m3_trap(), cb.bank_bf16_trap(), cb.bank_crowd(30)):
        S, _, _ = cb.model_scores(keys)
        _, _, ds = _oracle_top(keys)
        assert np.abs(S - ds).max() < 1e-12


def test_e4m3_trap_defeats_the_fixed_margin():
    keys = cb.bank_e4m3_trap()
    _unit_rounded(keys)
    S, F, F8 = cb.model_scores(keys)
    top, sc, _ = _oracle_top(keys)
    assert top[0] == len(keys) - 1 and sc[0] - sc[1] >= 1e-4       # X first, clear of the rest
    assert np.all(F8 == F8[0])                                      # the E4M3 filter sees one value
    best, certified = cb.old_rule_outcome(S, F8, margin=2.0 ** -6)
    assert certified and len(keys) - 1 not in best                  # fixed margin: wrong, certified
    # the derived bound for this query is at least u8 * sum_g ||q_g|| = 2^-4 (the e0 query's
    # group sums have norm 1/8 each): the 16th exact score is not that far above the 48th filter score
    s_kth = sorted(S[best])[0]
    assert not (s_kth > F8[47] + U_E4M3)
    # the bf16 filter puts X among its 48 candidates and certifies with its bound
    best2, _ = cb.old_rule_outcome(S, F, margin=0.0)
    assert set(best2) == set(top)


def test_bf16_trap_defeats_the_fixed_margin():
    keys = cb.bank_bf16_trap()
    _unit_rounded(keys)
    S, F, _ = cb.model_scores(keys)
    top, sc, _ = _oracle_top(keys)
    assert top[0] == len(keys) - 1 and sc[0] - sc[1] >= 1e-4
    best, certified = cb.old_rule_outcome(S, F, margin=1e-3)
    assert certified and len(keys) - 1 not in best
    order = sorted(range(len(F)), key=lambda d: (-F[d], d))
    s_kth = sorted(S[best])[0]
    assert not (s_kth > F[order[47]] + KEY_DEV)                      # the derived bound does not certify


def test_crowd_banks_hide_the_top_documents_behind_equal_filter_scores():
    for n in (100, 1100):
        keys = cb.bank_crowd(n)
        _unit_rounded(keys)
        S, F, F8 = cb.model_scores(keys)
        top, sc, _ = _oracle_top(keys)
        assert sorted(top) == list(range(n, n + cb.K))               # the last 16 documents
        assert sc[cb.K - 1] - np.sort(S)[::-1][cb.K] >= 4e-4          # clear of the crowd
        assert np.all(F == F[0]) and np.all(F8 == F8[0])              # both filters see one value
        assert S.max() - S.min() < KEY_DEV                            # all within the bf16 bound
