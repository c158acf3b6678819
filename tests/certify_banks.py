"""Routing banks built to sit on the tensor-core filter's rounding, for the certification
tests.  Every document is one block whose eight key heads are the bf16 rounding (nearest)
of a unit vector, as the pool step stores them; the query's 32 heads all point along
coordinate 0, so that

    exact score  S(d) = mean over key heads g of k_g[0] / ||k_g||
    bf16 filter  F(d) = mean over g of k_g[0]                  (the unnormalised stored key)
    E4M3 filter  F8(d) = mean over g of e4m3(256 k_g[0] / ||k_g||) / 256

and every rounding step of the filter is known exactly.  The banks make the filter order
disagree with the exact order by more than the earlier empirical error margins (1e-3 for
bf16 operands, 2^-6 for E4M3) while those margins would still have certified the wrong
selection, or put more near-ties inside the filter's error than any candidate list holds.
Plain numpy, seeded; no method arithmetic beyond these definitions.
"""
from __future__ import annotations

import numpy as np

import msa_synth as syn
from tests.helpers import e4m3

H, HQ, D = 8, 32, 128
K = 16


def bf16(x) -> np.ndarray:
    """Nearest-even bf16 rounding of float values, as float64."""
    return syn.bf16_bits_to_f32(syn.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))).astype(np.float64)


def _stored(y) -> np.ndarray:
    k = bf16(y)
    return k


def head_structured(c: float, n: int, t: float, direction: int) -> np.ndarray:
    """A stored key head: coordinate 0 = c (bf16-exact), n coordinates placed just past a
    bf16 rounding midpoint of t (direction -1: they round down, +1: up, 0: exactly t) and
    one coordinate closing the unit norm of the unrounded vector."""
    y = np.zeros(D)
    y[0] = c
    eps = 2.0 ** -14
    v = t * (1 + 2.0 ** -8 + direction * eps) if direction else t
    y[1:1 + n] = v
    rest = 1.0 - c * c - n * v * v
    assert rest > 0
    y[1 + n] = np.sqrt(rest)
    k = _stored(y)
    assert k[0] == c
    return k


def head_searched(c: float, dev_lo: float, dev_hi: float, rng, n: int = 12, tries: int = 200_000) -> np.ndarray:
    """A stored key head with coordinate 0 = c (bf16-exact) and ||k|| - 1 in [dev_lo, dev_hi]:
    random n-coordinate tails of the unit vector are drawn until the rounding lands there."""
    for _ in range(tries):
        y = np.zeros(D)
        y[0] = c
        tail = rng.standard_normal(n)
        y[1:1 + n] = tail / np.linalg.norm(tail) * np.sqrt(1.0 - c * c)
        k = _stored(y)
        dev = np.linalg.norm(k) - 1.0
        if k[0] == c and dev_lo <= dev <= dev_hi:
            return k
    raise RuntimeError("no tail found")


def stack(docs) -> np.ndarray:
    """docs: list of per-document head lists (8 heads each) -> keys [C][H][D] float32."""
    return np.asarray(docs, dtype=np.float32)


def e0_query(T: int = 1) -> np.ndarray:
    """[T][Hq][d] float32: every query head along coordinate 0."""
    q = np.zeros((T, HQ, D), dtype=np.float32)
    q[:, :, 0] = 1.0
    return q


def model_scores(keys: np.ndarray):
    """(S, F_bf16, F_e4m3) of every document for the e0 query, from the definitions above
    (float64; the E4M3 key uses the fp64 norm, which differs from the kernel's fp32 one by
    far less than a rounding step in these banks)."""
    k = keys.astype(np.float64)
    n = np.linalg.norm(k, axis=2)
    S = (k[:, :, 0] / n).mean(axis=1)
    F = k[:, :, 0].mean(axis=1)
    F8 = (e4m3(256.0 * k[:, :, 0] / n) / 256.0).mean(axis=1)
    return S, F, F8


def old_rule_outcome(S, F, k: int = K, k2: int = 48, margin: float = 1e-3):
    """What a selection certified with a fixed margin would return: the k2 best documents
    by filter score (equal scores: smaller id), their top k by exact score, and whether the
    fixed margin certified it (k-th exact > k2-th filter + margin)."""
    order = sorted(range(len(F)), key=lambda d: (-F[d], d))
    cand = order[:k2]
    best = sorted(cand, key=lambda d: (-S[d], d))[:k]
    certified = S[best[-1]] > F[cand[-1]] + margin
    return best, certified


def bank_e4m3_trap():
    """49 documents.  E4M3 filter: every document rounds to 144/256.  32 fillers (exact
    ~0.547), 16 decoys (~0.582-0.586) and, with the highest id, the true best document X
    (~0.590): the 48 candidates are fillers and decoys, the 16th exact score among them beats
    the 48th filter score by more than 2^-6, yet X belongs first in the top-16."""
    fill = head_structured(140 / 256, 10, 0.25, 0)
    docs = [[fill] * H for _ in range(32)]
    for c in [149 / 256] * 8 + [150 / 256] * 8:
        docs.append([head_structured(c, 10, 0.25, 0)] * H)
    docs.append([head_structured(151 / 256, 10, 0.25, 0)] * H)
    return stack(docs)


def bank_bf16_trap(seed: int = 7):
    """49 documents.  bf16 filter: X (highest id) has coordinate 0 = 0.5 in every head and
    key norms ~0.9974 (its tail rounds down), so F(X) = 0.5 < S(X) ~ 0.50132; 32 fillers have
    F = 0.5 (lower ids, exact below 0.5); 16 decoys have F ~ 0.50098 and exact scores in
    (0.501, S(X) - 1e-4).  The 48 candidates are fillers and decoys, and the 16th exact score
    beats the 48th filter score by more than 1e-3, yet X belongs first."""
    rng = np.random.default_rng(seed)
    x_head = head_structured(0.5, 11, 0.25, -1)
    fill_head = head_structured(0.5, 11, 0.25, +1)
    docs = [[fill_head] * H for _ in range(32)]
    hi = head_structured(0.50390625, 11, 0.25, 0)
    for _ in range(16):
        lo = head_searched(0.5, -5e-4, -4e-4, rng)
        docs.append([hi, hi] + [lo] * 6)
    docs.append([x_head] * H)
    return stack(docs)


def bank_crowd(n_crowd: int, seed: int = 11):
    """n_crowd + 16 documents whose coordinate 0 is the same bf16 value 0.2353515625 in every
    head.  The crowd (lower ids) has key norms within 2e-4 of 1; the last 16 documents have
    norms ~0.9964 (tails rounding down), so their exact scores are ~8e-4 above the crowd's
    while every filter score (bf16 and E4M3) is identical.  With more crowd documents than
    any candidate list, only the exact scan finds the last 16."""
    rng = np.random.default_rng(seed)
    c = 0.2353515625
    top = head_structured(c, 14, 0.25, -1)
    crowd = [head_searched(c, -2e-4, 2e-4, rng) for _ in range(64)]
    docs = [[crowd[(i + j) % 64] for j in range(H)] for i in range(n_crowd)]
    docs += [[top] * H for _ in range(K)]
    return stack(docs)
