"""Test-side helpers: tensor plumbing and the parity rules (no method arithmetic)."""
import numpy as np

import msa_synth as syn

SCORE_TOL = 1e-3        # routing scores, absolute (fp32 accumulate vs fp64 oracle)
GAP_TOL = 1e-4          # ids must agree wherever the oracle's consecutive gap is at least this
POOL_TOL = 1e-2         # pooled bf16 blocks, absolute
DEC_MAX_ABS = 1e-2      # decode output, absolute
DEC_REL_L2 = 5e-3       # decode output, relative L2


def bf16_tensor(bits: np.ndarray, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def bf16_to_np(t) -> np.ndarray:
    """bf16 torch tensor -> float32 numpy (exact)."""
    import torch
    return t.detach().to("cpu").view(torch.int16).numpy().view(np.uint16).astype(np.uint32).__lshift__(16).view(np.float32)


def ordered(doc_scores: np.ndarray, k: int):
    ids = sorted(range(len(doc_scores)), key=lambda i: (-doc_scores[i], i))
    ids = ids[:k + 1]
    sc = [doc_scores[i] for i in ids]
    while len(ids) < k + 1:
        ids.append(-1)
        sc.append(-np.inf)
    return ids, np.array(sc, dtype=np.float64)


def check_topk(gpu_ids, gpu_scores, oracle_doc_scores, k, gap=GAP_TOL, tol=SCORE_TOL):
    """The GPU's first i ids equal the oracle's first i ids (as sets) at every cut i whose
    oracle gap (score i-1 minus score i, position k being the (k+1)-th) is >= gap; every
    GPU score is within tol of the oracle's score for that id; scores are non-increasing."""
    gpu_ids = [int(x) for x in gpu_ids]
    gpu_scores = np.asarray(gpu_scores, dtype=np.float64)
    ref_ids, ref_sc = ordered(np.asarray(oracle_doc_scores, dtype=np.float64), k)
    n_docs = len(oracle_doc_scores)
    for i in range(1, k + 1):
        a, b = ref_sc[i - 1], ref_sc[i]
        g = (a - b) if np.isfinite(a) and np.isfinite(b) else (np.inf if np.isfinite(a) else 0.0)
        if g >= gap:
            assert set(gpu_ids[:i]) == set(ref_ids[:i]), (i, gpu_ids, ref_ids[:k], ref_sc[:k + 1])
    for r, d in enumerate(gpu_ids):
        if d < 0:
            assert r >= n_docs and gpu_scores[r] == -np.inf
            continue
        ref = oracle_doc_scores[d]
        if np.isfinite(ref):
            assert abs(gpu_scores[r] - ref) <= tol, (r, d, gpu_scores[r], ref)
        else:
            assert gpu_scores[r] == -np.inf
    fin = gpu_scores[np.isfinite(gpu_scores)]
    assert np.all(np.diff(fin) <= 0)
    sel = [x for x in gpu_ids if x >= 0]
    assert len(set(sel)) == len(sel)
    # near a tie the cut may fall either way, but only inside the tie: no document left out
    # beats the smallest selected oracle score by GAP_TOL, and every selected document is
    # within GAP_TOL of the oracle's k-th score
    ods = np.asarray(oracle_doc_scores, dtype=np.float64)
    if len(sel) == min(k, n_docs) and sel:
        low = min(ods[d] for d in sel)
        left = np.ones(n_docs, dtype=bool)
        left[sel] = False
        if left.any() and np.isfinite(low):
            assert ods[left].max() < low + gap, (float(ods[left].max()), float(low))
        kth = ref_sc[min(k, n_docs) - 1]
        if np.isfinite(kth):
            assert low > kth - gap, (float(low), float(kth))


# ---------------------------------------------------------------------------- E4M3 format
def e4m3(x) -> np.ndarray:
    """Nearest-even rounding of float64 values to OCP FP8 E4M3 (3 mantissa bits, exponent
    bias 7, subnormal step 2^-9, saturating at +-448), returned as float64.  A codec of the
    number format (the tensor-core filter's operand type), not of the method."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, e = np.frexp(np.where(a > 0, a, 1.0))  # a = m 2^e, m in [0.5, 1)
    step = np.where(a >= 2.0 ** -6, np.ldexp(1.0, e - 1 - 3), 2.0 ** -9)
    q = np.round(a / step) * step  # np.round: half to even
    q = np.minimum(q, 448.0)
    return np.copysign(q, x)


def rel_l2(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))
