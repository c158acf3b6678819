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
    assert len(set(x for x in gpu_ids if x >= 0)) == sum(1 for x in gpu_ids if x >= 0)


def rel_l2(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))
