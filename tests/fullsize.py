"""Test-side plumbing for the full-size configurations: device banks built the way the
benchmark builds them, host copies of selected documents for the oracle, and the sampled
parity rules.  No method arithmetic here beyond calls into the oracle and the product."""
from __future__ import annotations

import numpy as np
import torch

import msa_synth as syn
import oracle
from tests.helpers import GAP_TOL, SCORE_TOL, check_topk

H, HQ, D = 8, 32, 128
THETA = 1e6


class DeviceBank:
    """Pooled-level routing keys of every layer on the device, made unit per head by the
    pool kernel (1-token blocks, no rotation), plus the E4M3 filter copy."""

    def __init__(self, msa, seed: int, lens, L: int, f8: bool = True):
        self.msa = msa
        self.seed, self.L = seed, L
        self.bank = syn.make_bank(seed, len(lens), lens, L)
        self.C = self.bank.n_chunks
        self.n_docs = len(lens)
        self.coffs = self.bank.doc_chunk_offsets
        self.d_coffs = torch.from_numpy(self.coffs).cuda()
        self.topic = torch.from_numpy(self.bank.topic).cuda()
        C = self.C
        self.kr_hat = torch.empty((L, C, H, D), dtype=torch.bfloat16, device="cuda")
        scratch = torch.empty((C, H, D), dtype=torch.bfloat16, device="cuda")
        row_topic = torch.from_numpy(syn.chunk_docs(self.coffs)).cuda()
        ones = torch.arange(C + 1, dtype=torch.int64, device="cuda")
        for l in range(L):
            syn.device_fill(scratch, seed, syn.STREAM_KRBAR, l, 0, 0, C, H * D, syn.POOLED_NOISE, self.topic,
                            row_topic)
            msa.msa_pool_blocks(None, None, scratch, ones, ones, C, C, H, D, 1, 0.0, None, None, self.kr_hat[l], None,
                                None, in_dtype=msa.MSA_BF16)
        del scratch, row_topic, ones
        self.kr_f8 = None
        if f8:
            self.kr_f8 = torch.empty((L, C, H, D), dtype=torch.uint8, device="cuda")
            msa.msa_route_filter_keys(self.kr_hat, L, C, H, D, self.kr_f8)
        torch.cuda.synchronize()

    def queries(self, n_queries: int, T: int, targets_of, dtype=torch.float32, q_seed=None):
        """Planted router queries [L][n_queries * T][Hq][d] on the device: token t of query b
        carries the topic of targets_of(b)[t mod n] (same draw as msa_synth.query_router)."""
        q = torch.empty((self.L, n_queries * T, HQ, D), dtype=dtype, device="cuda")
        for b in range(n_queries):
            self.fill_segment(q[:, b * T:(b + 1) * T], b, 0, targets_of(b), q_seed)
        return q

    def fill_segment(self, dst, sub: int, tok0: int, targets, q_seed=None):
        """dst [L][n][Hq][d]: tokens tok0 .. tok0+n of router-query stream `sub`, token
        tok0 + t carrying the topic of targets[t mod len(targets)]."""
        n = dst.shape[1]
        tg = np.asarray(targets, dtype=np.int64)
        rt = torch.from_numpy(np.repeat(tg[np.arange(n) % len(tg)], HQ).astype(np.int32)).cuda()
        seed = self.seed if q_seed is None else q_seed
        for l in range(self.L):
            syn.device_fill(dst[l], seed, syn.STREAM_QR, l, sub, tok0 * HQ, n * HQ, D, 0.5, self.topic, rt)

    def route(self, qr, q_offsets, k: int, flags: int, ws=None):
        msa = self.msa
        B = len(q_offsets) - 1
        T = int(q_offsets[-1])
        if ws is None:
            ws = torch.empty(msa.msa_route_topk_workspace_size(self.L, B, T, H, self.C, self.n_docs, k),
                             dtype=torch.uint8, device="cuda")
        ids = torch.full((B, self.L, k), -7, dtype=torch.int32, device="cuda")
        sc = torch.full((B, self.L, k), float("nan"), device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        msa.msa_route_topk(qr, q_offsets, self.kr_hat, self.d_coffs, self.n_docs, self.C, self.L, HQ, H, D, k, ids,
                           sc, ws, flags=flags, dev_err=err,
                           kr_f8=self.kr_f8 if (flags & ~msa.MSA_ROUTE_LAYER_MEAN) in (msa.MSA_ROUTE_AUTO,
                                                                                       msa.MSA_ROUTE_TENSOR_F8)
                           else None)
        torch.cuda.synchronize()
        return ids.cpu().numpy(), sc.cpu().numpy(), int(err.item())


def host_doc_keys(bank, layer: int, docs):
    """Routing keys of the given documents on the host, in the oracle's hands: the same
    generator draw as the device, made unit per head by the oracle (1-token blocks) and
    rounded to bf16.  Returns (keys [n][H][d] float32, block offsets [len(docs)+1])."""
    coffs = bank.doc_chunk_offsets
    parts, offs = [], [0]
    for d in docs:
        c0, c1 = int(coffs[d]), int(coffs[d + 1])
        n = c1 - c0
        if n == 0:
            offs.append(offs[-1])
            continue
        raw = syn.fill(bank.seed, syn.STREAM_KRBAR, layer, 0, c0, n, H * D, sigma=syn.POOLED_NOISE,
                       topic=bank.topic, row_topic=np.full(n, d), dtype="bf16")
        unit = oracle.pool(None, None, syn.bf16_bits_to_f32(raw).reshape(n, H, D), np.arange(n + 1), H, D, 1, THETA,
                           rope_k=False)["kr_unit"]
        parts.append(syn.bf16_bits_to_f32(syn.f32_to_bf16_bits(unit.astype(np.float32))))
        offs.append(offs[-1] + n)
    keys = np.concatenate(parts) if parts else np.zeros((0, H, D), np.float32)
    return keys, np.asarray(offs, dtype=np.int64)


def host_query(bank, layer: int, b: int, T: int, targets, dtype: str = "f32", q_seed=None, tok0: int = 0):
    """The host draw of router-query stream b for one layer (tokens tok0 .. tok0+T),
    [T][Hq][d] float32 (the values of `dtype`)."""
    tg = np.asarray(targets, dtype=np.int64)
    rt = np.repeat(tg[np.arange(T) % len(tg)], HQ)
    x = syn.fill(bank.seed if q_seed is None else q_seed, syn.STREAM_QR, layer, b, tok0 * HQ, T * HQ, D, sigma=0.5,
                 topic=bank.topic, row_topic=rt, dtype=dtype)
    if dtype == "bf16":
        x = syn.bf16_bits_to_f32(x)
    return x.reshape(T, HQ, D)


def oracle_doc_scores(bank, layer: int, q, docs):
    """Exact document scores (oracle, grouped form) of the given documents for query q."""
    docs = sorted(set(int(d) for d in docs))
    keys, offs = host_doc_keys(bank, layer, docs)
    _, _, ds, _ = oracle.route(q, keys, offs, 1, grouped=True)
    return dict(zip(docs, ds.tolist()))


def check_sampled(gpu_ids, gpu_scores, ref: dict, k: int, planted=()):
    """Parity on sampled documents, valid at any bank size: every returned score equals the
    oracle's score of that document (within SCORE_TOL); scores do not increase; ids are
    unique; no sampled document left out beats the k-th returned one by GAP_TOL or more;
    every planted document is returned."""
    ids = [int(x) for x in gpu_ids]
    sel = [d for d in ids if d >= 0]
    assert len(sel) == len(set(sel))
    for r, d in enumerate(ids):
        if d >= 0:
            assert abs(float(gpu_scores[r]) - ref[d]) <= SCORE_TOL, (r, d, gpu_scores[r], ref[d])
    fin = np.asarray(gpu_scores, dtype=np.float64)[:len(sel)]
    assert np.all(np.diff(fin) <= 0)
    if len(sel) == k:
        kth = min(ref[d] for d in sel)
        for d, s in ref.items():
            if d not in sel:
                assert s < kth + GAP_TOL, (d, s, kth)
    assert set(int(p) for p in planted) <= set(sel), (sorted(planted), sel)


def check_full_layer(gpu_ids, gpu_scores, bank, layer, q, k):
    """Full oracle over every document of one layer (sizes the oracle covers in seconds)."""
    keys, offs = host_doc_keys(bank, layer, range(len(bank.lengths)))
    _, _, ds, _ = oracle.route(q, keys, offs, k, grouped=True)
    check_topk(gpu_ids, gpu_scores, ds, k)
    return ds


def random_docs(seed: int, n_docs: int, n: int, sub: int = 0):
    """n distinct document ids by the generator's hash (not the method's)."""
    return syn.pick_targets(seed + 1000, n_docs, min(n, n_docs), sub=sub + 500)


def host_store(seed: int, L: int, P: int):
    """Page-locked content store [L][P][2][H][d] bf16 drawn on the device (generator only)
    and copied to the host, the benchmark's construction.  Returns (pinned tensor, numpy
    uint16 view)."""
    store = torch.empty((L, P, 2, H, D), dtype=torch.bfloat16, pin_memory=True)
    stage = torch.empty((2, P, H * D), dtype=torch.bfloat16, device="cuda")
    for l in range(L):
        syn.device_fill(stage[0], seed, syn.STREAM_KBAR, l, 0, 0, P, H * D, syn.POOLED_NOISE)
        syn.device_fill(stage[1], seed, syn.STREAM_VBAR, l, 0, 0, P, H * D, syn.POOLED_NOISE)
        store[l].copy_(stage.permute(1, 0, 2).reshape(P, 2, H, D))
    del stage
    torch.cuda.synchronize()
    return store, store.view(torch.int16).numpy().view(np.uint16)


def oracle_gather_layer(store_np, layer: int, doc_chunk_offsets, store_off, ids_row, M_max: int):
    """The oracle's gather of one (query, layer) selection: the selected documents' store
    rows (first block store_off[d], or the block offset when store_off is None) as a small
    store of their own, gathered in rank order.  Returns (mem [2][H][M_max][d] float32, len)."""
    rows, offs, sel = [], [0], []
    for d in ids_row:
        d = int(d)
        if d < 0:
            sel.append(-1)
            continue
        n = int(doc_chunk_offsets[d + 1] - doc_chunk_offsets[d])
        s0 = int(doc_chunk_offsets[d] if store_off is None else store_off[d])
        rows.append(store_np[layer, s0:s0 + n])
        sel.append(len(offs) - 1)
        offs.append(offs[-1] + n)
    mini = np.concatenate(rows)[None] if rows else np.zeros((1, 0, 2, H, D), np.uint16)
    out, mlen = oracle.gather(mini, np.asarray(offs, np.int64), np.asarray(sel, np.int32)[None, None], M_max)
    return syn.bf16_bits_to_f32(out[0, 0]), int(mlen[0, 0])


def decode_inputs(seed: int, step: int, B: int, L: int, sub: int = 0):
    """bf16 bits of one decode step's q [B][L][Hq][d], k_new and v_new [B][L][H][d]."""
    q = syn.fill(seed, syn.STREAM_DEC_Q, step, sub, 0, B * L * HQ, D, dtype="bf16").reshape(B, L, HQ, D)
    k = syn.fill(seed, syn.STREAM_DEC_K, step, sub, 0, B * L * H, D, dtype="bf16").reshape(B, L, H, D)
    v = syn.fill(seed, syn.STREAM_DEC_V, step, sub, 0, B * L * H, D, dtype="bf16").reshape(B, L, H, D)
    return q, k, v
