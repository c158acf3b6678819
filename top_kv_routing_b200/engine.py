"""Query-serving plumbing over the four C-ABI steps (device buffers, streams, graphs).

``SparseMemory`` holds a resident bank (unit routing keys in HBM, content K/V in a
page-locked host store) plus every buffer one query needs, and runs

    route + top-k  ->  gather of the selected documents (side stream)  ->  n decode steps

as enqueued work on the current stream, optionally captured once as a CUDA graph and
replayed.  Everything computed runs in the libraries' kernels; this module only
allocates, sequences and moves bytes.
"""
from __future__ import annotations

import numpy as np
import torch

from .abi import (MSA_ROUTE_AUTO, msa_gather_kv, msa_route_topk, msa_route_topk_workspace_size,
                  msa_sparse_decode, msa_sparse_decode_workspace_size)


class SparseMemory:
    def __init__(self, kr_hat: torch.Tensor, doc_chunk_offsets: np.ndarray, host_kv: torch.Tensor,
                 doc_store_offsets: np.ndarray | None = None, *, n_q_heads: int = 32, top_k: int = 16,
                 query_tokens: int = 256, local_cap: int = 384, rope_theta: float = 1e6,
                 max_mem_chunks: int | None = None, route_flags: int = MSA_ROUTE_AUTO):
        assert kr_hat.is_cuda and kr_hat.dtype == torch.bfloat16 and kr_hat.dim() == 4
        assert host_kv.is_pinned() and host_kv.dim() == 5 and host_kv.shape[2] == 2
        dev = kr_hat.device
        self.dev = dev
        self.L, self.C, self.H, self.D = kr_hat.shape
        self.Hq = n_q_heads
        self.k = top_k
        self.T = query_tokens
        self.cap = local_cap
        self.theta = rope_theta
        self.flags = route_flags
        self.kr_hat = kr_hat
        offs = np.ascontiguousarray(doc_chunk_offsets, dtype=np.int64)
        self.n_docs = len(offs) - 1
        self.doc_chunk_offsets = torch.from_numpy(offs).to(dev)
        self.max_doc_chunks = int(np.diff(offs).max()) if self.n_docs else 0
        self.M = max_mem_chunks or max(1, top_k * self.max_doc_chunks)
        self.host_kv = host_kv
        self.n_store = host_kv.shape[1]
        self.doc_store_offsets = (None if doc_store_offsets is None else
                                  torch.from_numpy(np.ascontiguousarray(doc_store_offsets, dtype=np.int64)).to(dev))
        L, H, D = self.L, self.H, self.D
        ws = msa_route_topk_workspace_size(L, 1, self.T, H, self.C, self.n_docs, top_k)
        self.ws = torch.empty(ws, dtype=torch.uint8, device=dev)
        self.qr = torch.zeros((L, self.T, n_q_heads, D), dtype=torch.bfloat16, device=dev)
        self.ids = torch.empty((1, L, top_k), dtype=torch.int32, device=dev)
        self.scores = torch.empty((1, L, top_k), dtype=torch.float32, device=dev)
        self.mem_kv = torch.zeros((1, L, 2, H, self.M, D), dtype=torch.bfloat16, device=dev)
        self.mem_len = torch.zeros((1, L), dtype=torch.int32, device=dev)
        self.local_k = torch.zeros((1, L, H, local_cap, D), dtype=torch.bfloat16, device=dev)
        self.local_v = torch.zeros_like(self.local_k)
        self.local_len = torch.zeros(1, dtype=torch.int32, device=dev)
        self.local_len0 = torch.zeros(1, dtype=torch.int32, device=dev)
        self.dev_err = torch.zeros(1, dtype=torch.int32, device=dev)
        self.dec_ws = torch.zeros(msa_sparse_decode_workspace_size(1, L, n_q_heads, H), dtype=torch.uint8, device=dev)
        self.side = torch.cuda.Stream(device=dev)
        self.routed = torch.cuda.Event()
        self.gathered = torch.cuda.Event()
        self.graph = None
        self.launches_per_query = 0

    def set_local_prefix(self, k_prefix: torch.Tensor, v_prefix: torch.Tensor) -> None:
        """The query's own (already rotated) local K/V, [L][H][n][D]; decode appends after it."""
        n = k_prefix.shape[2]
        self.local_k[0, :, :, :n].copy_(k_prefix)
        self.local_v[0, :, :, :n].copy_(v_prefix)
        self.local_len0.fill_(n)

    def enqueue(self, dec_q: torch.Tensor, dec_k: torch.Tensor, dec_v: torch.Tensor,
                out: torch.Tensor) -> int:
        """Enqueues one query: route self.qr, gather on the side stream, then one decode step
        per row of dec_q [S][1][L][Hq][D] (dec_k/dec_v [S][1][L][H][D]) into out
        [S][1][L][Hq][D].  Returns the number of library kernels enqueued."""
        cur = torch.cuda.current_stream(self.dev)
        n = msa_route_topk(self.qr, [0, self.T], self.kr_hat, self.doc_chunk_offsets, self.n_docs, self.C, self.L,
                           self.Hq, self.H, self.D, self.k, self.ids, self.scores, self.ws, flags=self.flags,
                           dev_err=self.dev_err, stream=cur)
        self.routed.record(cur)
        self.side.wait_event(self.routed)
        msa_gather_kv(self.host_kv, self.n_store, self.doc_chunk_offsets, self.doc_store_offsets, self.n_docs,
                      self.ids, 1, self.L, self.k, self.H, self.D, self.M, self.mem_kv, self.mem_len,
                      dev_err=self.dev_err, stream=self.side)
        n += 1
        self.gathered.record(self.side)
        self.local_len.copy_(self.local_len0)
        cur.wait_event(self.gathered)
        for s in range(dec_q.shape[0]):
            msa_sparse_decode(dec_q[s], dec_k[s], dec_v[s], 1, self.L, self.Hq, self.H, self.D, self.local_k,
                              self.local_v, self.local_len, self.cap, self.mem_kv, self.mem_len, self.M, self.k,
                              self.theta, self.D ** -0.5, out[s], self.dec_ws, dev_err=self.dev_err, stream=cur)
            n += 1
        self.launches_per_query = n
        return n

    def capture(self, dec_q, dec_k, dec_v, out) -> torch.cuda.CUDAGraph:
        """Captures enqueue(...) on these static buffers as one CUDA graph."""
        self.enqueue(dec_q, dec_k, dec_v, out)  # warm-up outside capture (attributes, lazy init)
        torch.cuda.synchronize(self.dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.enqueue(dec_q, dec_k, dec_v, out)
        self.graph = g
        return g
