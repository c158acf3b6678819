"""Query-serving plumbing over the four C-ABI steps (device buffers, streams, graphs).

``SparseMemory`` holds a resident bank (unit routing keys in HBM, content K/V in a
page-locked host store) plus the buffers of ``slots`` queries in flight, and runs each
query as

    route + top-k  ->  gather of the selected documents  ->  n decode steps

Each slot is captured as two CUDA graphs: the route, and the tail (gather + decode).
Routes run back to back on one stream; a query's tail runs on a second stream as soon
as its route is done, so the latency-bound tail of query i overlaps the bandwidth-bound
route of query i+1.  A slot is reused only after its previous tail has finished.
Everything computed runs in the libraries' kernels; this module only allocates,
sequences and moves bytes.
"""
from __future__ import annotations

import numpy as np
import torch

from .abi import (MSA_ROUTE_AUTO, msa_gather_kv, msa_route_topk, msa_route_topk_workspace_size,
                  msa_sparse_decode, msa_sparse_decode_workspace_size)


class _Slot:
    def __init__(self, eng: "SparseMemory"):
        L, H, D, dev = eng.L, eng.H, eng.D, eng.dev
        ws = msa_route_topk_workspace_size(L, 1, eng.T, H, eng.C, eng.n_docs, eng.k)
        self.ws = torch.empty(ws, dtype=torch.uint8, device=dev)
        self.qr = torch.zeros((L, eng.T, eng.Hq, D), dtype=torch.bfloat16, device=dev)
        self.ids = torch.empty((1, L, eng.k), dtype=torch.int32, device=dev)
        self.scores = torch.empty((1, L, eng.k), dtype=torch.float32, device=dev)
        self.mem_kv = torch.zeros((1, L, 2, H, eng.M, D), dtype=torch.bfloat16, device=dev)
        self.mem_len = torch.zeros((1, L), dtype=torch.int32, device=dev)
        self.local_k = torch.zeros((1, L, H, eng.cap, D), dtype=torch.bfloat16, device=dev)
        self.local_v = torch.zeros_like(self.local_k)
        self.local_len = torch.zeros(1, dtype=torch.int32, device=dev)
        self.local_len0 = torch.zeros(1, dtype=torch.int32, device=dev)
        self.dev_err = torch.zeros(1, dtype=torch.int32, device=dev)
        self.dec_ws = torch.zeros(msa_sparse_decode_workspace_size(1, L, eng.Hq, H), dtype=torch.uint8, device=dev)
        self.route_graph = None
        self.tail_graph = None
        self.route_done = torch.cuda.Event(enable_timing=True)
        self.tail_done = torch.cuda.Event(enable_timing=True)
        self.route_start = torch.cuda.Event(enable_timing=True)
        self.used = False


class SparseMemory:
    def __init__(self, kr_hat: torch.Tensor, doc_chunk_offsets: np.ndarray, host_kv: torch.Tensor,
                 doc_store_offsets: np.ndarray | None = None, *, n_q_heads: int = 32, top_k: int = 16,
                 query_tokens: int = 256, local_cap: int = 384, rope_theta: float = 1e6,
                 max_mem_chunks: int | None = None, route_flags: int = MSA_ROUTE_AUTO, slots: int = 2,
                 kr_f8: torch.Tensor | None = None):
        """kr_f8: optional E4M3 filter copy of kr_hat (msa_route_filter_keys); with the
        default route flags, routes of long queries then filter on it."""
        assert kr_hat.is_cuda and kr_hat.dtype == torch.bfloat16 and kr_hat.dim() == 4
        assert kr_f8 is None or (kr_f8.is_cuda and kr_f8.dtype == torch.uint8 and kr_f8.shape == kr_hat.shape)
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
        self.kr_f8 = kr_f8
        offs = np.ascontiguousarray(doc_chunk_offsets, dtype=np.int64)
        self.n_docs = len(offs) - 1
        self.doc_chunk_offsets = torch.from_numpy(offs).to(dev)
        self.max_doc_chunks = int(np.diff(offs).max()) if self.n_docs else 0
        self.M = max_mem_chunks or max(1, top_k * self.max_doc_chunks)
        self.host_kv = host_kv
        self.n_store = host_kv.shape[1]
        self.doc_store_offsets = (None if doc_store_offsets is None else
                                  torch.from_numpy(np.ascontiguousarray(doc_store_offsets, dtype=np.int64)).to(dev))
        self.slots = [_Slot(self) for _ in range(slots)]
        self.route_stream = torch.cuda.Stream(device=dev)
        self.tail_stream = torch.cuda.Stream(device=dev)
        self.launches_per_query = 0

    # ------------------------------------------------------------------ enqueueing
    def set_local_prefix(self, k_prefix: torch.Tensor, v_prefix: torch.Tensor) -> None:
        """The query's own (already rotated) local K/V, [L][H][n][D]; decode appends after it."""
        n = k_prefix.shape[2]
        for s in self.slots:
            s.local_k[0, :, :, :n].copy_(k_prefix)
            s.local_v[0, :, :, :n].copy_(v_prefix)
            s.local_len0.fill_(n)

    def enqueue_route(self, slot: _Slot, stream) -> int:
        return msa_route_topk(slot.qr, [0, self.T], self.kr_hat, self.doc_chunk_offsets, self.n_docs, self.C,
                              self.L, self.Hq, self.H, self.D, self.k, slot.ids, slot.scores, slot.ws,
                              flags=self.flags, dev_err=slot.dev_err, stream=stream, kr_f8=self.kr_f8)

    def enqueue_tail(self, slot: _Slot, dec_q, dec_k, dec_v, out, stream) -> int:
        """Gather of slot's selection, then one decode step per row of dec_q [S][1][L][Hq][D]
        (dec_k/dec_v [S][1][L][H][D]) into out [S][1][L][Hq][D]."""
        msa_gather_kv(self.host_kv, self.n_store, self.doc_chunk_offsets, self.doc_store_offsets, self.n_docs,
                      slot.ids, 1, self.L, self.k, self.H, self.D, self.M, slot.mem_kv, slot.mem_len,
                      dev_err=slot.dev_err, stream=stream)
        with torch.cuda.stream(stream):
            slot.local_len.copy_(slot.local_len0)
        n = 1
        for s in range(dec_q.shape[0]):
            msa_sparse_decode(dec_q[s], dec_k[s], dec_v[s], 1, self.L, self.Hq, self.H, self.D, slot.local_k,
                              slot.local_v, slot.local_len, self.cap, slot.mem_kv, slot.mem_len, self.M, self.k,
                              self.theta, self.D ** -0.5, out[s], slot.dec_ws, dev_err=slot.dev_err, stream=stream)
            n += 1
        return n

    def capture(self, dec_inputs) -> None:
        """Captures every slot's route and tail as CUDA graphs.  dec_inputs: one
        (dec_q, dec_k, dec_v, out) tuple of static buffers per slot."""
        for slot, (dec_q, dec_k, dec_v, out) in zip(self.slots, dec_inputs):
            with torch.cuda.stream(self.route_stream):  # warm-up outside capture
                self.enqueue_route(slot, self.route_stream)
                self.enqueue_tail(slot, dec_q, dec_k, dec_v, out, self.route_stream)
            torch.cuda.synchronize(self.dev)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=self.route_stream):
                n = self.enqueue_route(slot, self.route_stream)
            slot.route_graph = g
            g2 = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g2, stream=self.tail_stream):
                n += self.enqueue_tail(slot, dec_q, dec_k, dec_v, out, self.tail_stream)
            slot.tail_graph = g2
            self.launches_per_query = n
        torch.cuda.synchronize(self.dev)

    # ------------------------------------------------------------------ running
    def launch(self, i: int, load=None, unload=None) -> _Slot:
        """Query i on slot i % slots: route on the route stream (after the slot's previous
        tail), tail on the tail stream (after this route).  load(slot, stream) copies the
        query's inputs into the slot on the route stream first; unload(slot, stream) reads
        results back on the tail stream after the tail."""
        slot = self.slots[i % len(self.slots)]
        rs, ts = self.route_stream, self.tail_stream
        if slot.used:
            rs.wait_event(slot.tail_done)
        slot.route_start.record(rs)
        with torch.cuda.stream(rs):
            if load is not None:
                load(slot, rs)
            slot.route_graph.replay()
        slot.route_done.record(rs)
        ts.wait_event(slot.route_done)
        with torch.cuda.stream(ts):
            slot.tail_graph.replay()
            if unload is not None:
                unload(slot, ts)
        slot.tail_done.record(ts)
        slot.used = True
        return slot

    def drain(self) -> None:
        torch.cuda.current_stream(self.dev).wait_stream(self.route_stream)
        torch.cuda.current_stream(self.dev).wait_stream(self.tail_stream)
