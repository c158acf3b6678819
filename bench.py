"""Benchmark of the MSA hot path on the 100M-token bank.

One step = one query through the whole online path: route + top-16 over all 18 routing
layers of a 100M-token bank (1.5625M blocks, routing keys resident in HBM), gather of the
selected documents' compressed K/V from page-locked host memory on a side stream, and 128
decode tokens of 32/8-head GQA attention over [gathered memory ; local KV].  The offline
block pooling of the bank runs once before the timed region (it is also timed on its own
and reported under "pool").

Prints one JSON line.  --impl reference times the CPU oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "bank tokens routed/s + K̄ᵣ scan GB/s vs HBM peak at 100M; p50 route+decode ms"
WORKLOAD = ("100M-token bank (100,000 docs, lognormal lengths rounded to 64, 1,562,500 blocks), "
            "18 routing layers x 8 heads x 128 bf16 unit routing keys in HBM (57.6 GB); "
            "query T=256 tokens with 16 planted target documents, top-16 per layer; gather of the "
            "selected blocks' K/V from a page-locked host store; 128-token GQA 32/8 decode, local KV 256")
N_DOCS, N_TOKENS, L, H, HQ, D, TOPK, T, DEC, SEED = 100_000, 100_000_000, 18, 8, 32, 128, 16, 256, 128, 3
TOKENS_PER_DOC = 1000
THETA = 1e6
# DRAM bytes per (block, layer) of the routing GEMM, read + write, from the ncu captures in
# profiles/ (2M-token bank, same kernels), scaled by blocks; None where not captured yet.
GEMM_TRAFFIC_PER_BLOCK_LAYER = {"bf16": None, "e4m3": 1039.5}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), float(j["bf16_tflops"]), float(j.get("bf16_tflops_sustained", 0)), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while running."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu = gpu_id
        self.proc = None
        self.rows = []
        self.thread = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([x.strip() for x in line.split(",")])

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=2)

    def summary(self):
        sm = [float(r[1]) for r in self.rows if len(r) >= 9 and r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if len(r) >= 9 and r[2].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in self.rows:
            if len(r) < 9:
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() in ("active", "0x1", "1"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(self.rows)}


def smi_id(dev) -> str:
    """nvidia-smi --id for a torch device: its PCI bus id when torch exposes it."""
    import torch
    p = torch.cuda.get_device_properties(dev)
    bus, devno, dom = getattr(p, "pci_bus_id", None), getattr(p, "pci_device_id", None), getattr(p, "pci_domain_id", 0)
    if bus is None or devno is None:
        return str(dev.index or 0)
    return f"{dom:08X}:{bus:02X}:{devno:02X}.0"


# ----------------------------------------------------------------------------- ranks

def rank_env():
    """(world, rank, local rank) from the launcher's environment (1, 0, 0 without one)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init_ranks(backend: str, timeout_s: int = 600):
    """One process per GPU: a process group when there is more than one rank."""
    import datetime

    import torch.distributed as dist
    world, rank, local = rank_env()
    if world > 1:
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return world, rank, local


def max_over_ranks(values, device):
    """Element-wise maximum of a list of floats over all ranks (the list itself with one)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def replica_throughput(units_per_rank: float, world: int, max_ms: float) -> float:
    """Whole-job units per second: every replica's units over the slowest rank's time."""
    return units_per_rank * world / (max_ms / 1e3)


# ----------------------------------------------------------------------------- workload

def set_bank_size(n_docs: int) -> None:
    """Scales the bank (documents x 1000 tokens); the default is the 100M-token bank."""
    global N_DOCS, N_TOKENS
    N_DOCS, N_TOKENS = n_docs, n_docs * TOKENS_PER_DOC


def build_keys(dev, seed: int, bank, f8: bool):
    """Routing keys of every layer on the device: pooled-level draws (topic + noise/8) made
    unit per head by the pool kernel with 1-token blocks (no rotation), plus the E4M3
    filter copy.  Returns (kr_hat, kr_f8 or None, filter-key ms or None, topic)."""
    import torch

    import msa_synth as syn
    import top_kv_routing_b200 as msa
    C = bank.n_chunks
    coffs = bank.doc_chunk_offsets
    topic = torch.from_numpy(bank.topic).to(dev)
    kr_hat = torch.empty((L, C, H, D), dtype=torch.bfloat16, device=dev)
    scratch = torch.empty((C, H, D), dtype=torch.bfloat16, device=dev)
    row_topic = torch.from_numpy(syn.chunk_docs(coffs)).to(dev)
    ones = torch.arange(C + 1, dtype=torch.int64, device=dev)
    for l in range(L):
        syn.device_fill(scratch, seed, syn.STREAM_KRBAR, l, 0, 0, C, H * D, syn.POOLED_NOISE, topic, row_topic)
        msa.msa_pool_blocks(None, None, scratch, ones, ones, C, C, H, D, 1, 0.0, None, None, kr_hat[l], None, None,
                            in_dtype=msa.MSA_BF16)
    del scratch, row_topic, ones
    kr_f8, f8_ms = None, None
    if f8:
        # the E4M3 filter copy of the keys (built once per bank, like the keys themselves)
        kr_f8 = torch.empty((L, C, H, D), dtype=torch.uint8, device=dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        msa.msa_route_filter_keys(kr_hat, L, C, H, D, kr_f8)
        e1.record()
        torch.cuda.synchronize(dev)
        f8_ms = e0.elapsed_time(e1)
    torch.cuda.synchronize(dev)
    return kr_hat, kr_f8, f8_ms, topic


def mem_available_gb() -> float | None:
    """MemAvailable of this host (GB), or None where /proc/meminfo is absent."""
    try:
        with open("/proc/meminfo") as f:
            for line in f:
                if line.startswith("MemAvailable:"):
                    return int(line.split()[1]) * 1024 / 1e9
    except OSError:
        return None
    return None


def host_cores() -> dict:
    try:
        aff = len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        aff = None
    return {"nproc": aff or os.cpu_count(), "cpu_count": os.cpu_count()}


def store_blocks_to_use(requested: int | None, C: int) -> tuple[int, str]:
    """Physical blocks per layer of the page-locked content store: the whole bank (every
    document at its own blocks) when the host has room for it with 24 GB to spare, else a
    smaller store read at hashed per-document offsets (the same bytes move per query)."""
    if requested is not None:
        return min(requested, C), "requested on the command line"
    need = L * C * 2 * H * D * 2 / 1e9
    avail = mem_available_gb()
    if avail is None or avail >= need + 24:
        return C, f"whole bank ({need:.1f} GB; host MemAvailable {avail if avail is None else round(avail, 1)} GB)"
    P = 163_840
    return min(P, C), (f"host MemAvailable {avail:.1f} GB < {need:.1f} GB + 24 GB: {P} blocks per layer at "
                       "hashed document offsets")


def make_workload(dev, host_store_chunks: int | None, f8: bool):
    import torch

    import msa_synth as syn

    t0 = time.time()
    lens = syn.doc_lengths_exact_total(SEED, N_DOCS, N_TOKENS)
    bank = syn.make_bank(SEED, N_DOCS, lens, L)
    C = bank.n_chunks
    coffs = bank.doc_chunk_offsets
    kr_hat, kr_f8, f8_ms, topic = build_keys(dev, SEED, bank, f8)
    log(f"routing keys ready: {C} blocks x {L} layers ({kr_hat.numel() * 2 / 1e9:.1f} GB) in {time.time() - t0:.1f}s")
    if f8_ms is not None:
        log(f"E4M3 filter keys: {kr_f8.numel() / 1e9:.1f} GB in {f8_ms:.1f} ms")
    # content store: P physical blocks per layer; with P < C document d reads the
    # contiguous physical range starting at a hashed offset (same bytes per selection)
    P, why = store_blocks_to_use(host_store_chunks, C)
    per_doc = np.diff(coffs)
    h = syn.hashes(syn.tensor_key(SEED, syn.STREAM_TARGETS, 0, 99), np.arange(N_DOCS, dtype=np.uint64))
    store_off = (h % np.uint64(max(1, P - int(per_doc.max())))).astype(np.int64) if P < C else coffs[:-1].copy()
    t1 = time.time()
    host_kv = torch.empty((L, P, 2, H, D), dtype=torch.bfloat16, pin_memory=True)
    pin_s = time.time() - t1
    stage = torch.empty((2, P, H * D), dtype=torch.bfloat16, device=dev)
    for l in range(L):
        syn.device_fill(stage[0], SEED, syn.STREAM_KBAR, l, 0, 0, P, H * D, syn.POOLED_NOISE)
        syn.device_fill(stage[1], SEED, syn.STREAM_VBAR, l, 0, 0, P, H * D, syn.POOLED_NOISE)
        host_kv[l].copy_(stage.permute(1, 0, 2).reshape(P, 2, H, D))
    del stage
    torch.cuda.empty_cache()
    store = {"blocks_per_layer": int(P), "gb_pinned": round(host_kv.numel() * 2 / 1e9, 1), "choice": why,
             "pin_s": round(pin_s, 1), "fill_s": round(time.time() - t1 - pin_s, 1)}
    log(f"host content store: {P} blocks x {L} layers ({store['gb_pinned']} GB pinned in {pin_s:.1f} s)")
    return bank, kr_hat, kr_f8, f8_ms, host_kv, store_off, topic, store


def make_queries(dev, bank, topic, n_queries: int):
    import torch

    import msa_synth as syn
    qs, targets = [], []
    for b in range(n_queries):
        tg = syn.pick_targets(SEED, N_DOCS, TOPK, sub=b)
        targets.append(tg)
        q = torch.empty((L, T, HQ, D), dtype=torch.bfloat16, device=dev)
        rt = torch.from_numpy(np.repeat(tg[np.arange(T) % TOPK], HQ).astype(np.int32)).to(dev)
        for l in range(L):
            syn.device_fill(q[l], SEED, syn.STREAM_QR, l, b, 0, T * HQ, D, 0.5, topic, rt)
        qs.append(q)
    return qs, targets


def make_decode_inputs(dev):
    import torch

    import msa_synth as syn
    dq = torch.empty((DEC, 1, L, HQ, D), dtype=torch.bfloat16, device=dev)
    dk = torch.empty((DEC, 1, L, H, D), dtype=torch.bfloat16, device=dev)
    dv = torch.empty_like(dk)
    for s in range(DEC):
        syn.device_fill(dq[s], SEED, syn.STREAM_DEC_Q, s, 0, 0, L * HQ, D)
        syn.device_fill(dk[s], SEED, syn.STREAM_DEC_K, s, 0, 0, L * H, D)
        syn.device_fill(dv[s], SEED, syn.STREAM_DEC_V, s, 0, 0, L * H, D)
    pk = torch.empty((L, H, T, D), dtype=torch.bfloat16, device=dev)
    pv = torch.empty_like(pk)
    syn.device_fill(pk, SEED, syn.STREAM_LOCAL_K, 0, 0, 0, L * H * T, D)
    syn.device_fill(pv, SEED, syn.STREAM_LOCAL_V, 0, 0, 0, L * H * T, D)
    return dq, dk, dv, pk, pv


def time_pool(dev):
    """Offline pooling throughput on raw bf16 tokens of a 1M-token bank, one layer."""
    import torch

    import msa_synth as syn
    import top_kv_routing_b200 as msa
    lens = syn.doc_lengths_lognormal(1, 1000)
    bank = syn.make_bank(1, 1000, lens, 1)
    n, C = bank.n_tokens, bank.n_chunks
    x = [torch.empty((n, H, D), dtype=torch.bfloat16, device=dev) for _ in range(3)]
    for i, st in enumerate((syn.STREAM_K, syn.STREAM_V, syn.STREAM_KR)):
        syn.device_fill(x[i], 1, st, 0, 0, 0, n, H * D, 1.0, torch.from_numpy(bank.topic).to(dev) if i == 2 else None,
                        torch.from_numpy(syn.token_docs(bank.doc_tok_offsets)).to(dev) if i == 2 else None)
    toff = torch.from_numpy(bank.doc_tok_offsets).to(dev)
    coff = torch.from_numpy(bank.doc_chunk_offsets).to(dev)
    out = [torch.empty((C, H, D), dtype=torch.bfloat16, device=dev) for _ in range(3)]
    nr = torch.empty((C, H), device=dev)

    def run():
        msa.msa_pool_blocks(x[0], x[1], x[2], toff, coff, 1000, C, H, D, 64, THETA, out[0], out[1], out[2], nr, None)
    for _ in range(3):
        run()
    torch.cuda.synchronize(dev)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 10
    s.record()
    for _ in range(reps):
        run()
    e.record()
    torch.cuda.synchronize(dev)
    ms = s.elapsed_time(e) / reps
    by = n * 3 * H * D * 2 + C * (3 * H * D * 2 + H * 4)
    hbm = measured_peaks()[0]
    return {"tokens": n, "blocks": C, "ms": round(ms, 4), "gbs": round(by / ms / 1e6, 1),
            "hbm_frac": round(by / ms / 1e6 / hbm, 4), "bytes_per_token": round(by / n, 1)}


PREFILL_MEM = 256  # gathered memory rows per (query, layer): 16 documents of about 16 blocks


def prefill_flops(n_layers: int, n_q_heads: int, T: int, M: int, prefix: int = 0) -> float:
    """Algorithmic FLOPs of one prefill block: token i of each (layer, query head) scores
    and weighs M + prefix + i + 1 keys, 2 d FLOPs each for QK^T and for PV."""
    keys = T * (M + prefix) + T * (T + 1) / 2
    return 4.0 * D * n_layers * n_q_heads * keys


def time_prefill(dev):
    """The query's own T tokens through sparse attention over 16 gathered documents: one
    query, every layer, no earlier local rows.  L2 is flushed before every timed launch."""
    import torch

    import msa_synth as syn
    import top_kv_routing_b200 as msa
    M = PREFILL_MEM
    q = torch.empty((1, L, T, HQ, D), dtype=torch.bfloat16, device=dev)
    kn = torch.empty((1, L, T, H, D), dtype=torch.bfloat16, device=dev)
    vn = torch.empty_like(kn)
    syn.device_fill(q, SEED, syn.STREAM_DEC_Q, 0, 1, 0, L * T * HQ, D)
    syn.device_fill(kn, SEED, syn.STREAM_DEC_K, 0, 1, 0, L * T * H, D)
    syn.device_fill(vn, SEED, syn.STREAM_DEC_V, 0, 1, 0, L * T * H, D)
    mem = torch.empty((1, L, 2, H, M, D), dtype=torch.bfloat16, device=dev)
    syn.device_fill(mem, SEED, syn.STREAM_KBAR, 0, 0, 0, L * 2 * H * M, D, syn.POOLED_NOISE)
    mlen = torch.full((1, L), M, dtype=torch.int32, device=dev)
    lk = torch.zeros((1, L, H, T, D), dtype=torch.bfloat16, device=dev)
    lv = torch.zeros_like(lk)
    llen = torch.zeros(1, dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def run():
        msa.msa_sparse_prefill(q, kn, vn, T, 1, L, HQ, H, D, lk, lv, llen, T, mem, mlen, M, TOPK, THETA, D ** -0.5, out,
                               err)
    ev = []
    for r in range(13):
        llen.zero_()
        flush.fill_(r & 0xFF)
        torch.cuda._sleep(2_000_000)  # the GPU is busy while the host prepares the call
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        run()
        e.record()
        if r >= 3:
            ev.append((s, e))
    torch.cuda.synchronize(dev)
    ms = sorted(a.elapsed_time(b) for a, b in ev)[len(ev) // 2]
    fl = prefill_flops(L, HQ, T, M)
    tf = fl / ms / 1e9
    peak = measured_peaks()[1]
    return {"tokens": T, "layers": L, "mem_rows": M, "ms_p50": round(ms, 4), "gflop": round(fl / 1e9, 2),
            "tflops": round(tf, 1), "tensor_frac_of_bf16_burst": round(tf / peak, 4),
            "launches": msa.LAUNCHES_PREFILL, "dev_err": int(err.item()), "l2": "flushed (256 MB write) before each"}


HIDDEN = 2560  # hidden size of the 4B backbone the pages' model is built on


def time_projection(dev, bank, kr_hat, kr_f8):
    """Routing from hidden states (msa_route_topk_hidden): the router query projection of
    the query's T tokens for every routing layer, fused with the normalisation and group
    sum, then the same routing as the step.  Synthetic bf16 weights.  Reports the
    projection kernel's device time (events around the query stage) and the whole call's."""
    import torch

    import msa_synth as syn
    import top_kv_routing_b200 as msa
    C, n_docs = bank.n_chunks, len(bank.lengths)
    # planted inputs: the first 128 hidden features carry a target document's topic (16
    # targets over the tokens) and every head's weights are near-identity on them, so the
    # projected queries find their documents and the E4M3 selections certify as in the step
    hid = torch.empty((T, HIDDEN), dtype=torch.bfloat16, device=dev)
    w = torch.empty((L, HQ * D, HIDDEN), dtype=torch.bfloat16, device=dev)
    syn.device_fill(hid, SEED, syn.STREAM_QR, 90, 0, 0, T, HIDDEN)
    targets = syn.pick_targets(SEED, n_docs, 16, sub=77)
    rt = torch.from_numpy(np.asarray(targets)[np.arange(T) % 16].astype(np.int32)).to(dev)
    head = torch.empty((T, D), dtype=torch.bfloat16, device=dev)
    syn.device_fill(head, SEED, syn.STREAM_QR, 91, 0, 0, T, D, 0.5, torch.from_numpy(bank.topic).to(dev), rt)
    hid[:, :D].copy_(head)
    syn.device_fill(w, SEED, syn.STREAM_KBAR, 92, 0, 0, L * HQ * D, HIDDEN, 0.02)
    eye = torch.eye(D, dtype=torch.bfloat16, device=dev)
    w.view(L, HQ, D, HIDDEN)[..., :D] += eye
    coffs = torch.from_numpy(bank.doc_chunk_offsets).to(dev)
    ws = torch.empty(msa.msa_route_topk_workspace_size(L, 1, T, H, C, n_docs, TOPK), dtype=torch.uint8, device=dev)
    ids = torch.empty((1, L, TOPK), dtype=torch.int32, device=dev)
    sc = torch.empty((1, L, TOPK), device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    flags = msa.MSA_ROUTE_TENSOR_F8 if kr_f8 is not None else msa.MSA_ROUTE_TENSOR
    q0, q1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    q0.record()  # (creates the events; the route library re-records them around the query stage)
    q1.record()
    torch.cuda.synchronize(dev)
    proj, whole = [], []
    msa.msa_route_set_query_profile_events(q0, q1)
    try:
        for r in range(8):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda._sleep(2_000_000)  # the GPU is busy while the host prepares the call
            a.record()
            msa.msa_route_topk_hidden(hid, w, HIDDEN, [0, T], kr_hat, coffs, n_docs, C, L, HQ, H, D, TOPK, ids, sc, ws,
                                      flags=flags, dev_err=err, kr_f8=kr_f8)
            b.record()
            torch.cuda.synchronize(dev)
            if r >= 3:
                proj.append(q0.elapsed_time(q1))
                whole.append(a.elapsed_time(b))
    finally:
        msa.msa_route_set_query_profile_events(None, None)
    ms = sorted(proj)[len(proj) // 2]
    fl = 2.0 * T * HIDDEN * HQ * D * L
    peak = measured_peaks()[1]
    want = set(np.asarray(targets).tolist())
    found = float(np.mean([len(want & set(x.tolist())) / 16 for x in ids[0].cpu().numpy()]))
    return {"hidden": HIDDEN, "tokens": T, "layers": L, "proj_ms_p50": round(ms, 4), "gflop": round(fl / 1e9, 1),
            "planted_recall": round(found, 4),
            "tflops": round(fl / ms / 1e9, 1), "tensor_frac_of_bf16_burst": round(fl / ms / 1e9 / peak, 4),
            "route_hidden_ms_p50": round(sorted(whole)[len(whole) // 2], 3), "dev_err": int(err.item())}


def time_tail_parts(eng, slot, dq, dk, dv, dev):
    """Gather and decode timed apart on the slot's current selection (direct calls, CUDA
    events, after the timed regions): the gather's GB/s against one large pinned
    host-to-device copy (the PCIe ceiling), and decode microseconds per step with the key and
    value bytes each step reads."""
    import torch

    import top_kv_routing_b200 as msa
    L, H, D = eng.L, eng.H, eng.D
    ev = lambda: torch.cuda.Event(enable_timing=True)
    n = 256 << 20
    src = torch.empty(n, dtype=torch.uint8, pin_memory=True)
    dst = torch.empty(n, dtype=torch.uint8, device=dev)
    dst.copy_(src, non_blocking=True)
    a, b = ev(), ev()
    a.record()
    dst.copy_(src, non_blocking=True)
    b.record()
    torch.cuda.synchronize(dev)
    pcie = n / (a.elapsed_time(b) / 1e3) / 1e9
    del src, dst
    gms = []
    for r in range(4):
        a, b = ev(), ev()
        torch.cuda._sleep(2_000_000)  # the GPU is busy while the host prepares the call
        a.record()
        msa.msa_gather_kv(eng.host_kv, eng.n_store, eng.doc_chunk_offsets, eng.doc_store_offsets, eng.n_docs,
                          slot.ids, 1, L, eng.k, H, D, eng.M, slot.mem_kv, slot.mem_len, dev_err=slot.dev_err)
        b.record()
        torch.cuda.synchronize(dev)
        if r:
            gms.append(a.elapsed_time(b))
    g_ms = sorted(gms)[len(gms) // 2]
    mem_blocks = int(slot.mem_len.sum().item())
    g_bytes = mem_blocks * 2 * H * D * 2
    slot.local_len.copy_(slot.local_len0)
    len0 = int(slot.local_len0.item())
    steps = min(32, dq.shape[0], eng.cap - len0)
    out = torch.empty((1, L, eng.Hq, D), dtype=torch.bfloat16, device=dev)
    a, b = ev(), ev()
    torch.cuda._sleep(20_000_000)  # all the steps are enqueued before the GPU reaches the start event
    a.record()
    for st in range(steps):
        msa.msa_sparse_decode(dq[st], dk[st], dv[st], 1, L, eng.Hq, H, D, slot.local_k, slot.local_v, slot.local_len,
                              eng.cap, slot.mem_kv, slot.mem_len, eng.M, eng.k, eng.theta, D ** -0.5, out, slot.dec_ws,
                              dev_err=slot.dev_err)
    b.record()
    torch.cuda.synchronize(dev)
    us = a.elapsed_time(b) * 1e3 / steps
    # per step: every memory row and every local row (the new one included), K and V, bf16
    d_bytes = (mem_blocks * H + L * H * (len0 + (steps + 1) / 2)) * 2 * D * 2
    return {"gather": {"ms": round(g_ms, 4), "bytes": g_bytes, "gbs": round(g_bytes / g_ms / 1e6, 1),
                       "pcie_h2d_gbs": round(pcie, 1), "frac_of_pcie_copy": round(g_bytes / g_ms / 1e6 / pcie, 4)},
            "decode": {"us_per_step": round(us, 2), "steps": steps, "bytes_per_step": int(d_bytes),
                       "gbs": round(d_bytes / (us / 1e6) / 1e9, 1),
                       "note": "direct launches queued behind a GPU sleep, so back to back as in the graph; K/V "
                               "are L2-resident after the first step"}}


def _route_timed(msa, dev, qr, q_off, kr_hat, kr_f8, coffs, n_docs, C, k, flags, ws, reps=4, warm=2):
    """Direct route calls: median device time of the whole call and of its score kernel
    (the library's events around the scan or the GEMM), plus the last ids / dev_err."""
    import torch
    B = len(q_off) - 1
    ids = torch.empty((B, L, k), dtype=torch.int32, device=dev)
    sc = torch.empty((B, L, k), device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0.record()
    g1.record()
    torch.cuda.synchronize(dev)
    whole, score = [], []
    msa.msa_route_set_profile_events(g0, g1)
    try:
        for r in range(warm + reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda._sleep(1_000_000)  # the GPU is busy while the host prepares the call
            a.record()
            msa.msa_route_topk(qr, q_off, kr_hat, coffs, n_docs, C, L, HQ, H, D, k, ids, sc, ws, flags=flags,
                               dev_err=err, kr_f8=kr_f8)
            b.record()
            torch.cuda.synchronize(dev)
            if r >= warm:
                whole.append(a.elapsed_time(b))
                score.append(g0.elapsed_time(g1))
    finally:
        msa.msa_route_set_profile_events(None, None)
    return sorted(whole)[len(whole) // 2], sorted(score)[len(score) // 2], ids, int(err.item())


def _roof(C: int, T: int, ms: float, elem: int, f8: bool):
    """Algorithmic bytes / flops of one routing pass over C blocks x L layers for a T-token
    query, and the fractions of the measured peaks they reach in ms (tensor peak: bf16
    burst, x 2 for E4M3 operands, the nominal dense ratio)."""
    hbm, bf16_burst, _, src = measured_peaks()
    by = L * C * H * D * elem
    fl = 2.0 * T * H * D * L * C
    gbs = by / ms / 1e6
    tf = fl / ms / 1e9
    tc_peak = bf16_burst * (2.0 if f8 else 1.0)
    return {"ms": round(ms, 4), "gbs": round(gbs, 1), "hbm_frac": round(gbs / hbm, 4),
            "frac_of_nominal_8tbs": round(gbs / 8000.0, 4), "tflops": round(tf, 1),
            "tensor_frac_of_burst": round(tf / tc_peak, 4), "peaks": src}


def time_bf16_filter(dev, eng, qs):
    """The step's route with the bf16 filter (MSA_ROUTE_TENSOR) instead of E4M3, on the same
    bank and query, timed by direct calls: whole route and its GEMM."""
    import top_kv_routing_b200 as msa
    slot = eng.slots[0]
    slot.qr.copy_(qs[0])
    whole, gemm, ids, err = _route_timed(msa, dev, slot.qr, [0, T], eng.kr_hat, None, eng.doc_chunk_offsets,
                                         eng.n_docs, eng.C, eng.k, msa.MSA_ROUTE_TENSOR, slot.ws)
    out = {"route_ms": round(whole, 4), "gemm": _roof(eng.C, T, gemm, 2, False), "dev_err": err,
           "timing": "direct calls, CUDA events (library hook around the GEMM); median of 4 after 2 warm-up"}
    return out


SWEEP_T = (1, 2, 4, 8, 16, 32, 64, 256, 1024)  # the workload's sweep {1, 8, 64, 256, 1024} plus 2, 4, 16, 32


def time_sweep(dev, f8: bool):
    """Query-length sweep on the 10M-token bank (10,000 documents, lognormal lengths, seed
    2): for every T the scan (T <= 64), the bf16 GEMM filter and the E4M3 GEMM filter, each
    timed as a whole route and as its score kernel, with the planted documents' recall;
    and which path MSA_ROUTE_AUTO takes."""
    import torch

    import msa_synth as syn
    import top_kv_routing_b200 as msa
    seed, n_docs = 2, 10_000
    lens = syn.doc_lengths_lognormal(seed, n_docs)
    bank = syn.make_bank(seed, n_docs, lens, L)
    C = bank.n_chunks
    kr_hat, kr_f8, _, topic = build_keys(dev, seed, bank, f8)
    coffs = torch.from_numpy(bank.doc_chunk_offsets).to(dev)
    targets = syn.pick_targets(seed, n_docs, TOPK, sub=0)
    points = []
    for Tq in SWEEP_T:
        q = torch.empty((L, Tq, HQ, D), dtype=torch.bfloat16, device=dev)
        rt = torch.from_numpy(np.repeat(targets[np.arange(Tq) % TOPK], HQ).astype(np.int32)).to(dev)
        for l in range(L):
            syn.device_fill(q[l], seed, syn.STREAM_QR, l, 0, 0, Tq * HQ, D, 0.5, topic, rt)
        ws = torch.empty(msa.msa_route_topk_workspace_size(L, 1, Tq, H, C, n_docs, TOPK), dtype=torch.uint8,
                         device=dev)
        want = set(targets[:min(Tq, TOPK)].tolist())
        row = {"T": Tq, "auto_path": "scan" if Tq <= 4 else ("tensor_e4m3" if f8 and Tq >= 16 else "tensor_bf16")}
        paths = [("scan", msa.MSA_ROUTE_SCAN, None, 2, False)] if Tq <= 64 else []
        paths += [("tensor_bf16", msa.MSA_ROUTE_TENSOR, None, 2, False)]
        if f8:
            paths += [("tensor_e4m3", msa.MSA_ROUTE_TENSOR_F8, kr_f8, 1, True)]
        for name, flags, f8k, elem, is_f8 in paths:
            whole, score, ids, err = _route_timed(msa, dev, q, [0, Tq], kr_hat, f8k, coffs, n_docs, C, TOPK, flags, ws)
            got = ids.cpu().numpy()[0]
            rec = float(np.mean([len(want & set(got[l].tolist())) / len(want) for l in range(L)]))
            row[name] = {"route_ms": round(whole, 4), "score_kernel": _roof(C, Tq, score, elem, is_f8),
                         "planted_recall": round(rec, 4), "dev_err": err}
        points.append(row)
        del q, ws
    # crossover: the smallest T at which a tensor path's whole route beats the scan's
    cross = None
    for row in points:
        if "scan" in row:
            best_t = min(row[n]["route_ms"] for n in ("tensor_bf16", "tensor_e4m3") if n in row)
            if best_t < row["scan"]["route_ms"] and cross is None:
                cross = row["T"]
    del kr_hat, kr_f8
    torch.cuda.empty_cache()
    return {"bank": f"10M-token bank: {n_docs} documents, lognormal lengths (median 900, sigma 0.5), {C} blocks x "
                    f"{L} layers", "blocks": C, "points": points,
            "first_T_where_tensor_route_beats_scan": cross,
            "timing": "direct calls, CUDA events; score_kernel = the scan or GEMM alone (library hook)"}


def time_scan(dev, n_blocks: int = 1_000_000, calls: int = 3):
    """The streaming scan alone on one layer of n_blocks blocks x 8 key heads (2 GB of bf16
    routing keys at 1M blocks, larger than L2): a one-token query, documents of 10 blocks,
    MSA_ROUTE_SCAN, `calls` whole routes timed with CUDA events.  The workload of the scan
    kernel's ncu capture."""
    import torch

    import msa_synth as syn
    import top_kv_routing_b200 as msa
    C, seed = n_blocks, 5
    kr = torch.empty((1, C, H, D), dtype=torch.bfloat16, device=dev)
    scratch = torch.empty((C, H, D), dtype=torch.bfloat16, device=dev)
    syn.device_fill(scratch, seed, syn.STREAM_KRBAR, 0, 0, 0, C, H * D, syn.POOLED_NOISE)
    ones = torch.arange(C + 1, dtype=torch.int64, device=dev)
    msa.msa_pool_blocks(None, None, scratch, ones, ones, C, C, H, D, 1, 0.0, None, None, kr[0], None, None,
                        in_dtype=msa.MSA_BF16)
    del scratch, ones
    n_docs = C // 10
    coffs = torch.arange(0, C + 1, 10, dtype=torch.int64, device=dev)
    q = torch.from_numpy(syn.fill(seed, syn.STREAM_QR, 0, 0, 0, HQ, D).reshape(1, 1, HQ, D).astype(np.float32)).to(dev)
    ws = torch.empty(msa.msa_route_topk_workspace_size(1, 1, 1, H, C, n_docs, TOPK), dtype=torch.uint8, device=dev)
    ids = torch.empty((1, 1, TOPK), dtype=torch.int32, device=dev)
    sc = torch.empty((1, 1, TOPK), dtype=torch.float32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    ms = []
    for _ in range(calls):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        n = msa.msa_route_topk(q, [0, 1], kr, coffs, n_docs, C, 1, HQ, H, D, TOPK, ids, sc, ws,
                               flags=msa.MSA_ROUTE_SCAN, dev_err=err)
        e1.record()
        torch.cuda.synchronize(dev)
        ms.append(e0.elapsed_time(e1))
    key_bytes = C * H * D * 2
    best = min(ms)
    out = {"blocks": C, "key_bytes": key_bytes, "route_ms": [round(x, 4) for x in ms], "launches": n,
           "route_GBps_best": round(key_bytes / best / 1e6, 1), "dev_err": int(err.item())}
    del kr, q, ws
    torch.cuda.empty_cache()
    return out


def time_interleave(dev, host_kv, f8: bool):
    """Multi-round interleave on the 10M-token bank: 64 queries of 128 router tokens, each
    planted with a chain of three documents A -> B -> C (the router vectors of the first
    128 tokens carry A); round r routes over all of each query's tokens so far (128 + 512 r),
    gathers the selections for all 64 queries, decodes 32 tokens; between rounds 512 local
    tokens are appended per query whose router vectors carry the next chain document.
    Reports per round the route, gather and decode device times and the chain recovery
    (fraction of (query, layer) selections holding the chain so far)."""
    import torch

    import msa_synth as syn
    import top_kv_routing_b200 as msa
    seed, n_docs, B, T0, A, R, DEC_R, k = 4, 10_000, 64, 128, 512, 3, 32, 16
    lens = syn.doc_lengths_lognormal(2, n_docs)
    bank = syn.make_bank(2, n_docs, lens, L)
    C = bank.n_chunks
    coffs_np = bank.doc_chunk_offsets
    kr_hat, kr_f8, _, topic = build_keys(dev, 2, bank, f8)
    coffs = torch.from_numpy(coffs_np).to(dev)
    P = host_kv.shape[1]
    per_doc = np.diff(coffs_np)
    h = syn.hashes(syn.tensor_key(seed, syn.STREAM_TARGETS, 0, 98), np.arange(n_docs, dtype=np.uint64))
    store_off = torch.from_numpy((h % np.uint64(max(1, P - int(per_doc.max())))).astype(np.int64)).to(dev)
    chains = [syn.pick_targets(seed, n_docs, 3, sub=b) for b in range(B)]
    cap = T0 + R * DEC_R + (R - 1) * A
    M = k * int(per_doc.max())
    mem = torch.zeros((B, L, 2, H, M, D), dtype=torch.bfloat16, device=dev)
    mem_len = torch.zeros((B, L), dtype=torch.int32, device=dev)
    lk = torch.zeros((B, L, H, cap, D), dtype=torch.bfloat16, device=dev)
    lv = torch.zeros_like(lk)
    llen = torch.zeros(B, dtype=torch.int32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    ws_dec = torch.zeros(msa.msa_sparse_decode_workspace_size(B, L, HQ, H), dtype=torch.uint8, device=dev)
    seg = torch.empty((L * H * A, D), dtype=torch.bfloat16, device=dev)
    dq = torch.empty((DEC_R, B, L, HQ, D), dtype=torch.bfloat16, device=dev)
    dk = torch.empty((DEC_R, B, L, H, D), dtype=torch.bfloat16, device=dev)
    dv = torch.empty_like(dk)
    out = torch.empty((B, L, HQ, D), dtype=torch.bfloat16, device=dev)

    def append_local(r, n):
        for b in range(B):
            pos = int(llen[b].item())
            for stream, cache in ((syn.STREAM_LOCAL_K, lk), (syn.STREAM_LOCAL_V, lv)):
                syn.device_fill(seg[:L * H * n], seed, stream, r, b, 0, L * H * n, D)
                cache[b, :, :, pos:pos + n] = seg[:L * H * n].view(L, H, n, D)
            llen[b] += n

    def fill_q(dst, b, tok0, n, doc):
        rt = torch.full((n * HQ,), int(doc), dtype=torch.int32, device=dev)
        for l in range(L):
            syn.device_fill(dst[l], seed, syn.STREAM_QR, l, b, tok0 * HQ, n * HQ, D, 0.5, topic, rt)

    append_local(0, T0)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    rounds = []
    for r in range(R):
        Tq = T0 + r * A
        qr = torch.empty((L, B * Tq, HQ, D), dtype=torch.bfloat16, device=dev)
        for b in range(B):
            fill_q(qr[:, b * Tq:b * Tq + T0], b, 0, T0, chains[b][0])
            for rr in range(1, r + 1):
                t0 = T0 + (rr - 1) * A
                fill_q(qr[:, b * Tq + t0:b * Tq + t0 + A], b, t0, A, chains[b][rr])
        offs = [b * Tq for b in range(B + 1)]
        ws = torch.empty(msa.msa_route_topk_workspace_size(L, B, B * Tq, H, C, n_docs, k), dtype=torch.uint8,
                         device=dev)
        ids = torch.empty((B, L, k), dtype=torch.int32, device=dev)
        sc = torch.empty((B, L, k), device=dev)
        for s_ in range(DEC_R):
            step = r * DEC_R + s_
            syn.device_fill(dq[s_], seed, syn.STREAM_DEC_Q, step, 0, 0, B * L * HQ, D)
            syn.device_fill(dk[s_], seed, syn.STREAM_DEC_K, step, 0, 0, B * L * H, D)
            syn.device_fill(dv[s_], seed, syn.STREAM_DEC_V, step, 0, 0, B * L * H, D)
        torch.cuda.synchronize(dev)
        e = [ev() for _ in range(4)]
        e[0].record()
        msa.msa_route_topk(qr, offs, kr_hat, coffs, n_docs, C, L, HQ, H, D, k, ids, sc, ws, dev_err=err, kr_f8=kr_f8)
        e[1].record()
        msa.msa_gather_kv(host_kv, P, coffs, store_off, n_docs, ids, B, L, k, H, D, M, mem, mem_len, dev_err=err)
        e[2].record()
        for s_ in range(DEC_R):
            msa.msa_sparse_decode(dq[s_], dk[s_], dv[s_], B, L, HQ, H, D, lk, lv, llen, cap, mem, mem_len, M, k, THETA,
                                  D ** -0.5, out, ws_dec, dev_err=err)
        e[3].record()
        torch.cuda.synchronize(dev)
        got = ids.cpu().numpy()
        rec = float(np.mean([set(chains[b][:r + 1].tolist()) <= set(got[b, l].tolist())
                             for b in range(B) for l in range(L)]))
        g_bytes = int(mem_len.sum().item()) * 2 * H * D * 2
        g_ms = e[1].elapsed_time(e[2])
        rounds.append({"round": r, "router_tokens_per_query": Tq, "route_ms": round(e[0].elapsed_time(e[1]), 3),
                       "gather_ms": round(g_ms, 3), "gather_gbs": round(g_bytes / g_ms / 1e6, 1),
                       "decode_ms": round(e[2].elapsed_time(e[3]), 3),
                       "decode_us_per_step": round(e[2].elapsed_time(e[3]) * 1e3 / DEC_R, 2),
                       "round_ms": round(e[0].elapsed_time(e[3]), 3), "chain_recovery": round(rec, 4),
                       "dev_err": int(err.item())})
        del qr, ws
        if r + 1 < R:
            append_local(r + 1, A)
    del kr_hat, kr_f8, mem, lk, lv, seg
    torch.cuda.empty_cache()
    return {"bank": f"10M-token bank ({n_docs} documents, {C} blocks x {L} layers)", "queries": B,
            "first_tokens": T0, "appended_per_round": A, "decode_per_round": DEC_R, "rounds": rounds,
            "filter": "E4M3" if f8 else "bf16",
            "store": f"page-locked host store of {P} blocks per layer at hashed document offsets",
            "timing": "CUDA events around one route (64 queries), one gather, 32 decode launches per round"}


# ----------------------------------------------------------------------------- GPU arm

def run_gpu(args):
    import torch
    import torch.distributed as dist

    import top_kv_routing_b200 as msa
    from top_kv_routing_b200.engine import SparseMemory

    world, rank, local = init_ranks("nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    hbm_peak, bf16_peak, bf16_sus, peak_src = measured_peaks()

    # pooling is an offline pass of its own: timed first, on the idle GPU
    pool = time_pool(dev) if (rank == 0 and not args.no_pool) else None
    prefill = time_prefill(dev) if (rank == 0 and not args.no_prefill) else None
    torch.cuda.empty_cache()
    f8 = args.filter == "e4m3"
    bank, kr_hat, kr_f8, f8_ms, host_kv, store_off, topic, store = make_workload(dev, args.host_store_blocks, f8)
    qs, targets = make_queries(dev, bank, topic, args.queries)
    n_distinct = len(qs)
    dq, dk, dv, pk, pv = make_decode_inputs(dev)
    n_slots = args.pipeline
    dec_inputs = [(dq.clone(), dk.clone(), dv.clone(), torch.empty((DEC, 1, L, HQ, D), dtype=torch.bfloat16,
                                                                   device=dev)) for _ in range(n_slots)]
    eng = SparseMemory(kr_hat, bank.doc_chunk_offsets, host_kv, store_off, n_q_heads=HQ, top_k=TOPK,
                       query_tokens=T, local_cap=T + DEC, rope_theta=THETA, slots=n_slots, kr_f8=kr_f8)
    eng.set_local_prefix(pk, pv)
    for s_ in eng.slots:
        s_.qr.copy_(qs[0])
    eng.capture(dec_inputs)
    launches = eng.launches_per_query
    slot0 = eng.slots[0]

    def score_kernel_ms(reps=5):
        # the score kernel's own device time: CUDA events the route library records right
        # before and after it, on the route stream, for direct (non-graph) calls of the same
        # route on the same buffers
        ev_a, ev_b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev_a.record()
        ev_b.record()
        torch.cuda.synchronize(dev)
        msa.msa_route_set_profile_events(ev_a, ev_b)
        vals = []
        try:
            for i in range(reps):
                slot0.qr.copy_(qs[i % len(qs)])
                torch.cuda.synchronize(dev)
                with torch.cuda.stream(eng.route_stream):
                    eng.enqueue_route(slot0, eng.route_stream)
                torch.cuda.synchronize(dev)
                vals.append(ev_a.elapsed_time(ev_b))
        finally:
            msa.msa_route_set_profile_events(None, None)
        return float(np.mean(vals))

    def run(n, times=None):
        """n queries from device-resident inputs; times: per-query (start, end) events."""
        for i in range(n):
            def load(slot, st, i=i):
                slot.qr.copy_(qs[i % len(qs)])
                if times is not None:
                    times[i][0].record(st)

            def unload(slot, st, i=i):
                if times is not None:
                    times[i][1].record(st)
            eng.launch(i, load, unload)
        eng.drain()

    # correctness guard on the benchmark's own output: planted documents are selected
    slot0.dev_err.zero_()
    run(1)
    torch.cuda.synchronize(dev)
    got = slot0.ids.cpu().numpy()[0]
    hits = np.mean([len(set(got[l].tolist()) & set(targets[0].tolist())) / TOPK for l in range(L)])
    dev_err = int(slot0.dev_err.item())
    same_as_bf16 = None
    if f8:
        # the same query through the bf16 filter: both end in exact rescoring, so the
        # selections must agree
        ids2 = torch.empty_like(slot0.ids)
        sc2 = torch.empty_like(slot0.scores)
        msa.msa_route_topk(slot0.qr, [0, T], kr_hat, eng.doc_chunk_offsets, eng.n_docs, eng.C, L, HQ, H, D, TOPK,
                           ids2, sc2, slot0.ws, flags=msa.MSA_ROUTE_TENSOR, dev_err=slot0.dev_err)
        torch.cuda.synchronize(dev)
        same_as_bf16 = bool(torch.equal(ids2, slot0.ids) and torch.equal(sc2, slot0.scores))
        dev_err |= int(slot0.dev_err.item())

    # isolated latency of one query (route + gather + decode, nothing overlapping)
    iso = []
    for i in range(5):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        tm = [(e0, e1)]
        run(1, times=tm)
        torch.cuda.synchronize(dev)
        iso.append(e0.elapsed_time(e1))

    run(args.warmup)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    times = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with ClockSampler(smi_id(dev)) as clk:
        run(args.steps, times=times)
        torch.cuda.synchronize(dev)
    per_query = [a.elapsed_time(b) for a, b in times]
    total_ms = times[0][0].elapsed_time(times[-1][1])
    gemm_avg = score_kernel_ms()

    # end to end: pinned host inputs in, results out, every query.  Query i+1's inputs
    # cross PCIe on a copy stream while query i runs (double-buffered device staging, then
    # one device-to-device copy into the slot); results leave through a staging buffer on
    # a second copy stream.  The timed region runs from the first host-to-device copy to
    # the last device-to-host copy.
    host = {"qr": [q.cpu().pin_memory() for q in qs], "dq": dq.cpu().pin_memory(), "dk": dk.cpu().pin_memory(),
            "dv": dv.cpu().pin_memory(),
            "ids": [torch.empty((1, L, TOPK), dtype=torch.int32).pin_memory() for _ in range(2)],
            "scores": [torch.empty((1, L, TOPK), dtype=torch.float32).pin_memory() for _ in range(2)],
            "out": [torch.empty((DEC, 1, L, HQ, D), dtype=torch.bfloat16).pin_memory() for _ in range(2)]}
    copy_in, copy_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    stage_in = [{"qr": torch.empty_like(slot0.qr), "dq": torch.empty_like(dq), "dk": torch.empty_like(dk),
                 "dv": torch.empty_like(dv)} for _ in range(2)]
    stage_out = [{"ids": torch.empty_like(slot0.ids), "scores": torch.empty_like(slot0.scores),
                  "out": torch.empty_like(dec_inputs[0][3])} for _ in range(2)]
    ev = lambda: torch.cuda.Event()
    h2d_done, consumed = [ev(), ev()], [ev(), ev()]
    out_ready, d2h_done = [ev(), ev()], [ev(), ev()]

    def run_host(n, e_start=None, e_end=None):
        def issue_h2d(i):
            b = i % 2
            with torch.cuda.stream(copy_in):
                copy_in.wait_event(consumed[b])  # query i-2 has moved these buffers into its slot
                st = stage_in[b]
                st["qr"].copy_(host["qr"][i % len(qs)], non_blocking=True)
                for k in ("dq", "dk", "dv"):
                    st[k].copy_(host[k], non_blocking=True)
                h2d_done[b].record(copy_in)

        if e_start is not None:
            e_start.record(copy_in)
        issue_h2d(0)
        for i in range(n):
            if i + 1 < n:
                issue_h2d(i + 1)

            def load(slot, st, i=i):
                b = i % 2
                st.wait_event(h2d_done[b])
                k = eng.slots.index(slot)
                slot.qr.copy_(stage_in[b]["qr"], non_blocking=True)
                for src, dst in zip((stage_in[b]["dq"], stage_in[b]["dk"], stage_in[b]["dv"]), dec_inputs[k][:3]):
                    dst.copy_(src, non_blocking=True)
                consumed[b].record(st)

            def unload(slot, st, i=i):
                b = i % 2
                st.wait_event(d2h_done[b])  # query i-2's results have left this staging buffer
                k = eng.slots.index(slot)
                so = stage_out[b]
                so["ids"].copy_(slot.ids, non_blocking=True)
                so["scores"].copy_(slot.scores, non_blocking=True)
                so["out"].copy_(dec_inputs[k][3], non_blocking=True)
                out_ready[b].record(st)
                with torch.cuda.stream(copy_out):
                    copy_out.wait_event(out_ready[b])
                    for name in ("ids", "scores", "out"):
                        host[name][b].copy_(so[name], non_blocking=True)
                    d2h_done[b].record(copy_out)
            eng.launch(i, load, unload)
        if e_end is not None:
            copy_out.wait_stream(eng.tail_stream)
            e_end.record(copy_out)
        eng.drain()
        torch.cuda.current_stream(dev).wait_stream(copy_in)
        torch.cuda.current_stream(dev).wait_stream(copy_out)

    run_host(2)
    torch.cuda.synchronize(dev)
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    run_host(args.steps, e_start, e_end)
    torch.cuda.synchronize(dev)
    e2e_ms = e_start.elapsed_time(e_end)
    # the results read back match the device-resident run's
    host_ok = bool(torch.equal(host["ids"][(args.steps - 1) % 2].to(dev),
                               eng.slots[(args.steps - 1) % n_slots].ids))
    h2d = host["qr"][0].numel() * 2 + (dq.numel() + dk.numel() + dv.numel()) * 2
    d2h = host["ids"][0].numel() * 4 + host["scores"][0].numel() * 4 + host["out"][0].numel() * 2
    # routing from hidden states (fused router projection), after the timed regions
    projection = time_projection(dev, bank, kr_hat, kr_f8) if (rank == 0 and not args.no_projection) else None
    tail_parts = bf16_filter = sweep = interleave = None
    if rank == 0:
        def guarded(fn, *a):
            try:
                return fn(*a)
            except Exception as e:  # (a separate measurement: never at the cost of the line)
                return {"error": f"{type(e).__name__}: {e}"}
        tail_parts = guarded(time_tail_parts, eng, slot0, dq, dk, dv, dev)
        if f8 and not args.no_bf16_filter:
            bf16_filter = guarded(time_bf16_filter, dev, eng, qs)
    # the 100M bank's device buffers go before the 10M-bank measurements (the host store stays)
    del eng, slot0, kr_hat, kr_f8, qs, dec_inputs, stage_in, stage_out
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    if rank == 0:
        if not args.no_sweep:
            sweep = guarded(time_sweep, dev, f8)
        if not args.no_interleave:
            interleave = guarded(time_interleave, dev, host_kv, f8)

    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], dev)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    ms = total_ms / args.steps
    units = N_TOKENS * args.steps * world
    value = replica_throughput(N_TOKENS * args.steps, world, total_ms)
    elem = 1 if f8 else 2
    algo_bytes = L * bank.n_chunks * H * D * elem
    achieved = algo_bytes / (gemm_avg / 1e3) / 1e9
    flops = 2.0 * T * H * D * L * bank.n_chunks
    tflops = flops / (gemm_avg / 1e3) / 1e12
    # tensor peak of the operand type: E4M3 = 2 x the measured bf16 figure (the nominal
    # dense ratio); the burst figure, as the GEMM is timed by isolated direct calls
    tc_peak = bf16_peak * (2.0 if f8 else 1.0)
    t_hbm = algo_bytes / (hbm_peak * 1e9)
    t_tc = flops / (tc_peak * 1e12)
    bound = "tensor" if t_tc > t_hbm else "hbm"
    traffic_pbl = GEMM_TRAFFIC_PER_BLOCK_LAYER["e4m3" if f8 else "bf16"]
    p = sorted(per_query)
    iso_s = sorted(iso)
    line = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "bank tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3 filter + fp32 rescoring" if f8 else "bf16 filter + fp32 rescoring",
        "data": "synthetic",
        "config": {"workload": WORKLOAD if N_DOCS == 100_000 else f"{N_TOKENS:,}-token bank (profiling size)",
                   "filter": ("E4M3 copy of the unit keys (x256), tcgen05 kind::f8f6f4; top candidates rescored "
                              "exactly in fp32 from the bf16 keys" if f8 else
                              "bf16 keys, tcgen05 kind::f16; top candidates rescored exactly in fp32"),
                   "n_docs": N_DOCS, "n_tokens": N_TOKENS, "n_blocks": bank.n_chunks,
                   "layers": L, "kv_heads": H, "q_heads": HQ, "head_dim": D, "query_tokens": T, "top_k": TOPK,
                   "decode_tokens": DEC, "distinct_queries": n_distinct, "host_store_blocks": int(host_kv.shape[1]),
                   "host_store": store,
                   "l2": f"inputs larger than L2 ({algo_bytes / 1e9:.1f} GB of routing keys stream through every step)",
                   "graph": "per query two CUDA graphs: route; gather + 128 decode steps",
                   "pipeline": (f"{n_slots} query slots: the gather+decode of query i overlaps the route of "
                                "query i+1" if n_slots > 1 else "one query at a time"),
                   "parallelism": f"replicas x{world}" if world > 1 else "1 GPU"},
        "scan_gbs": round(achieved, 1),
        "scan_frac_of_nominal_8tbs": round(achieved / 8000.0, 4),
        "p50_route_decode_ms": round(p[len(p) // 2], 4),
        "p99_route_decode_ms": round(p[min(len(p) - 1, int(0.99 * len(p)))], 4),
        "p50_isolated_ms": round(iso_s[len(iso_s) // 2], 4),
        "roofline": {"bound": bound, "kernel": "route score GEMM (tcgen05, %s)" % ("E4M3" if f8 else "bf16"),
                     "achieved": round(tflops if bound == "tensor" else achieved, 1),
                     "peak": round(tc_peak if bound == "tensor" else hbm_peak, 1),
                     "unit": "TFLOP/s" if bound == "tensor" else "GB/s",
                     "frac": round(tflops / tc_peak if bound == "tensor" else achieved / hbm_peak, 4),
                     "peak_source": (f"{peak_src}: " + ("bf16 burst x 2 (E4M3/bf16 nominal ratio)" if f8 else
                                                        "bf16 burst") if bound == "tensor" else
                                     f"{peak_src}: HBM copy"),
                     "timing": "score GEMM alone, direct calls between steps (CUDA events the route library "
                               "records around it); burst peak for an isolated kernel",
                     "tensor_frac_of_sustained": round(tflops / (bf16_sus * (2.0 if f8 else 1.0)), 4)
                     if bf16_sus else None,
                     "traffic": None if traffic_pbl is None else round(traffic_pbl * L * bank.n_chunks),
                     "traffic_source": ("ncu dram bytes of a 2M-token launch scaled by blocks" if traffic_pbl
                                        else "not captured for this kernel yet"),
                     "algorithmic_bytes": algo_bytes, "kernel_ms": round(gemm_avg, 4),
                     "gbs": round(achieved, 1), "hbm_frac": round(achieved / hbm_peak, 4),
                     "tflops": round(tflops, 1), "tensor_frac": round(tflops / tc_peak, 4),
                     "roofline_ms": round(max(t_hbm, t_tc) * 1e3, 4)},
        "e2e": {"value": round(replica_throughput(N_TOKENS * args.steps, world, e2e_ms), 1), "unit": "bank tokens/s",
                "overlap": "next query's inputs copied in while the current one runs", "host_ids_match": host_ok,
                "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": launches * args.steps,
        "clocks": clk.summary(),
        "pool": pool,
        "prefill": prefill,
        "router_projection": projection,
        "tail_parts": tail_parts,
        "planted_recall": round(float(hits), 4),
        "dev_err": dev_err,
        "filter_keys_ms": None if f8_ms is None else round(f8_ms, 2),
        "ids_match_bf16_filter": same_as_bf16,
        "bf16_filter": bf16_filter,
        "sweep": sweep,
        "interleave": interleave,
        "host": dict(host_cores(), mem_available_gb=None if mem_available_gb() is None else
                     round(mem_available_gb(), 1)),
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- CPU oracle arm

def _oracle_sample(n_blocks: int):
    """Layer-0 routing keys of the first n_blocks blocks of the 100M bank and the T=256 query."""
    import msa_synth as syn
    lens = syn.doc_lengths_exact_total(SEED, N_DOCS, N_TOKENS)
    bank = syn.make_bank(SEED, N_DOCS, lens, L)
    coffs = bank.doc_chunk_offsets
    n_docs = int(np.searchsorted(coffs, n_blocks, side="right")) - 1
    n_docs = max(1, n_docs)
    nb = int(coffs[n_docs])
    keys = syn.bf16_bits_to_f32(syn.pooled_router_keys(bank, 0, 0, nb))
    tg = syn.pick_targets(SEED, N_DOCS, TOPK, sub=0)
    q = syn.query_router(SEED, 0, 0, T, HQ, D, bank.topic, tg, dtype="bf16")
    return syn.bf16_bits_to_f32(q), keys, coffs[:n_docs + 1].copy(), nb


def cpu_baseline(seconds: float):
    """The CPU oracle's routing (explicit cosine form, one core) on a bounded sample."""
    import oracle
    t_probe = time.time()
    q, keys, offs, nb = _oracle_sample(64)
    t0 = time.time()
    oracle.route(q, keys, offs, TOPK)
    per_block = (time.time() - t0) / nb
    n = max(64, int(seconds / max(per_block, 1e-9)))
    q, keys, offs, nb = _oracle_sample(n)
    t0 = time.time()
    oracle.route(q, keys, offs, TOPK)
    dt = time.time() - t0
    # bank tokens routed per second over all 18 layers: 64 tokens per block, 1 of 18 layers
    value = nb * 64 / L / dt
    return {"value": round(value, 3), "unit": "bank tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"layer 0 of 18, first {nb} of 1,562,500 blocks, T=256 query, explicit cosine form "
                      f"({dt:.1f} s); rate scaled to all 18 layers", "setup_s": round(t0 - t_probe, 1),
            "host_nproc": host_cores()["nproc"]}


def run_reference(args):
    """The oracle on a bounded sample, on rank 0; with several ranks (gloo, host only) the
    others wait for it at a barrier and print nothing."""
    world, rank, _ = rank_env()
    if world > 1:
        import torch.distributed as dist
        init_ranks("gloo", timeout_s=1800)
        try:
            if rank == 0:
                _reference_line(args, world)
            dist.barrier()
        finally:
            dist.destroy_process_group()
        return
    _reference_line(args, 1)


def _reference_line(args, world: int):
    vals = []
    for _ in range(args.warmup):
        cpu_baseline(min(2.0, args.cpu_seconds))
    t0 = time.time()
    for _ in range(args.steps):
        vals.append(cpu_baseline(args.cpu_seconds / max(1, args.steps)))
    step_ms = (time.time() - t0) * 1e3 / max(1, args.steps)
    v = float(np.mean([x["value"] for x in vals]))
    line = {"impl": "reference", "metric": METRIC, "value": round(v, 3), "unit": "bank tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(step_ms, 1), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD},
            "cpu_baseline": {"value": round(v, 3), "unit": "bank tokens/s", "cores": 1, "kind": "oracle",
                             "sample": vals[0]["sample"], "host_nproc": host_cores()["nproc"]},
            "e2e": {"value": round(v, 3), "unit": "bank tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--queries", type=int, default=16, help="distinct synthetic queries cycled over the steps")
    ap.add_argument("--host-store-blocks", type=int, default=None,
                    help="physical blocks per layer in the page-locked content store (default: the whole bank "
                         "when the host has room for it)")
    ap.add_argument("--no-bf16-filter", action="store_true", help="skip the bf16-filter route measurement")
    ap.add_argument("--no-sweep", action="store_true", help="skip the query-length sweep on the 10M-token bank")
    ap.add_argument("--no-interleave", action="store_true",
                    help="skip the multi-round interleave measurement on the 10M-token bank")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-pool", action="store_true", help="skip the separate pooling measurement")
    ap.add_argument("--no-prefill", action="store_true", help="skip the separate prefill measurement")
    ap.add_argument("--no-projection", action="store_true",
                    help="skip the separate routing-from-hidden-states measurement")
    ap.add_argument("--pipeline", type=int, default=1, choices=[1, 2],
                    help="queries in flight (2 overlaps a query's gather+decode with the next route)")
    ap.add_argument("--filter", default="e4m3", choices=["e4m3", "bf16"],
                    help="operands of the routing filter GEMM (both end in exact fp32 rescoring)")
    ap.add_argument("--docs", type=int, default=N_DOCS,
                    help="documents in the bank (x1000 tokens); smaller banks serve profiling captures")
    args = ap.parse_args()
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        sys.exit(spawn_ranks(args.gpus))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world != args.gpus:
        log(f"bench.py: --gpus {args.gpus} but the launcher started {world} ranks")
        sys.exit(2)
    set_bank_size(args.docs)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


def spawn_ranks(n: int) -> int:
    """--gpus N without a launcher: starts N local ranks of this same command under
    torch.distributed.run (rendezvous on 127.0.0.1); rank 0 prints the line.  Returns the
    launcher's exit status."""
    import socket
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", f"--master-port={port}", os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


if __name__ == "__main__":
    main()
