"""Seeded synthetic inputs for the Memory Sparse Attention hot path.

This module only draws numbers.  It holds none of the method's arithmetic (no
RoPE, pooling, normalisation of routing keys, cosine, top-k or attention); both
the CPU oracle's tests and the CUDA path take their inputs from here, so that
the two sides see bit-identical data.

Generator (defined here, mirrored for the GPU in ``csrc/synth.h``):

* ``mix64`` is the splitmix64 output finaliser.
* A tensor is identified by (seed, stream, layer, sub); its 64-bit key is
  ``mix64(mix64(seed*G + stream + 2^32*sub) + (layer+1)*L)``.
* Element ``idx`` (row-major flat index inside the tensor) draws
  ``h = mix64(key + (idx+1)*G)``, i.e. the (idx+1)-th splitmix64 output with
  state ``key``.
* The four 16-bit fields of ``h`` are summed; ``(sum - 131070) * sqrt(3)/65536``
  (one fp32 multiply of an exactly representable integer) is an Irwin-Hall(4)
  variate with mean 0 and variance 1, standing in for N(0, 1).  Being integer
  arithmetic plus a single IEEE multiply, host and device produce the same bits.
* ``x = ih * sigma`` (fp32, skipped when sigma == 1) then ``x = x + topic[j]``
  (fp32, when the row has a topic), then optional round-to-nearest-even bf16.

Workload recipes (document-length laws, topic vectors, planted needles) are at
the bottom; they follow the pages' workload shapes: ~1000-token documents, 64
tokens per memory block, 8 KV heads x 128, 32 query heads, top-16.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

MASK64 = (1 << 64) - 1
GOLDEN = 0x9E3779B97F4A7C15
LAYER_MUL = 0xD1B54A32D192ED03
M1 = 0xBF58476D1CE4E5B9
M2 = 0x94D049BB133111EB

# fp32 bits of sqrt(3)/65536 rounded to nearest; the device header carries the same bits.
IH_SCALE_BITS = int(np.float32(math.sqrt(3.0) / 65536.0).view(np.uint32))
IH_SCALE = np.uint32(IH_SCALE_BITS).view(np.float32)

# Streams: one per kind of tensor.
STREAM_K = 1          # raw K tokens            [tok][H][d]
STREAM_V = 2          # raw V tokens            [tok][H][d]
STREAM_KR = 3         # raw router keys         [tok][H][d]
STREAM_QR = 4         # router queries          [t][Hq][d]      (sub = query index)
STREAM_TOPIC = 5      # topic vectors           [doc][d]
STREAM_DOCLEN = 6     # document lengths
STREAM_DEC_Q = 7      # decode q                [step][B][L][Hq][d] (layer = step)
STREAM_DEC_K = 8      # decode new k            [step][B][L][H][d]
STREAM_DEC_V = 9      # decode new v
STREAM_LOCAL_K = 10   # pre-filled local K      [B][L][H][len][d]
STREAM_LOCAL_V = 11
STREAM_KBAR = 12      # pooled-level content K  [chunk][H][d]
STREAM_VBAR = 13      # pooled-level content V
STREAM_KRBAR = 14     # pooled-level router key [chunk][H][d]
STREAM_TARGETS = 15   # planted target choice


def _mix64_int(z: int) -> int:
    z &= MASK64
    z ^= z >> 30
    z = (z * M1) & MASK64
    z ^= z >> 27
    z = (z * M2) & MASK64
    z ^= z >> 31
    return z


def mix64(z: np.ndarray) -> np.ndarray:
    """splitmix64 finaliser over a uint64 array (wrapping arithmetic)."""
    z = z.astype(np.uint64, copy=True)
    with np.errstate(over="ignore"):
        z ^= z >> np.uint64(30)
        z *= np.uint64(M1)
        z ^= z >> np.uint64(27)
        z *= np.uint64(M2)
        z ^= z >> np.uint64(31)
    return z


def tensor_key(seed: int, stream: int, layer: int = 0, sub: int = 0) -> int:
    k = _mix64_int(seed * GOLDEN + stream + (sub << 32))
    return _mix64_int(k + (layer + 1) * LAYER_MUL)


def hashes(key: int, idx: np.ndarray) -> np.ndarray:
    idx = np.asarray(idx, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(key) + (idx + np.uint64(1)) * np.uint64(GOLDEN)
    return mix64(z)


def irwin_hall(h: np.ndarray) -> np.ndarray:
    """Unit-variance Irwin-Hall(4) variate from 64 random bits (fp32, exact)."""
    m = np.uint64(0xFFFF)
    s = ((h & m) + ((h >> np.uint64(16)) & m) + ((h >> np.uint64(32)) & m)
         + (h >> np.uint64(48))).astype(np.int64) - 131070
    return s.astype(np.float32) * IH_SCALE


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16 bit pattern (finite inputs)."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((b >> np.uint64(16)) & np.uint64(1)) + np.uint64(0x7FFF)
    return ((b + r) >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def fill(seed: int, stream: int, layer: int, sub: int, row0: int, n_rows: int, row_len: int,
         sigma: float = 1.0, topic: np.ndarray | None = None, row_topic: np.ndarray | None = None,
         dtype: str = "f32") -> np.ndarray:
    """Rows [row0, row0+n_rows) of a [rows][row_len] tensor.

    ``topic`` is [n_topics][tlen] fp32; row r adds ``topic[row_topic[r - row0]][j % tlen]``
    when ``row_topic[r - row0] >= 0``.  Returns fp32 values, or bf16 bit patterns
    (uint16) when ``dtype == "bf16"``.
    """
    key = tensor_key(seed, stream, layer, sub)
    idx = (np.arange(row0, row0 + n_rows, dtype=np.uint64)[:, None] * np.uint64(row_len)
           + np.arange(row_len, dtype=np.uint64)[None, :])
    x = irwin_hall(hashes(key, idx))
    if sigma != 1.0:
        x = x * np.float32(sigma)
    if topic is not None and row_topic is not None:
        topic = np.asarray(topic, dtype=np.float32)
        tlen = topic.shape[1]
        rt = np.asarray(row_topic, dtype=np.int64)
        has = rt >= 0
        if np.any(has):
            cols = np.arange(row_len) % tlen
            add = topic[np.where(has, rt, 0)][:, cols]
            x = np.where(has[:, None], x + add, x).astype(np.float32)
    if dtype == "bf16":
        return f32_to_bf16_bits(x)
    return x


def uniform01(seed: int, stream: int, layer: int, sub: int, n: int) -> np.ndarray:
    """n doubles in (0, 1] from 53-bit draws."""
    h = hashes(tensor_key(seed, stream, layer, sub), np.arange(n, dtype=np.uint64))
    return ((h >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)


# ----------------------------------------------------------------------------- recipes

def doc_lengths_uniform(seed: int, n_docs: int, lo: int, hi: int) -> np.ndarray:
    h = hashes(tensor_key(seed, STREAM_DOCLEN), np.arange(n_docs, dtype=np.uint64))
    return (lo + (h % np.uint64(hi - lo + 1)).astype(np.int64)).astype(np.int64)


def doc_lengths_lognormal(seed: int, n_docs: int, median: float = 900.0, sigma: float = 0.5,
                          lo: int = 64, hi: int = 8192) -> np.ndarray:
    """Box-Muller normal -> lognormal(ln median, sigma) -> round -> clip."""
    u1 = uniform01(seed, STREAM_DOCLEN, 0, 1, n_docs)
    u2 = uniform01(seed, STREAM_DOCLEN, 0, 2, n_docs)
    z = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)
    n = np.rint(median * np.exp(sigma * z)).astype(np.int64)
    return np.clip(n, lo, hi)


def doc_lengths_exact_total(seed: int, n_docs: int, total: int, block: int = 64,
                            median: float = 900.0, sigma: float = 0.5,
                            lo: int = 64, hi: int = 8192) -> np.ndarray:
    """Lognormal lengths rounded to multiples of ``block`` and nudged by +-block on
    hashed documents until they sum to ``total`` exactly."""
    assert total % block == 0
    n = doc_lengths_lognormal(seed, n_docs, median, sigma, lo, hi)
    n = np.clip(np.rint(n / block).astype(np.int64) * block, block, (hi // block) * block)
    excess = (int(n.sum()) - total) // block
    step = -block if excess > 0 else block
    key = tensor_key(seed, STREAM_DOCLEN, 0, 3)
    cand = (hashes(key, np.arange(8 * abs(excess) + 64, dtype=np.uint64))
            % np.uint64(n_docs)).astype(np.int64)
    i = 0
    while excess != 0:
        d = int(cand[i])
        i += 1
        nv = n[d] + step
        if block <= nv <= (hi // block) * block:
            n[d] = nv
            excess += -1 if step < 0 else 1
    return n


def offsets(lengths: np.ndarray) -> np.ndarray:
    o = np.zeros(len(lengths) + 1, dtype=np.int64)
    np.cumsum(lengths, out=o[1:])
    return o


def topics(seed: int, n_docs: int, d: int = 128, norm: float = 4.0) -> np.ndarray:
    """One d-vector per document, Irwin-Hall draws rescaled to the given norm."""
    t = fill(seed, STREAM_TOPIC, 0, 0, 0, n_docs, d).astype(np.float64)
    t *= norm / np.linalg.norm(t, axis=1, keepdims=True)
    return t.astype(np.float32)


def pick_targets(seed: int, n_docs: int, n_targets: int, sub: int = 0) -> np.ndarray:
    """n_targets distinct document ids chosen by hashing."""
    key = tensor_key(seed, STREAM_TARGETS, 0, sub)
    out: list[int] = []
    i = 0
    while len(out) < n_targets:
        d = int(hashes(key, np.array([i], dtype=np.uint64))[0] % np.uint64(n_docs))
        i += 1
        if d not in out:
            out.append(d)
    return np.array(out, dtype=np.int64)


def token_docs(doc_tok_offsets: np.ndarray) -> np.ndarray:
    """Document id of every token (the per-token doc_ids array of the pages)."""
    lens = np.diff(doc_tok_offsets)
    return np.repeat(np.arange(len(lens), dtype=np.int32), lens)


def query_router(seed: int, layer: int, q_index: int, T: int, n_q_heads: int, d: int,
                 topic: np.ndarray, targets: np.ndarray, noise: float = 0.5,
                 dtype: str = "f32") -> np.ndarray:
    """Router queries Q_r [T][Hq][d]: token t carries topic(targets[t mod n]) plus noise
    in every query head."""
    rt = np.asarray(targets, dtype=np.int64)[np.arange(T) % len(targets)]
    # row = (t, h): the topic row index repeats over heads
    row_topic = np.repeat(rt, n_q_heads)
    x = fill(seed, STREAM_QR, layer, q_index, 0, T * n_q_heads, d, sigma=noise,
             topic=topic, row_topic=row_topic, dtype=dtype)
    return x.reshape(T, n_q_heads, d)


@dataclass
class BankSpec:
    """A synthetic memory bank: document lengths and the draw parameters."""
    seed: int
    n_docs: int
    lengths: np.ndarray
    n_layers: int
    n_heads: int = 8
    head_dim: int = 128
    chunk: int = 64
    topic_norm: float = 4.0
    topic: np.ndarray = field(default=None, repr=False)

    @property
    def doc_tok_offsets(self) -> np.ndarray:
        return offsets(self.lengths)

    @property
    def chunks_per_doc(self) -> np.ndarray:
        return (self.lengths + self.chunk - 1) // self.chunk

    @property
    def doc_chunk_offsets(self) -> np.ndarray:
        return offsets(self.chunks_per_doc)

    @property
    def n_tokens(self) -> int:
        return int(self.lengths.sum())

    @property
    def n_chunks(self) -> int:
        return int(self.chunks_per_doc.sum())


def make_bank(seed: int, n_docs: int, lengths: np.ndarray, n_layers: int, **kw) -> BankSpec:
    b = BankSpec(seed=seed, n_docs=n_docs, lengths=np.asarray(lengths, dtype=np.int64),
                 n_layers=n_layers, **kw)
    b.topic = topics(seed, n_docs, b.head_dim, b.topic_norm)
    return b


def raw_tokens(bank: BankSpec, layer: int, stream: int, tok0: int, n_tok: int,
               dtype: str = "f32") -> np.ndarray:
    """Raw per-token K, V or K_r rows [n_tok][H][d]; K_r rows add their document's topic."""
    rl = bank.n_heads * bank.head_dim
    rt = None
    if stream == STREAM_KR:
        rt = token_docs(bank.doc_tok_offsets)[tok0:tok0 + n_tok]
    x = fill(bank.seed, stream, layer, 0, tok0, n_tok, rl, topic=bank.topic if rt is not None else None,
             row_topic=rt, dtype=dtype)
    return x.reshape(n_tok, bank.n_heads, bank.head_dim)


def chunk_docs(doc_chunk_offsets: np.ndarray) -> np.ndarray:
    lens = np.diff(doc_chunk_offsets)
    return np.repeat(np.arange(len(lens), dtype=np.int32), lens)


POOLED_NOISE = 0.125  # noise std of the mean of 64 unit-variance tokens


def pooled_router_keys(bank: BankSpec, layer: int, c0: int, n_c: int, dtype: str = "bf16") -> np.ndarray:
    """Pooled-level routing keys [n_c][H][d]: document topic + noise/8, drawn directly
    (used where materialising the raw tokens is out of reach)."""
    rl = bank.n_heads * bank.head_dim
    rt = chunk_docs(bank.doc_chunk_offsets)[c0:c0 + n_c]
    x = fill(bank.seed, STREAM_KRBAR, layer, 0, c0, n_c, rl, sigma=POOLED_NOISE,
             topic=bank.topic, row_topic=rt, dtype=dtype)
    return x.reshape(n_c, bank.n_heads, bank.head_dim)


def pooled_content(bank: BankSpec, layer: int, c0: int, n_c: int, dtype: str = "bf16") -> np.ndarray:
    """Pooled-level content rows [n_c][2][H][d] (K-bar then V-bar), noise/8."""
    rl = bank.n_heads * bank.head_dim
    k = fill(bank.seed, STREAM_KBAR, layer, 0, c0, n_c, rl, sigma=POOLED_NOISE, dtype=dtype)
    v = fill(bank.seed, STREAM_VBAR, layer, 0, c0, n_c, rl, sigma=POOLED_NOISE, dtype=dtype)
    return np.stack([k, v], axis=1).reshape(n_c, 2, bank.n_heads, bank.head_dim)


# ----------------------------------------------------------------------------- device fill

_dev_lib = None


def _device_lib():
    import ctypes
    import os
    global _dev_lib
    if _dev_lib is None:
        path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmsa_synth.so")
        if not os.path.exists(path):
            raise ImportError(f"{path} missing: run python -m top_kv_routing_b200.build")
        lib = ctypes.CDLL(path)
        lib.msa_synth_fill.argtypes = [ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint64, ctypes.c_uint32,
                                       ctypes.c_uint32, ctypes.c_uint32, ctypes.c_int64, ctypes.c_int64,
                                       ctypes.c_int32, ctypes.c_float, ctypes.c_void_p, ctypes.c_int32,
                                       ctypes.c_void_p, ctypes.c_void_p]
        lib.msa_synth_fill.restype = ctypes.c_int32
        _dev_lib = lib
    return _dev_lib


def device_fill(dst, seed: int, stream: int, layer: int, sub: int, row0: int, n_rows: int, row_len: int,
                sigma: float = 1.0, topic=None, row_topic=None, cuda_stream=None) -> None:
    """Same values as ``fill`` written by a GPU kernel into the torch tensor ``dst``
    (fp32 or bf16, contiguous, >= n_rows*row_len elements).  topic / row_topic are
    device tensors (fp32 [n][tlen], int32 [n_rows]) or None."""
    import torch
    dtype = 1 if dst.dtype == torch.bfloat16 else 0
    s = torch.cuda.current_stream().cuda_stream if cuda_stream is None else cuda_stream
    tl = 0 if topic is None else int(topic.shape[-1])
    r = _device_lib().msa_synth_fill(dst.data_ptr(), dtype, seed, stream, layer, sub, row0, n_rows, row_len,
                                     sigma, None if topic is None else topic.data_ptr(), tl,
                                     None if row_topic is None else row_topic.data_ptr(), s)
    if r != 0:
        raise RuntimeError(f"msa_synth_fill failed ({r})")
