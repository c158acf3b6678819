"""ctypes wrapper of the CPU oracle (oracle.cpp).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and bench.py's
``cpu_baseline`` / ``--impl reference`` legs are the only callers.  Nothing in the
product package imports this module, and this module imports nothing from it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")

_i32 = ctypes.c_int32
_i64 = ctypes.c_int64
_dbl = ctypes.c_double
_p = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile oracle.cpp (g++, -O2, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math",
                               "-shared", "-fPIC", "-o", _LIB, _SRC])
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.oracle_rope.argtypes = [_p, _i32, _i64, _dbl, _p]
        _lib.oracle_rope.restype = None
        _lib.oracle_count_chunks.argtypes = [_p, _i32, _i32, _p]
        _lib.oracle_count_chunks.restype = _i64
        _lib.oracle_pool.argtypes = [_p, _p, _p, _p, _i32, _i32, _i32, _i32, _dbl, _i32,
                                     _p, _p, _p, _p, _p, _i64]
        _lib.oracle_pool.restype = _i64
        _lib.oracle_topk.argtypes = [_p, _i32, _i32, _p, _p]
        _lib.oracle_topk.restype = None
        for name in ("oracle_route_explicit", "oracle_route_grouped"):
            f = getattr(_lib, name)
            f.argtypes = [_p, _i32, _i32, _p, _i64, _i32, _i32, _p, _i32, _i32, _p, _p, _p, _p]
            f.restype = _i32
        _lib.oracle_gather.argtypes = [_p, _i32, _i64, _i32, _i32, _p, _i32, _p, _i32, _i32, _i32,
                                       _p, _p]
        _lib.oracle_gather.restype = _i32
        _lib.oracle_decode.argtypes = [_p, _p, _p, _p, _i32, _i32, _p, _p, _i32, _i32, _i64, _dbl,
                                       _dbl, _i32, _i32, _i32, _p]
        _lib.oracle_decode.restype = _i32
        _lib.oracle_prefill.argtypes = [_p, _p, _p, _i32, _p, _i32, _i32, _p, _p, _i32, _i32, _i64, _dbl, _dbl,
                                        _i32, _i32, _i32, _p]
        _lib.oracle_prefill.restype = _i32
        _lib.oracle_query_sums.argtypes = [_p, _i32, _i32, _i32, _i32, _p]
        _lib.oracle_query_sums.restype = _i32
        _lib.oracle_router_project.argtypes = [_p, _i32, _i32, _p, _i32, _p]
        _lib.oracle_router_project.restype = None
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f32(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float32)


def rope(x: np.ndarray, pos: int, theta: float) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty_like(x)
    lib().oracle_rope(_ptr(x), x.shape[-1], pos, theta, _ptr(out))
    return out


def count_chunks(doc_tok_offsets: np.ndarray, chunk: int = 64):
    o = np.ascontiguousarray(doc_tok_offsets, dtype=np.int64)
    n_docs = len(o) - 1
    out = np.empty(n_docs + 1, dtype=np.int64)
    total = lib().oracle_count_chunks(_ptr(o), n_docs, chunk, _ptr(out))
    return int(total), out


def pool(k, v, kr, doc_tok_offsets, n_heads: int, head_dim: int, chunk: int = 64,
         theta: float = 1e6, rope_k: bool = True):
    """Returns dict of k_bar, v_bar, kr_bar, kr_unit [C][H][d] and kr_norm [C][H] (double)."""
    o = np.ascontiguousarray(doc_tok_offsets, dtype=np.int64)
    n_docs = len(o) - 1
    C, _ = count_chunks(o, chunk)
    k, v, kr = _f32(k), _f32(v), _f32(kr)
    shape = (C, n_heads, head_dim)
    out = {
        "k_bar": np.zeros(shape) if k is not None else None,
        "v_bar": np.zeros(shape) if v is not None else None,
        "kr_bar": np.zeros(shape) if kr is not None else None,
        "kr_unit": np.zeros(shape) if kr is not None else None,
        "kr_norm": np.zeros((C, n_heads)) if kr is not None else None,
    }
    r = lib().oracle_pool(_ptr(k), _ptr(v), _ptr(kr), _ptr(o), n_docs, n_heads, head_dim, chunk, theta,
                          1 if rope_k else 0, _ptr(out["k_bar"]), _ptr(out["v_bar"]),
                          _ptr(out["kr_bar"]), _ptr(out["kr_unit"]), _ptr(out["kr_norm"]), C)
    assert r == C
    return out


def topk(doc_score: np.ndarray, k: int):
    s = np.ascontiguousarray(doc_score, dtype=np.float64)
    ids = np.empty(k, dtype=np.int32)
    sc = np.empty(k, dtype=np.float64)
    lib().oracle_topk(_ptr(s), len(s), k, _ptr(ids), _ptr(sc))
    return ids, sc


def route(qr, kr, doc_chunk_offsets, top_k: int, grouped: bool = False):
    """One layer, one query.  qr [T][Hq][d], kr [C][H][d].
    Returns (ids [k], scores [k], doc_score [D], chunk_score [C])."""
    qr = _f32(qr)
    kr = _f32(kr)
    o = np.ascontiguousarray(doc_chunk_offsets, dtype=np.int64)
    T, Hq, d = qr.shape
    C, H, d2 = kr.shape
    assert d == d2 and o[-1] == C
    n_docs = len(o) - 1
    doc_score = np.empty(n_docs, dtype=np.float64)
    chunk_score = np.empty(C, dtype=np.float64)
    ids = np.empty(top_k, dtype=np.int32)
    sc = np.empty(top_k, dtype=np.float64)
    f = lib().oracle_route_grouped if grouped else lib().oracle_route_explicit
    r = f(_ptr(qr), T, Hq, _ptr(kr), C, H, d, _ptr(o), n_docs, top_k, _ptr(doc_score),
          _ptr(chunk_score), _ptr(ids), _ptr(sc))
    if r != 0:
        raise ValueError("oracle route: bad head counts")
    return ids, sc, doc_score, chunk_score


def query_sums(qr, n_kv_heads: int):
    """The grouped routing form's query operand: qr [T][Hq][d] -> qt [T][H][d] (double),
    qt[t][g] = (1/Hq) sum of the unit query heads h with h / (Hq/H) == g."""
    qr = _f32(qr)
    T, Hq, d = qr.shape
    out = np.empty((T, n_kv_heads, d), dtype=np.float64)
    if lib().oracle_query_sums(_ptr(qr), T, Hq, n_kv_heads, d, _ptr(out)) != 0:
        raise ValueError("oracle query_sums: bad head counts")
    return out


def gather(host_kv_bits, doc_chunk_offsets, ids, max_mem_chunks: int):
    """host_kv_bits [L][C][2][H][d] uint16; ids [B][L][k] int32.
    Returns (out [B][L][2][H][M_max][d] uint16 (zeros past mem_len), mem_len [B][L])."""
    hk = np.ascontiguousarray(host_kv_bits, dtype=np.uint16)
    L, C, two, H, d = hk.shape
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    B, L2, k = ids.shape
    assert L2 == L and two == 2
    o = np.ascontiguousarray(doc_chunk_offsets, dtype=np.int64)
    out = np.zeros((B, L, 2, H, max_mem_chunks, d), dtype=np.uint16)
    mem_len = np.zeros((B, L), dtype=np.int32)
    r = lib().oracle_gather(_ptr(hk), L, C, H, d, _ptr(o), len(o) - 1, _ptr(ids), B, k, max_mem_chunks,
                            _ptr(out), _ptr(mem_len))
    if r == -1:
        raise ValueError("oracle gather: bad document id")
    if r == -2:
        raise OverflowError("oracle gather: selection exceeds max_mem_chunks")
    return out, mem_len


def decode(q, k_new, v_new, mem_kv, mem_len: int, local_k, local_v, local_len: int, pos: int,
           theta: float, scale: float):
    """One token for one (sequence, layer).  q [Hq][d], k_new/v_new [H][d],
    mem_kv [2][H][M_stride][d], local_k/local_v [H][Lcap][d] float64 (updated in place).
    Returns out [Hq][d] (double)."""
    q, k_new, v_new, mem_kv = _f32(q), _f32(k_new), _f32(v_new), _f32(mem_kv)
    Hq, d = q.shape
    H = k_new.shape[0]
    M_stride = mem_kv.shape[2]
    assert local_k.dtype == np.float64 and local_k.flags.c_contiguous
    assert local_v.dtype == np.float64 and local_v.flags.c_contiguous
    Lcap = local_k.shape[1]
    out = np.empty((Hq, d), dtype=np.float64)
    r = lib().oracle_decode(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(mem_kv), mem_len, M_stride,
                            _ptr(local_k), _ptr(local_v), local_len, Lcap, pos, theta, scale, Hq, H, d,
                            _ptr(out))
    if r != 0:
        raise OverflowError("oracle decode: local cache full")
    return out


def prefill(q, k_new, v_new, mem_kv, mem_len: int, local_k, local_v, local_len: int, pos: int, theta: float,
            scale: float):
    """n new tokens for one (sequence, layer): token i is the decode step at local index
    local_len + i, position pos + i.  q [n][Hq][d], k_new/v_new [n][H][d], mem_kv
    [2][H][M_stride][d], local_k/local_v [H][Lcap][d] float64 (updated in place).
    Returns out [n][Hq][d] (double)."""
    q, k_new, v_new, mem_kv = _f32(q), _f32(k_new), _f32(v_new), _f32(mem_kv)
    n, Hq, d = q.shape
    H = k_new.shape[1]
    M_stride = mem_kv.shape[2]
    assert local_k.dtype == np.float64 and local_k.flags.c_contiguous
    assert local_v.dtype == np.float64 and local_v.flags.c_contiguous
    Lcap = local_k.shape[1]
    out = np.empty((n, Hq, d), dtype=np.float64)
    r = lib().oracle_prefill(_ptr(q), _ptr(k_new), _ptr(v_new), n, _ptr(mem_kv), mem_len, M_stride, _ptr(local_k),
                             _ptr(local_v), local_len, Lcap, pos, theta, scale, Hq, H, d, _ptr(out))
    if r != 0:
        raise OverflowError("oracle prefill: local cache full")
    return out


def router_project(h, w, n_q_heads: int):
    """Router query projection of one layer ("【MSA】突破100M Token 上下文：记忆稀疏注意力架构深度解析",
    section 5.1: the decoupled, bias-free router_q_proj): h [T][hidden] times
    w [n_q_heads * d][hidden] transposed.  Returns Q_r [T][n_q_heads][d] (double)."""
    h, w = _f32(h), _f32(w)
    T, hidden = h.shape
    F, hidden2 = w.shape
    assert hidden == hidden2 and F % n_q_heads == 0
    out = np.empty((T, F), dtype=np.float64)
    lib().oracle_router_project(_ptr(h), T, hidden, _ptr(w), F, _ptr(out))
    return out.reshape(T, n_q_heads, F // n_q_heads)


def layer_mean_topk(doc_scores, k: int):
    """Layer-aggregated selection: one top-k shared by every routing layer, ranking the
    documents by the mean over layers of their per-layer document scores (a document with
    no block scores -inf in every layer and so in the mean).  doc_scores [L][n_docs].
    Returns (ids [k], scores [k], mean [n_docs]).

    The pages give the per-layer document score ("MSA端到端可训练记忆模型完整开源，支持亿级Token
    上下文", section 架构: mean over heads, max over tokens) and one top-16 selection per query
    (MSA paper reading notes, section 路由投影器 + Top-k 稀疏注意力); where one selection is to
    serve all routing layers, this takes the plain reading that the layers' document scores
    are averaged, and ranks as the per-layer top-k does (score descending, then id)."""
    ds = np.asarray(doc_scores, dtype=np.float64)
    L = ds.shape[0]
    mean = np.empty(ds.shape[1], dtype=np.float64)
    for d in range(ds.shape[1]):  # in layer order, as written
        col = ds[:, d]
        mean[d] = -np.inf if np.isneginf(col).any() else sum(float(x) for x in col) / L
    ids, sc = topk(mean, k)
    return ids, sc, mean


def route_layer_mean(q_layers, kr_layers, doc_chunk_offsets, top_k: int):
    """Routing of one query with the layer-aggregated selection: q_layers [L][T][Hq][d],
    kr_layers [L][C][H][d].  Each layer's document scores are the grouped routing form
    (route(..., grouped=True)), then layer_mean_topk.  Returns (ids [k], scores [k], mean
    doc scores [n_docs])."""
    per_layer = [route(q, kr, doc_chunk_offsets, top_k, grouped=True)[2] for q, kr in zip(q_layers, kr_layers)]
    return layer_mean_topk(np.stack(per_layer), top_k)
