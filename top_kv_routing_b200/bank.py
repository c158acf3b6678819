"""A pooled memory bank as one object: encode documents, append new ones without
re-encoding the old, save to and load from a bank file (include/msa_bank.h).

Follows "【MSA】突破100M Token 上下文：记忆稀疏注意力架构深度解析", section 8.3 (documents encoded
once into K̄/V̄/K̄ᵣ, saved, loaded for inference) and "把一亿 token 装进模型的“记忆”里…", section
5.2 (documents are encoded independently, so new ones can be appended).  The arithmetic
runs in the pool and filter-key kernels; this module allocates, sequences and moves bytes.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from .abi import (MSA_BANK_KR, MSA_BANK_KR_F8, MSA_BANK_KV, MSA_BANK_NORM, MSA_BF16, MSA_F32, MsaBankInfo,
                  msa_bank_append_offsets, msa_bank_load, msa_bank_read_info, msa_bank_relayout, msa_bank_save,
                  msa_count_chunks, msa_pool_blocks, msa_route_filter_keys)

STAGING_BYTES = 64 << 20


@dataclass
class PooledBank:
    """kr_hat bf16 [L][C][H][d] (device), kr_f8 uint8 [L][C][H][d] or None (device),
    content bf16 [L][C][2][H][d] (page-locked host or device), kr_norm fp32 [L][C][H]
    (device), doc_chunk_offsets int64 [n_docs + 1] (host)."""
    kr_hat: torch.Tensor
    kr_f8: torch.Tensor | None
    content: torch.Tensor
    kr_norm: torch.Tensor
    doc_chunk_offsets: np.ndarray
    block_tokens: int = 64

    @property
    def n_layers(self) -> int:
        return self.kr_hat.shape[0]

    @property
    def n_blocks(self) -> int:
        return int(self.doc_chunk_offsets[-1])

    @property
    def n_docs(self) -> int:
        return len(self.doc_chunk_offsets) - 1


def _pool_layers(k, v, kr, doc_tok_offsets, n_docs, theta, block_tokens, kr_hat_rows, kr_norm_rows, content_rows,
                 f8_rows, stream=None):
    """Pools every layer of raw tokens k, v, kr [L][n_tok][H][d] into the given row views
    (each [L][C_new][...], contiguous per layer)."""
    L, _, H, D = kr.shape
    C, coffs = msa_count_chunks(doc_tok_offsets, block_tokens)
    if C == 0:
        return
    dev = kr.device
    toff = torch.from_numpy(np.ascontiguousarray(doc_tok_offsets, dtype=np.int64)).to(dev)
    coff = torch.from_numpy(coffs).to(dev)
    kb = torch.empty((C, H, D), dtype=torch.bfloat16, device=dev)
    vb = torch.empty_like(kb)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    dt = MSA_BF16 if kr.dtype == torch.bfloat16 else MSA_F32
    for l in range(L):
        msa_pool_blocks(k[l], v[l], kr[l], toff, coff, n_docs, C, H, D, block_tokens, theta, kb, vb, kr_hat_rows[l],
                        kr_norm_rows[l], err, in_dtype=dt, stream=stream)
        content_rows[l, :, 0].copy_(kb, non_blocking=True)
        content_rows[l, :, 1].copy_(vb, non_blocking=True)
        if f8_rows is not None:
            msa_route_filter_keys(kr_hat_rows[l], 1, C, H, D, f8_rows[l], stream=stream)
    torch.cuda.synchronize(dev)
    if int(err.item()):
        raise RuntimeError(f"pooling reported device error bits {int(err.item())}")


def encode(k, v, kr, doc_tok_offsets, theta: float = 1e6, block_tokens: int = 64, with_f8: bool = True,
           content_on_host: bool = False) -> PooledBank:
    """Pools raw tokens k, v, kr [L][n_tok][H][d] (device, bf16 or fp32) of documents with
    token offsets doc_tok_offsets [n_docs + 1] into a new bank."""
    L, _, H, D = kr.shape
    n_docs = len(doc_tok_offsets) - 1
    C, coffs = msa_count_chunks(doc_tok_offsets, block_tokens)
    dev = kr.device
    kr_hat = torch.empty((L, C, H, D), dtype=torch.bfloat16, device=dev)
    kr_norm = torch.empty((L, C, H), dtype=torch.float32, device=dev)
    content = torch.empty((L, C, 2, H, D), dtype=torch.bfloat16, device="cpu" if content_on_host else dev,
                          pin_memory=content_on_host)
    kr_f8 = torch.empty((L, C, H, D), dtype=torch.uint8, device=dev) if with_f8 else None
    _pool_layers(k, v, kr, doc_tok_offsets, n_docs, theta, block_tokens, kr_hat, kr_norm, content, kr_f8)
    return PooledBank(kr_hat, kr_f8, content, kr_norm, coffs, block_tokens)


def append(bank: PooledBank, k, v, kr, doc_tok_offsets, theta: float = 1e6) -> PooledBank:
    """A new bank = bank's documents followed by the documents of the raw tokens k, v, kr
    [L][n_tok][H][d] (token offsets doc_tok_offsets): the old blocks are copied, not
    re-encoded; only the new documents are pooled (and given E4M3 filter keys)."""
    L, C0 = bank.n_layers, bank.n_blocks
    n_new = len(doc_tok_offsets) - 1
    Cn, coffs = msa_count_chunks(doc_tok_offsets, bank.block_tokens)
    C = C0 + Cn
    H, D = bank.kr_hat.shape[2], bank.kr_hat.shape[3]
    dev = bank.kr_hat.device

    def grown(old, shape_tail, dtype, device, pin=False):
        new = torch.empty((L, C) + shape_tail, dtype=dtype, device=device, pin_memory=pin)
        row = int(np.prod(shape_tail)) * new.element_size()
        msa_bank_relayout(old, new, L, C0, C, row)
        return new

    kr_hat = grown(bank.kr_hat, (H, D), torch.bfloat16, dev)
    kr_norm = grown(bank.kr_norm, (H,), torch.float32, dev)
    host = bank.content.device.type == "cpu"
    content = grown(bank.content, (2, H, D), torch.bfloat16, bank.content.device, pin=host)
    kr_f8 = grown(bank.kr_f8, (H, D), torch.uint8, dev) if bank.kr_f8 is not None else None
    _pool_layers(k, v, kr, doc_tok_offsets, n_new, theta, bank.block_tokens, kr_hat[:, C0:], kr_norm[:, C0:],
                 content[:, C0:], kr_f8[:, C0:] if kr_f8 is not None else None)
    offs = msa_bank_append_offsets(bank.doc_chunk_offsets, coffs)
    return PooledBank(kr_hat, kr_f8, content, kr_norm, offs, bank.block_tokens)


def save(bank: PooledBank, path) -> None:
    fields = MSA_BANK_KR | MSA_BANK_KV | MSA_BANK_NORM | (MSA_BANK_KR_F8 if bank.kr_f8 is not None else 0)
    info = MsaBankInfo(n_layers=bank.n_layers, n_heads=bank.kr_hat.shape[2], head_dim=bank.kr_hat.shape[3],
                       block_tokens=bank.block_tokens, n_docs=bank.n_docs, n_blocks=bank.n_blocks, fields=fields)
    staging = torch.empty(STAGING_BYTES, dtype=torch.uint8, pin_memory=True)
    msa_bank_save(path, info, bank.doc_chunk_offsets, bank.kr_hat, bank.kr_f8, bank.content, bank.kr_norm, staging)


def load(path, device="cuda", content_on_host: bool = True) -> PooledBank:
    info = msa_bank_read_info(path)
    L, C, H, D = info.n_layers, info.n_blocks, info.n_heads, info.head_dim
    if not (info.fields & MSA_BANK_KR and info.fields & MSA_BANK_KV and info.fields & MSA_BANK_NORM):
        raise ValueError(f"{path}: a bank file needs routing keys, content and norms")
    offs = np.empty(info.n_docs + 1, dtype=np.int64)
    kr_hat = torch.empty((L, C, H, D), dtype=torch.bfloat16, device=device)
    kr_norm = torch.empty((L, C, H), dtype=torch.float32, device=device)
    content = torch.empty((L, C, 2, H, D), dtype=torch.bfloat16, device="cpu" if content_on_host else device,
                          pin_memory=content_on_host)
    kr_f8 = torch.empty((L, C, H, D), dtype=torch.uint8, device=device) if info.fields & MSA_BANK_KR_F8 else None
    staging = torch.empty(STAGING_BYTES, dtype=torch.uint8, pin_memory=True)
    msa_bank_load(path, offs, kr_hat, kr_f8, content, kr_norm, staging)
    return PooledBank(kr_hat, kr_f8, content, kr_norm, offs, info.block_tokens)
