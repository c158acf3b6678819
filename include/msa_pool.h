/* Step 1 of the MSA hot path: offline block compression of one layer of the memory bank.
 *
 * Defined by: "MSA端到端可训练记忆模型完整开源，支持亿级Token上下文", section 架构 (document
 * hidden states K/V/K_r are compressed by block-wise mean pooling; 并行 RoPE restarts
 * positions at 0 in every document) and section 推理流水线 step 1 (global memory encoding
 * caches the pooled K-bar, V-bar, K-bar_r); MSA paper reading notes, section 路由投影器 +
 * Top-k 稀疏注意力 (fixed blocks of 64 tokens, 64 -> 1) and section 文档级 RoPE.
 */
#ifndef MSA_POOL_H
#define MSA_POOL_H

#include "msa_common.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Number of memory blocks of a bank: sum over documents of ceil(n_tokens / chunk).
 * doc_tok_offsets_host: HOST [n_docs + 1], non-decreasing, starting at 0.
 * doc_chunk_offsets_host: HOST [n_docs + 1] output (may be NULL).
 * Returns the block count, or -1 on a bad argument. */
int64_t msa_count_chunks(const int64_t* doc_tok_offsets_host, int32_t n_docs, int32_t chunk,
                         int64_t* doc_chunk_offsets_host);

/* Pools one layer.  For each document d and its token i (position i - start_d):
 *   K'_i   = RoPE(K_i, i - start_d)     rotate-half pairing (j, j + d/2), angle
 *                                        pos * theta^(-2j/d); skipped when rope_theta == 0
 *   block j of document d covers tokens [chunk*j, min(chunk*(j+1), n_d)) of the document;
 *   k_bar  = mean K', v_bar = mean V over the block's real tokens (a trailing partial
 *            block averages only its own tokens);
 *   kr_hat = m / max(||m||, 1e-8) per head, with m the mean of K_r (the routing key stored
 *            unit-normalised, i.e. with its inverse norm applied at encode time);
 *   kr_norm = ||m|| per (block, head).
 * Arithmetic: fp32 (RoPE angle reduced in fp64), outputs rounded to nearest-even bf16.
 *
 * k, v, kr       DEVICE [n_tok][n_heads][head_dim] in in_dtype (MSA_F32 or MSA_BF16),
 *                token t of the bank at row t; any of the three may be NULL (skipped).
 *                16-byte aligned.
 * doc_tok_offsets, doc_chunk_offsets  DEVICE int64 [n_docs + 1] (see msa_count_chunks).
 * n_chunks       doc_chunk_offsets[n_docs]; a mismatch sets MSA_DEVERR_BAD_OFFSETS.
 * head_dim       must be 128; n_heads in [1, 16]; chunk in [1, 64].
 * k_bar, v_bar, kr_hat  DEVICE bf16 [n_chunks][n_heads][head_dim], NULL to skip (must be
 *                non-NULL when the matching input is); kr_norm DEVICE fp32 [n_chunks][n_heads]
 *                or NULL.
 * dev_err        DEVICE int32 error word (see msa_common.h), or NULL.
 * No workspace.  Asynchronous on stream. */
msa_status msa_pool_blocks(const void* k, const void* v, const void* kr, msa_dtype in_dtype,
                           const int64_t* doc_tok_offsets, const int64_t* doc_chunk_offsets,
                           int32_t n_docs, int64_t n_chunks, int32_t n_heads, int32_t head_dim,
                           int32_t chunk, float rope_theta, void* k_bar, void* v_bar, void* kr_hat,
                           float* kr_norm, int32_t* dev_err, msa_stream_t stream);

const char* msa_pool_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* MSA_POOL_H */
