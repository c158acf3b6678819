/* Query prefill through sparse attention: a block of n_new tokens per query attends to
 * [selected compressed memory ; the query's local KV up to and including each token].
 *
 * Defined by: "MSA端到端可训练记忆模型完整开源，支持亿级Token上下文", section 推理流水线 (the
 * question is processed over the retrieved documents' compressed K/V joined to the local
 * context, then generation proceeds token by token) and section 架构 (全局 RoPE: positions of
 * the query's tokens are offset by k); MSA paper reading notes, section 推理全流程 (memory
 * KV fixed, local KV grows).  Token i of the block is exactly the decode step at local
 * index local_len + i (msa_decode.h); the block computes all n_new of them at once.
 */
#ifndef MSA_PREFILL_H
#define MSA_PREFILL_H

#include "msa_common.h"

#ifdef __cplusplus
extern "C" {
#endif

/* For every query b and layer l, with i0 = local_len[b] (read on the device) and, for
 * token i in [0, n_new), local index i0 + i and position p_i = rope_pos_offset + i0 + i:
 *   k'_i = RoPE(k_new_i, p_i), q'_i = RoPE(q_i, p_i)  (rotate-half, angle p * theta^(-2j/d),
 *                                                       fp64-reduced)
 *   local_k[b][l][h][i0 + i] = bf16(k'_i), local_v[b][l][h][i0 + i] = v_new_i   (append)
 *   keys/values of token i = mem_kv[b][l][0/1][h][0 .. mem_len[b][l]) followed by local
 *                            rows 0 .. i0 + i (causal inside the block; the memory and the
 *                            earlier local rows are visible to every token)
 *   out[b][l][i][hq] = softmax(softmax_scale * <q'_i,hq, K_j>) . V_j, key head h = hq / G
 *                      (fp32 scores, running max and sums; output rounded to bf16)
 * then local_len[b] += n_new.
 *   q       DEVICE bf16 [n_queries][n_layers][n_new][n_q_heads][head_dim]
 *   k_new, v_new  DEVICE bf16 [n_queries][n_layers][n_new][n_kv_heads][head_dim]
 *   local_k, local_v  DEVICE bf16 [n_queries][n_layers][n_kv_heads][local_cap][head_dim]
 *   local_len DEVICE int32 [n_queries], read and advanced by the call
 *   mem_kv  DEVICE bf16 [n_queries][n_layers][2][n_kv_heads][max_mem_chunks][head_dim]
 *           (msa_gather_kv output); mem_len DEVICE int32 [n_queries][n_layers]
 *   out     DEVICE bf16 [n_queries][n_layers][n_new][n_q_heads][head_dim]
 *   head_dim = 128; n_q_heads / n_kv_heads in {1, 2, 4, 8}; n_kv_heads <= 16;
 *   n_queries * n_layers <= 65535.  q, k_new, v_new, mem_kv, local_k, local_v, out 16-byte
 *   aligned.
 *   The caller owns every buffer; the call allocates nothing.
 * Three kernel launches on `stream` (append, attention, advance), asynchronous and
 * graph-capturable (every per-call quantity that changes is read on the device).  The
 * attention kernel runs on the tcgen05 tensor cores: at most one CTA per SM, each walking
 * units of 128 (token, query head) rows (the MMA's M) of its share of the (query, layer,
 * key head, token tile) list, K/V streaming in tiles of 64 keys, the query, scores,
 * weights and output in tensor memory.
 * A query whose cache cannot hold the whole block (local_len + n_new > local_cap) is
 * skipped (out and cache untouched, length not advanced) and sets MSA_DEVERR_LOCAL_FULL;
 * mem_len > max_mem_chunks is clamped with MSA_DEVERR_CAPACITY.  Host-checked argument
 * errors return MSA_ERR_INVALID_ARG before any launch; a device other than sm_100
 * returns MSA_ERR_UNSUPPORTED. */
msa_status msa_sparse_prefill(const void* q, const void* k_new, const void* v_new, int32_t n_new, int32_t n_queries,
                              int32_t n_layers, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                              void* local_k, void* local_v, int32_t* local_len, int32_t local_cap,
                              const void* mem_kv, const int32_t* mem_len, int32_t max_mem_chunks,
                              int32_t rope_pos_offset, float rope_theta, float softmax_scale, void* out,
                              int32_t* dev_err, msa_stream_t stream);

const char* msa_prefill_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* MSA_PREFILL_H */
