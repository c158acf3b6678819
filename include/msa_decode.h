/* Step 4 of the MSA hot path: sparse decode attention of one new token over
 * [selected compressed memory ; the query's local KV], with global RoPE offset by k.
 *
 * Defined by: "MSA端到端可训练记忆模型完整开源，支持亿级Token上下文", section 架构 (the selected
 * documents' compressed K/V are concatenated with the query's local K/V for autoregressive
 * decoding; 全局 RoPE: the query's start index is offset by k, keeping the order background
 * -> query -> generation) and section 推理流水线 step 3 (sparse generation); MSA paper
 * reading notes, section 推理全流程 (attention context = [Top-16 compressed KV ; local KV];
 * the local KV grows per token while the memory KV stays fixed).
 */
#ifndef MSA_DECODE_H
#define MSA_DECODE_H

#include "msa_common.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Workspace bytes of one msa_sparse_decode call (partial softmax sums of up to 4 key
 * splits per (query, layer, key head), and the arrival counters). */
msa_status msa_sparse_decode_workspace_size(int32_t n_queries, int32_t n_layers, int32_t n_q_heads,
                                            int32_t n_kv_heads, size_t* bytes);

/* One decode step for every query b and layer l.  With i = local_len[b] (read on the
 * device) and p = rope_pos_offset + i:
 *   q' = RoPE(q, p), k' = RoPE(k_new, p)  (rotate-half, angle p * theta^(-2j/d), fp64-reduced)
 *   local_k[b][l][h][i] = bf16(k'), local_v[b][l][h][i] = v_new       (append)
 *   keys/values = mem_kv[b][l][0/1][h][0 .. mem_len[b][l]) followed by local[0 .. i]
 *                 (memory keys keep the document-wise rotation applied at encode time;
 *                  no mask: the memory precedes the query)
 *   out[b][l][hq] = softmax(softmax_scale * <q'_hq, K_j>) . V_j with key head h = hq / G
 *                 (fp32 scores, running max and sums; output rounded to bf16)
 * then local_len[b] += 1.
 *   q       DEVICE bf16 [n_queries][n_layers][n_q_heads][head_dim]
 *   k_new, v_new  DEVICE bf16 [n_queries][n_layers][n_kv_heads][head_dim]
 *   local_k, local_v  DEVICE bf16 [n_queries][n_layers][n_kv_heads][local_cap][head_dim]
 *   local_len DEVICE int32 [n_queries], read and advanced by the call
 *   mem_kv  DEVICE bf16 [n_queries][n_layers][2][n_kv_heads][max_mem_chunks][head_dim]
 *           (msa_gather_kv output); mem_len DEVICE int32 [n_queries][n_layers]
 *   out     DEVICE bf16 [n_queries][n_layers][n_q_heads][head_dim]
 *   head_dim = 128; n_q_heads / n_kv_heads in {1, 2, 4, 8}; n_kv_heads <= 16.
 *   q, mem_kv, local_k, local_v  16-byte aligned.
 *   workspace  DEVICE, >= msa_sparse_decode_workspace_size bytes, 16-byte aligned, zeroed
 *              (e.g. cudaMemset) once before its first use; every call leaves it ready for
 *              the next (its arrival counters return to zero).  Calls that share a
 *              workspace must not overlap on the device.
 * One CTA per (query, layer, key head) streams its keys in tiles of 16 through the tensor
 * cores; when there are fewer such units than SMs, the keys of each are split over up to
 * 4 CTAs and the last of them to finish merges the partial softmax sums.  Every CTA of
 * a query announces on an arrival counter that it has read local_len; the last one
 * advances it.
 * A query whose cache is full (local_len >= local_cap) is skipped (out untouched, length
 * not advanced) and sets MSA_DEVERR_LOCAL_FULL; mem_len > max_mem_chunks is clamped with
 * MSA_DEVERR_CAPACITY.  One kernel launch, asynchronous on stream, graph-capturable
 * (every per-step quantity is read on the device).  The kernel is launched as a
 * programmatic dependent of the kernel before it on the stream: it may be scheduled while
 * that kernel finishes, and it reads every input only after waiting for it, so inputs that
 * the preceding kernel or copy writes (msa_gather_kv's mem_len, this step's q) are seen. */
msa_status msa_sparse_decode(const void* q, const void* k_new, const void* v_new, int32_t n_queries,
                             int32_t n_layers, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                             void* local_k, void* local_v, int32_t* local_len, int32_t local_cap,
                             const void* mem_kv, const int32_t* mem_len, int32_t max_mem_chunks,
                             int32_t rope_pos_offset, float rope_theta, float softmax_scale, void* out,
                             void* workspace, size_t workspace_bytes, int32_t* dev_err, msa_stream_t stream);

/* msa_sparse_decode without a caller workspace.  There is no counterpart in the MSA
 * pages: this exists for callers that cannot allocate device memory at all (for example
 * a host that hands the library only the buffers it already owns, or code running where
 * allocation is forbidden mid-stream).  The scratch is a fixed array inside this library,
 * MSA_DECODE_STATIC_SCRATCH_BYTES in size, which every GPU that loads the library keeps
 * until the process exits; sizes that need more fail with MSA_ERR_CAPACITY.  A call needs
 * n_queries * n_layers * n_kv_heads * (2080 * G + 4) + 4 * n_queries bytes (G = n_q_heads /
 * n_kv_heads): at 18 layers, 8 key heads and G = 4, six queries fit.  The first
 * call on a device looks the array's device address up (issue that first call before any
 * stream capture).  Each call clears the part that must start at zero with one
 * cudaMemsetAsync on `stream` and allocates nothing.  All calls share the one array:
 * calls that overlap on the GPU (other streams, other threads) race and must be
 * serialised by the caller.  Same arguments, results and errors as msa_sparse_decode. */
#define MSA_DECODE_STATIC_SCRATCH_BYTES (8u << 20)
msa_status msa_sparse_decode_static(const void* q, const void* k_new, const void* v_new, int32_t n_queries,
                                    int32_t n_layers, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                    void* local_k, void* local_v, int32_t* local_len, int32_t local_cap,
                                    const void* mem_kv, const int32_t* mem_len, int32_t max_mem_chunks,
                                    int32_t rope_pos_offset, float rope_theta, float softmax_scale, void* out,
                                    int32_t* dev_err, msa_stream_t stream);

const char* msa_decode_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* MSA_DECODE_H */
