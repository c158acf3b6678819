/* Step 2 of the MSA hot path: online routing of queries over the pooled routing keys
 * with fused top-k document selection.
 *
 * Defined by: "MSA端到端可训练记忆模型完整开源，支持亿级Token上下文", section 架构 (cosine
 * similarity of router query Q_r and pooled router key K-bar_r, mean over attention heads
 * first, then max over query tokens, Top-k documents) and section 推理流水线 step 2 (the
 * query is projected to Q_r and matched against K-bar_r); MSA paper reading notes, section
 * 路由投影器 + Top-k 稀疏注意力 (Top-16 documents, cosine against every document) and
 * section KV 缓存压缩 + Memory Parallel (routing keys stay in GPU memory and every query
 * scans them all).
 *
 * For query b, layer l, query token t, query head h (G = n_q_heads / n_kv_heads):
 *   s[t][c]  = (1/Hq) sum_h cos(Q_r[t][h], K-bar_r[c][h / G])
 *   m[c]     = max over the query's tokens of s[t][c]
 *   S[doc]   = max over the document's blocks of m[c]     (a document with no block: -inf)
 *   ids      = the top_k documents by S, descending, equal scores -> smaller id first;
 *              fewer than top_k documents -> id -1, score -inf.
 * The [T x C] score matrix is never stored.  Computed as
 *   s[t][c] = < (1/Hq) sum_{h: h/G = g} Q_r[t][h] / max(||Q_r[t][h]||, 1e-8) , kr_hat[c][g] >
 * summed over key heads g, with kr_hat the unit routing keys written by msa_pool_blocks,
 * in fp32 accumulation (bf16 operands on the tensor-core path).
 */
#ifndef MSA_ROUTE_H
#define MSA_ROUTE_H

#include "msa_common.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Path selection for msa_route_topk (flags argument). */
#define MSA_ROUTE_AUTO 0    /* pick by query length                                  */
#define MSA_ROUTE_SCAN 1    /* CUDA-core streaming scan (few query tokens)           */
#define MSA_ROUTE_TENSOR 2  /* tcgen05 tensor-core GEMM with fused token-max epilogue */
#define MSA_ROUTE_TENSOR_F8 3 /* the same GEMM on the E4M3 copy of the keys            */
/* OR-ed with a path: one selection shared by every routing layer (the layer-aggregated
 * variant).  Documents are ranked by the mean over the layers of their document scores
 * (each layer's score defined as above), and the same top_k ids and mean scores are
 * written for every layer.  A reading of the pages' single-selection variant: the
 * "MSA端到端可训练记忆模型完整开源，支持亿级Token上下文" page, section 架构, and the MSA paper
 * reading notes, section 路由投影器 + Top-k 稀疏注意力, state the selection per query; where
 * the layers' selections are to be one, their scores are averaged.  Runs on the tensor
 * path (AUTO picks it at any query length; with MSA_ROUTE_SCAN it is MSA_ERR_INVALID_ARG;
 * needs n_kv_heads = 8): the mean filter scores choose the candidates, every layer rescores
 * them exactly, and the final top-k is certified on the mean exact scores against the
 * best mean filter score left out by the mean of the layers' bounds (plus the fp32
 * rounding of the means).  An uncertified query sends every layer through the same
 * further stages as the per-layer selection (bf16 filter, widened rescoring, exact scan
 * of every layer). */
#define MSA_ROUTE_LAYER_MEAN 16
/* OR-ed with MSA_ROUTE_TENSOR or MSA_ROUTE_TENSOR_F8 (not with the layer-aggregated
 * variant): returns the top_k documents by the tensor-core FILTER score and those filter
 * scores, without the exact rescoring.  The MSA pages have no counterpart; it exposes the
 * filter whose error the certification bounds, so that the bound can be checked. */
#define MSA_ROUTE_FILTER_SCORES 32

/* Workspace bytes for one msa_route_topk call with these sizes. */
msa_status msa_route_topk_workspace_size(int32_t n_layers, int32_t n_queries, int32_t total_q_tokens,
                                         int32_t n_kv_heads, int64_t n_chunks, int32_t n_docs, int32_t top_k,
                                         size_t* bytes);

/* E4M3 filter copy of the unit routing keys, for MSA_ROUTE_TENSOR_F8.  The MSA pages have
 * no counterpart: this is an index the tensor-core filter streams instead of kr_hat
 * (half the bytes, twice the tensor-core rate); the selection is still decided on exact
 * fp32 scores of kr_hat.  Every head of kr_hat is renormalised in fp32 (scale
 * 1 / max(||k||, 1e-8)), multiplied by 256 and rounded to E4M3 (OCP FP8, nearest even,
 * saturating at 448).
 *   kr_hat  DEVICE bf16 [n_layers][n_chunks][n_kv_heads][head_dim], 16-byte aligned
 *   kr_f8   DEVICE bytes, same shape, 16-byte aligned (caller-owned, written)
 *   head_dim = 128.  One kernel, asynchronous on stream. */
msa_status msa_route_filter_keys(const void* kr_hat, int32_t n_layers, int64_t n_chunks, int32_t n_kv_heads,
                                 int32_t head_dim, void* kr_f8, msa_stream_t stream);

/* Routes n_queries queries over n_layers routing layers (each layer selects its own
 * top_k documents).
 *   qr               DEVICE [n_layers][total_q_tokens][n_q_heads][head_dim], q_dtype
 *                    (MSA_F32 or MSA_BF16); the tokens of query b are rows
 *                    [q_offsets_host[b], q_offsets_host[b+1]).
 *   q_offsets_host   HOST int32 [n_queries + 1], q_offsets_host[0] = 0, strictly increasing
 *                    (every query has at least one token); read during the call only.
 *   kr_hat           DEVICE bf16 [n_layers][n_chunks][n_kv_heads][head_dim], unit-norm
 *                    routing keys (msa_pool_blocks), 16-byte aligned.
 *   kr_f8            DEVICE, msa_route_filter_keys(kr_hat), or NULL.  Required by
 *                    MSA_ROUTE_TENSOR_F8; with MSA_ROUTE_AUTO its presence selects that path
 *                    for queries beyond the scan length that average at least 16 tokens
 *                    (shorter ones take the bf16 filter).
 *   doc_chunk_offsets DEVICE int64 [n_docs + 1], doc_chunk_offsets[n_docs] = n_chunks.
 *   head_dim = 128; n_kv_heads = 8 on the tensor-core path; n_q_heads % n_kv_heads = 0;
 *   1 <= top_k <= 64; 1 <= n_queries <= 256; n_kv_heads in {2, 4, 8, 16}; n_q_heads <= 64.
 *   out_ids, out_scores DEVICE [n_queries][n_layers][top_k] int32 / fp32.
 *   workspace        DEVICE, >= msa_route_topk_workspace_size bytes, 256-byte aligned.
 *   flags            MSA_ROUTE_AUTO / _SCAN / _TENSOR / _TENSOR_F8, optionally OR-ed with
 *                    MSA_ROUTE_LAYER_MEAN or MSA_ROUTE_FILTER_SCORES.
 * The tensor paths score with low-precision operands as a filter, rescore the best
 * candidates (K2 = max(2 top_k, top_k + 32), at most 128) exactly and take the top_k
 * from the exact scores.  A selection is certified when its k-th exact score beats the
 * best filter score left out by more than a bound on |filter - exact| derived from the
 * operands' rounding (Cauchy-Schwarz over each key head, computed per query token from the
 * query's own operand rows and rounding residuals; the key side enters through its
 * format: E4M3 keys at most 2^-4 relative per element, bf16 keys the nearest rounding of
 * unit vectors).  That bound holds under two preconditions: kr_hat heads are the bf16
 * rounding of unit vectors (or zero), as msa_pool_blocks writes them, and the tensor
 * cores accumulate in fp32 (each addition rounded to nearest or toward zero).
 * Layers that are not certified go, within the same call, through further stages, each
 * of whose kernels return at once when no layer is marked for it: E4M3 filter -> bf16
 * filter -> the 1024 best documents by bf16 filter score rescored exactly -> an exact
 * scan of the layer.  The result is therefore always the exact top_k (up to the fp32
 * rounding of the exact scores, about 1e-6); MSA_DEVERR_UNCERTIFIED is not raised.
 * MSA_ROUTE_SCAN is exact from the start.
 * Asynchronous on stream; no host synchronisation. */
msa_status msa_route_topk(const void* qr, msa_dtype q_dtype, const int32_t* q_offsets_host,
                          int32_t n_queries, const void* kr_hat, const void* kr_f8, const int64_t* doc_chunk_offsets,
                          int32_t n_docs, int64_t n_chunks, int32_t n_layers, int32_t n_q_heads,
                          int32_t n_kv_heads, int32_t head_dim, int32_t top_k, int32_t* out_ids,
                          float* out_scores, void* workspace, size_t workspace_bytes, int32_t flags,
                          int32_t* dev_err, msa_stream_t stream);

/* msa_route_topk with the router's query projection fused in.  Defined by "【MSA】突破100M
 * Token 上下文：记忆稀疏注意力架构深度解析", section 5.1 (each routing layer's decoupled
 * router_q_proj: hidden -> n_q_heads x head_dim, no bias) and section 5.2 (the router
 * query is that projection of the layer's input hidden states).  Per layer l and token t:
 *   Q_r[l][t] = hidden[t] . w_router_q[l]^T          (head q = features q*128 .. q*128+127)
 * computed on the tensor cores (bf16 operands, fp32 accumulation) and normalised per head
 * and summed per key-head group inside the same kernel, straight into the routing
 * operand; Q_r is never written to memory.  Everything after that, and every other
 * argument, result and error, is as msa_route_topk with q_dtype bf16.
 *   hidden      DEVICE bf16 [total tokens][hidden_size], 16-byte aligned (the tokens of
 *               all queries back to back, as qr)
 *   w_router_q  DEVICE bf16 [n_layers][n_q_heads * head_dim][hidden_size], 16-byte aligned
 *   hidden_size a multiple of 64; n_q_heads / n_kv_heads in {1, 2, 4}.
 * The workspace is msa_route_topk_workspace_size's.  One launch replaces the query
 * preparation kernel (the launch count is unchanged). */
msa_status msa_route_topk_hidden(const void* hidden, const void* w_router_q, int32_t hidden_size,
                                 const int32_t* q_offsets_host, int32_t n_queries, const void* kr_hat,
                                 const void* kr_f8, const int64_t* doc_chunk_offsets, int32_t n_docs,
                                 int64_t n_chunks, int32_t n_layers, int32_t n_q_heads, int32_t n_kv_heads,
                                 int32_t head_dim, int32_t top_k, int32_t* out_ids, float* out_scores,
                                 void* workspace, size_t workspace_bytes, int32_t flags, int32_t* dev_err,
                                 msa_stream_t stream);

/* Self test of the bounded waits that every tensor-core routing kernel uses (the MSA
 * pages have no counterpart).  Enqueues one small kernel that takes tensor memory as those
 * kernels do and waits on a barrier that nothing completes (unless release_first != 0,
 * which completes it first), the wait bounded by wait_ns on the GPU's global timer.  On
 * expiry the kernel ORs MSA_DEVERR_TIMEOUT into *dev_err (DEVICE int32), frees its tensor
 * memory and returns, leaving the context usable: the exit path of the routing kernels,
 * whose own limit is 2 s.  1 <= wait_ns <= 1e10.  Asynchronous on stream. */
msa_status msa_route_wait_selftest(int64_t wait_ns, int32_t release_first, int32_t* dev_err, msa_stream_t stream);

/* Number of kernel launches the last successful msa_route_topk on this thread enqueued
 * (for launch accounting). */
int32_t msa_route_last_launch_count(void);

/* Measurement hook: when both are non-NULL (cudaEvent_t handles created by the caller),
 * every later msa_route_topk call on this thread records start_event right before and
 * stop_event right after its score kernel (scan or tensor-core GEMM) on the call's
 * stream, so cudaEventElapsedTime gives that kernel's device time (also inside a CUDA
 * graph capture).  NULL, NULL turns it off.  Returns MSA_OK. */
msa_status msa_route_set_profile_events(void* start_event, void* stop_event);

/* The same hook around the query stage: the query preparation kernel of msa_route_topk,
 * or the fused projection kernel of msa_route_topk_hidden. */
msa_status msa_route_set_query_profile_events(void* start_event, void* stop_event);

/* Tensor-core path tiling on this thread: 1 (default) runs N tiles of 128 / 256 query
 * tokens as M=256 tiles on pairs of SMs (tcgen05 cta_group::2, each SM streaming half of
 * the query tile); 0 keeps one CTA per M=128 tile.  Results are identical.  Returns MSA_OK. */
msa_status msa_route_set_pair_mode(int32_t enabled);

const char* msa_route_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* MSA_ROUTE_H */
