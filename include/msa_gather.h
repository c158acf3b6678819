/* Step 3 of the MSA hot path: load only the selected documents' compressed K/V from
 * pinned host memory into a packed device buffer.
 *
 * Defined by: "MSA端到端可训练记忆模型完整开源，支持亿级Token上下文", section 推理流水线 step 2
 * (only the selected K-bar/V-bar are loaded and joined to the local context) and section
 * 记忆并行 (content K-bar/V-bar live in host memory and are fetched asynchronously when
 * selected); MSA paper reading notes, section KV 缓存压缩 + Memory Parallel (content KV in
 * CPU memory, ~19 MB per query for the Top-16 documents).
 *
 * The copy is done by a kernel that reads the host store directly over PCIe (zero-copy
 * loads from page-locked memory), driven by the device-resident ids of msa_route_topk, so
 * no host synchronisation sits between routing and the load.  Run it on a side stream and
 * hand off to decode with an event.
 */
#ifndef MSA_GATHER_H
#define MSA_GATHER_H

#include "msa_common.h"

#ifdef __cplusplus
extern "C" {
#endif

/* For every query b and layer l, packs the blocks of the documents ids[b][l][0..top_k)
 * (in rank order, skipping -1) into
 *   dev_kv[b][l][kv][h][m][:]   kv = 0 (K-bar) / 1 (V-bar), m < mem_len[b][l]
 * and writes mem_len[b][l] = number of packed blocks.
 *   host_kv        HOST, page-locked and device-mapped (cudaHostAlloc / cudaHostRegister),
 *                  bf16 [n_layers][n_store_chunks][2][n_heads][head_dim]: every block of every
 *                  layer stores K-bar then V-bar.  16-byte aligned.
 *   doc_chunk_offsets  DEVICE int64 [n_docs + 1]: document d has blocks
 *                  [doc_chunk_offsets[d], doc_chunk_offsets[d+1]) (the count is what moves).
 *   doc_store_offsets  DEVICE int64 [n_docs] or NULL: first block of document d in the host
 *                  store (NULL = doc_chunk_offsets[d]).  Lets several logical documents share
 *                  physical blocks when the host store is smaller than the logical bank.
 *   ids            DEVICE int32 [n_queries][n_layers][top_k] (msa_route_topk output).
 *   head_dim = 128; n_heads in [1, 16]; top_k in [1, 64].
 *   dev_kv         DEVICE bf16 [n_queries][n_layers][2][n_heads][max_mem_chunks][head_dim].
 *   mem_len        DEVICE int32 [n_queries][n_layers].
 * A selection with more than max_mem_chunks blocks is clamped and sets
 * MSA_DEVERR_CAPACITY; an id outside [-1, n_docs) is skipped with MSA_DEVERR_BAD_DOC; a
 * block outside the store is skipped with MSA_DEVERR_BAD_OFFSETS.  Asynchronous on stream. */
msa_status msa_gather_kv(const void* host_kv, int64_t n_store_chunks, const int64_t* doc_chunk_offsets,
                         const int64_t* doc_store_offsets, int32_t n_docs, const int32_t* ids,
                         int32_t n_queries, int32_t n_layers, int32_t top_k, int32_t n_heads, int32_t head_dim,
                         int32_t max_mem_chunks, void* dev_kv, int32_t* mem_len, int32_t* dev_err,
                         msa_stream_t stream);

const char* msa_gather_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* MSA_GATHER_H */
