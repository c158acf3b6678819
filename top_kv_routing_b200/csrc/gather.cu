// Step 3: zero-copy gather of the selected documents' compressed K/V from pinned host
// memory (PCIe-bound).
//
// Follows "MSA端到端可训练记忆模型完整开源，支持亿级Token上下文", sections 推理流水线 and 记忆并行
// (only the selected K-bar/V-bar are fetched from host memory) and the MSA paper reading
// notes, section KV 缓存压缩 + Memory Parallel (~19 MB per Top-16 query).
//
// One CTA per (rank r, layer l, query b) copies its document's blocks.  The destination
// offset is the block count of the higher-ranked documents of the same (b, l), so all
// CTAs run independently.  Every thread moves 16-byte words; each CTA keeps several
// PCIe reads in flight per thread.
#include "common.cuh"
#include "msa_gather.h"

MSA_DEFINE_LAST_ERROR(msa_gather_last_error)

namespace {

constexpr int kD = 128;

__global__ void __launch_bounds__(256) gather_kernel(const uint4* __restrict__ host_kv, int64_t n_store,
                                                     const int64_t* __restrict__ doc_chunk_off,
                                                     const int64_t* __restrict__ doc_store_off, int n_docs,
                                                     const int32_t* __restrict__ ids, int L, int k, int H,
                                                     int M_max, uint4* __restrict__ dev_kv,
                                                     int32_t* __restrict__ mem_len, int32_t* dev_err) {
  const int r = blockIdx.x, l = blockIdx.y, b = blockIdx.z;
  const int32_t* sel = ids + ((int64_t)b * L + l) * k;
  __shared__ int64_t s_dst, s_n, s_src;
  if (threadIdx.x == 0) {
    int64_t before = 0;
    for (int i = 0; i < r; ++i) {
      const int d = sel[i];
      if (d >= 0 && d < n_docs) before += doc_chunk_off[d + 1] - doc_chunk_off[d];
    }
    const int d = sel[r];
    int64_t n = 0, src = 0;
    if (d >= n_docs || d < -1) {
      msa::set_err(dev_err, MSA_DEVERR_BAD_DOC);
    } else if (d >= 0) {
      n = doc_chunk_off[d + 1] - doc_chunk_off[d];
      src = doc_store_off ? doc_store_off[d] : doc_chunk_off[d];
      if (src < 0 || src + n > n_store) {
        msa::set_err(dev_err, MSA_DEVERR_BAD_OFFSETS);
        n = 0;
      }
    }
    if (before + n > M_max) {
      msa::set_err(dev_err, MSA_DEVERR_CAPACITY);
      n = before >= M_max ? 0 : M_max - before;
    }
    s_dst = before;
    s_n = n;
    s_src = src;
    if (r == k - 1) {
      int64_t total = before + (d >= 0 && d < n_docs ? doc_chunk_off[d + 1] - doc_chunk_off[d] : 0);
      mem_len[(int64_t)b * L + l] = (int32_t)(total > M_max ? M_max : total);
    }
  }
  __syncthreads();
  const int64_t n = s_n;
  if (n == 0) return;
  const int64_t dst0 = s_dst, src0 = s_src;
  // one block = 2 * H * 128 bf16 = 32 * H words of 16 bytes; a row of one head = 16 words
  const int words_per_block = 2 * H * (kD / 8);
  const int64_t total = n * words_per_block;
  const uint4* src = host_kv + ((int64_t)l * n_store + src0) * words_per_block;
  uint4* dst_base = dev_kv + ((int64_t)b * L + l) * (int64_t)2 * H * M_max * (kD / 8);
  constexpr int kUnroll = 4;
  for (int64_t base = threadIdx.x; base < total; base += (int64_t)blockDim.x * kUnroll) {
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t w = base + (int64_t)u * blockDim.x;
      if (w < total) v[u] = src[w];
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t w = base + (int64_t)u * blockDim.x;
      if (w < total) {
        const int64_t blk = w / words_per_block;
        const int rem = (int)(w % words_per_block);
        const int kvh = rem / (kD / 8);        // kv * H + h
        const int part = rem % (kD / 8);
        const int64_t m = dst0 + blk;
        dst_base[((int64_t)kvh * M_max + m) * (kD / 8) + part] = v[u];
      }
    }
  }
}

}  // namespace

extern "C" msa_status msa_gather_kv(const void* host_kv, int64_t n_store_chunks, const int64_t* doc_chunk_offsets,
                                    const int64_t* doc_store_offsets, int32_t n_docs, const int32_t* ids,
                                    int32_t n_queries, int32_t n_layers, int32_t top_k, int32_t n_heads,
                                    int32_t head_dim, int32_t max_mem_chunks, void* dev_kv, int32_t* mem_len,
                                    int32_t* dev_err, msa_stream_t stream) {
  if (!host_kv || !doc_chunk_offsets || !ids || !dev_kv || !mem_len) return msa_fail(MSA_ERR_INVALID_ARG, "null pointer");
  if (head_dim != kD) return msa_fail(MSA_ERR_INVALID_ARG, "head_dim must be 128");
  if (n_heads < 1 || n_heads > 16) return msa_fail(MSA_ERR_INVALID_ARG, "n_heads in [1,16]");
  if (top_k < 1 || top_k > 64) return msa_fail(MSA_ERR_INVALID_ARG, "top_k in [1,64]");
  if (n_queries < 1 || n_layers < 1 || n_store_chunks < 0 || n_docs < 0 || max_mem_chunks < 1)
    return msa_fail(MSA_ERR_INVALID_ARG, "bad counts");
  if (n_queries > 65535 || n_layers > 65535) return msa_fail(MSA_ERR_INVALID_ARG, "too many queries/layers");
  if (!msa::aligned16(host_kv) || !msa::aligned16(dev_kv)) return msa_fail(MSA_ERR_INVALID_ARG, "16-byte alignment");
  const int arch = msa::current_device_is_sm100(nullptr);
  if (arch < 0) return msa_fail(MSA_ERR_CUDA, "no CUDA device");
  if (arch == 0) return msa_fail(MSA_ERR_UNSUPPORTED, "device is not sm_100");
  cudaPointerAttributes attr;
  MSA_CUDA_TRY(cudaPointerGetAttributes(&attr, host_kv));
  if (attr.type != cudaMemoryTypeHost || attr.devicePointer == nullptr)
    return msa_fail(MSA_ERR_INVALID_ARG, "host_kv must be page-locked, device-mapped host memory");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  gather_kernel<<<dim3(top_k, n_layers, n_queries), 256, 0, s>>>(
      reinterpret_cast<const uint4*>(attr.devicePointer), n_store_chunks, doc_chunk_offsets, doc_store_offsets,
      n_docs, ids, n_layers, top_k, n_heads, max_mem_chunks, reinterpret_cast<uint4*>(dev_kv), mem_len, dev_err);
  MSA_CUDA_TRY(cudaGetLastError());
  return msa_ok();
}
