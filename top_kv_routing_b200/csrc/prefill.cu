// Prefill: a block of new tokens per query (the query's own tokens) through sparse
// attention over [gathered memory blocks ; the local cache up to each token].
//
// Follows "MSA端到端可训练记忆模型完整开源，支持亿级Token上下文", section 推理流水线 (the query is
// processed over the selected documents' compressed K/V joined to its local context;
// 全局 RoPE offset by k) and the MSA paper reading notes, section 推理全流程.  Token i of a
// block is the decode step at local index local_len + i: it sees the whole memory and the
// local keys 0 .. local_len + i.
//
// Three launches: (1) the new keys are rotated (RoPE at position offset + local index),
// rounded to the cache's bf16 and appended with the new values; (2) attention on the
// tcgen05 tensor cores (prefill_tc.cu), persistent CTAs taking 128 (token, query head)
// rows at a time; (3) local_len += n_new.
#include "common.cuh"
#include "msa_prefill.h"
#include "prefill_tc.cuh"

MSA_DEFINE_LAST_ERROR(msa_prefill_last_error)

namespace {

constexpr int kD = 128;
constexpr int kHalf = 64;
constexpr int kThreads = 128;
constexpr float kLog2e = 1.4426950408889634f;


// (1) grid (ceil(n_new / 8), H, B * L), 128 threads: 16 threads per token (4 rotation pairs
// and 8 values each) rotate, round and append 8 tokens' keys and values; the 64 frequencies
// are computed once per CTA.
constexpr int kAppendTok = 8;
__global__ void __launch_bounds__(kThreads) prefill_append_kernel(
    const __nv_bfloat16* __restrict__ k_new, const __nv_bfloat16* __restrict__ v_new, int T, int L, int H,
    __nv_bfloat16* __restrict__ local_k, __nv_bfloat16* __restrict__ local_v, const int32_t* __restrict__ local_len,
    int cap, const int32_t* __restrict__ mem_len, int M_max, int pos_off, double log2_theta, int32_t* dev_err) {
  __shared__ double s_w[kHalf];  // theta^(-2j/d) / pi
  const int h = blockIdx.y;
  const int64_t bl = blockIdx.z;
  const int b = (int)(bl / L);
  const int tid = threadIdx.x;
  const int len = local_len[b];
  if (len < 0 || len + T > cap) {
    if (blockIdx.x == 0 && h == 0 && (bl % L) == 0 && tid == 0) msa::set_err(dev_err, MSA_DEVERR_LOCAL_FULL);
    return;
  }
  if (blockIdx.x == 0 && h == 0 && tid == 0 && mem_len[bl] > M_max) msa::set_err(dev_err, MSA_DEVERR_CAPACITY);
  if (tid < kHalf) s_w[tid] = exp2(-2.0 * (double)tid / (double)kD * log2_theta) * 0.31830988618379067154;
  __syncthreads();
  const int i = blockIdx.x * kAppendTok + tid / 16, q16 = tid % 16;
  if (i >= T) return;
  const int64_t src = ((bl * T + i) * H + h) * kD;
  const int64_t dst = ((bl * H + h) * (int64_t)cap + len + i) * kD;
  const double pos = (double)pos_off + (double)(len + i);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int j = 4 * q16 + e;
    double u = pos * s_w[j];  // angle / pi, reduced to [-1, 1]
    u -= 2.0 * rint(0.5 * u);
    float c, sn;
    sincospif((float)u, &sn, &c);
    const float a = __bfloat162float(k_new[src + j]), bb = __bfloat162float(k_new[src + j + kHalf]);
    local_k[dst + j] = __float2bfloat16_rn(a * c - bb * sn);
    local_k[dst + j + kHalf] = __float2bfloat16_rn(bb * c + a * sn);
  }
  *reinterpret_cast<uint4*>(local_v + dst + 8 * q16) = *reinterpret_cast<const uint4*>(v_new + src + 8 * q16);
}

// (3) one thread per query: the length advances by the block (unless the cache was full).
__global__ void prefill_advance_kernel(int32_t* local_len, int B, int T, int cap) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B && local_len[b] >= 0 && local_len[b] + T <= cap) local_len[b] += T;
}

}  // namespace

extern "C" msa_status msa_sparse_prefill(const void* q, const void* k_new, const void* v_new, int32_t n_new,
                                         int32_t n_queries, int32_t n_layers, int32_t n_q_heads, int32_t n_kv_heads,
                                         int32_t head_dim, void* local_k, void* local_v, int32_t* local_len,
                                         int32_t local_cap, const void* mem_kv, const int32_t* mem_len,
                                         int32_t max_mem_chunks, int32_t rope_pos_offset, float rope_theta,
                                         float softmax_scale, void* out, int32_t* dev_err, msa_stream_t stream) {
  if (!q || !k_new || !v_new || !local_k || !local_v || !local_len || !mem_kv || !mem_len || !out)
    return msa_fail(MSA_ERR_INVALID_ARG, "null pointer");
  if (head_dim != kD) return msa_fail(MSA_ERR_INVALID_ARG, "head_dim must be 128");
  if (n_kv_heads < 1 || n_kv_heads > 16 || n_q_heads % n_kv_heads != 0)
    return msa_fail(MSA_ERR_INVALID_ARG, "n_q_heads must be a multiple of n_kv_heads (<= 16)");
  const int G = n_q_heads / n_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return msa_fail(MSA_ERR_INVALID_ARG, "n_q_heads / n_kv_heads in {1,2,4,8}");
  if (n_new < 1 || n_queries < 1 || n_layers < 1 || (int64_t)n_queries * n_layers > 65535 || local_cap < 1 ||
      max_mem_chunks < 1)
    return msa_fail(MSA_ERR_INVALID_ARG, "bad counts (n_queries * n_layers <= 65535)");
  if (!(rope_theta > 1.0f)) return msa_fail(MSA_ERR_INVALID_ARG, "rope_theta must be > 1");
  if (!msa::aligned16(q) || !msa::aligned16(k_new) || !msa::aligned16(v_new) || !msa::aligned16(mem_kv) ||
      !msa::aligned16(local_k) || !msa::aligned16(local_v) ||
      !msa::aligned16(out))
    return msa_fail(MSA_ERR_INVALID_ARG, "16-byte alignment (q, k_new, v_new, mem_kv, local_k, local_v, out)");
  const int arch = msa::current_device_is_sm100(nullptr);
  if (arch < 0) return msa_fail(MSA_ERR_CUDA, "no CUDA device");
  if (arch == 0) return msa_fail(MSA_ERR_UNSUPPORTED, "device is not sm_100");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const double log2_theta = log2((double)rope_theta);
  const float qscale = softmax_scale * kLog2e;
  const int BL = n_queries * n_layers;
  prefill_append_kernel<<<dim3((n_new + kAppendTok - 1) / kAppendTok, n_kv_heads, BL), kThreads, 0, s>>>(
      (const __nv_bfloat16*)k_new, (const __nv_bfloat16*)v_new, n_new, n_layers, n_kv_heads, (__nv_bfloat16*)local_k,
      (__nv_bfloat16*)local_v, local_len, local_cap, mem_len, max_mem_chunks, rope_pos_offset, log2_theta, dev_err);
  MSA_CUDA_TRY(cudaGetLastError());
  prefill_tc::Args ta;
  ta.q = (const __nv_bfloat16*)q;
  ta.out = (__nv_bfloat16*)out;
  ta.local_k = (const __nv_bfloat16*)local_k;
  ta.local_v = (const __nv_bfloat16*)local_v;
  ta.local_len = local_len;
  ta.mem_kv = (const __nv_bfloat16*)mem_kv;
  ta.mem_len = mem_len;
  ta.T = n_new;
  ta.B = n_queries;
  ta.L = n_layers;
  ta.H = n_kv_heads;
  ta.G = G;
  ta.cap = local_cap;
  ta.M_max = max_mem_chunks;
  ta.pos_off = rope_pos_offset;
  ta.log2_theta = log2_theta;
  ta.qscale = qscale;
  ta.dev_err = dev_err;
  if (!prefill_tc::supported(ta))
    return msa_fail(MSA_ERR_CAPACITY, "caches beyond 2^31 rows of 128 elements");
  {
    const char* why = nullptr;
    if (prefill_tc::launch(ta, s, &why) != 0) return msa_fail(MSA_ERR_CUDA, "prefill attention: %s", why);
  }
  MSA_CUDA_TRY(cudaGetLastError());
  prefill_advance_kernel<<<(n_queries + 127) / 128, 128, 0, s>>>(local_len, n_queries, n_new, local_cap);
  MSA_CUDA_TRY(cudaGetLastError());
  return msa_ok();
}
