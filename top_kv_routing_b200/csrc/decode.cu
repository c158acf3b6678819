// Step 4: sparse decode attention over [gathered memory blocks ; local KV] (GQA).
//
// Follows "MSA端到端可训练记忆模型完整开源，支持亿级Token上下文", section 架构 (concatenate the
// selected compressed K/V with the local K/V; 全局 RoPE offset by k) and the MSA paper
// reading notes, section 推理全流程 (memory KV fixed, local KV grows per token).
//
// One CTA per (kv head h, layer l, query b) serves the G query heads of that key head.
// Keys are processed in tiles of 256 (one key per thread for the scores, one
// (head, dim) output pair per thread for P.V) with an online softmax across tiles.
#include "common.cuh"
#include "msa_decode.h"

MSA_DEFINE_LAST_ERROR(msa_decode_last_error)

namespace {

constexpr int kD = 128;
constexpr int kHalf = 64;
constexpr int kThreads = 256;
constexpr int kTile = kThreads;

template <int G>
__global__ void __launch_bounds__(kThreads) decode_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k_new,
    const __nv_bfloat16* __restrict__ v_new, int L, int H,
    // written (the appended row) and read back in this kernel: plain, coherent loads only
    __nv_bfloat16* local_k, __nv_bfloat16* local_v, const int32_t* __restrict__ local_len, int cap,
    const __nv_bfloat16* __restrict__ mem_kv, const int32_t* __restrict__ mem_len, int M_max, int pos_off,
    double log2_theta, float scale, __nv_bfloat16* __restrict__ out, int32_t* dev_err) {
  constexpr int kOut = G * kD;                          // outputs of this CTA
  constexpr int kPer = (kOut + kThreads - 1) / kThreads;  // outputs per thread
  __shared__ __align__(16) float qs[G][kD];
  __shared__ float lg[G][kTile];
  __shared__ float2 cs[kHalf];
  __shared__ float s_max[G], s_sum[G], s_fac[G];
  const int h = blockIdx.x, l = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  const int Hq = H * G;
  const int len = local_len[b];
  if (len >= cap) {
    if (tid == 0 && h == 0 && l == 0) msa::set_err(dev_err, MSA_DEVERR_LOCAL_FULL);
    return;
  }
  int M = mem_len[(int64_t)b * L + l];
  if (M > M_max) {
    if (tid == 0) msa::set_err(dev_err, MSA_DEVERR_CAPACITY);
    M = M_max;
  }
  if (M < 0) M = 0;
  const double pos = (double)pos_off + (double)len;
  if (tid < kHalf) {
    const double w = exp2(-2.0 * (double)tid / (double)kD * log2_theta);
    float c, s;
    msa::angle_sincos(pos, w, &c, &s);
    cs[tid] = make_float2(c, s);
  }
  if (tid < G) {
    s_max[tid] = -INFINITY;
    s_sum[tid] = 0.f;
  }
  __syncthreads();
  // rotate q (scaled) into smem; rotate k_new and append k', v_new to the local cache
  const int64_t bl = (int64_t)b * L + l;
  for (int e = tid; e < G * kHalf; e += kThreads) {
    const int g = e / kHalf, j = e % kHalf;
    const __nv_bfloat16* qp = q + (bl * Hq + (int64_t)h * G + g) * kD;
    const float a = __bfloat162float(qp[j]), bb = __bfloat162float(qp[j + kHalf]);
    const float2 c = cs[j];
    qs[g][j] = (a * c.x - bb * c.y) * scale;
    qs[g][j + kHalf] = (bb * c.x + a * c.y) * scale;
  }
  const int64_t cache_row = ((bl * H + h) * (int64_t)cap + len) * kD;
  if (tid < kHalf) {
    const __nv_bfloat16* kp = k_new + (bl * H + h) * kD;
    const float a = __bfloat162float(kp[tid]), bb = __bfloat162float(kp[tid + kHalf]);
    const float2 c = cs[tid];
    local_k[cache_row + tid] = __float2bfloat16_rn(a * c.x - bb * c.y);
    local_k[cache_row + tid + kHalf] = __float2bfloat16_rn(bb * c.x + a * c.y);
  } else if (tid < kHalf + kD) {
    const int j = tid - kHalf;
    local_v[cache_row + j] = v_new[(bl * H + h) * kD + j];
  }
  __syncthreads();

  const int n_keys = M + len + 1;
  const __nv_bfloat16* memk = mem_kv + ((bl * 2 + 0) * H + h) * (int64_t)M_max * kD;
  const __nv_bfloat16* memv = mem_kv + ((bl * 2 + 1) * H + h) * (int64_t)M_max * kD;
  const __nv_bfloat16* lock = local_k + (bl * H + h) * (int64_t)cap * kD;
  const __nv_bfloat16* locv = local_v + (bl * H + h) * (int64_t)cap * kD;
  float acc[kPer];
#pragma unroll
  for (int u = 0; u < kPer; ++u) acc[u] = 0.f;

  for (int t0 = 0; t0 < n_keys; t0 += kTile) {
    // scores: one key per thread
    const int i = t0 + tid;
    if (i < n_keys) {
      const __nv_bfloat16* kr = i < M ? memk + (int64_t)i * kD : lock + (int64_t)(i - M) * kD;
      float dotv[G];
#pragma unroll
      for (int g = 0; g < G; ++g) dotv[g] = 0.f;
#pragma unroll 4
      for (int v8 = 0; v8 < kD / 8; ++v8) {
        const uint4 w = *reinterpret_cast<const uint4*>(kr + 8 * v8);
        const float2 f0 = msa::bf16x2_to_float2(w.x), f1 = msa::bf16x2_to_float2(w.y);
        const float2 f2 = msa::bf16x2_to_float2(w.z), f3 = msa::bf16x2_to_float2(w.w);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float4 qa = *reinterpret_cast<const float4*>(&qs[g][8 * v8]);
          const float4 qb = *reinterpret_cast<const float4*>(&qs[g][8 * v8 + 4]);
          float d = dotv[g];
          d = fmaf(f0.x, qa.x, d); d = fmaf(f0.y, qa.y, d); d = fmaf(f1.x, qa.z, d); d = fmaf(f1.y, qa.w, d);
          d = fmaf(f2.x, qb.x, d); d = fmaf(f2.y, qb.y, d); d = fmaf(f3.x, qb.z, d); d = fmaf(f3.y, qb.w, d);
          dotv[g] = d;
        }
      }
#pragma unroll
      for (int g = 0; g < G; ++g) lg[g][tid] = dotv[g];
    } else {
#pragma unroll
      for (int g = 0; g < G; ++g) lg[g][tid] = -INFINITY;
    }
    __syncthreads();
    // per-head tile max, rescale factor, probabilities and sums (warp g handles head g)
    const int warp = tid / 32, lane = tid % 32;
    for (int g = warp; g < G; g += kThreads / 32) {
      float mx = -INFINITY;
      for (int u = lane; u < kTile; u += 32) mx = fmaxf(mx, lg[g][u]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float old = s_max[g];
      const float nm = fmaxf(old, mx);
      float sum = 0.f;
      for (int u = lane; u < kTile; u += 32) {
        const float p = expf(lg[g][u] - nm);
        lg[g][u] = p;
        sum += p;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0) {
        const float fac = expf(old - nm);  // old = -inf on the first tile -> 0
        s_fac[g] = fac;
        s_sum[g] = s_sum[g] * fac + sum;
        s_max[g] = nm;
      }
    }
    __syncthreads();
    // P.V: thread owns outputs o = tid + 256 u, (head o / 128, dim o % 128)
    const int nt = min(kTile, n_keys - t0);
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int o = tid + kThreads * u;
      if (o < kOut) {
        const int g = o / kD, j = o % kD;
        float a = acc[u] * s_fac[g];
        for (int kk = 0; kk < nt; ++kk) {
          const int ii = t0 + kk;
          const __nv_bfloat16* vr = ii < M ? memv + (int64_t)ii * kD : locv + (int64_t)(ii - M) * kD;
          a = fmaf(lg[g][kk], __bfloat162float(vr[j]), a);
        }
        acc[u] = a;
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int o = tid + kThreads * u;
    if (o < kOut) {
      const int g = o / kD, j = o % kD;
      out[(bl * Hq + (int64_t)h * G + g) * kD + j] = __float2bfloat16_rn(acc[u] / s_sum[g]);
    }
  }
}

__global__ void advance_kernel(int32_t* local_len, int n, int cap) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < n && local_len[b] < cap) local_len[b] += 1;
}

}  // namespace

extern "C" msa_status msa_sparse_decode(const void* q, const void* k_new, const void* v_new, int32_t n_queries,
                                        int32_t n_layers, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                        void* local_k, void* local_v, int32_t* local_len, int32_t local_cap,
                                        const void* mem_kv, const int32_t* mem_len, int32_t max_mem_chunks,
                                        int32_t rope_pos_offset, float rope_theta, float softmax_scale, void* out,
                                        int32_t* dev_err, msa_stream_t stream) {
  if (!q || !k_new || !v_new || !local_k || !local_v || !local_len || !mem_kv || !mem_len || !out)
    return msa_fail(MSA_ERR_INVALID_ARG, "null pointer");
  if (head_dim != kD) return msa_fail(MSA_ERR_INVALID_ARG, "head_dim must be 128");
  if (n_kv_heads < 1 || n_kv_heads > 16 || n_q_heads % n_kv_heads != 0)
    return msa_fail(MSA_ERR_INVALID_ARG, "n_q_heads must be a multiple of n_kv_heads (<= 16)");
  const int G = n_q_heads / n_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return msa_fail(MSA_ERR_INVALID_ARG, "n_q_heads / n_kv_heads in {1,2,4,8}");
  if (n_queries < 1 || n_queries > 65535 || n_layers < 1 || n_layers > 65535 || local_cap < 1 || max_mem_chunks < 1)
    return msa_fail(MSA_ERR_INVALID_ARG, "bad counts");
  if (!(rope_theta > 1.0f)) return msa_fail(MSA_ERR_INVALID_ARG, "rope_theta must be > 1");
  if (!msa::aligned16(mem_kv) || !msa::aligned16(local_k)) return msa_fail(MSA_ERR_INVALID_ARG, "16-byte alignment");
  const int arch = msa::current_device_is_sm100(nullptr);
  if (arch < 0) return msa_fail(MSA_ERR_CUDA, "no CUDA device");
  if (arch == 0) return msa_fail(MSA_ERR_UNSUPPORTED, "device is not sm_100");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const dim3 grid(n_kv_heads, n_layers, n_queries);
  const double l2t = log2((double)rope_theta);
#define MSA_DECODE_LAUNCH(GG)                                                                              \
  decode_kernel<GG><<<grid, kThreads, 0, s>>>(                                                             \
      (const __nv_bfloat16*)q, (const __nv_bfloat16*)k_new, (const __nv_bfloat16*)v_new, n_layers, n_kv_heads, \
      (__nv_bfloat16*)local_k, (__nv_bfloat16*)local_v, local_len, local_cap, (const __nv_bfloat16*)mem_kv,  \
      mem_len, max_mem_chunks, rope_pos_offset, l2t, softmax_scale, (__nv_bfloat16*)out, dev_err)
  switch (G) {
    case 1: MSA_DECODE_LAUNCH(1); break;
    case 2: MSA_DECODE_LAUNCH(2); break;
    case 4: MSA_DECODE_LAUNCH(4); break;
    default: MSA_DECODE_LAUNCH(8); break;
  }
#undef MSA_DECODE_LAUNCH
  MSA_CUDA_TRY(cudaGetLastError());
  advance_kernel<<<(n_queries + 255) / 256, 256, 0, s>>>(local_len, n_queries, local_cap);
  MSA_CUDA_TRY(cudaGetLastError());
  return msa_ok();
}
