// Step 4: sparse decode attention over [gathered memory blocks ; local KV] (GQA).
//
// Follows "MSA端到端可训练记忆模型完整开源，支持亿级Token上下文", section 架构 (concatenate the
// selected compressed K/V with the local K/V; 全局 RoPE offset by k) and the MSA paper
// reading notes, section 推理全流程 (memory KV fixed, local KV grows per token).
//
// Flash-decoding in one launch: the keys of every (query b, layer l, key head h) are cut
// into kSplits contiguous ranges, one 128-thread CTA each: one key per thread for the
// scores of the CTA's G query heads, a local softmax, and P.V with each warp taking 32
// keys and each lane 4 dims (coalesced 8-byte rows).  Each CTA publishes its
// unnormalised partial output with its running max and sum; the last CTA of a (b, l, h)
// to finish (a self-resetting arrival counter) merges the splits and writes the output,
// and the last merging CTA of query b advances local_len[b].  Only the CTA whose range
// holds the new key appends it (rotated) to the cache, and it uses its own copy of it.
// RoPE angles: p * w_j with w_j / pi precomputed in fp64 on the host; the product is
// reduced modulo 2 pi in fp64 and evaluated by fp32 sincospif.
#include "common.cuh"
#include "msa_decode.h"

#include <mutex>

MSA_DEFINE_LAST_ERROR(msa_decode_last_error)

namespace {

constexpr int kD = 128;
constexpr int kHalf = 64;
constexpr int kThreads = 128;
constexpr int kTile = kThreads;
constexpr int kWarps = kThreads / 32;
constexpr int kSplits = 5;  // 5 x 8 heads x 18 layers fits one wave of 5 CTAs per SM

struct RopeTable {
  double w_over_pi[kHalf];  // theta^(-2j/d) / pi
};

// Workspace: per (b, l, h, split) the partial output [G][128] and (max, sum) per head,
// then one arrival counter per (b, l, h) and one per query b.
size_t ws_floats(int B, int L, int Hq, int H) {
  const size_t units = (size_t)B * L * H * kSplits;
  const int G = Hq / H;
  return units * (size_t)G * (kD + 2);
}
size_t ws_bytes(int B, int L, int Hq, int H) {
  return ws_floats(B, L, Hq, H) * sizeof(float) + ((size_t)B * L * H + (size_t)B) * sizeof(int);
}

template <int G>
__global__ void __launch_bounds__(kThreads, 5) decode_split_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k_new,
    const __nv_bfloat16* __restrict__ v_new, int L, int H,
    // the CTA that appends the new row never reads it back from memory
    __nv_bfloat16* local_k, __nv_bfloat16* local_v, int32_t* local_len, int cap,
    const __nv_bfloat16* __restrict__ mem_kv, const int32_t* __restrict__ mem_len, int M_max, int pos_off,
    const __grid_constant__ RopeTable rope, float scale, float* part, float2* stat, int* unit_count,
    int* query_count, __nv_bfloat16* __restrict__ out, int32_t* dev_err) {
  __shared__ __align__(16) float qs[G][kD];
  __shared__ __align__(16) float knew[kD];
  __shared__ __align__(16) float vnew[kD];
  __shared__ float lg[G][kTile];
  __shared__ float2 cs[kHalf];
  __shared__ float s_max[G], s_sum[G], s_fac[G];
  __shared__ __align__(16) float red[kWarps][G][kD];
  const int split = blockIdx.x, h = blockIdx.y;
  const int b = blockIdx.z / L, l = blockIdx.z % L;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int Hq = H * G;
  const int64_t bl = (int64_t)b * L + l;
  const int64_t unit = (bl * H + h) * kSplits + split;
  float* my_part = part + unit * G * kD;
  float2* my_stat = stat + unit * G;
  const int len = local_len[b];
  const bool full = len >= cap;
  int M = mem_len[bl];
  if (M > M_max) {
    if (tid == 0 && split == 0 && h == 0 && !full) msa::set_err(dev_err, MSA_DEVERR_CAPACITY);
    M = M_max;
  }
  if (M < 0) M = 0;
  const int n_keys = M + len + 1;
  const int per = (n_keys + kSplits - 1) / kSplits;
  const int k0 = split * per, k1 = min(n_keys, k0 + per);
  const int new_key = M + len;
  const bool has_new = new_key >= k0 && new_key < k1;
  if (full) {
    if (tid == 0 && split == 0 && h == 0 && l == 0) msa::set_err(dev_err, MSA_DEVERR_LOCAL_FULL);
    if (tid < G) my_stat[tid] = make_float2(-INFINITY, -1.f);  // unit skipped
  } else if (k0 >= k1) {
    if (tid < G) my_stat[tid] = make_float2(-INFINITY, 0.f);   // empty split
  } else {
  const double pos = (double)pos_off + (double)len;
  if (tid < kHalf) {
    double u = pos * rope.w_over_pi[tid];  // angle / pi
    u -= 2.0 * rint(0.5 * u);             // in [-1, 1]
    float sn, c;
    sincospif((float)u, &sn, &c);
    cs[tid] = make_float2(c, sn);
  }
  if (tid < G) {
    s_max[tid] = -INFINITY;
    s_sum[tid] = 0.f;
  }
  __syncthreads();
  for (int e = tid; e < G * kHalf; e += kThreads) {
    const int g = e / kHalf, j = e % kHalf;
    const __nv_bfloat16* qp = q + (bl * Hq + (int64_t)h * G + g) * kD;
    const float a = __bfloat162float(qp[j]), bb = __bfloat162float(qp[j + kHalf]);
    const float2 c = cs[j];
    qs[g][j] = (a * c.x - bb * c.y) * scale;
    qs[g][j + kHalf] = (bb * c.x + a * c.y) * scale;
  }
  if (has_new) {
    // rotate k_new, round to the cache's bf16 (the value every later step reads) and append
    const int64_t cache_row = ((bl * H + h) * (int64_t)cap + len) * kD;
    if (tid < kHalf) {
      const __nv_bfloat16* kp = k_new + (bl * H + h) * kD;
      const float a = __bfloat162float(kp[tid]), bb = __bfloat162float(kp[tid + kHalf]);
      const float2 c = cs[tid];
      const __nv_bfloat16 lo = __float2bfloat16_rn(a * c.x - bb * c.y);
      const __nv_bfloat16 hi = __float2bfloat16_rn(bb * c.x + a * c.y);
      local_k[cache_row + tid] = lo;
      local_k[cache_row + tid + kHalf] = hi;
      knew[tid] = __bfloat162float(lo);
      knew[tid + kHalf] = __bfloat162float(hi);
    }
    const __nv_bfloat16 vv = v_new[(bl * H + h) * kD + tid];
    local_v[cache_row + tid] = vv;
    vnew[tid] = __bfloat162float(vv);
  }
  __syncthreads();

  const __nv_bfloat16* memk = mem_kv + ((bl * 2 + 0) * H + h) * (int64_t)M_max * kD;
  const __nv_bfloat16* memv = mem_kv + ((bl * 2 + 1) * H + h) * (int64_t)M_max * kD;
  const __nv_bfloat16* lock = local_k + (bl * H + h) * (int64_t)cap * kD;
  const __nv_bfloat16* locv = local_v + (bl * H + h) * (int64_t)cap * kD;
  float acc[G][4];
#pragma unroll
  for (int g = 0; g < G; ++g) {
#pragma unroll
    for (int u = 0; u < 4; ++u) acc[g][u] = 0.f;
  }

  for (int t0 = k0; t0 < k1; t0 += kTile) {
    const int i = t0 + tid;
    if (i < k1) {
      float dotv[G];
#pragma unroll
      for (int g = 0; g < G; ++g) dotv[g] = 0.f;
      if (i == new_key) {
        for (int j = 0; j < kD; j += 4) {
          const float4 kk = *reinterpret_cast<const float4*>(&knew[j]);
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float4 qa = *reinterpret_cast<const float4*>(&qs[g][j]);
            float d = dotv[g];
            d = fmaf(kk.x, qa.x, d); d = fmaf(kk.y, qa.y, d); d = fmaf(kk.z, qa.z, d); d = fmaf(kk.w, qa.w, d);
            dotv[g] = d;
          }
        }
      } else {
        const __nv_bfloat16* kr = i < M ? memk + (int64_t)i * kD : lock + (int64_t)(i - M) * kD;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
        uint4 w[kD / 16];
#pragma unroll
        for (int v8 = 0; v8 < kD / 16; ++v8) w[v8] = *reinterpret_cast<const uint4*>(kr + 64 * half + 8 * v8);
#pragma unroll
        for (int v8 = 0; v8 < kD / 16; ++v8) {
          const int e8 = 64 * half + 8 * v8;
          const float2 f0 = msa::bf16x2_to_float2(w[v8].x), f1 = msa::bf16x2_to_float2(w[v8].y);
          const float2 f2 = msa::bf16x2_to_float2(w[v8].z), f3 = msa::bf16x2_to_float2(w[v8].w);
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float4 qa = *reinterpret_cast<const float4*>(&qs[g][e8]);
            const float4 qb = *reinterpret_cast<const float4*>(&qs[g][e8 + 4]);
            float d = dotv[g];
            d = fmaf(f0.x, qa.x, d); d = fmaf(f0.y, qa.y, d); d = fmaf(f1.x, qa.z, d); d = fmaf(f1.y, qa.w, d);
            d = fmaf(f2.x, qb.x, d); d = fmaf(f2.y, qb.y, d); d = fmaf(f3.x, qb.z, d); d = fmaf(f3.y, qb.w, d);
            dotv[g] = d;
          }
        }
        }
      }
#pragma unroll
      for (int g = 0; g < G; ++g) lg[g][tid] = dotv[g];
    } else {
#pragma unroll
      for (int g = 0; g < G; ++g) lg[g][tid] = -INFINITY;
    }
    __syncthreads();
    for (int g = warp; g < G; g += kWarps) {
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
        const float fac = expf(old - nm);  // 0 on the first tile (old = -inf)
        s_fac[g] = fac;
        s_sum[g] = s_sum[g] * fac + sum;
        s_max[g] = nm;
      }
    }
    __syncthreads();
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float f = s_fac[g];
#pragma unroll
      for (int u = 0; u < 4; ++u) acc[g][u] *= f;
    }
    const int kbeg = warp * 32;
    const int kend = min(kbeg + 32, k1 - t0);
    for (int kk0 = kbeg; kk0 < kend; kk0 += 8) {
      uint2 vw[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int ii = t0 + kk0 + u;
        vw[u] = make_uint2(0u, 0u);
        if (kk0 + u < kend && ii != new_key) {
          const __nv_bfloat16* vr = ii < M ? memv + (int64_t)ii * kD : locv + (int64_t)(ii - M) * kD;
          vw[u] = *reinterpret_cast<const uint2*>(vr + 4 * lane);
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int kk = kk0 + u;
        if (kk < kend) {
          float v0, v1, v2, v3;
          if (t0 + kk == new_key) {
            const float4 x = *reinterpret_cast<const float4*>(&vnew[4 * lane]);
            v0 = x.x; v1 = x.y; v2 = x.z; v3 = x.w;
          } else {
            const float2 a = msa::bf16x2_to_float2(vw[u].x), c = msa::bf16x2_to_float2(vw[u].y);
            v0 = a.x; v1 = a.y; v2 = c.x; v3 = c.y;
          }
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float p = lg[g][kk];
            acc[g][0] = fmaf(p, v0, acc[g][0]);
            acc[g][1] = fmaf(p, v1, acc[g][1]);
            acc[g][2] = fmaf(p, v2, acc[g][2]);
            acc[g][3] = fmaf(p, v3, acc[g][3]);
          }
        }
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int g = 0; g < G; ++g)
    *reinterpret_cast<float4*>(&red[warp][g][4 * lane]) = make_float4(acc[g][0], acc[g][1], acc[g][2], acc[g][3]);
  __syncthreads();
  for (int o = tid; o < G * kD; o += kThreads) {
    const int g = o / kD, j = o % kD;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) v += red[w][g][j];
    my_part[o] = v;
  }
  if (tid < G) my_stat[tid] = make_float2(s_max[tid], s_sum[tid]);
  }  // work of a non-empty split

  // ---- arrival: the last split CTA of (b, l, h) merges the splits
  __shared__ int s_last;
  __threadfence();
  __syncthreads();
  const int64_t uh = bl * H + h;
  if (tid == 0) s_last = atomicAdd(&unit_count[uh], 1) == kSplits - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int64_t unit0 = uh * kSplits;
  const bool skipped = __ldcg(&stat[unit0 * G]).y < 0.f;
  if (!skipped) {
    for (int o = tid; o < G * kD; o += kThreads) {
      const int g = o / kD;
      float mx = -INFINITY;
#pragma unroll
      for (int sp = 0; sp < kSplits; ++sp) mx = fmaxf(mx, __ldcg(&stat[(unit0 + sp) * G + g]).x);
      float num = 0.f, den = 0.f;
#pragma unroll
      for (int sp = 0; sp < kSplits; ++sp) {
        const float2 st = __ldcg(&stat[(unit0 + sp) * G + g]);
        if (st.y > 0.f) {
          const float w = expf(st.x - mx);
          num = fmaf(w, __ldcg(&part[(unit0 + sp) * G * kD + o]), num);
          den = fmaf(w, st.y, den);
        }
      }
      out[(bl * Hq + (int64_t)h * G + g) * kD + (o % kD)] = __float2bfloat16_rn(num / den);
    }
  }
  if (tid == 0) {
    unit_count[uh] = 0;  // ready for the next call
    // the last merged (l, h) of query b advances its local length (every CTA of this
    // call that reads local_len[b] has arrived by then)
    __threadfence();
    if (atomicAdd(&query_count[b], 1) == L * H - 1) {
      if (!skipped) local_len[b] = len + 1;
      query_count[b] = 0;
    }
  }
}

}  // namespace

extern "C" msa_status msa_sparse_decode_workspace_size(int32_t n_queries, int32_t n_layers, int32_t n_q_heads,
                                                       int32_t n_kv_heads, size_t* bytes) {
  if (!bytes || n_queries < 1 || n_layers < 1 || n_kv_heads < 1 || n_q_heads < n_kv_heads ||
      n_q_heads % n_kv_heads != 0)
    return msa_fail(MSA_ERR_INVALID_ARG, "bad sizes");
  *bytes = ws_bytes(n_queries, n_layers, n_q_heads, n_kv_heads);
  return msa_ok();
}

extern "C" msa_status msa_sparse_decode(const void* q, const void* k_new, const void* v_new, int32_t n_queries,
                                        int32_t n_layers, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                        void* local_k, void* local_v, int32_t* local_len, int32_t local_cap,
                                        const void* mem_kv, const int32_t* mem_len, int32_t max_mem_chunks,
                                        int32_t rope_pos_offset, float rope_theta, float softmax_scale, void* out,
                                        void* workspace, size_t workspace_bytes, int32_t* dev_err,
                                        msa_stream_t stream) {
  if (!q || !k_new || !v_new || !local_k || !local_v || !local_len || !mem_kv || !mem_len || !out || !workspace)
    return msa_fail(MSA_ERR_INVALID_ARG, "null pointer");
  if (head_dim != kD) return msa_fail(MSA_ERR_INVALID_ARG, "head_dim must be 128");
  if (n_kv_heads < 1 || n_kv_heads > 16 || n_q_heads % n_kv_heads != 0)
    return msa_fail(MSA_ERR_INVALID_ARG, "n_q_heads must be a multiple of n_kv_heads (<= 16)");
  const int G = n_q_heads / n_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return msa_fail(MSA_ERR_INVALID_ARG, "n_q_heads / n_kv_heads in {1,2,4,8}");
  if (n_queries < 1 || n_layers < 1 || (int64_t)n_queries * n_layers > 65535 || local_cap < 1 || max_mem_chunks < 1)
    return msa_fail(MSA_ERR_INVALID_ARG, "bad counts (n_queries * n_layers <= 65535)");
  if (!(rope_theta > 1.0f)) return msa_fail(MSA_ERR_INVALID_ARG, "rope_theta must be > 1");
  if (!msa::aligned16(mem_kv) || !msa::aligned16(local_k) || !msa::aligned16(workspace))
    return msa_fail(MSA_ERR_INVALID_ARG, "16-byte alignment");
  const size_t need = ws_bytes(n_queries, n_layers, n_q_heads, n_kv_heads);
  if (workspace_bytes < need)
    return msa_fail(MSA_ERR_CAPACITY, "workspace too small (%zu < %zu)", workspace_bytes, need);
  const int arch = msa::current_device_is_sm100(nullptr);
  if (arch < 0) return msa_fail(MSA_ERR_CUDA, "no CUDA device");
  if (arch == 0) return msa_fail(MSA_ERR_UNSUPPORTED, "device is not sm_100");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t units = (size_t)n_queries * n_layers * n_kv_heads * kSplits;
  float* part = reinterpret_cast<float*>(workspace);
  float2* stat = reinterpret_cast<float2*>(part + units * G * kD);
  int* unit_count = reinterpret_cast<int*>(part + ws_floats(n_queries, n_layers, n_q_heads, n_kv_heads));
  int* query_count = unit_count + (size_t)n_queries * n_layers * n_kv_heads;
  const dim3 grid(kSplits, n_kv_heads, n_queries * n_layers);
  RopeTable rope;
  for (int j = 0; j < kHalf; ++j)
    rope.w_over_pi[j] = pow((double)rope_theta, -2.0 * (double)j / (double)kD) / 3.14159265358979323846;
#define MSA_DECODE_LAUNCH(GG)                                                                                    \
  decode_split_kernel<GG><<<grid, kThreads, 0, s>>>(                                                             \
      (const __nv_bfloat16*)q, (const __nv_bfloat16*)k_new, (const __nv_bfloat16*)v_new, n_layers, n_kv_heads,     \
      (__nv_bfloat16*)local_k, (__nv_bfloat16*)local_v, local_len, local_cap, (const __nv_bfloat16*)mem_kv,        \
      mem_len, max_mem_chunks, rope_pos_offset, rope, softmax_scale, part, stat, unit_count, query_count,         \
      (__nv_bfloat16*)out, dev_err)
  switch (G) {
    case 1: MSA_DECODE_LAUNCH(1); break;
    case 2: MSA_DECODE_LAUNCH(2); break;
    case 4: MSA_DECODE_LAUNCH(4); break;
    default: MSA_DECODE_LAUNCH(8); break;
  }
#undef MSA_DECODE_LAUNCH
  MSA_CUDA_TRY(cudaGetLastError());
  return msa_ok();
}

// ---------------------------------------------------------------------------- no-allocation entry
// Decode scratch that lives in the library itself, for callers that cannot allocate
// device memory.  Every GPU that loads this library holds these bytes until the process
// exits.  The host-side symbol is only a stand-in for the device address, so the address
// is looked up once per device (cudaGetSymbolAddress, that device current) and passed to
// the kernel.
static __device__ __align__(256) unsigned char g_decode_scratch[MSA_DECODE_STATIC_SCRATCH_BYTES];

namespace {
std::mutex g_scratch_mutex;
void* g_scratch_addr[64];  // per device ordinal; nullptr until looked up
}  // namespace

extern "C" msa_status msa_sparse_decode_static(const void* q, const void* k_new, const void* v_new,
                                               int32_t n_queries, int32_t n_layers, int32_t n_q_heads,
                                               int32_t n_kv_heads, int32_t head_dim, void* local_k, void* local_v,
                                               int32_t* local_len, int32_t local_cap, const void* mem_kv,
                                               const int32_t* mem_len, int32_t max_mem_chunks,
                                               int32_t rope_pos_offset, float rope_theta, float softmax_scale,
                                               void* out, int32_t* dev_err, msa_stream_t stream) {
  if (n_queries < 1 || n_layers < 1 || n_kv_heads < 1 || n_q_heads < n_kv_heads || n_q_heads % n_kv_heads != 0)
    return msa_fail(MSA_ERR_INVALID_ARG, "bad sizes");
  const size_t need = ws_bytes(n_queries, n_layers, n_q_heads, n_kv_heads);
  if (need > MSA_DECODE_STATIC_SCRATCH_BYTES)
    return msa_fail(MSA_ERR_CAPACITY, "static decode scratch holds %u bytes, these sizes need %zu",
                    MSA_DECODE_STATIC_SCRATCH_BYTES, need);
  int dev = 0;
  MSA_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return msa_fail(MSA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_addr[dev] == nullptr) {
      void* p = nullptr;
      MSA_CUDA_TRY(cudaGetSymbolAddress(&p, g_decode_scratch));
      g_scratch_addr[dev] = p;
    }
    scratch = g_scratch_addr[dev];
  }
  // the arrival counters must start at zero: their place depends on the sizes, and the
  // array keeps whatever the previous call left there
  const size_t counters_at = ws_floats(n_queries, n_layers, n_q_heads, n_kv_heads) * sizeof(float);
  MSA_CUDA_TRY(cudaMemsetAsync(static_cast<unsigned char*>(scratch) + counters_at, 0, need - counters_at,
                               reinterpret_cast<cudaStream_t>(stream)));
  return msa_sparse_decode(q, k_new, v_new, n_queries, n_layers, n_q_heads, n_kv_heads, head_dim, local_k, local_v,
                           local_len, local_cap, mem_kv, mem_len, max_mem_chunks, rope_pos_offset, rope_theta,
                           softmax_scale, out, scratch, MSA_DECODE_STATIC_SCRATCH_BYTES, dev_err, stream);
}
