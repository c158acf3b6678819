// Step 1: document-wise RoPE + block mean pooling of one bank layer (HBM-bound stream).
//
// Follows "MSA端到端可训练记忆模型完整开源，支持亿级Token上下文", section 架构 (block mean
// pooling of K/V/K_r; 并行 RoPE: positions restart at 0 per document) and the MSA paper
// reading notes, section 路由投影器 + Top-k 稀疏注意力 (64-token blocks).
//
// Design: persistent CTAs, one memory block (<= 64 tokens x H heads) per iteration.
// Thread (parity p, head h, part q) owns dims [8q, 8q+8) and their rotate-half partners
// [64+8q, 64+8q+8) of head h for tokens p, p+2, ... of the block, so a 16-byte load of
// each half feeds the rotation with no exchange.  RoPE cos/sin for the block's 64
// positions x 64 frequencies are built once per block in shared memory from a per-CTA
// table cos/sin(i w_j) and the block's base angle (fp64 reduced), by angle addition.
#include "common.cuh"
#include "msa_pool.h"

MSA_DEFINE_LAST_ERROR(msa_pool_last_error)

namespace {

constexpr int kD = 128;      // head_dim
constexpr int kHalf = 64;    // rotate-half partner distance
constexpr int kMaxChunk = 64;

struct PoolSmem {
  float2 inner[kMaxChunk][kHalf];   // (cos, sin)(i * w_j)
  float2 table[kMaxChunk][kHalf];   // (cos, sin)((p0 + i) * w_j) for the current block
  float2 base[kHalf];               // (cos, sin)(p0 * w_j)
  double w[kHalf];                  // theta^(-2j/d)
  float partial[3][8 * 16][16];     // odd-parity partial sums, [stream][thread][value]
  int64_t tok0, n_tok, pos0;
  int skip;
};

template <typename T>
struct Loader;

template <>
struct Loader<float> {
  // 8 consecutive fp32 values
  static __device__ __forceinline__ void load8(const float* p, float* x) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
};

template <>
struct Loader<__nv_bfloat16> {
  static __device__ __forceinline__ void load8(const __nv_bfloat16* p, float* x) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
    float2 f;
    f = msa::bf16x2_to_float2(a.x); x[0] = f.x; x[1] = f.y;
    f = msa::bf16x2_to_float2(a.y); x[2] = f.x; x[3] = f.y;
    f = msa::bf16x2_to_float2(a.z); x[4] = f.x; x[5] = f.y;
    f = msa::bf16x2_to_float2(a.w); x[6] = f.x; x[7] = f.y;
  }
};

__device__ __forceinline__ void store8_bf16(__nv_bfloat16* p, const float* x) {
  uint4 o;
  o.x = msa::float2_to_bf16x2(x[0], x[1]);
  o.y = msa::float2_to_bf16x2(x[2], x[3]);
  o.z = msa::float2_to_bf16x2(x[4], x[5]);
  o.w = msa::float2_to_bf16x2(x[6], x[7]);
  *reinterpret_cast<uint4*>(p) = o;
}

template <typename TIn>
__global__ void __launch_bounds__(256) pool_kernel(
    const TIn* __restrict__ k, const TIn* __restrict__ v, const TIn* __restrict__ kr,
    const int64_t* __restrict__ doc_tok_off, const int64_t* __restrict__ doc_chunk_off, int n_docs,
    int64_t n_chunks, int H, int chunk, double log2_theta, int use_rope,
    __nv_bfloat16* __restrict__ k_bar, __nv_bfloat16* __restrict__ v_bar,
    __nv_bfloat16* __restrict__ kr_hat, float* __restrict__ kr_norm, int32_t* dev_err) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  PoolSmem& sm = *reinterpret_cast<PoolSmem*>(smem_raw);
  const int tid = threadIdx.x;
  const int per_parity = 8 * H;
  const int parity = tid / per_parity;
  const int r = tid % per_parity;
  const int h = r / 8;
  const int q = r % 8;
  const int64_t row = (int64_t)H * kD;

  if (blockIdx.x == 0 && tid == 0 && __ldg(doc_chunk_off + n_docs) != n_chunks)
    msa::set_err(dev_err, MSA_DEVERR_BAD_OFFSETS);

  if (use_rope) {
    for (int j = tid; j < kHalf; j += blockDim.x) sm.w[j] = exp2(-2.0 * (double)j / (double)kD * log2_theta);
    __syncthreads();
    for (int e = tid; e < chunk * kHalf; e += blockDim.x) {
      const int i = e / kHalf, j = e % kHalf;
      float c, s;
      msa::angle_sincos((double)i, sm.w[j], &c, &s);
      sm.inner[i][j] = make_float2(c, s);
    }
  }

  for (int64_t blk = blockIdx.x; blk < n_chunks; blk += gridDim.x) {
    __syncthreads();  // previous block's smem readers are done
    if (tid == 0) {
      const int d = msa::upper_doc(doc_chunk_off, n_docs, blk);
      const int64_t j = blk - __ldg(doc_chunk_off + d);
      const int64_t t_begin = __ldg(doc_tok_off + d), t_end = __ldg(doc_tok_off + d + 1);
      const int64_t start = t_begin + j * chunk;
      sm.skip = 0;
      if (start >= t_end || start < t_begin) {
        msa::set_err(dev_err, MSA_DEVERR_BAD_OFFSETS);
        sm.skip = 1;
      }
      sm.tok0 = start;
      sm.n_tok = min((int64_t)chunk, t_end - start);
      sm.pos0 = start - t_begin;
    }
    __syncthreads();
    if (sm.skip) continue;
    const int64_t tok0 = sm.tok0;
    const int n = (int)sm.n_tok;
    if (use_rope && k != nullptr) {
      for (int j = tid; j < kHalf; j += blockDim.x) {
        float c, s;
        msa::angle_sincos((double)sm.pos0, sm.w[j], &c, &s);
        sm.base[j] = make_float2(c, s);
      }
      __syncthreads();
      for (int e = tid; e < n * kHalf; e += blockDim.x) {
        const int i = e / kHalf, j = e % kHalf;
        const float2 b = sm.base[j], in = sm.inner[i][j];
        sm.table[i][j] = make_float2(b.x * in.x - b.y * in.y, b.y * in.x + b.x * in.y);
      }
      __syncthreads();
    }

    float ak[16], av[16], ar[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) { ak[u] = 0.f; av[u] = 0.f; ar[u] = 0.f; }
    if (parity < 2) {
      const int64_t lo_off = (int64_t)h * kD + 8 * q;
      const int64_t hi_off = lo_off + kHalf;
#pragma unroll 2
      for (int i = parity; i < n; i += 2) {
        const int64_t base = (tok0 + i) * row;
        float lo[8], hi[8];
        if (k != nullptr) {
          Loader<TIn>::load8(k + base + lo_off, lo);
          Loader<TIn>::load8(k + base + hi_off, hi);
          if (use_rope) {
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const float2 cs = sm.table[i][8 * q + u];
              ak[u] += lo[u] * cs.x - hi[u] * cs.y;
              ak[8 + u] += hi[u] * cs.x + lo[u] * cs.y;
            }
          } else {
#pragma unroll
            for (int u = 0; u < 8; ++u) { ak[u] += lo[u]; ak[8 + u] += hi[u]; }
          }
        }
        if (v != nullptr) {
          Loader<TIn>::load8(v + base + lo_off, lo);
          Loader<TIn>::load8(v + base + hi_off, hi);
#pragma unroll
          for (int u = 0; u < 8; ++u) { av[u] += lo[u]; av[8 + u] += hi[u]; }
        }
        if (kr != nullptr) {
          Loader<TIn>::load8(kr + base + lo_off, lo);
          Loader<TIn>::load8(kr + base + hi_off, hi);
#pragma unroll
          for (int u = 0; u < 8; ++u) { ar[u] += lo[u]; ar[8 + u] += hi[u]; }
        }
      }
    }
    if (parity == 1) {
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        sm.partial[0][r][u] = ak[u];
        sm.partial[1][r][u] = av[u];
        sm.partial[2][r][u] = ar[u];
      }
    }
    __syncthreads();
    if (parity == 0) {
      const float cnt = (float)n;
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        ak[u] = (ak[u] + sm.partial[0][r][u]) / cnt;
        av[u] = (av[u] + sm.partial[1][r][u]) / cnt;
        ar[u] = (ar[u] + sm.partial[2][r][u]) / cnt;
      }
      const int64_t o = blk * row + (int64_t)h * kD + 8 * q;
      if (k != nullptr && k_bar != nullptr) {
        store8_bf16(k_bar + o, ak);
        store8_bf16(k_bar + o + kHalf, ak + 8);
      }
      if (v != nullptr && v_bar != nullptr) {
        store8_bf16(v_bar + o, av);
        store8_bf16(v_bar + o + kHalf, av + 8);
      }
      if (kr != nullptr) {
        float ss = 0.f;
#pragma unroll
        for (int u = 0; u < 16; ++u) ss += ar[u] * ar[u];
        // the 8 threads of head h are 8 consecutive lanes (an aligned group) of one warp
        const unsigned grp = 0xFFu << (threadIdx.x & 24);
        ss += __shfl_xor_sync(grp, ss, 1);
        ss += __shfl_xor_sync(grp, ss, 2);
        ss += __shfl_xor_sync(grp, ss, 4);
        const float nrm = sqrtf(ss);
        const float inv = 1.0f / fmaxf(nrm, 1e-8f);
        if (kr_hat != nullptr) {
          float x[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) x[u] = ar[u] * inv;
          store8_bf16(kr_hat + o, x);
          store8_bf16(kr_hat + o + kHalf, x + 8);
        }
        if (kr_norm != nullptr && q == 0) kr_norm[blk * H + h] = nrm;
      }
    }
  }
}

// 1-token blocks without rotation: block c is token c, so each output row is its input
// row (K, V copied to bf16; K_r made unit per head).  One warp per row; lane owns the
// 8-element vectors lane + 32 i of the H*128-element row (head = (lane + 32 i) / 16).
template <typename TIn, int NV>
__global__ void __launch_bounds__(256) pool_rows_kernel(const TIn* __restrict__ k, const TIn* __restrict__ v,
                                                        const TIn* __restrict__ kr, int64_t n_rows,
                                                        __nv_bfloat16* __restrict__ k_bar,
                                                        __nv_bfloat16* __restrict__ v_bar,
                                                        __nv_bfloat16* __restrict__ kr_hat,
                                                        float* __restrict__ kr_norm) {
  constexpr int R = NV * 256;
  const int lane = threadIdx.x % 32;
  const int64_t w0 = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) / 32;
  const int64_t nw = (int64_t)gridDim.x * blockDim.x / 32;
  for (int64_t row = w0; row < n_rows; row += nw) {
    const int64_t base = row * R;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int64_t e = base + 8 * (lane + 32 * i);
      float x[8];
      if (k != nullptr && k_bar != nullptr) {
        Loader<TIn>::load8(k + e, x);
        store8_bf16(k_bar + e, x);
      }
      if (v != nullptr && v_bar != nullptr) {
        Loader<TIn>::load8(v + e, x);
        store8_bf16(v_bar + e, x);
      }
    }
    if (kr != nullptr) {
      float x[NV][8];
#pragma unroll
      for (int i = 0; i < NV; ++i) Loader<TIn>::load8(kr + base + 8 * (lane + 32 * i), x[i]);
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        float ss = 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) ss += x[i][u] * x[i][u];
        ss += __shfl_xor_sync(0xffffffffu, ss, 1);   // 16 lanes share a head
        ss += __shfl_xor_sync(0xffffffffu, ss, 2);
        ss += __shfl_xor_sync(0xffffffffu, ss, 4);
        ss += __shfl_xor_sync(0xffffffffu, ss, 8);
        const float nrm = sqrtf(ss);
        const float inv = 1.0f / fmaxf(nrm, 1e-8f);
#pragma unroll
        for (int u = 0; u < 8; ++u) x[i][u] *= inv;
        if (kr_hat != nullptr) store8_bf16(kr_hat + base + 8 * (lane + 32 * i), x[i]);
        if (kr_norm != nullptr && (lane & 15) == 0) kr_norm[row * (2 * NV) + ((lane + 32 * i) >> 4)] = nrm;
      }
    }
  }
}

template <typename TIn>
bool launch_rows(int H, const void* k, const void* v, const void* kr, int64_t n, void* kb, void* vb, void* krh,
                 float* krn, cudaStream_t s) {
  int64_t blocks = (n + 7) / 8;
  const int64_t cap = (int64_t)msa::sm_count() * 8;
  if (blocks > cap) blocks = cap;
#define MSA_ROWS(NV)                                                                                         \
  pool_rows_kernel<TIn, NV><<<(unsigned)blocks, 256, 0, s>>>((const TIn*)k, (const TIn*)v, (const TIn*)kr, n, \
                                                            (__nv_bfloat16*)kb, (__nv_bfloat16*)vb,           \
                                                            (__nv_bfloat16*)krh, krn)
  switch (H) {
    case 2: MSA_ROWS(1); return true;
    case 4: MSA_ROWS(2); return true;
    case 8: MSA_ROWS(4); return true;
    case 16: MSA_ROWS(8); return true;
    default: return false;
  }
#undef MSA_ROWS
}

}  // namespace

extern "C" int64_t msa_count_chunks(const int64_t* doc_tok_offsets_host, int32_t n_docs, int32_t chunk,
                                    int64_t* doc_chunk_offsets_host) {
  if (doc_tok_offsets_host == nullptr || n_docs < 0 || chunk <= 0) return -1;
  if (doc_tok_offsets_host[0] != 0) return -1;
  int64_t total = 0;
  if (doc_chunk_offsets_host) doc_chunk_offsets_host[0] = 0;
  for (int32_t d = 0; d < n_docs; ++d) {
    const int64_t n = doc_tok_offsets_host[d + 1] - doc_tok_offsets_host[d];
    if (n < 0) return -1;
    total += (n + chunk - 1) / chunk;
    if (doc_chunk_offsets_host) doc_chunk_offsets_host[d + 1] = total;
  }
  return total;
}

extern "C" msa_status msa_pool_blocks(const void* k, const void* v, const void* kr, msa_dtype in_dtype,
                                      const int64_t* doc_tok_offsets, const int64_t* doc_chunk_offsets,
                                      int32_t n_docs, int64_t n_chunks, int32_t n_heads, int32_t head_dim,
                                      int32_t chunk, float rope_theta, void* k_bar, void* v_bar,
                                      void* kr_hat, float* kr_norm, int32_t* dev_err,
                                      msa_stream_t stream) {
  if (head_dim != kD) return msa_fail(MSA_ERR_INVALID_ARG, "head_dim must be 128 (got %d)", head_dim);
  if (n_heads < 1 || n_heads > 16) return msa_fail(MSA_ERR_INVALID_ARG, "n_heads must be in [1,16]");
  if (chunk < 1 || chunk > kMaxChunk) return msa_fail(MSA_ERR_INVALID_ARG, "chunk must be in [1,64]");
  if (n_docs < 0 || n_chunks < 0) return msa_fail(MSA_ERR_INVALID_ARG, "negative count");
  if (in_dtype != MSA_F32 && in_dtype != MSA_BF16) return msa_fail(MSA_ERR_UNSUPPORTED, "in_dtype");
  if (!(rope_theta == 0.0f || rope_theta > 1.0f))
    return msa_fail(MSA_ERR_INVALID_ARG, "rope_theta must be 0 (no rotation) or > 1");
  if (doc_tok_offsets == nullptr || doc_chunk_offsets == nullptr)
    return msa_fail(MSA_ERR_INVALID_ARG, "null offsets");
  if ((k && !k_bar) || (v && !v_bar) || (kr && !kr_hat && !kr_norm))
    return msa_fail(MSA_ERR_INVALID_ARG, "an input stream has no output");
  const void* ptrs[6] = {k, v, kr, k_bar, v_bar, kr_hat};
  for (const void* p : ptrs)
    if (p && !msa::aligned16(p)) return msa_fail(MSA_ERR_INVALID_ARG, "buffers must be 16-byte aligned");
  const int arch = msa::current_device_is_sm100(nullptr);
  if (arch < 0) return msa_fail(MSA_ERR_CUDA, "no CUDA device");
  if (arch == 0) return msa_fail(MSA_ERR_UNSUPPORTED, "device is not sm_100");
  if (n_chunks == 0 || n_docs == 0 || (!k && !v && !kr)) return msa_ok();

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (chunk == 1 && (k == nullptr || rope_theta == 0.0f)) {
    // every block is one token: row-wise fast path (no positions, so no offsets needed)
    const bool ok = in_dtype == MSA_F32 ? launch_rows<float>(n_heads, k, v, kr, n_chunks, k_bar, v_bar, kr_hat, kr_norm, s)
                                        : launch_rows<__nv_bfloat16>(n_heads, k, v, kr, n_chunks, k_bar, v_bar, kr_hat,
                                                                     kr_norm, s);
    if (ok) {
      MSA_CUDA_TRY(cudaGetLastError());
      return msa_ok();
    }
  }
  const size_t smem = sizeof(PoolSmem);
  const int threads = 16 * n_heads;
  const int use_rope = (rope_theta != 0.0f && k != nullptr) ? 1 : 0;
  const double log2_theta = use_rope ? log2((double)rope_theta) : 0.0;
  const int per_sm = 2;
  int64_t grid = (int64_t)msa::sm_count() * per_sm;
  if (grid > n_chunks) grid = n_chunks;
  if (in_dtype == MSA_F32) {
    MSA_CUDA_TRY(cudaFuncSetAttribute(pool_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    pool_kernel<float><<<(unsigned)grid, threads, smem, s>>>(
        (const float*)k, (const float*)v, (const float*)kr, doc_tok_offsets, doc_chunk_offsets, n_docs,
        n_chunks, n_heads, chunk, log2_theta, use_rope, (__nv_bfloat16*)k_bar, (__nv_bfloat16*)v_bar,
        (__nv_bfloat16*)kr_hat, kr_norm, dev_err);
  } else {
    MSA_CUDA_TRY(cudaFuncSetAttribute(pool_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem));
    pool_kernel<__nv_bfloat16><<<(unsigned)grid, threads, smem, s>>>(
        (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, (const __nv_bfloat16*)kr, doc_tok_offsets,
        doc_chunk_offsets, n_docs, n_chunks, n_heads, chunk, log2_theta, use_rope, (__nv_bfloat16*)k_bar,
        (__nv_bfloat16*)v_bar, (__nv_bfloat16*)kr_hat, kr_norm, dev_err);
  }
  MSA_CUDA_TRY(cudaGetLastError());
  return msa_ok();
}
