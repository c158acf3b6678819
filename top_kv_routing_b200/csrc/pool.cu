// Step 1: document-wise RoPE + block mean pooling of one bank layer (HBM-bound stream).
//
// Follows "MSA端到端可训练记忆模型完整开源，支持亿级Token上下文", section 架构 (block mean
// pooling of K/V/K_r; 并行 RoPE: positions restart at 0 per document) and the MSA paper
// reading notes, section 路由投影器 + Top-k 稀疏注意力 (64-token blocks).
//
// Design: a streaming kernel, one CTA per SM, each owning a contiguous range of memory
// blocks (so a block's document is found once by binary search and then advanced
// incrementally).  A producer warp copies the blocks' token rows of K, V and K_r with
// bulk asynchronous copies (cp.async.bulk, completion on mbarriers) into a ring of
// shared-memory stages of S tokens; one consumer warp per head h accumulates them.
// Lane (g, q) of that warp (g = lane / 8) owns dims [8q, 8q+8) and their rotate-half
// partners [64+8q, 64+8q+8) of head h for the block's tokens g, g+4, g+8, ...; its 8
// frequencies' cos/sin live in registers, exact at the lane's first token of the block
// (angle / pi reduced in fp64, fp32 sincospif) and advanced by the fixed rotation of 4
// positions per token.  At the block's end the four token groups meet through warp
// shuffles.  Every wait is bounded (2 s); a timeout sets MSA_DEVERR_TIMEOUT.
#include "common.cuh"
#include "msa_pool.h"

MSA_DEFINE_LAST_ERROR(msa_pool_last_error)

namespace {

constexpr int kD = 128;      // head_dim
constexpr int kHalf = 64;    // rotate-half partner distance
constexpr int kMaxChunk = 64;

template <typename T>
struct Loader;

// 8 consecutive elements: raw() reads them (16 or 32 bytes), unpack() widens to fp32.
template <>
struct Loader<float> {
  struct Raw {
    float4 a, b;
  };
  static __device__ __forceinline__ void raw(const float* p, Raw& r) {
    r.a = __ldg(reinterpret_cast<const float4*>(p));
    r.b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  }
  static __device__ __forceinline__ void unpack(const Raw& r, float* x) {
    x[0] = r.a.x; x[1] = r.a.y; x[2] = r.a.z; x[3] = r.a.w;
    x[4] = r.b.x; x[5] = r.b.y; x[6] = r.b.z; x[7] = r.b.w;
  }
  static __device__ __forceinline__ void load8(const float* p, float* x) {
    Raw r;
    raw(p, r);
    unpack(r, x);
  }
  static __device__ __forceinline__ void load8_smem(const unsigned char* p, float* x) {
    Raw r;
    r.a = *reinterpret_cast<const float4*>(p);
    r.b = *reinterpret_cast<const float4*>(p + 16);
    unpack(r, x);
  }
};

template <>
struct Loader<__nv_bfloat16> {
  using Raw = uint4;
  static __device__ __forceinline__ void raw(const __nv_bfloat16* p, Raw& r) {
    r = __ldg(reinterpret_cast<const uint4*>(p));
  }
  static __device__ __forceinline__ void unpack(const Raw& a, float* x) {
    float2 f;
    f = msa::bf16x2_to_float2(a.x); x[0] = f.x; x[1] = f.y;
    f = msa::bf16x2_to_float2(a.y); x[2] = f.x; x[3] = f.y;
    f = msa::bf16x2_to_float2(a.z); x[4] = f.x; x[5] = f.y;
    f = msa::bf16x2_to_float2(a.w); x[6] = f.x; x[7] = f.y;
  }
  static __device__ __forceinline__ void load8(const __nv_bfloat16* p, float* x) {
    Raw r;
    raw(p, r);
    unpack(r, x);
  }
  static __device__ __forceinline__ void load8_smem(const unsigned char* p, float* x) {
    unpack(*reinterpret_cast<const uint4*>(p), x);
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

constexpr int kStageBytesTarget = 48 * 1024;  // K, V and K_r rows of one stage
constexpr int kRingBytes = 192 * 1024;
constexpr unsigned long long kTimeoutNs = 2000000000ull;

struct SliceMeta {
  int64_t blk;    // memory block
  int first;      // index in the block of the slice's first token
  int rows;       // tokens in the slice
  int n_block;    // tokens in the block
  int pos0;       // position (in its document) of the block's first token
  int last;       // last slice of the block
  int state;      // 0 = tokens, 1 = skipped block (bad offsets), 2 = end of the sequence
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t global_timer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Waits for the phase with this parity; false after 2 s or once another warp has given up.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*abort_flag) return false;
      if (global_timer() - t0 > kTimeoutNs) return false;
    }
  }
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// global -> shared bulk copy (no multicast), completing on an mbarrier of this CTA
__device__ __forceinline__ void bulk_copy(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

template <typename TIn, int kWarps>  // kWarps: heads + 1 at most
__global__ void __launch_bounds__(kWarps * 32) pool_kernel(
    const TIn* __restrict__ k, const TIn* __restrict__ v, const TIn* __restrict__ kr,
    const int64_t* __restrict__ doc_tok_off, const int64_t* __restrict__ doc_chunk_off, int n_docs,
    int64_t n_chunks, int64_t blocks_per_cta, int H, int chunk, int S, int n_stages, double log2_theta, int use_rope,
    __nv_bfloat16* __restrict__ k_bar, __nv_bfloat16* __restrict__ v_bar,
    __nv_bfloat16* __restrict__ kr_hat, float* __restrict__ kr_norm, int32_t* dev_err) {
  extern __shared__ __align__(128) unsigned char ring[];
  __shared__ SliceMeta meta[8];
  __shared__ __align__(8) uint64_t full[8], empty[8];
  __shared__ int abort_flag;
  __shared__ double s_wpi[kHalf];  // theta^(-2j/d) / pi
  __shared__ float2 s_r4[kHalf];   // (cos, sin) of 4 positions' angle, per frequency
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (use_rope)
    for (int j = threadIdx.x; j < kHalf; j += blockDim.x) {
      const double w = exp2(-2.0 * (double)j / (double)kD * log2_theta) * 0.31830988618379067154;
      double x = 4.0 * w;
      x -= 2.0 * rint(0.5 * x);
      float sn, cs;
      sincospif((float)x, &sn, &cs);
      s_wpi[j] = w;
      s_r4[j] = make_float2(cs, sn);
    }
  const int64_t row_elems = (int64_t)H * kD;
  const uint32_t row_bytes = (uint32_t)(row_elems * sizeof(TIn));
  const uint32_t region = (uint32_t)S * row_bytes;  // one stream's rows in a stage
  const uint32_t stage_bytes = 3u * region;
  if (threadIdx.x == 0) {
    for (int i = 0; i < n_stages; ++i) {
      mbar_init(smem_u32(&full[i]), 1);
      mbar_init(smem_u32(&empty[i]), (uint32_t)H);
    }
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    if (blockIdx.x == 0 && __ldg(doc_chunk_off + n_docs) != n_chunks) msa::set_err(dev_err, MSA_DEVERR_BAD_OFFSETS);
  }
  __syncthreads();
  const int64_t b_begin = blockIdx.x * blocks_per_cta;
  const int64_t b_end = min(n_chunks, b_begin + blocks_per_cta);

  if (warp == H) {
    // ------------------------------------------------------------ producer
    if (lane != 0) return;
    int stage = 0;
    uint32_t phase = 0;
    uint32_t armed = 0u, armed_phase = 0u;  // stages with a copy issued, and its phase bit
    bool ok = true;
    auto next_stage = [&]() -> bool {  // waits for a free stage
      if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, &abort_flag)) return false;
      return true;
    };
    auto advance = [&]() {
      armed |= 1u << stage;
      armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
      if (++stage == n_stages) {
        stage = 0;
        phase ^= 1u;
      }
    };
    int d = b_begin < b_end ? msa::upper_doc(doc_chunk_off, n_docs, b_begin) : 0;
    for (int64_t blk = b_begin; blk < b_end && ok; ++blk) {
      while (d + 1 < n_docs && __ldg(doc_chunk_off + d + 1) <= blk) ++d;
      const int64_t j = blk - __ldg(doc_chunk_off + d);
      const int64_t t_begin = __ldg(doc_tok_off + d), t_end = __ldg(doc_tok_off + d + 1);
      const int64_t tok0 = t_begin + j * chunk;
      const bool bad = tok0 >= t_end || tok0 < t_begin;
      const int nb = bad ? 0 : (int)min((int64_t)chunk, t_end - tok0);
      const int n_slices = bad ? 1 : (nb + S - 1) / S;
      for (int sl = 0; sl < n_slices; ++sl) {
        if (!next_stage()) {
          ok = false;
          break;
        }
        SliceMeta& m = meta[stage];
        m.blk = blk;
        m.first = sl * S;
        m.rows = bad ? 0 : min(S, nb - sl * S);
        m.n_block = nb;
        m.pos0 = (int)(j * chunk);
        m.last = sl == n_slices - 1;
        m.state = bad ? 1 : 0;
        if (bad) msa::set_err(dev_err, MSA_DEVERR_BAD_OFFSETS);
        const uint32_t bytes = (uint32_t)m.rows * row_bytes;
        const uint32_t fb = smem_u32(&full[stage]);
        const uint32_t dst = smem_u32(ring) + stage * stage_bytes;
        const int64_t src = (tok0 + sl * S) * row_elems;
        mbar_arrive_expect_tx(fb, bytes * ((k != nullptr) + (v != nullptr) + (kr != nullptr)));
        if (bytes > 0) {
          if (k != nullptr) bulk_copy(dst, k + src, bytes, fb);
          if (v != nullptr) bulk_copy(dst + region, v + src, bytes, fb);
          if (kr != nullptr) bulk_copy(dst + 2 * region, kr + src, bytes, fb);
        }
        advance();
      }
    }
    if (ok && next_stage()) {  // the end marker
      meta[stage].state = 2;
      mbar_arrive_expect_tx(smem_u32(&full[stage]), 0u);
      advance();
    } else {
      ok = false;
    }
    if (!ok) {
      abort_flag = 1;
      msa::set_err(dev_err, MSA_DEVERR_TIMEOUT);
    }
    // no copy may still be writing this CTA's shared memory when it exits
    for (int i = 0; i < n_stages; ++i) {
      if (!((armed >> i) & 1u)) continue;
      const uint64_t t0 = global_timer();
      while (!mbar_try_wait(smem_u32(&full[i]), (armed_phase >> i) & 1u))
        if (global_timer() - t0 > kTimeoutNs) break;
    }
    return;
  }

  // -------------------------------------------------------------- consumers: warp h = head
  const int h = warp, g = lane >> 3, q = lane & 7;
  float ak[16], av[16], ar[16], c[8], sn[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) { c[u] = 1.f; sn[u] = 0.f; }
  const uint32_t lo_byte = (uint32_t)((h * kD + 8 * q) * (int)sizeof(TIn));
  const uint32_t hi_byte = lo_byte + (uint32_t)(kHalf * sizeof(TIn));
  int stage = 0;
  uint32_t phase = 0;
  while (true) {
    if (!mbar_wait(smem_u32(&full[stage]), phase, &abort_flag)) {
      if (lane == 0) {
        abort_flag = 1;
        msa::set_err(dev_err, MSA_DEVERR_TIMEOUT);
      }
      break;
    }
    const SliceMeta m = meta[stage];
    if (m.state == 2) break;
    if (m.state == 0) {
      if (m.first == 0) {  // a new block
#pragma unroll
        for (int u = 0; u < 16; ++u) { ak[u] = 0.f; av[u] = 0.f; ar[u] = 0.f; }
        if (use_rope && k != nullptr) {
          const double pos = (double)(m.pos0 + g);
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            double x = pos * s_wpi[8 * q + u];  // angle / pi
            x -= 2.0 * rint(0.5 * x);
            sincospif((float)x, &sn[u], &c[u]);
          }
        }
      }
      const unsigned char* st = ring + stage * stage_bytes;
      for (int rr = g; rr < m.rows; rr += 4) {
        const unsigned char* rowp = st + rr * row_bytes;
        float lo[8], hi[8];
        if (k != nullptr) {
          Loader<TIn>::load8_smem(rowp + lo_byte, lo);
          Loader<TIn>::load8_smem(rowp + hi_byte, hi);
          if (use_rope) {
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              ak[u] += lo[u] * c[u] - hi[u] * sn[u];
              ak[8 + u] += hi[u] * c[u] + lo[u] * sn[u];
              const float2 r4 = s_r4[8 * q + u];  // advance 4 positions
              const float cn = c[u] * r4.x - sn[u] * r4.y;
              sn[u] = sn[u] * r4.x + c[u] * r4.y;
              c[u] = cn;
            }
          } else {
#pragma unroll
            for (int u = 0; u < 8; ++u) { ak[u] += lo[u]; ak[8 + u] += hi[u]; }
          }
        }
        if (v != nullptr) {
          Loader<TIn>::load8_smem(rowp + region + lo_byte, lo);
          Loader<TIn>::load8_smem(rowp + region + hi_byte, hi);
#pragma unroll
          for (int u = 0; u < 8; ++u) { av[u] += lo[u]; av[8 + u] += hi[u]; }
        }
        if (kr != nullptr) {
          Loader<TIn>::load8_smem(rowp + 2 * region + lo_byte, lo);
          Loader<TIn>::load8_smem(rowp + 2 * region + hi_byte, hi);
#pragma unroll
          for (int u = 0; u < 8; ++u) { ar[u] += lo[u]; ar[8 + u] += hi[u]; }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&empty[stage]));  // the stage may be refilled
    if (m.state == 0 && m.last) {
      // the four token groups (lanes q, q+8, q+16, q+24) meet
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        ak[u] += __shfl_xor_sync(0xffffffffu, ak[u], 8);
        ak[u] += __shfl_xor_sync(0xffffffffu, ak[u], 16);
        av[u] += __shfl_xor_sync(0xffffffffu, av[u], 8);
        av[u] += __shfl_xor_sync(0xffffffffu, av[u], 16);
        ar[u] += __shfl_xor_sync(0xffffffffu, ar[u], 8);
        ar[u] += __shfl_xor_sync(0xffffffffu, ar[u], 16);
      }
      const float inv_n = 1.0f / (float)m.n_block;
      const int64_t o = m.blk * row_elems + (int64_t)h * kD + 8 * q;
      float ss = 0.f;
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        ak[u] *= inv_n;
        av[u] *= inv_n;
        ar[u] *= inv_n;
        ss += ar[u] * ar[u];
      }
      ss += __shfl_xor_sync(0xffffffffu, ss, 1);  // the 8 q-lanes of the head
      ss += __shfl_xor_sync(0xffffffffu, ss, 2);
      ss += __shfl_xor_sync(0xffffffffu, ss, 4);
      if (g == 0) {
        if (k != nullptr && k_bar != nullptr) {
          store8_bf16(k_bar + o, ak);
          store8_bf16(k_bar + o + kHalf, ak + 8);
        }
        if (v != nullptr && v_bar != nullptr) {
          store8_bf16(v_bar + o, av);
          store8_bf16(v_bar + o + kHalf, av + 8);
        }
        if (kr != nullptr) {
          const float nrm = sqrtf(ss);
          const float inv = 1.0f / fmaxf(nrm, 1e-8f);
          if (kr_hat != nullptr) {
            float x[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) x[u] = ar[u] * inv;
            store8_bf16(kr_hat + o, x);
            store8_bf16(kr_hat + o + kHalf, x + 8);
          }
          if (kr_norm != nullptr && q == 0) kr_norm[m.blk * H + h] = nrm;
        }
      }
    }
    if (++stage == n_stages) {
      stage = 0;
      phase ^= 1u;
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
  const int use_rope = (rope_theta != 0.0f && k != nullptr) ? 1 : 0;
  const double log2_theta = use_rope ? log2((double)rope_theta) : 0.0;
  // stages of S tokens of each stream (S a multiple of 4, the token groups of a warp)
  const size_t esz = in_dtype == MSA_F32 ? 4 : 2;
  const size_t row_bytes = (size_t)n_heads * kD * esz;
  int S = (int)(kStageBytesTarget / (3 * row_bytes)) / 4 * 4;
  if (S < 4) S = 4;
  if (S > 64) S = 64;
  int n_stages = (int)(kRingBytes / (3 * (size_t)S * row_bytes));
  if (n_stages > 8) n_stages = 8;
  if (n_stages < 2) return msa_fail(MSA_ERR_UNSUPPORTED, "token rows too large for the staging ring");
  const size_t smem = (size_t)n_stages * 3 * S * row_bytes;
  const int threads = 32 * (n_heads + 1);  // a warp per head + the producer warp
  int64_t grid = msa::sm_count();           // one CTA per SM (the ring fills shared memory)
  if (grid > n_chunks) grid = n_chunks;
  const int64_t per_cta = (n_chunks + grid - 1) / grid;
  grid = (n_chunks + per_cta - 1) / per_cta;
#define MSA_POOL_LAUNCH(T, W)                                                                                   \
  do {                                                                                                         \
    MSA_CUDA_TRY(cudaFuncSetAttribute(pool_kernel<T, W>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)); \
    pool_kernel<T, W><<<(unsigned)grid, threads, smem, s>>>(                                                    \
        (const T*)k, (const T*)v, (const T*)kr, doc_tok_offsets, doc_chunk_offsets, n_docs, n_chunks, per_cta, \
        n_heads, chunk, S, n_stages, log2_theta, use_rope, (__nv_bfloat16*)k_bar, (__nv_bfloat16*)v_bar,       \
        (__nv_bfloat16*)kr_hat, kr_norm, dev_err);                                                              \
  } while (0)
  if (in_dtype == MSA_F32) {
    if (n_heads <= 8) MSA_POOL_LAUNCH(float, 9);
    else MSA_POOL_LAUNCH(float, 17);
  } else {
    if (n_heads <= 8) MSA_POOL_LAUNCH(__nv_bfloat16, 9);
    else MSA_POOL_LAUNCH(__nv_bfloat16, 17);
  }
#undef MSA_POOL_LAUNCH
  MSA_CUDA_TRY(cudaGetLastError());
  return msa_ok();
}
