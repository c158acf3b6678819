// Prefill attention on the tcgen05 tensor cores.
//
// Computes what the prefill's attention step defines (msa_prefill.h): for every (query b,
// layer l, key head h) and every row (token t of the block, query head q of the group),
// softmax over [memory keys 0 .. M ; local keys 0 .. len + t] of the scaled dot products,
// times the values.  Follows "MSA端到端可训练记忆模型完整开源，支持亿级Token上下文", section
// 推理流水线, and the MSA paper reading notes, section 推理全流程.
//
// One CTA (192 threads) per 128 rows: 128 / G tokens x the G query heads of key head h.
//   warp 5, one thread   TMA producer: tiles of 64 keys (K as two 64-column boxes, then V
//                        the same), 128-byte swizzle, a 3-stage ring; memory tiles first,
//                        then local tiles up to the CTA's last token
//   warp 4, one thread   MMA issuer: S_i = Q K_i^T (M = 128, N = 64, K = 128) into one of two
//                        TMEM score buffers, then O += P_{i-1} V_{i-1} (M = 128, N = 128,
//                        K = 64) into the TMEM output.  The rotated queries and the softmax
//                        weights are each a bf16 value plus a bf16 residual (two MMAs), the
//                        keys and values exact bf16; V is read MN-major straight from its
//                        [key][d] rows
//   warps 0..3           thread = row (TMEM lane): builds its rotated, scaled query row in
//                        shared memory; per tile reads its score row, masks it (memory keys
//                        < M, local keys <= its own local index), keeps a running maximum
//                        that is raised (and O rescaled in TMEM) only when a score exceeds it
//                        by more than 2^8, writes its weights exp2(s - m) as the A operand of
//                        the next PV, and at the end divides O by the running sum.
// Key rows past a tile's valid count are zeroed in shared memory before the PV that reads
// them (the cache rows beyond the valid length may hold anything).  Every wait is bounded
// (2 s); a timeout sets MSA_DEVERR_TIMEOUT and the CTA drains and frees its TMEM.
#include <cuda.h>

#include "common.cuh"
#include "prefill_tc.cuh"
#include "tc_common.cuh"

namespace prefill_tc {
namespace {
using namespace tc;

constexpr int kD = 128;
constexpr int kHalf = 64;
constexpr int kRows = 128;
constexpr int kKeys = 64;
constexpr int kStages = 3;
constexpr int kThreads = 192;
constexpr int kQHalf = kRows * 128;      // 16 KB: 64 bf16 of every row
constexpr int kQBytes = 2 * kQHalf;      // 32 KB: one bf16 copy of the CTA's queries
constexpr int kPBytes = kRows * 128;     // 16 KB: 64 bf16 weights of every row
constexpr int kKVHalf = kKeys * 128;     // 8 KB: 64 keys x 64 elements
constexpr int kTileBytes = 4 * kKVHalf;  // K (two halves) then V (two halves)
constexpr int kOffQhi = 0;
constexpr int kOffQlo = kQBytes;
constexpr int kOffPhi = 2 * kQBytes;
constexpr int kOffPlo = 2 * kQBytes + kPBytes;
constexpr int kOffRing = 2 * kQBytes + 2 * kPBytes;
constexpr int kSmemData = kOffRing + kStages * kTileBytes;
constexpr int kSmem = kSmemData + 1024 + 256;
constexpr uint32_t kTmemCols = 256;  // S0 [0, 64) | S1 [64, 128) | O [128, 256)
constexpr uint32_t kColO = 128;
constexpr float kHeadroom = 8.0f;    // log2 growth of a row's maximum tolerated before rescaling

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  const __nv_bfloat162 l =
      __floats2bfloat162_rn(x0 - __uint_as_float(hi << 16), x1 - __uint_as_float(hi & 0xFFFF0000u));
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

template <int G>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_mem, const __grid_constant__ CUtensorMap tm_lk,
                      const __grid_constant__ CUtensorMap tm_lv, const __nv_bfloat16* __restrict__ q, int T, int L,
                      int H, const int32_t* __restrict__ local_len, int cap, const int32_t* __restrict__ mem_len,
                      int M_max, int pos_off, double log2_theta, float qscale, __nv_bfloat16* __restrict__ out,
                      int32_t* dev_err) {
  constexpr int kTok = kRows / G;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSmemData);
  uint64_t* full = bars;                 // [kStages]
  uint64_t* empty = bars + kStages;      // [kStages]
  uint64_t* bar_q = empty + kStages;     // queries written (4 warps)
  uint64_t* bar_s = bar_q + 1;           // [2] scores ready
  uint64_t* bar_p = bar_s + 2;           // weights ready (4 warps)
  uint64_t* bar_pv = bar_p + 1;          // PV done
  uint64_t* drain = bar_pv + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  __shared__ double s_w[kHalf];          // theta^(-2j/d) / pi

  const int h = blockIdx.y;
  const int64_t bl = blockIdx.z;
  const int b = (int)(bl / L);
  const int tok0 = blockIdx.x * kTok;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Hq = H * G;
  const int len = local_len[b];
  if (len < 0 || len + T > cap) return;  // (the append kernel has set MSA_DEVERR_LOCAL_FULL)
  int M = mem_len[bl];
  M = M < 0 ? 0 : (M > M_max ? M_max : M);
  const int tok_last = min(T, tok0 + kTok) - 1;
  const int n_local = len + tok_last + 1;
  const int nt_mem = (M + kKeys - 1) / kKeys;
  const int nt = nt_mem + (n_local + kKeys - 1) / kKeys;

  if (tid < kHalf) s_w[tid] = exp2(-2.0 * (double)tid / (double)kD * log2_theta) * 0.31830988618379067154;
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(bar_q), 4);
    mbar_init(smem_u32(&bar_s[0]), 1);
    mbar_init(smem_u32(&bar_s[1]), 1);
    mbar_init(smem_u32(bar_p), 4);
    mbar_init(smem_u32(bar_pv), 1);
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_async_smem();
  }
  if (warp == 4) {
    tmem_alloc<false>(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish<false>();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t sbase = smem_u32(smem);

  if (warp == 5) {
    if (lane == 0) {
      // ---------------- TMA producer
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_mem)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_lk)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_lv)) : "memory");
      const uint64_t pol = policy_evict_last();
      int armed[kStages] = {-1, -1, -1};
      bool ok = true;
      for (int i = 0; i < nt && ok; ++i) {
        const int stage = i % kStages;
        const uint32_t ph = (uint32_t)((i / kStages) & 1);
        if (!mbar_wait(smem_u32(&empty[stage]), ph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t fb = smem_u32(&full[stage]);
        const uint32_t dst = sbase + kOffRing + stage * kTileBytes;
        mbar_arrive_expect_tx(fb, kTileBytes);
        if (i < nt_mem) {
          const int rk = (int)((((bl * 2 + 0) * H + h) * (int64_t)M_max) + i * kKeys);
          const int rv = (int)((((bl * 2 + 1) * H + h) * (int64_t)M_max) + i * kKeys);
          tma_load_2d(dst, &tm_mem, fb, 0, rk, pol);
          tma_load_2d(dst + kKVHalf, &tm_mem, fb, kHalf, rk, pol);
          tma_load_2d(dst + 2 * kKVHalf, &tm_mem, fb, 0, rv, pol);
          tma_load_2d(dst + 3 * kKVHalf, &tm_mem, fb, kHalf, rv, pol);
        } else {
          const int r = (int)((bl * H + h) * (int64_t)cap + (int64_t)(i - nt_mem) * kKeys);
          tma_load_2d(dst, &tm_lk, fb, 0, r, pol);
          tma_load_2d(dst + kKVHalf, &tm_lk, fb, kHalf, r, pol);
          tma_load_2d(dst + 2 * kKVHalf, &tm_lv, fb, 0, r, pol);
          tma_load_2d(dst + 3 * kKVHalf, &tm_lv, fb, kHalf, r, pol);
        }
        armed[stage] = (int)ph;
      }
      if (!ok) {
        *abort_flag = 1;
        msa::set_err(dev_err, MSA_DEVERR_TIMEOUT);
        for (int s = 0; s < kStages; ++s)
          if (armed[s] >= 0) mbar_drain(smem_u32(&full[s]), (uint32_t)armed[s]);
      }
    }
  } else if (warp == 4) {
    if (lane == 0) {
      // ---------------- MMA issuer
      constexpr uint32_t idesc_s = idesc_make(kRows, kKeys, false);
      constexpr uint32_t idesc_pv = idesc_make_bmn(kRows, kD);
      bool ok = mbar_wait(smem_u32(bar_q), 0u, abort_flag), issued = false;
      tc_fence_after();
      for (int i = 0; i <= nt && ok; ++i) {
        if (i < nt) {
          const int stage = i % kStages;
          if (!mbar_wait(smem_u32(&full[stage]), (uint32_t)((i / kStages) & 1), abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t kt = sbase + kOffRing + stage * kTileBytes;
          const uint32_t d_s = tmem_base + (uint32_t)((i & 1) * kKeys);
#pragma unroll
          for (int ks = 0; ks < kD / 16; ++ks) {
            const uint32_t off = (uint32_t)((ks >> 2) * kQHalf);
            const uint64_t kdesc = sw128_desc(kt + (uint32_t)((ks >> 2) * kKVHalf)) + (uint64_t)(2 * (ks & 3));
            umma<false, false>(d_s, sw128_desc(sbase + kOffQhi + off) + (uint64_t)(2 * (ks & 3)), kdesc, idesc_s,
                               ks > 0 ? 1u : 0u);
            umma<false, false>(d_s, sw128_desc(sbase + kOffQlo + off) + (uint64_t)(2 * (ks & 3)), kdesc, idesc_s, 1u);
          }
          issued = true;
          umma_commit<false>(smem_u32(&bar_s[i & 1]));
        }
        if (i >= 1) {
          const int j = i - 1, stage = j % kStages;
          if (!mbar_wait(smem_u32(bar_p), (uint32_t)(j & 1), abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t vt = sbase + kOffRing + stage * kTileBytes + 2 * kKVHalf;
#pragma unroll
          for (int ks = 0; ks < kKeys / 16; ++ks) {
            const uint64_t vdesc = sw128_desc_mn(vt + (uint32_t)(ks * 2048), kKVHalf, 1024);
            umma<false, false>(tmem_base + kColO, sw128_desc(sbase + kOffPhi) + (uint64_t)(2 * ks), vdesc, idesc_pv,
                               (j > 0 || ks > 0) ? 1u : 0u);
            umma<false, false>(tmem_base + kColO, sw128_desc(sbase + kOffPlo) + (uint64_t)(2 * ks), vdesc, idesc_pv,
                               1u);
          }
          umma_commit<false>(smem_u32(bar_pv));
          umma_commit<false>(smem_u32(&empty[stage]));
        }
      }
      if (!ok) {
        *abort_flag = 1;
        msa::set_err(dev_err, MSA_DEVERR_TIMEOUT);
        if (issued) {
          umma_commit<false>(smem_u32(drain));
          mbar_drain(smem_u32(drain), 0u);
        }
      }
    }
  } else {
    // ---------------- rows (warps 0..3, thread = TMEM lane = row)
    const int r = tid;
    const int tl = r / G, hd = r % G;
    const int tok = tok0 + tl;
    const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
    {  // rotated, scaled query row: bf16 value and residual, 128-byte swizzled rows
      float x[kD];
      if (tok < T) {
        const uint4* src = reinterpret_cast<const uint4*>(q + ((bl * T + tok) * Hq + (int64_t)h * G + hd) * kD);
#pragma unroll
        for (int c = 0; c < kD / 8; ++c) {
          const uint4 w = __ldg(src + c);
          const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            x[8 * c + 2 * e] = __uint_as_float(ww[e] << 16);
            x[8 * c + 2 * e + 1] = __uint_as_float(ww[e] & 0xFFFF0000u);
          }
        }
        const double pos = (double)pos_off + (double)(len + tok);
#pragma unroll
        for (int j = 0; j < kHalf; ++j) {
          double u = pos * s_w[j];
          u -= 2.0 * rint(0.5 * u);
          float sn, cs;
          sincospif((float)u, &sn, &cs);
          const float a = x[j], bb = x[j + kHalf];
          x[j] = (a * cs - bb * sn) * qscale;
          x[j + kHalf] = (bb * cs + a * sn) * qscale;
        }
      } else {
#pragma unroll
        for (int j = 0; j < kD; ++j) x[j] = 0.f;
      }
#pragma unroll
      for (int c = 0; c < kD / 8; ++c) {  // chunk c: elements 8c .. 8c+7
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) split2(x[8 * c + 2 * e], x[8 * c + 2 * e + 1], hw[e], lw[e]);
        const uint32_t off = (uint32_t)((c >> 3) * kQHalf + r * 128 + (((c & 7) ^ (r & 7)) << 4));
        st_shared_v4(sbase + kOffQhi + off, hw[0], hw[1], hw[2], hw[3]);
        st_shared_v4(sbase + kOffQlo + off, lw[0], lw[1], lw[2], lw[3]);
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(bar_q));
    }
    const int lim = len + min(tok, T - 1);
    float m_used = -INFINITY, l_sum = 0.f;
    bool ok = true;
    for (int i = 0; i < nt; ++i) {
      // (waits are made warp-uniform: the TMEM accesses below are warp-collective)
      if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&bar_s[i & 1]), (uint32_t)((i >> 1) & 1), abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sa[32], sb[32];
      tmem_ld32(tmem_base + lane_addr + (uint32_t)((i & 1) * kKeys), sa);
      tmem_ld32(tmem_base + lane_addr + (uint32_t)((i & 1) * kKeys + 32), sb);
      tmem_wait_ld();
      const bool local = i >= nt_mem;
      const int key0 = local ? (i - nt_mem) * kKeys : i * kKeys;
      const int n_valid = local ? min(kKeys, n_local - key0) : min(kKeys, M - key0);
      float mx = -INFINITY;
      float s[kKeys];
#pragma unroll
      for (int e = 0; e < kKeys; ++e) {
        const int key = key0 + e;
        const bool v = local ? key <= lim : key < M;
        s[e] = v ? __uint_as_float(e < 32 ? sa[e] : sb[e - 32]) : -INFINITY;
        mx = fmaxf(mx, s[e]);
      }
      const bool need = mx > m_used + kHeadroom;
      if (i > 0) {  // PV of the previous tile done: O is stable and the weight buffer free
        if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(bar_pv), (uint32_t)((i - 1) & 1), abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, need)) {
          const float alpha = need ? exp2f(m_used - mx) : 1.0f;
#pragma unroll 1
          for (int c = 0; c < kD / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(tmem_base + lane_addr + kColO + (uint32_t)(c * 32), o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(tmem_base + lane_addr + kColO + (uint32_t)(c * 32), o);
          }
          tmem_wait_st();
          if (need) l_sum *= alpha;
        }
      }
      if (need) m_used = mx;
      // key rows past the valid count: zero their V rows (all four warps share the rows)
      if (n_valid < kKeys) {
        const uint32_t vt = sbase + kOffRing + (i % kStages) * kTileBytes + 2 * kKVHalf;
        for (int idx = r; idx < (kKeys - n_valid) * 16; idx += kRows) {
          const int row = n_valid + (idx >> 4), c16 = idx & 15;
          st_shared_v4(vt + (uint32_t)((c16 >> 3) * kKVHalf + row * 128 + (((c16 & 7) ^ (row & 7)) << 4)), 0u, 0u, 0u,
                       0u);
        }
      }
      float psum = 0.f;
#pragma unroll
      for (int c = 0; c < kKeys / 8; ++c) {
        float p[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          p[e] = exp2f(s[8 * c + e] - m_used);
          psum += p[e];
        }
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) split2(p[2 * e], p[2 * e + 1], hw[e], lw[e]);
        const uint32_t off = (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
        st_shared_v4(sbase + kOffPhi + off, hw[0], hw[1], hw[2], hw[3]);
        st_shared_v4(sbase + kOffPlo + off, lw[0], lw[1], lw[2], lw[3]);
      }
      l_sum += psum;
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(bar_p));
    }
    if (ok && nt > 0 &&
        !__all_sync(0xffffffffu, mbar_wait(smem_u32(bar_pv), (uint32_t)((nt - 1) & 1), abort_flag)))
      ok = false;
    if (ok) {
      tc_fence_after();
      const float inv = 1.0f / l_sum;
      __nv_bfloat16* dst = out + ((bl * T + tok) * Hq + (int64_t)h * G + hd) * kD;
#pragma unroll 1
      for (int c = 0; c < kD / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem_base + lane_addr + kColO + (uint32_t)(c * 32), o);
        tmem_wait_ld();
        if (tok < T) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            uint32_t w[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(o[8 * e + 2 * u]) * inv,
                                                             __uint_as_float(o[8 * e + 2 * u + 1]) * inv);
              w[u] = *reinterpret_cast<const uint32_t*>(&v);
            }
            d4[e] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
    } else {
      *abort_flag = 1;
      if (lane == 0) msa::set_err(dev_err, MSA_DEVERR_TIMEOUT);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc<false>(tmem_base, kTmemCols);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// bf16 rows of 128 elements, box [64 rows][64 elements], 128-byte swizzle; rows past the
// end read as zero
bool make_map(CUtensorMap* m, const void* base, uint64_t rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kHalf, (cuuint32_t)kKeys};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int G>
int launch_g(const Args& a, cudaStream_t s, const char** why) {
  CUtensorMap tm_mem, tm_lk, tm_lv;
  const uint64_t mem_rows = (uint64_t)a.B * a.L * 2 * a.H * a.M_max;
  const uint64_t loc_rows = (uint64_t)a.B * a.L * a.H * a.cap;
  if (!make_map(&tm_mem, a.mem_kv, mem_rows) || !make_map(&tm_lk, a.local_k, loc_rows) ||
      !make_map(&tm_lv, a.local_v, loc_rows)) {
    *why = "cuTensorMapEncodeTiled failed";
    return 1;
  }
  if (cudaFuncSetAttribute(prefill_tc_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) != cudaSuccess) {
    *why = "cudaFuncSetAttribute (shared memory)";
    return 1;
  }
  const int tiles = (a.T + kRows / G - 1) / (kRows / G);
  prefill_tc_kernel<G><<<dim3(tiles, a.H, a.B * a.L), kThreads, kSmem, s>>>(
      tm_mem, tm_lk, tm_lv, a.q, a.T, a.L, a.H, a.local_len, a.cap, a.mem_len, a.M_max, a.pos_off, a.log2_theta,
      a.qscale, a.out, a.dev_err);
  if (cudaGetLastError() != cudaSuccess) {
    *why = "kernel launch";
    return 1;
  }
  return 0;
}

}  // namespace

bool supported(const Args& a) {
  const uint64_t mem_rows = (uint64_t)a.B * a.L * 2 * a.H * a.M_max;
  const uint64_t loc_rows = (uint64_t)a.B * a.L * a.H * a.cap;
  return mem_rows < (1ull << 31) && loc_rows + kKeys < (1ull << 31);
}

int launch(const Args& a, cudaStream_t s, const char** why) {
  switch (a.G) {
    case 1: return launch_g<1>(a, s, why);
    case 2: return launch_g<2>(a, s, why);
    case 4: return launch_g<4>(a, s, why);
    default: return launch_g<8>(a, s, why);
  }
}

}  // namespace prefill_tc
