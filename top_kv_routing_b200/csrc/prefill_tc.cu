// Prefill attention on the tcgen05 tensor cores.
//
// Computes what the prefill's attention step defines (msa_prefill.h): for every (query b,
// layer l, key head h) and every row (token t of the block, query head q of the group),
// softmax over [memory keys 0 .. M ; local keys 0 .. len + t] of the scaled dot products,
// times the values.  Follows "MSA端到端可训练记忆模型完整开源，支持亿级Token上下文", section
// 推理流水线, and the MSA paper reading notes, section 推理全流程.
//
// One CTA (320 threads) per 128 rows: 128 / G tokens x the G query heads of key head h.
//   warp 9, one thread   TMA producer: tiles of 64 keys (K as two 64-column boxes, then V
//                        the same), 128-byte swizzle, a 3-stage ring; memory tiles first,
//                        then local tiles up to the CTA's last token
//   warp 8, one thread   MMA issuer: S_i = Q K_i^T (M = 128, N = 64, K = 128) into one of two
//                        TMEM score buffers, then O += P_{i-1} V_{i-1} (M = 128, N = 128,
//                        K = 64) into the TMEM output, with P read from tensor memory (it
//                        replaces the scores it was computed from) and V read MN-major
//                        straight from its [key][d] rows.  The rotated queries and the
//                        weights are each a bf16 value plus a bf16 residual (two MMAs); keys
//                        and values exact bf16; fp32 accumulation
//   warps 0..7           two threads per row (TMEM lane), each with half of the row's dims
//                        and half of every tile's keys: build the rotated, scaled query row
//                        in shared memory; per tile read the score row, mask it (memory keys
//                        < M, local keys <= its own local index), keep a running maximum
//                        that is raised (and O rescaled in TMEM) only when a score exceeds
//                        it by more than 2^8, write the weights exp2(s - m) into the tile's
//                        score columns (values in the first 32, residuals in the last 32),
//                        and at the end divide O by the running sum.
// Weights of a tile are written while the previous tile's PV runs: the row threads wait
// for PV_{i-1} after releasing P_i (before, only when O must be rescaled).  Key rows past a
// tile's valid count are zeroed in shared memory before the PV that reads them (the cache
// rows beyond the valid length may hold anything).  Every wait is bounded (2 s); a timeout
// sets MSA_DEVERR_TIMEOUT and the CTA drains and frees its TMEM.
#include <cuda.h>

#include <math.h>

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
constexpr int kRowWarps = 8;                  // two threads per row: 32 keys of a tile each
constexpr int kMmaWarp = kRowWarps, kTmaWarp = kRowWarps + 1;
constexpr int kThreads = (kRowWarps + 2) * 32;
constexpr int kQHalf = kRows * 128;      // 16 KB: 64 bf16 of every row
constexpr int kQBytes = 2 * kQHalf;      // 32 KB: one bf16 copy of the CTA's queries
constexpr int kKVHalf = kKeys * 128;     // 8 KB: 64 keys x 64 elements
constexpr int kTileBytes = 4 * kKVHalf;  // K (two halves) then V (two halves)
constexpr int kOffQ = 0;                 // values
constexpr int kOffQlo = kQBytes;         // residuals
constexpr int kOffRing = 2 * kQBytes;
constexpr int kOffTab = kOffRing + kStages * kTileBytes;  // cos / sin of the block's tokens (G > 1)
constexpr int kTabBytes = 64 * kHalf * 8;                 // up to 64 tokens x 64 angles x float2
constexpr int kSmemData = kOffTab + kTabBytes;
constexpr int kSmem = kSmemData + 1024 + 256 + 4 * 128 * 4;  // + barriers, the row pairs' exchange buffer
constexpr uint32_t kTmemCols = 256;  // S0 / P0 [0, 64) | S1 / P1 [64, 128) | O [128, 256)
constexpr uint32_t kColPlo = 32;     // residuals of a tile's weights, after its 32 value columns
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

__device__ __forceinline__ uint32_t pack2(float x0, float x1) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// D (TMEM) += A (TMEM, K-major, 2 bf16 per column) x B (shared-memory descriptor).
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

template <int G>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_mem, const __grid_constant__ CUtensorMap tm_lk,
                      const __grid_constant__ CUtensorMap tm_lv, const __nv_bfloat16* __restrict__ q, int T, int L,
                      int H, const int32_t* __restrict__ local_len, int cap, const int32_t* __restrict__ mem_len,
                      int M_max, int pos_off, const __grid_constant__ RopeW rw, float qscale,
                      __nv_bfloat16* __restrict__ out, int32_t* dev_err) {
  constexpr int kTok = kRows / G;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSmemData);
  uint64_t* full = bars;                 // [kStages]
  uint64_t* empty = bars + kStages;      // [kStages]
  uint64_t* bar_q = empty + kStages;     // queries written (8 warps)
  uint64_t* bar_s = bar_q + 1;           // [2] scores ready
  uint64_t* bar_p = bar_s + 2;           // weights ready (8 warps)
  uint64_t* bar_pv = bar_p + 1;          // PV done
  uint64_t* drain = bar_pv + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

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

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(bar_q), kRowWarps);
    mbar_init(smem_u32(&bar_s[0]), 1);
    mbar_init(smem_u32(&bar_s[1]), 1);
    mbar_init(smem_u32(bar_p), kRowWarps);
    mbar_init(smem_u32(bar_pv), 1);
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_async_smem();
  }
  if (warp == kMmaWarp) {
    tmem_alloc<false>(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish<false>();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t sbase = smem_u32(smem);

  if (warp == kTmaWarp) {
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
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      // ---------------- MMA issuer (tensor-core operations from this thread run in order,
      // so S_{i+2}, written over P_i, follows the PV that reads P_i)
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
            umma<false, false>(d_s, sw128_desc(sbase + kOffQ + off) + (uint64_t)(2 * (ks & 3)), kdesc, idesc_s,
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
          const uint32_t p_tmem = tmem_base + (uint32_t)((j & 1) * kKeys);  // P_j: 64 bf16 in 32 columns
#pragma unroll
          for (int ks = 0; ks < kKeys / 16; ++ks) {
            const uint64_t vdesc = sw128_desc_mn(vt + (uint32_t)(ks * 2048), kKVHalf, 1024);
            umma_ts(tmem_base + kColO, p_tmem + (uint32_t)(8 * ks), vdesc, idesc_pv, (j > 0 || ks > 0) ? 1u : 0u);
            umma_ts(tmem_base + kColO, p_tmem + kColPlo + (uint32_t)(8 * ks), vdesc, idesc_pv, 1u);
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
    // ---------------- rows (warps 0..7): thread (row r = TMEM lane, half hf) takes the row's
    // dims 32 hf .. 32 hf + 31 and 64 + 32 hf .. 95 + 32 hf of the query, and keys
    // 32 hf .. 32 hf + 31 of every tile; the pair meets in shared memory (warps w, w + 4)
    const int r = tid & (kRows - 1), hf = tid >> 7;
    const int tl = r / G, hd = r % G;
    const int tok = tok0 + tl;
    const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
    const int pair_bar = 1 + (warp & 3);  // named barrier of warps w and w + 4
    auto pair_sync = [&]() { asm volatile("bar.sync %0, 64;" ::"r"(pair_bar) : "memory"); };
    {  // rotated, scaled query row (bf16 value and residual), 128-byte swizzled, 8 dims (and
       // their partners) at a time; with G > 1 the cos / sin of each token are computed once
       // into a table its G rows share
      const __nv_bfloat16* src = q + ((bl * T + tok) * Hq + (int64_t)h * G + hd) * kD;
      const double pos = (double)pos_off + (double)(len + tok);
      float2* tab = reinterpret_cast<float2*>(smem + kOffTab);
      if (G > 1) {
        for (int e = tid; e < kTok * kHalf; e += kRowWarps * 32) {
          const int t2 = e / kHalf, j = e % kHalf;
          double u = ((double)pos_off + (double)(len + tok0 + t2)) * rw.w_over_pi[j];
          u -= 2.0 * rint(0.5 * u);
          float sn, cs;
          sincospif((float)u, &sn, &cs);
          tab[e] = make_float2(cs, sn);
        }
        asm volatile("bar.sync 5, %0;" ::"n"(kRowWarps * 32) : "memory");
      }
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float xa[8], xb[8];  // dims 32 hf + 8c + e and 64 + 32 hf + 8c + e
        if (tok < T) {
          const uint4 wa = __ldg(reinterpret_cast<const uint4*>(src + 32 * hf + 8 * c));
          const uint4 wb = __ldg(reinterpret_cast<const uint4*>(src + kHalf + 32 * hf + 8 * c));
          const uint32_t va[4] = {wa.x, wa.y, wa.z, wa.w}, vb[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            xa[2 * e] = __uint_as_float(va[e] << 16);
            xa[2 * e + 1] = __uint_as_float(va[e] & 0xFFFF0000u);
            xb[2 * e] = __uint_as_float(vb[e] << 16);
            xb[2 * e + 1] = __uint_as_float(vb[e] & 0xFFFF0000u);
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            float sn, cs;
            if (G > 1) {
              const float2 t2 = tab[tl * kHalf + 32 * hf + 8 * c + e];
              cs = t2.x;
              sn = t2.y;
            } else {
              double u = pos * rw.w_over_pi[32 * hf + 8 * c + e];
              u -= 2.0 * rint(0.5 * u);
              sincospif((float)u, &sn, &cs);
            }
            const float a = xa[e], bb = xb[e];
            xa[e] = (a * cs - bb * sn) * qscale;
            xb[e] = (bb * cs + a * sn) * qscale;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) xa[e] = xb[e] = 0.f;
        }
        // chunk 4 hf + c of the first half, 8 + 4 hf + c of the second
        const int ca = 4 * hf + c, cb = 8 + 4 * hf + c;
        const uint32_t oa = (uint32_t)((ca >> 3) * kQHalf + r * 128 + (((ca & 7) ^ (r & 7)) << 4));
        const uint32_t ob = (uint32_t)((cb >> 3) * kQHalf + r * 128 + (((cb & 7) ^ (r & 7)) << 4));
        uint32_t ha[4], la[4], hb[4], lb[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          split2(xa[2 * e], xa[2 * e + 1], ha[e], la[e]);
          split2(xb[2 * e], xb[2 * e + 1], hb[e], lb[e]);
        }
        st_shared_v4(sbase + kOffQ + oa, ha[0], ha[1], ha[2], ha[3]);
        st_shared_v4(sbase + kOffQlo + oa, la[0], la[1], la[2], la[3]);
        st_shared_v4(sbase + kOffQ + ob, hb[0], hb[1], hb[2], hb[3]);
        st_shared_v4(sbase + kOffQlo + ob, lb[0], lb[1], lb[2], lb[3]);
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(bar_q));
    }
    float* xch = reinterpret_cast<float*>(smem + kSmemData + 256);  // [2 tiles][2 halves][128 rows]
    const int lim = len + min(tok, T - 1);
    float m_used = -INFINITY, l_sum = 0.f;
    bool ok = true;
    // Every row thread runs every iteration and every pair barrier, whatever happens: a
    // failed (timed-out) wait only clears `ok` and raises the abort flag, after which the
    // remaining waits return at once and the work is skipped.  So the pair barriers, which
    // cannot time out, always meet.
    auto fail = [&]() {
      ok = false;
      *abort_flag = 1;
    };
    // PV_{i-1} done (the bar_pv phases are waited one by one, in order)
    auto wait_pv = [&](int j) {
      if (ok && !__all_sync(0xffffffffu, mbar_wait(smem_u32(bar_pv), (uint32_t)(j & 1), abort_flag))) fail();
      if (ok) tc_fence_after();
    };
    for (int i = 0; i < nt; ++i) {
      // (waits are made warp-uniform: the TMEM accesses below are warp-collective)
      if (ok && !__all_sync(0xffffffffu, mbar_wait(smem_u32(&bar_s[i & 1]), (uint32_t)((i >> 1) & 1), abort_flag)))
        fail();
      const bool local = i >= nt_mem;
      const int key0 = local ? (i - nt_mem) * kKeys : i * kKeys;
      const int n_valid = local ? min(kKeys, n_local - key0) : min(kKeys, M - key0);
      float mx = -INFINITY;
      float sv[32];
      if (ok) {
        tc_fence_after();
        uint32_t sa[32];
        tmem_ld32(tmem_base + lane_addr + (uint32_t)((i & 1) * kKeys + 32 * hf), sa);
        tmem_wait_ld();
        // this thread's 32 keys: all visible (a memory tile's first keys below M, or local
        // keys up to the row's limit), or masked one by one
        const int kfirst = key0 + 32 * hf;
        const bool all_in = local ? kfirst + 31 <= lim : kfirst + 31 < M;
        if (all_in) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            sv[e] = __uint_as_float(sa[e]);
            mx = fmaxf(mx, sv[e]);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int key = kfirst + e;
            const bool v = local ? key <= lim : key < M;
            sv[e] = v ? __uint_as_float(sa[e]) : -INFINITY;
            mx = fmaxf(mx, sv[e]);
          }
        }
      }
      xch[((i & 1) * 2 + hf) * kRows + r] = mx;
      pair_sync();  // (also: both threads of the row have read the score row before either writes P)
      mx = fmaxf(mx, xch[((i & 1) * 2 + (hf ^ 1)) * kRows + r]);
      if (!ok) continue;
      const bool need = mx > m_used + kHeadroom;  // (the same in both threads of the row)
      const float m_old = m_used;
      if (need) m_used = mx;
      uint32_t pw[16], plw[16];
      float psum = 0.f;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float p0 = exp2f(sv[2 * e] - m_used), p1 = exp2f(sv[2 * e + 1] - m_used);
        psum += p0 + p1;
        split2(p0, p1, pw[e], plw[e]);
      }
      // key rows past the valid count: zero their V rows (this tile's stage; all row threads)
      if (n_valid < kKeys) {
        const uint32_t vt = sbase + kOffRing + (i % kStages) * kTileBytes + 2 * kKVHalf;
        for (int idx = tid; idx < (kKeys - n_valid) * 16; idx += kRowWarps * 32) {
          const int row = n_valid + (idx >> 4), c16 = idx & 15;
          st_shared_v4(vt + (uint32_t)((c16 >> 3) * kKVHalf + row * 128 + (((c16 & 7) ^ (row & 7)) << 4)), 0u, 0u, 0u,
                       0u);
        }
      }
      const bool rescale = __any_sync(0xffffffffu, need);
      if (i > 0 && rescale) {  // O must be stable: PV_{i-1} done before it is rescaled
        wait_pv(i - 1);
        if (!ok) continue;
        const float alpha = need ? exp2f(m_old - m_used) : 1.0f;
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {  // this thread's 64 of the 128 output columns
          uint32_t o[32];
          const uint32_t col = kColO + (uint32_t)(64 * hf + 32 * c);
          tmem_ld32(tmem_base + lane_addr + col, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(tmem_base + lane_addr + col, o);
        }
        if (need) l_sum *= alpha;
      }
      // P_i over the scores it came from: values in columns 16 hf .. 16 hf + 15 of the
      // tile's buffer, residuals 32 columns further
      tmem_st16(tmem_base + lane_addr + (uint32_t)((i & 1) * kKeys + 16 * hf), pw);
      tmem_st16(tmem_base + lane_addr + (uint32_t)((i & 1) * kKeys + kColPlo + 16 * hf), plw);
      tmem_wait_st();
      l_sum += psum;
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(bar_p));
      if (i > 0 && !rescale) wait_pv(i - 1);  // (one wait per tile, in order)
    }
    if (nt > 0) wait_pv(nt - 1);
    // the row's sum of weights: both halves (the exchange slot of tile nt is free)
    xch[((nt & 1) * 2 + hf) * kRows + r] = l_sum;
    pair_sync();
    l_sum += xch[((nt & 1) * 2 + (hf ^ 1)) * kRows + r];
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      const float inv = 1.0f / l_sum;
      __nv_bfloat16* dst = out + ((bl * T + tok) * Hq + (int64_t)h * G + hd) * kD;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t o[32];
        const int col = 64 * hf + 32 * c;
        tmem_ld32(tmem_base + lane_addr + kColO + (uint32_t)col, o);
        tmem_wait_ld();
        if (tok < T) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + col);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            uint32_t w[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
              w[u] = pack2(__uint_as_float(o[8 * e + 2 * u]) * inv, __uint_as_float(o[8 * e + 2 * u + 1]) * inv);
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
  if (warp == kMmaWarp) {
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
  RopeW rw;
  for (int j = 0; j < kHalf; ++j) rw.w_over_pi[j] = exp2(-2.0 * (double)j / (double)kD * a.log2_theta) / M_PI;
  prefill_tc_kernel<G><<<dim3(tiles, a.H, a.B * a.L), kThreads, kSmem, s>>>(
      tm_mem, tm_lk, tm_lv, a.q, a.T, a.L, a.H, a.local_len, a.cap, a.mem_len, a.M_max, a.pos_off, rw, a.qscale,
      a.out, a.dev_err);
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
