// Step 4: sparse decode attention over [gathered memory blocks ; local KV] (GQA).
//
// Follows "MSA端到端可训练记忆模型完整开源，支持亿级Token上下文", section 架构 (concatenate the
// selected compressed K/V with the local K/V; 全局 RoPE offset by k) and the MSA paper
// reading notes, section 推理全流程 (memory KV fixed, local KV grows per token).
//
// One 256-thread CTA per (query b, layer l, key head h) and key split (several splits
// only when there are fewer (b, l, h) units than SMs).  The keys are cut into tiles of
// 16 (memory rows, then local rows); warp w of the CTA takes tiles w, w + 8, ... and
// streams each through its own 3-stage cp.async ring in shared memory (16 K rows and
// 16 V rows, 16-byte chunks XOR-swizzled by row so ldmatrix reads are conflict-free).
// Per tile, on the tensor cores (mma.sync m16n8k16, bf16 in, fp32 accumulate):
//   S = Q K^T   with the G query heads of h as A rows: row g carries bf16(q'_g) and row
//               g + 8 the bf16 residual q'_g - bf16(q'_g), so S_g = row g + row g + 8 keeps
//               about 16 mantissa bits of the rotated query (K is exact bf16);
//   O += P V    with P split the same way (row g = bf16(p), row g + 8 = residual), the S
//               accumulators being reused as the A fragments and V read by ldmatrix.trans.
// Online softmax per warp in the log2 domain (softmax_scale * log2 e folded into q'),
// then the 8 warps' (max, sum, O) are merged in shared memory.  With one split the CTA
// writes the output; with several, each publishes its partial and the last CTA of the
// (b, l, h) to arrive (a self-resetting counter) merges them.  The last CTA of query b
// advances local_len[b].  The rotated new key (rounded to the cache's bf16) and the new
// value go to the cache (split 0) and into the zero-filled row of the last local tile
// in shared memory, so they are scored like every other key.  RoPE angles: position times
// a 64-bit fixed-point step per frequency (turns, modulo 1 by integer wrap-around), fp32
// sincospif.  The query fragments are built once per CTA in shared memory in MMA order (the
// kernel's per-launch path is kept short: it runs with a cold instruction cache on every
// launch).
#include "attn_common.cuh"
#include "common.cuh"
#include "msa_decode.h"

#include <algorithm>
#include <mutex>

MSA_DEFINE_LAST_ERROR(msa_decode_last_error)

namespace {
using namespace attn;

constexpr int kD = 128;
constexpr int kHalf = 64;
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kTileKeys = 16;
constexpr int kStages = 3;
constexpr int kRowBytes = kD * 2;                        // one bf16 key or value row
constexpr int kStageBytes = 2 * kTileKeys * kRowBytes;   // 16 K rows then 16 V rows
constexpr int kRingBytes = kWarps * kStages * kStageBytes;
constexpr int kMaxSplits = 4;
constexpr int kRedStride = kD + 4;                       // merge rows, padded against bank conflicts
constexpr float kLog2e = 1.4426950408889634f;
static_assert(kWarps * 8 * kRedStride * 4 <= kRingBytes, "merge buffer reuses the ring");

// Workspace: per (b, l, h, split slot) the partial output [G][128] and (max, sum) per head,
// then one arrival counter per (b, l, h) and one per query b.
size_t ws_floats(int B, int L, int Hq, int H) {
  const size_t units = (size_t)B * L * H * kMaxSplits;
  const int G = Hq / H;
  return units * (size_t)G * (kD + 2);
}
size_t ws_bytes(int B, int L, int Hq, int H) {
  return ws_floats(B, L, Hq, H) * sizeof(float) + ((size_t)B * L * H + (size_t)B) * sizeof(int);
}

// RoPE frequencies of one call in fixed point: step[j] = round(2^64 theta^(-2j/128) / (2 pi)),
// the rotation of frequency j per position in units of 2^-64 turns, so that the angle of
// position p is p * step[j] mod 2^64 turns (exact integer arithmetic, no range reduction).
struct RopeFreq {
  unsigned long long step[kHalf];
};

// 2^x by the hardware approximation (relative error about 2^-22, results below 2^-126
// flushed to zero, 2^-inf = 0): the weights exp2(s - m) with s <= m, and the rescale factors.
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int G>
__global__ void __launch_bounds__(kThreads, 1) decode_mma_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k_new,
    const __nv_bfloat16* __restrict__ v_new, int L, int H,
    // rows [0, len) are read; row len is written by split 0 and read by nobody here
    __nv_bfloat16* local_k, __nv_bfloat16* local_v, int32_t* local_len, int cap,
    const __nv_bfloat16* __restrict__ mem_kv, const int32_t* __restrict__ mem_len, int M_max, int pos_off,
    const __grid_constant__ RopeFreq rf, float qscale, int splits, float* part, float2* stat, int* unit_count,
    int* query_count,
    __nv_bfloat16* __restrict__ out, int32_t* dev_err) {
  extern __shared__ __align__(128) unsigned char ring[];
  // query fragments in MMA order: row g*4 + t holds thread (g, t)'s 8 k-steps x 4 words,
  // the 16-byte chunk of k-step ks at position ks ^ (row & 7)
  __shared__ __align__(16) uint32_t qfrag[32][32];
  __shared__ __align__(16) __nv_bfloat16 knew[kD];  // the rotated new key (as cached)
  __shared__ __align__(16) __nv_bfloat16 vnew[kD];
  __shared__ float2 cs[kHalf];
  __shared__ float2 wml[kWarps][8];
  __shared__ float fac[kWarps][8];
  __shared__ float s_mx[8], s_den[8];
  __shared__ int s_last;
  const int split = blockIdx.x, h = blockIdx.y;
  const int b = blockIdx.z / L;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int Hq = H * G;
  const int64_t bl = blockIdx.z;
  const int64_t uh = bl * H + h;
  // Launched as a programmatic dependent of the kernel before it on the stream (the
  // previous decode step, or whatever kernel or copy wrote this step's inputs: the gather
  // writes mem_len, a copy may write q): every input is read after the wait, past which that
  // grid's writes are complete and visible.  The next step may then be scheduled onto SMs as
  // this one's CTAs leave.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // thread (head gg, m) takes q dims 2m, 2m+1 and their rotate-half partners 2m+64, 2m+65
  const int gg = tid >> 5, mq = tid & 31;
  uint32_t qlo = 0u, qhi = 0u;
  if (gg < G) {
    const __nv_bfloat16* qp = q + (bl * Hq + (int64_t)h * G + gg) * kD;
    qlo = *reinterpret_cast<const uint32_t*>(qp + 2 * mq);
    qhi = *reinterpret_cast<const uint32_t*>(qp + 2 * mq + kHalf);
  }
  float kx0 = 0.f, kx1 = 0.f;
  __nv_bfloat16 vx = __float2bfloat16_rn(0.f);
  if (tid < kHalf) {
    kx0 = __bfloat162float(k_new[uh * kD + tid]);
    kx1 = __bfloat162float(k_new[uh * kD + tid + kHalf]);
  } else if (tid < kHalf + kD) {
    vx = v_new[uh * kD + tid - kHalf];
  }
  int M = mem_len[bl];
  const int len = local_len[b];
  const bool full = len < 0 || len >= cap;  // (a negative length is treated as unusable too)
  if (M > M_max) {
    if (tid == 0 && split == 0 && h == 0 && !full) msa::set_err(dev_err, MSA_DEVERR_CAPACITY);
    M = M_max;
  }
  if (M < 0) M = 0;
  // once every thread has read local_len[b], lane 0 of the last warp announces it (arrivals
  // before this CTA's are counted in `arrived`); the last CTA of the query to arrive
  // advances the length at its end.  That lane loads no new key or value and has no tile
  // copy pending yet, so the release costs it little, and nothing waits for the atomic's
  // result until the end.
  constexpr int kAnnouncer = kThreads - 32;
  static_assert(kAnnouncer >= kHalf + kD, "the announcer loads no new key or value");
  int arrived = 0;
  __syncthreads();
  if (tid == kAnnouncer) arrived = arrive_release(&query_count[b]);

  if (full) {
    if (tid == 0 && split == 0 && h == 0 && (bl % L) == 0) msa::set_err(dev_err, MSA_DEVERR_LOCAL_FULL);
    if (splits > 1 && tid < G) stat[(uh * kMaxSplits + split) * G + tid] = make_float2(-INFINITY, -1.f);
  } else {
    // ---- this warp's tiles (memory tiles, then local tiles; the new key, row len, rides
    // in the last local tile): the first ones are requested before anything else
    const int nt_mem = (M + kTileKeys - 1) / kTileKeys;
    const int nt = nt_mem + len / kTileKeys + 1;
    const int per = (nt + splits - 1) / splits;
    const int t0 = min(nt, split * per), t1 = min(nt, t0 + per);
    const int first = t0 + warp;
    const int my_n = first < t1 ? (t1 - first + kWarps - 1) / kWarps : 0;
    const __nv_bfloat16* memk = mem_kv + ((bl * 2 + 0) * H + h) * (int64_t)M_max * kD;
    const __nv_bfloat16* memv = mem_kv + ((bl * 2 + 1) * H + h) * (int64_t)M_max * kD;
    const __nv_bfloat16* lock = local_k + uh * (int64_t)cap * kD;
    const __nv_bfloat16* locv = local_v + uh * (int64_t)cap * kD;
    const uint32_t my_ring = smem_u32(ring) + warp * (kStages * kStageBytes);

    struct Tile {
      const __nv_bfloat16 *kp, *vp;
      int n_copy;   // rows read from memory
      int nvalid;   // rows that are keys
      int new_row;  // row of the new key, or -1
    };
    auto tile = [&](int i) -> Tile {
      const int ti = first + i * kWarps;
      Tile tl;
      if (ti < nt_mem) {
        tl.kp = memk + (int64_t)ti * kTileKeys * kD;
        tl.vp = memv + (int64_t)ti * kTileKeys * kD;
        tl.n_copy = tl.nvalid = min(kTileKeys, M - ti * kTileKeys);
        tl.new_row = -1;
      } else {
        const int r0 = (ti - nt_mem) * kTileKeys;
        tl.kp = lock + (int64_t)r0 * kD;
        tl.vp = locv + (int64_t)r0 * kD;
        tl.n_copy = max(0, min(kTileKeys, len - r0));
        tl.nvalid = min(kTileKeys, len + 1 - r0);
        tl.new_row = len - r0 < kTileKeys ? len - r0 : -1;
      }
      return tl;
    };
    auto issue = [&](int i) {
      const Tile tl = tile(i);
      const uint32_t st = my_ring + (i % kStages) * kStageBytes;
      const int chunk = lane & 15;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int row = 2 * j + (lane >> 4);  // 0..15 K rows, 16..31 V rows
        const int key = row & 15;
        const bool ok = key < tl.n_copy;
        const __nv_bfloat16* src = (j < 8 ? tl.kp : tl.vp) + (ok ? key * kD + chunk * 8 : 0);
        cp_async16(st + row * kRowBytes + ((chunk ^ (row & 7)) << 4), src, ok ? 16u : 0u);
      }
    };
    // all three stages requested at once (a stage is refilled as soon as its tile is used)
#pragma unroll
    for (int p = 0; p < kStages; ++p) {
      if (p < my_n) issue(p);
      cp_async_commit();
    }

    // ---- RoPE angles of this step's position p: the top 32 bits of p * step[j] mod 2^64,
    // read as signed, are the angle / pi in [-1, 1) x 2^31; fp32 sincospif
    if (tid < kHalf) {
      const unsigned long long pos = (unsigned long long)((long long)pos_off + len);
      const int top = (int)((pos * rf.step[tid]) >> 32);
      float sn, c;
      sincospif((float)top * 4.656612873077392578125e-10f, &sn, &c);  // x 2^-31
      cs[tid] = make_float2(c, sn);
    }
    __syncthreads();
    {  // rotated, scaled query pairs -> MMA fragments (bf16 value and bf16 residual)
      float r[4] = {0.f, 0.f, 0.f, 0.f};  // dims 2m, 2m+1, 2m+64, 2m+65
      if (gg < G) {
        const float2 a = msa::bf16x2_to_float2(qlo), bb = msa::bf16x2_to_float2(qhi);
        const float2 c0 = cs[2 * mq], c1 = cs[2 * mq + 1];
        r[0] = (a.x * c0.x - bb.x * c0.y) * qscale;
        r[1] = (a.y * c1.x - bb.y * c1.y) * qscale;
        r[2] = (bb.x * c0.x + a.x * c0.y) * qscale;
        r[3] = (bb.y * c1.x + a.y * c1.y) * qscale;
      }
#pragma unroll
      for (int p2 = 0; p2 < 2; ++p2) {
        const int d = 2 * mq + p2 * kHalf;  // first dim of the pair
        const int ks = d >> 4, c = d & 15, tq = (c & 7) >> 1, half = c >> 3;
        const int row = gg * 4 + tq;
        uint32_t hi, lo;
        split_pair(r[2 * p2], r[2 * p2 + 1], hi, lo);
        uint32_t* w = &qfrag[row][((ks ^ (row & 7)) << 2)];
        w[half ? 2 : 0] = hi;
        w[half ? 3 : 1] = lo;
      }
    }
    if (tid < kHalf) {  // the new key, rotated and rounded to the cache's bf16
      const float2 c = cs[tid];
      const __nv_bfloat16 lo = __float2bfloat16_rn(kx0 * c.x - kx1 * c.y);
      const __nv_bfloat16 hi = __float2bfloat16_rn(kx1 * c.x + kx0 * c.y);
      knew[tid] = lo;
      knew[tid + kHalf] = hi;
      if (split == 0) {
        const int64_t cache_row = (uh * (int64_t)cap + len) * kD;
        local_k[cache_row + tid] = lo;
        local_k[cache_row + tid + kHalf] = hi;
      }
    } else if (tid < kHalf + kD) {
      const int j = tid - kHalf;
      vnew[j] = vx;
      if (split == 0) local_v[(uh * (int64_t)cap + len) * kD + j] = vx;
    }
    __syncthreads();

    uint32_t qa[8][4];
    {
      const int row = g * 4 + t;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint4 w = *reinterpret_cast<const uint4*>(&qfrag[row][(ks ^ (row & 7)) << 2]);
        qa[ks][0] = w.x;
        qa[ks][1] = w.y;
        qa[ks][2] = w.z;
        qa[ks][3] = w.w;
      }
    }

    float o[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float m = -INFINITY, lsum = 0.f;
    for (int i = 0; i < my_n; ++i) {
      cp_async_wait<kStages - 1>();  // (3 + i groups committed: tile i has landed)
      __syncwarp();
      const Tile tl = tile(i);
      const uint32_t st = my_ring + (i % kStages) * kStageBytes;
      if (tl.new_row >= 0) {  // the new key and value into their (zero-filled) rows
        const int row = (lane < 16 ? 0 : kTileKeys) + tl.new_row, chunk = lane & 15;
        const uint4 w = *reinterpret_cast<const uint4*>((lane < 16 ? knew : vnew) + 8 * chunk);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(st + row * kRowBytes +
                                                                          ((chunk ^ (row & 7)) << 4)),
                     "r"(w.x), "r"(w.y), "r"(w.z), "r"(w.w)
                     : "memory");
        __syncwarp();
      }
      const int nvalid = tl.nvalid;

      // two accumulators per 8-key half (even / odd k-steps) keep the MMA chains short
      float s[2][2][4];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
#pragma unroll
        for (int u = 0; u < 2; ++u) s[j][u][0] = s[j][u][1] = s[j][u][2] = s[j][u][3] = 0.f;
      }
#pragma unroll
      for (int ks2 = 0; ks2 < 4; ++ks2) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int row = 8 * j + (lane & 7);
          const int chunk = 4 * ks2 + (lane >> 3);
          uint32_t b0, b1, b2, b3;
          ldsm_x4(st + row * kRowBytes + ((chunk ^ (row & 7)) << 4), b0, b1, b2, b3);
          mma_bf16(s[j][0], qa[2 * ks2], b0, b1);
          mma_bf16(s[j][1], qa[2 * ks2 + 1], b2, b3);
        }
      }
      float sc[4];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int key = 8 * j + 2 * t + e;
          sc[2 * j + e] = key < nvalid ? (s[j][0][e] + s[j][0][2 + e]) + (s[j][1][e] + s[j][1][2 + e]) : -INFINITY;
        }
      }
      float mx = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m, mx);
      const float alpha = ex2_ftz(m - m_new);  // 0 while m is still -inf
      float pr[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) pr[u] = ex2_ftz(sc[u] - m_new);
      lsum = fmaf(lsum, alpha, (pr[0] + pr[1]) + (pr[2] + pr[3]));
      m = m_new;
      if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
        for (int n = 0; n < 16; ++n) {
          o[n][0] *= alpha; o[n][1] *= alpha; o[n][2] *= alpha; o[n][3] *= alpha;
        }
      }
      uint32_t pa[4];
      split_pair(pr[0], pr[1], pa[0], pa[1]);
      split_pair(pr[2], pr[3], pa[2], pa[3]);
      const int vkey = (lane & 7) + 8 * ((lane >> 3) & 1);
      const int vrow = kTileKeys + vkey;
#pragma unroll
      for (int i2 = 0; i2 < 8; ++i2) {
        const int chunk = 2 * i2 + (lane >> 4);
        uint32_t v0, v1, v2, v3;
        ldsm_x4_t(st + vrow * kRowBytes + ((chunk ^ (vrow & 7)) << 4), v0, v1, v2, v3);
        mma_bf16(o[2 * i2], pa, v0, v1);
        mma_bf16(o[2 * i2 + 1], pa, v2, v3);
      }
      __syncwarp();  // every lane is done with the stage: refill it with tile i + 3
      if (i + kStages < my_n) issue(i + kStages);
      cp_async_commit();
    }
    cp_async_wait<0>();
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);

    // ---- merge the warps (the ring is free once every warp is here)
    __syncthreads();
    float* red = reinterpret_cast<float*>(ring);
    if (t == 0) wml[warp][g] = make_float2(m, lsum);
#pragma unroll
    for (int n = 0; n < 16; ++n)
      *reinterpret_cast<float2*>(&red[(warp * 8 + g) * kRedStride + 8 * n + 2 * t]) =
          make_float2(o[n][0] + o[n][2], o[n][1] + o[n][3]);
    __syncthreads();
    if (tid < 64) {  // per head (8 lanes each): every warp's weight, and the sum
      const int hg = tid >> 3, w = tid & 7;
      const float2 st = wml[w][hg];
      float mx = st.x;
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      const float f = st.y > 0.f ? exp2f(st.x - mx) : 0.f;
      float den = f * st.y;
      den += __shfl_xor_sync(0xffffffffu, den, 1);
      den += __shfl_xor_sync(0xffffffffu, den, 2);
      den += __shfl_xor_sync(0xffffffffu, den, 4);
      fac[w][hg] = splits == 1 ? f / den : f;
      if (w == 0) {
        s_mx[hg] = mx;
        s_den[hg] = den;
      }
    }
    __syncthreads();
    const int64_t unit = uh * kMaxSplits + split;
    for (int oi = tid; oi < G * kD; oi += kThreads) {
      const int hg = oi / kD, d = oi % kD;
      float num = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) num = fmaf(fac[w][hg], red[(w * 8 + hg) * kRedStride + d], num);
      if (splits == 1) {
        out[(bl * Hq + (int64_t)h * G + hg) * kD + d] = __float2bfloat16_rn(num);
      } else {
        part[unit * G * kD + oi] = num;
        if (d == 0) stat[unit * G + hg] = make_float2(s_mx[hg], s_den[hg]);
      }
    }
  }

  if (splits > 1) {
    // ---- the last split CTA of (b, l, h) to finish merges the splits
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(&unit_count[uh], 1) == splits - 1;
    __syncthreads();
    if (s_last) {
      __threadfence();
      const int64_t unit0 = uh * kMaxSplits;
      if (!full) {
        for (int oi = tid; oi < G * kD; oi += kThreads) {
          const int hg = oi / kD;
          float mx = -INFINITY;
          for (int sp = 0; sp < splits; ++sp) mx = fmaxf(mx, __ldcg(&stat[(unit0 + sp) * G + hg]).x);
          float num = 0.f, den = 0.f;
          for (int sp = 0; sp < splits; ++sp) {
            const float2 st = __ldcg(&stat[(unit0 + sp) * G + hg]);
            if (st.y > 0.f) {
              const float w = exp2f(st.x - mx);
              num = fmaf(w, __ldcg(&part[(unit0 + sp) * G * kD + oi]), num);
              den = fmaf(w, st.y, den);
            }
          }
          out[(bl * Hq + (int64_t)h * G + hg) * kD + (oi % kD)] = __float2bfloat16_rn(num / den);
        }
      }
      if (tid == 0) unit_count[uh] = 0;  // ready for the next call
    }
  }
  // every CTA of query b arrived after reading local_len[b]; the last one advances it
  if (tid == kAnnouncer && arrived == L * H * splits - 1) {
    if (!full) local_len[b] = len + 1;
    query_count[b] = 0;  // ready for the next call
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

namespace {
// Host-side argument and device checks of a decode call (nothing is enqueued).
msa_status check_decode(const void* q, const void* k_new, const void* v_new, int32_t n_queries, int32_t n_layers,
                        int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, const void* local_k,
                        const void* local_v, const int32_t* local_len, int32_t local_cap, const void* mem_kv,
                        const int32_t* mem_len, int32_t max_mem_chunks, float rope_theta, const void* out,
                        const void* workspace, size_t workspace_bytes) {
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
  if (!msa::aligned16(q) || !msa::aligned16(mem_kv) || !msa::aligned16(local_k) || !msa::aligned16(local_v) ||
      !msa::aligned16(workspace))
    return msa_fail(MSA_ERR_INVALID_ARG, "16-byte alignment (q, mem_kv, local_k, local_v, workspace)");
  const size_t need = ws_bytes(n_queries, n_layers, n_q_heads, n_kv_heads);
  if (workspace_bytes < need)
    return msa_fail(MSA_ERR_CAPACITY, "workspace too small (%zu < %zu)", workspace_bytes, need);
  const int arch = msa::current_device_is_sm100(nullptr);
  if (arch < 0) return msa_fail(MSA_ERR_CUDA, "no CUDA device");
  if (arch == 0) return msa_fail(MSA_ERR_UNSUPPORTED, "device is not sm_100");
  return msa_ok();
}

// Enqueues the decode kernel (arguments already checked).
msa_status launch_decode(const void* q, const void* k_new, const void* v_new, int32_t n_queries, int32_t n_layers,
                         int32_t n_q_heads, int32_t n_kv_heads, void* local_k, void* local_v, int32_t* local_len,
                         int32_t local_cap, const void* mem_kv, const int32_t* mem_len, int32_t max_mem_chunks,
                         int32_t rope_pos_offset, float rope_theta, float softmax_scale, void* out, void* workspace,
                         int32_t* dev_err, msa_stream_t stream) {
  const int G = n_q_heads / n_kv_heads;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t units = (int64_t)n_queries * n_layers * n_kv_heads;
  const int splits = (int)std::min<int64_t>(kMaxSplits, std::max<int64_t>(1, msa::sm_count() / units));
  float* part = reinterpret_cast<float*>(workspace);
  float2* stat = reinterpret_cast<float2*>(part + (size_t)units * kMaxSplits * G * kD);
  int* unit_count = reinterpret_cast<int*>(part + ws_floats(n_queries, n_layers, n_q_heads, n_kv_heads));
  int* query_count = unit_count + units;
  const dim3 grid(splits, n_kv_heads, n_queries * n_layers);
  RopeFreq rf;
  const long double log2_theta = log2l((long double)rope_theta);
  for (int j = 0; j < kHalf; ++j) {
    const long double turns = exp2l(-2.0L * j / kD * log2_theta) / (2.0L * 3.14159265358979323846264338L);
    rf.step[j] = (unsigned long long)llroundl(ldexpl(turns, 64));
  }
  const float qscale = softmax_scale * kLog2e;
  // programmatic stream serialisation: the kernel may be scheduled before the previous
  // kernel on the stream finishes and waits for it (griddepcontrol.wait) before reading
  // any input
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kRingBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
#define MSA_DECODE_LAUNCH(GG)                                                                                    \
  MSA_CUDA_TRY(cudaFuncSetAttribute(decode_mma_kernel<GG>, cudaFuncAttributeMaxDynamicSharedMemorySize,           \
                                    kRingBytes));                                                                 \
  MSA_CUDA_TRY(cudaLaunchKernelEx(                                                                                \
      &cfg, decode_mma_kernel<GG>, (const __nv_bfloat16*)q, (const __nv_bfloat16*)k_new,                          \
      (const __nv_bfloat16*)v_new, n_layers, n_kv_heads, (__nv_bfloat16*)local_k, (__nv_bfloat16*)local_v,        \
      local_len, local_cap, (const __nv_bfloat16*)mem_kv, mem_len, max_mem_chunks, rope_pos_offset, rf,          \
      qscale, splits, part, stat, unit_count, query_count, (__nv_bfloat16*)out, dev_err))
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
}  // namespace

extern "C" msa_status msa_sparse_decode(const void* q, const void* k_new, const void* v_new, int32_t n_queries,
                                        int32_t n_layers, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                        void* local_k, void* local_v, int32_t* local_len, int32_t local_cap,
                                        const void* mem_kv, const int32_t* mem_len, int32_t max_mem_chunks,
                                        int32_t rope_pos_offset, float rope_theta, float softmax_scale, void* out,
                                        void* workspace, size_t workspace_bytes, int32_t* dev_err,
                                        msa_stream_t stream) {
  const msa_status st = check_decode(q, k_new, v_new, n_queries, n_layers, n_q_heads, n_kv_heads, head_dim, local_k,
                                     local_v, local_len, local_cap, mem_kv, mem_len, max_mem_chunks, rope_theta, out,
                                     workspace, workspace_bytes);
  if (st != MSA_OK) return st;
  return launch_decode(q, k_new, v_new, n_queries, n_layers, n_q_heads, n_kv_heads, local_k, local_v, local_len,
                       local_cap, mem_kv, mem_len, max_mem_chunks, rope_pos_offset, rope_theta, softmax_scale, out,
                       workspace, dev_err, stream);
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
  const int arch = msa::current_device_is_sm100(nullptr);
  if (arch < 0) return msa_fail(MSA_ERR_CUDA, "no CUDA device");
  if (arch == 0) return msa_fail(MSA_ERR_UNSUPPORTED, "device is not sm_100");
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
  // every check before anything is enqueued: a rejected call leaves the stream (and a
  // graph being captured) untouched
  const msa_status st = check_decode(q, k_new, v_new, n_queries, n_layers, n_q_heads, n_kv_heads, head_dim, local_k,
                                     local_v, local_len, local_cap, mem_kv, mem_len, max_mem_chunks, rope_theta, out,
                                     scratch, MSA_DECODE_STATIC_SCRATCH_BYTES);
  if (st != MSA_OK) return st;
  // the arrival counters must start at zero: their place depends on the sizes, and the
  // array keeps whatever the previous call left there
  const size_t counters_at = ws_floats(n_queries, n_layers, n_q_heads, n_kv_heads) * sizeof(float);
  MSA_CUDA_TRY(cudaMemsetAsync(static_cast<unsigned char*>(scratch) + counters_at, 0, need - counters_at,
                               reinterpret_cast<cudaStream_t>(stream)));
  return launch_decode(q, k_new, v_new, n_queries, n_layers, n_q_heads, n_kv_heads, local_k, local_v, local_len,
                       local_cap, mem_kv, mem_len, max_mem_chunks, rope_pos_offset, rope_theta, softmax_scale, out,
                       scratch, dev_err, stream);
}
