// Prefill attention on the tcgen05 tensor cores.
//
// Computes what the prefill's attention step defines (msa_prefill.h): for every (query b,
// layer l, key head h) and every row (token t of the block, query head q of the group),
// softmax over [memory keys 0 .. M ; local keys 0 .. len + t] of the scaled dot products,
// times the values.  Follows "MSA端到端可训练记忆模型完整开源，支持亿级Token上下文", section
// 推理流水线, and the MSA paper reading notes, section 推理全流程.
//
// Persistent CTAs of 608 threads, at most one per SM.  A unit is 128 rows: 128 / G tokens x
// the G query heads of key head h.  CTA c walks the tile pairs c, c + gridDim.x, ... of the
// (query x layer, key head, pair) list, pair j holding token tiles j and n_tiles - 1 - j (a
// short and a long one under the causal mask), one unit at a time:
//   warp 17, one thread  TMA producer: per unit its query rows as a 4D box (once the
//                        previous unit's queries are in tensor memory), then its tiles of
//                        128 keys (memory tiles first, then local tiles up to the unit's last
//                        token) as 64-key boxes, 128-byte swizzle, into a ring of two slots:
//                        the K of tile g once the scores of tile g - 2 have read that slot's
//                        K, then the V of tile g - 1 once PV_{g-3} has read its V.  A tile
//                        with at most 64 valid keys is loaded as one box.
//   warp 16              MMA issuer (the warp waits, one elected lane issues): S_g = Q K_g^T
//                        (M = 128, N = 128, or 64 for a half tile, K = 128, the query read
//                        from tensor memory) into score buffer g % 2, one tile ahead of the
//                        weights; O += P_g V_g (M = 128, N = 128, K = the tile's keys) into
//                        the TMEM output, P read from tensor memory (it replaces the scores
//                        it was computed from), V read MN-major from its [key][d] rows.  The
//                        rotated queries are a bf16 value plus a bf16 residual (two MMAs);
//                        the weights are bf16, rounded to nearest, and the row sums are taken
//                        over the rounded weights, so numerator and denominator use the same
//                        ones; keys and values exact bf16; fp32 accumulation.  g runs on from
//                        unit to unit.
//   warp 18              (G >= 4) the RoPE table of a unit's 128 / G tokens (64-bit
//                        fixed-point angles, hardware sin / cos of the reduced angle), written
//                        once the rows have staged the previous unit's queries
//   warps 0..15          four threads per row (TMEM lane), each with a quarter of the row's
//                        dims and 32 keys of every tile.  Per unit: rotate and scale the
//                        query rows into tensor memory (from the table; G <= 2 computes the
//                        angles in place); then the previous unit's output: O / sum as bf16
//                        through a shared-memory box, one TMA store; then per tile read the
//                        score row, mask it (memory keys < M, local keys <= its own local
//                        index), keep a running maximum that is raised (and O rescaled in
//                        TMEM) only when a score exceeds it by more than 2^8, and write the
//                        weights exp2(s - m) as bf16 over the first 64 of the tile's score
//                        columns.
// The row threads wait for a PV only before rescaling O and before the output; one score,
// weight and PV barrier per score buffer keeps every wait's phase unambiguous.  Key rows
// past a tile's valid count are zeroed in shared memory before the PV that reads them (the
// cache rows beyond the valid length may hold anything).  Every wait is bounded (2 s); a
// timeout sets MSA_DEVERR_TIMEOUT and the CTA drains and frees its TMEM.
#include <cuda.h>

#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "prefill_tc.cuh"
#include "tc_common.cuh"

namespace prefill_tc {
namespace {
using namespace tc;

constexpr int kD = 128;
constexpr int kHalf = 64;
constexpr int kRows = 128;
constexpr int kKeys = 64;   // keys per TMA box (half a tile)
constexpr int kTile = 128;  // keys per score tile
constexpr int kRowWarps = 16;                 // four threads per row: 16 keys of a tile each
constexpr int kParts = kRowWarps / 4;
constexpr int kMmaWarp = kRowWarps, kTmaWarp = kRowWarps + 1;
constexpr int kTabWarp = kRowWarps + 2;  // the next unit's RoPE table, off the row warps' path
constexpr int kThreads = (kRowWarps + 3) * 32;
constexpr int kKVHalf = kTile * 128;     // 16 KB: a tile's 128 keys x 64 elements
constexpr int kTileBytes = 4 * kKVHalf;  // 64 KB: K (two 64-dim halves) then V (two halves)
constexpr int kSlots = 2;                // ring slots of one tile
constexpr int kOffRing = 0;
constexpr int kQBoxHalf = kRows * 128;                    // 16 KB: 64 dims of the CTA's 128 rows
constexpr int kQBox = 2 * kQBoxHalf;                      // 32 KB: one unit's query rows

constexpr int kTabStride = kHalf + 1;                     // (a token's 64 angles + 1: the G-row groups of
                                                           // a warp read 8 tokens in distinct banks)
constexpr int kOffXch = 256;                                 // after the barriers: the rows' exchange buffer
constexpr int kOffW = kOffXch + 2 * kParts * kRows * 4;      // then the RoPE frequencies (64 x 8 bytes)
// Shared memory per group size: the K / V ring (two tiles), a unit's query box, its output
// box, the RoPE table of its 128 / G tokens (G >= 4; smaller groups compute their angles in
// place), then barriers, exchange buffer and the frequencies.
template <int G>
struct Lay {
  static constexpr bool kUseTab = G >= 4;
  static constexpr int kTabBytes = kUseTab ? (kRows / G) * kTabStride * 8 : 0;
  static constexpr int kTail = 1024 + kOffW + kHalf * 8;  // (+ alignment of the dynamic base)
  static constexpr int kOffQraw = kOffRing + kSlots * kTileBytes;  // a unit's queries as loaded
  static constexpr int kOffOut = kOffQraw + kQBox;                  // a unit's output rows on their way out
  static constexpr int kOffTab = kOffOut + kQBox;                   // cos / sin of a unit's tokens (G >= 4)
  static constexpr int kSmemData = kOffTab + kTabBytes;
  static constexpr int kSmem = kSmemData + kTail;
  static_assert(kSmem <= 227 * 1024, "shared memory");
};
// S0 / P0 [0, 128) | S1 / P1 [128, 256) | O [256, 384) | the unit's query value [384, 448) and
// residual [448, 512)
constexpr int kSBufs = 2;         // score buffers: the MMA runs one tile ahead of the weights
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 256;
constexpr uint32_t kColQ = 384;   // the rotated, scaled query rows: dims 2c, 2c + 1 in column c
constexpr uint32_t kColQlo = 448;
constexpr float kHeadroom = 8.0f;    // log2 growth of a row's maximum tolerated before rescaling

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// x = value + residual, both bf16: the value is x with its low 16 bits cleared (exact), the
// residual x - value (exact in fp32, at most 2^-7 |x|) rounded to bf16, so |error| <= 2^-16 |x|.
// Packed in pairs (x0 in the low half); one float-to-bf16 conversion per pair.
__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const uint32_t b0 = __float_as_uint(x0), b1 = __float_as_uint(x1);
  hi = __byte_perm(b0, b1, 0x7632);
  const __nv_bfloat162 l =
      __floats2bfloat162_rn(x0 - __uint_as_float(b0 & 0xFFFF0000u), x1 - __uint_as_float(b1 & 0xFFFF0000u));
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// 2^x by the hardware approximation (relative error about 2^-22, results below 2^-126
// flushed to zero, 2^-inf = 0): the weights exp2(s - m), with s - m <= 8 or -inf.
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// cos / sin of the RoPE angle of position p at frequency step s (2^-64 turns per position):
// the top 32 bits of p * s mod 2^64, read as signed, are the angle in [-pi, pi) x 2^31 / pi.
// The hardware sine / cosine is used on that reduced angle (absolute error about 2^-21 on
// [-pi, pi], far below the query's value + residual precision of 2^-16).
__device__ __forceinline__ void rope_cs(unsigned long long p, unsigned long long s, float& cs, float& sn) {
  const int top = (int)((p * s) >> 32);
  __sincosf((float)top * 1.4629180792671596e-09f, &sn, &cs);  // x pi / 2^31
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

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// 4D tiled TMA load (no multicast) completing on an mbarrier of this CTA: the box of a
// CTA's query rows, [128 / G tokens][G heads][64 dims].
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y, int z,
                                            int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], "
      "[%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}

// The matching 4D tiled TMA store (elements outside the tensor are not written).
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, uint32_t src, int x, int y, int z, int w) {
  asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(x), "r"(y), "r"(z), "r"(w)
               : "memory");
}

// The CTA's work, in order: the valid units of the tile pairs p = blockIdx.x, + gridDim.x, ...
// of the grid's (query, layer, key head) x pair list.  Pair j of (b, l, h) holds token tiles j
// and n_tiles - 1 - j (a short and a long one under the causal mask; one unit when they
// coincide).  Every role walks the same sequence; a pair whose cache cannot take the block
// is skipped by all of them.
struct UnitWalk {
  int T, L, H, cap, M_max, n_tiles, pairs_x, n_pairs, kTok;
  const int32_t* local_len;
  const int32_t* mem_len;
  // the current unit
  int p, k, nu;       // pair, unit within it, units in it
  int64_t bl;
  int h, len, M, tok0, nt_mem, n_local, nt;
  __device__ bool load_pair() {  // from p: the first pair whose cache takes the block
    for (; p < n_pairs; p += gridDim.x) {
      const int j = p % pairs_x;
      h = (p / pairs_x) % H;
      bl = p / (pairs_x * H);
      len = local_len[bl / L];
      if (len < 0 || len + T > cap) continue;  // (the append kernel has set MSA_DEVERR_LOCAL_FULL)
      const int m = mem_len[bl];
      M = m < 0 ? 0 : (m > M_max ? M_max : m);
      nt_mem = (M + kTile - 1) / kTile;
      nu = j == n_tiles - 1 - j ? 1 : 2;
      k = 0;
      return true;
    }
    return false;
  }
  __device__ void set_unit() {
    const int j = p % pairs_x;
    tok0 = (k == 0 ? j : n_tiles - 1 - j) * kTok;
    n_local = len + min(T, tok0 + kTok);
    nt = nt_mem + (n_local + kTile - 1) / kTile;
  }
  // tile i of the unit: its first key (within the memory rows or the local rows) and its
  // number of valid keys (a tile with at most 64 is loaded, scored and summed half-size)
  __device__ int key0(int i) const { return i >= nt_mem ? (i - nt_mem) * kTile : i * kTile; }
  __device__ int n_valid(int i) const {
    return i >= nt_mem ? min(kTile, n_local - key0(i)) : min(kTile, M - key0(i));
  }
  __device__ bool first() {
    p = blockIdx.x;
    if (!load_pair()) return false;
    set_unit();
    return true;
  }
  __device__ bool next() {
    if (++k < nu) {
      set_unit();
      return true;
    }
    p += gridDim.x;
    if (!load_pair()) return false;
    set_unit();
    return true;
  }
};

template <int G>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_mem, const __grid_constant__ CUtensorMap tm_lk,
                      const __grid_constant__ CUtensorMap tm_lv, const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_out, int T, int L,
                      int H, const int32_t* __restrict__ local_len, int cap, const int32_t* __restrict__ mem_len,
                      int M_max, int pos_off, const __grid_constant__ RopeW rw, float qscale, int n_bl,
                      int32_t* dev_err) {
  constexpr int kTok = kRows / G;
  constexpr int kStages = kSlots, kOffQraw = Lay<G>::kOffQraw, kOffOut = Lay<G>::kOffOut;
  constexpr bool kUseTab = Lay<G>::kUseTab;
  constexpr int kOffTab = Lay<G>::kOffTab, kSmemData = Lay<G>::kSmemData;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSmemData);
  // per ring slot: its K landed / read by the score MMAs, its V landed / read by the PV MMAs
  uint64_t* full_k = bars;               // [kStages]
  uint64_t* empty_k = bars + kStages;    // [kStages]
  uint64_t* full_v = bars + 2 * kStages;   // [kStages]
  uint64_t* empty_v = bars + 3 * kStages;  // [kStages]
  uint64_t* bar_q = bars + 4 * kStages;  // a unit's queries in tensor memory (16 warps; a phase per unit)
  uint64_t* bar_s = bar_q + 1;           // [kSBufs] scores ready
  // weights ready (16 warps) and PV done, one of each per score buffer: tile g's phases are
  // g / 2 of barrier g % 2, so neither side can complete a phase the other has not waited
  // for yet (the MMA thread issues scores one tile ahead)
  uint64_t* bar_p = bar_s + kSBufs;      // [kSBufs]
  uint64_t* bar_pv = bar_p + kSBufs;     // [kSBufs]
  uint64_t* drain = bar_pv + kSBufs;
  uint64_t* bar_qraw = drain + 1;        // a unit's query box has landed (a phase per unit)
  uint64_t* bar_tab = bar_qraw + 1;      // a unit's RoPE table is written (a phase per unit)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_tab + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  unsigned long long* wsm = reinterpret_cast<unsigned long long*>(smem + kSmemData + kOffW);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sbase = smem_u32(smem);
  const int n_tiles = (T + kTok - 1) / kTok;
  const int pairs_x = (n_tiles + 1) / 2;
  UnitWalk walk{T, L, H, cap, M_max, n_tiles, pairs_x, pairs_x * H * n_bl, kTok, local_len, mem_len};

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&full_k[s]), 1);
      mbar_init(smem_u32(&empty_k[s]), 1);
      mbar_init(smem_u32(&full_v[s]), 1);
      mbar_init(smem_u32(&empty_v[s]), 1);
    }
    mbar_init(smem_u32(bar_q), kRowWarps);
    for (int s = 0; s < kSBufs; ++s) {
      mbar_init(smem_u32(&bar_s[s]), 1);
      mbar_init(smem_u32(&bar_p[s]), kRowWarps);
      mbar_init(smem_u32(&bar_pv[s]), 1);
    }
    mbar_init(smem_u32(drain), 1);
    mbar_init(smem_u32(bar_qraw), 1);
    mbar_init(smem_u32(bar_tab), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_async_smem();
  }
  if (tid < kHalf) wsm[tid] = rw.step[tid];  // (indexed per lane: read from shared memory below)
  if (warp == kMmaWarp) {
    tmem_alloc<false>(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish<false>();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == kTmaWarp) {
    if (lane == 0) {
      // ---------------- TMA producer: per unit its query box (once the previous unit's
      // queries have been read out of the box's space), then its tiles in 64-key boxes: the
      // K of tile g once S_{g-2} has read the slot's K, then the V of tile g - 1 once
      // PV_{g-3} has read that slot's V (so a tile's keys land a softmax step before its
      // scores are due, and its values a step later still)
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_q)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_mem)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_lk)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_lv)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_out)) : "memory");
      const uint64_t pol = policy_evict_last();
      int armed_k[kStages], armed_v[kStages];
#pragma unroll
      for (int st = 0; st < kStages; ++st) armed_k[st] = armed_v[st] = -1;
      int qarmed = -1;
      bool ok = true;
      // a tile's source: the memory rows (K and V in one tensor) or the local cache's
      struct Src {
        int g, krow, vrow, boxes;
        bool mem;
      };
      // its K (is_v false) or V into slot g % 2: `boxes` 64-key boxes of both 64-dim halves
      auto load = [&](const Src& t, bool is_v) -> bool {
        const int stage = t.g % kStages;
        const uint32_t ph = (uint32_t)((t.g / kStages) & 1);
        if (!mbar_wait(smem_u32(is_v ? &empty_v[stage] : &empty_k[stage]), ph ^ 1u, abort_flag)) return false;
        const uint32_t fb = smem_u32(is_v ? &full_v[stage] : &full_k[stage]);
        const CUtensorMap* map = t.mem ? &tm_mem : (is_v ? &tm_lv : &tm_lk);
        const int row = is_v ? t.vrow : t.krow;
        const uint32_t dst = sbase + kOffRing + stage * kTileBytes + (is_v ? 2 * kKVHalf : 0);
        mbar_arrive_expect_tx(fb, t.boxes * (kTileBytes / 4));
        for (int hb = 0; hb < t.boxes; ++hb) {
          const uint32_t d = dst + (uint32_t)(hb * kKeys * 128);
          tma_load_2d(d, map, fb, 0, row + hb * kKeys, pol);
          tma_load_2d(d + kKVHalf, map, fb, kHalf, row + hb * kKeys, pol);
        }
        (is_v ? armed_v : armed_k)[stage] = (int)ph;
        return true;
      };
      Src prev{0, 0, 0, 0, false};
      bool have_prev = false;
      int g = 0, vu = 0;
      for (bool more = walk.first(); more && ok; more = walk.next(), ++vu) {
        if (vu > 0 && !mbar_wait(smem_u32(bar_q), (uint32_t)((vu - 1) & 1), abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t qb = smem_u32(bar_qraw);
        mbar_arrive_expect_tx(qb, kQBox);
        tma_load_4d(sbase + kOffQraw, &tm_q, qb, 0, walk.h * G, walk.tok0, (int)walk.bl);
        tma_load_4d(sbase + kOffQraw + kQBoxHalf, &tm_q, qb, kHalf, walk.h * G, walk.tok0, (int)walk.bl);
        qarmed = vu & 1;
        for (int i = 0; i < walk.nt && ok; ++i, ++g) {
          Src t;
          t.g = g;
          t.boxes = walk.n_valid(i) > kKeys ? 2 : 1;
          t.mem = i < walk.nt_mem;
          if (t.mem) {
            t.krow = (int)((((walk.bl * 2 + 0) * H + walk.h) * (int64_t)M_max) + i * kTile);
            t.vrow = (int)((((walk.bl * 2 + 1) * H + walk.h) * (int64_t)M_max) + i * kTile);
          } else {
            t.krow = t.vrow = (int)((walk.bl * H + walk.h) * (int64_t)cap + (int64_t)(i - walk.nt_mem) * kTile);
          }
          ok = load(t, false);
          if (ok && have_prev) ok = load(prev, true);
          prev = t;
          have_prev = true;
        }
      }
      if (ok && have_prev) ok = load(prev, true);
      if (!ok) {
        *abort_flag = 1;
        msa::set_err(dev_err, MSA_DEVERR_TIMEOUT);
        for (int s = 0; s < kStages; ++s) {
          if (armed_k[s] >= 0) mbar_drain(smem_u32(&full_k[s]), (uint32_t)armed_k[s]);
          if (armed_v[s] >= 0) mbar_drain(smem_u32(&full_v[s]), (uint32_t)armed_v[s]);
        }
        if (qarmed >= 0) mbar_drain(smem_u32(bar_qraw), (uint32_t)qarmed);
      }
    }
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issuer: the warp waits together, one elected lane issues.  The
    // tensor-core operations of that lane run in order.  S_g goes to score buffer g % 2 as
    // soon as its tile has landed and PV_{g-2} has been issued (S_g is written over P_{g-2}
    // and follows the PV that reads it): the scores run one tile ahead of the weights.  A
    // tile of at most 64 valid keys is scored with N = 64 and summed over its first 64 keys.
    // A unit's first score tile waits for its queries, and only after every PV of the
    // previous unit has been issued.
    const bool leader = elect_one();
    constexpr uint32_t idesc_s = idesc_make(kRows, kTile, false), idesc_s_half = idesc_make(kRows, kKeys, false);
    constexpr uint32_t idesc_pv = idesc_make_bmn(kRows, kD);
    bool ok = true, issued = false;
    // score side: the walk is one unit ahead of the PV side at most
    UnitWalk sw = walk, pw = walk;
    bool s_more = sw.first(), p_more = pw.first();
    int s_i = 0, s_vu = 0, g_s = 0;  // next S: tile s_i of unit s_vu (global g_s)
    int p_i = 0, g_pv = 0;           // next PV: tile p_i of the PV side's unit (global g_pv)
    auto issue_s = [&]() -> bool {
      if (s_i == 0) {
        if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(bar_q), (uint32_t)(s_vu & 1), abort_flag))) return false;
        tc_fence_after();
      }
      const int stage = g_s % kStages;
      if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&full_k[stage]), (uint32_t)((g_s / kStages) & 1), abort_flag)))
        return false;
      tc_fence_after();
      if (leader) {
        const uint32_t kt = sbase + kOffRing + stage * kTileBytes;
        const uint32_t d_s = tmem_base + (uint32_t)((g_s % kSBufs) * kTile);
        const uint32_t idesc = sw.n_valid(s_i) > kKeys ? idesc_s : idesc_s_half;
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks) {
          const uint64_t kdesc = sw128_desc(kt + (uint32_t)((ks >> 2) * kKVHalf)) + (uint64_t)(2 * (ks & 3));
          umma_ts(d_s, tmem_base + kColQ + (uint32_t)(8 * ks), kdesc, idesc, ks > 0 ? 1u : 0u);
          umma_ts(d_s, tmem_base + kColQlo + (uint32_t)(8 * ks), kdesc, idesc, 1u);
        }
        umma_commit<false>(smem_u32(&bar_s[g_s % kSBufs]));
        umma_commit<false>(smem_u32(&empty_k[stage]));
      }
      issued = true;
      __syncwarp();
      ++g_s;
      if (++s_i == sw.nt) {
        s_i = 0;
        ++s_vu;
        s_more = sw.next();
      }
      return true;
    };
    auto issue_pv = [&]() -> bool {
      const int j = g_pv, stage = j % kStages;
      if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&bar_p[j % kSBufs]), (uint32_t)((j / kSBufs) & 1), abort_flag)))
        return false;
      if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&full_v[stage]), (uint32_t)((j / kStages) & 1), abort_flag)))
        return false;
      tc_fence_after();
      if (leader) {
        const uint32_t vt = sbase + kOffRing + stage * kTileBytes + 2 * kKVHalf;
        const uint32_t p_tmem = tmem_base + (uint32_t)((j % kSBufs) * kTile);  // P_j: 128 bf16 in 64 columns
        const int n_ks = pw.n_valid(p_i) > kKeys ? kTile / 16 : kKeys / 16;
        for (int ks = 0; ks < n_ks; ++ks) {
          const uint64_t vdesc = sw128_desc_mn(vt + (uint32_t)(ks * 2048), kKVHalf, 1024);
          umma_ts(tmem_base + kColO, p_tmem + (uint32_t)(8 * ks), vdesc, idesc_pv, (p_i > 0 || ks > 0) ? 1u : 0u);
        }
        umma_commit<false>(smem_u32(&bar_pv[j % kSBufs]));
        umma_commit<false>(smem_u32(&empty_v[stage]));
      }
      __syncwarp();
      ++g_pv;
      if (++p_i == pw.nt) {
        p_i = 0;
        p_more = pw.next();
      }
      return true;
    };
    while (ok && p_more) {
      // scores first while allowed: up to one ahead of the next PV; a unit's first one only
      // once every PV of the previous unit has been issued (g_pv >= g_s), so that the last
      // PV, which the previous unit's output waits for, does not queue behind the next
      // unit's scores
      while (ok && s_more && g_s <= g_pv + 1 && (s_i != 0 || g_s <= g_pv))
        ok = issue_s();
      if (ok) ok = issue_pv();
    }
    if (!ok) {
      if (lane == 0) {
        *abort_flag = 1;
        msa::set_err(dev_err, MSA_DEVERR_TIMEOUT);
      }
      if (issued) {
        if (leader) umma_commit<false>(smem_u32(drain));
        __syncwarp();
        mbar_drain(smem_u32(drain), 0u);
      }
    }
  } else if (warp == kTabWarp) {
    // ---------------- RoPE table (G >= 4): per unit the cos / sin of its 128 / G tokens at
    // the 64 frequencies, written once the rows have staged the previous unit's queries
    if (kUseTab) {
      float2* tab = reinterpret_cast<float2*>(smem + kOffTab);
      int vu = 0;
      for (bool more = walk.first(); more; more = walk.next(), ++vu) {
        if (vu > 0 && !__all_sync(0xffffffffu, mbar_wait(smem_u32(bar_q), (uint32_t)((vu - 1) & 1), abort_flag))) {
          if (lane == 0) {
            *abort_flag = 1;
            msa::set_err(dev_err, MSA_DEVERR_TIMEOUT);
          }
          break;
        }
        for (int e = lane; e < kTok * kHalf; e += 32) {
          const int t2 = e / kHalf, j = e % kHalf;
          float sn, cs;
          rope_cs((unsigned long long)((long long)pos_off + walk.len + walk.tok0 + t2), wsm[j], cs, sn);
          tab[t2 * kTabStride + j] = make_float2(cs, sn);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(bar_tab));
      }
    }
  } else {
    // ---------------- rows (warps 0..15): thread (row r = TMEM lane, part hf of 4) takes the
    // row's dims 16 hf .. 16 hf + 15 and 64 + 16 hf .. 79 + 16 hf of the query, and keys
    // 16 hf .. 16 hf + 15 of every tile; the four meet in shared memory (warps w, w + 4,
    // w + 8, w + 12).  Per unit: its queries (so that its first score tiles run under what
    // follows), the previous unit's output, its tiles.
    const int r = tid & (kRows - 1), hf = tid >> 7;
    const int tl = r / G;
    const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
    const int pair_bar = 1 + (warp & 3);  // named barrier of the row's four warps
    auto pair_sync = [&]() { asm volatile("bar.sync %0, 128;" ::"r"(pair_bar) : "memory"); };
    auto rows_sync = [&]() { asm volatile("bar.sync 5, %0;" ::"n"(kRowWarps * 32) : "memory"); };
    bool ok = true;
    // Every row thread runs every iteration and every barrier, whatever happens: a failed
    // (timed-out) wait only clears `ok` and raises the abort flag, after which the remaining
    // waits return at once and the work is skipped.  So the named barriers, which cannot time
    // out, always meet.
    auto fail = [&]() {
      ok = false;
      *abort_flag = 1;
    };
    float* xch = reinterpret_cast<float*>(smem + kSmemData + kOffXch);  // [2 tiles][4 parts][128 rows]
    // PV_g done (the PV phases are waited one by one, in order)
    auto wait_pv = [&](int g) {
      if (ok && !__all_sync(0xffffffffu,
                            mbar_wait(smem_u32(&bar_pv[g % kSBufs]), (uint32_t)((g / kSBufs) & 1), abort_flag)))
        fail();
      if (ok) tc_fence_after();
    };

    // unit v's rotated, scaled query rows (bf16 value and residual) into its tensor-memory
    // columns, 8 dims (and their partners) at a time; with G >= 4 the cos / sin of each token
    // come from the table the table warp has written for the G rows that share them
    auto stage_q = [&](const UnitWalk& w, int v) {
      const int tok0 = w.tok0, tok = tok0 + tl;
      const unsigned long long pos = (unsigned long long)((long long)pos_off + w.len + tok);
      const float2* tab = reinterpret_cast<const float2*>(smem + kOffTab);
      if (kUseTab && ok && !__all_sync(0xffffffffu, mbar_wait(smem_u32(bar_tab), (uint32_t)(v & 1), abort_flag)))
        fail();  // (the table warp has written the unit's table)
      // the query box (TMA, 128-byte swizzle): row r's 16-byte chunk c of each 64-dim half at
      // 128 r + 16 (c ^ (r & 7))
      if (ok && !__all_sync(0xffffffffu, mbar_wait(smem_u32(bar_qraw), (uint32_t)(v & 1), abort_flag))) fail();
      uint32_t qh[16], ql[16];  // bf16 pairs of the row's dims (values, residuals)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float xa[8], xb[8];  // dims 16 hf + 8c + e and 64 + 16 hf + 8c + e
        if (tok < T && ok) {
          const uint32_t qoff = sbase + kOffQraw + (uint32_t)(r * 128 + (((2 * hf + c) ^ (r & 7)) << 4));
          const uint4 wa = ld_shared_v4(qoff), wb = ld_shared_v4(qoff + kQBoxHalf);
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
            if (kUseTab) {
              const float2 t2 = tab[tl * kTabStride + 16 * hf + 8 * c + e];
              cs = t2.x;
              sn = t2.y;
            } else {
              rope_cs(pos, wsm[16 * hf + 8 * c + e], cs, sn);
            }
            const float a = xa[e], bb = xb[e];
            xa[e] = (a * cs - bb * sn) * qscale;
            xb[e] = (bb * cs + a * sn) * qscale;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) xa[e] = xb[e] = 0.f;
        }
        // dims 16 hf + 8c .. + 7 -> columns 8 hf + 4c .. + 3 (and 32 further for the second half)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          split2(xa[2 * e], xa[2 * e + 1], qh[4 * c + e], ql[4 * c + e]);
          split2(xb[2 * e], xb[2 * e + 1], qh[8 + 4 * c + e], ql[8 + 4 * c + e]);
        }
      }
      const uint32_t qcol = tmem_base + lane_addr + kColQ + (uint32_t)(8 * hf);
      tmem_st8(qcol, *reinterpret_cast<const uint32_t(*)[8]>(qh));
      tmem_st8(qcol + 32, *reinterpret_cast<const uint32_t(*)[8]>(qh + 8));
      tmem_st8(qcol + (kColQlo - kColQ), *reinterpret_cast<const uint32_t(*)[8]>(ql));
      tmem_st8(qcol + (kColQlo - kColQ) + 32, *reinterpret_cast<const uint32_t(*)[8]>(ql + 8));
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(bar_q));
    };

    // a unit's tiles (global numbers g0 ..): masked scores, weights into tensor memory, the
    // running maximum and sum; the wait for its last PV is left to its output step
    float m_used = -INFINITY, l_sum = 0.f;
    auto run_tiles = [&](const UnitWalk& w, int g0) {
      const int tok = w.tok0 + tl;
      const int lim = w.len + min(tok, T - 1);
      m_used = -INFINITY;
      l_sum = 0.f;
      for (int i = 0; i < w.nt; ++i) {
        const int g = g0 + i;
        // (waits are made warp-uniform: the TMEM accesses below are warp-collective)
        if (ok && !__all_sync(0xffffffffu,
                              mbar_wait(smem_u32(&bar_s[g % kSBufs]), (uint32_t)((g / kSBufs) & 1), abort_flag)))
          fail();
        const bool local = i >= w.nt_mem;
        const int key0 = w.key0(i), n_valid = w.n_valid(i);
        const int n_keys = n_valid > kKeys ? kTile : kKeys;  // keys scored and summed
        const uint32_t s_col = tmem_base + lane_addr + (uint32_t)((g % kSBufs) * kTile);
        // this thread's 32 keys: none valid (left out: weights 0), all visible (a memory
        // tile's first keys below M, or local keys up to the row's limit), or masked one by one
        const bool none = 32 * hf >= n_valid;  // (the same in the whole warp)
        const int kfirst = key0 + 32 * hf;
        const bool all_in = local ? kfirst + 31 <= lim : kfirst + 31 < w.M;
        uint32_t sv[32];  // (fp32 bits; a masked key is -inf)
        float mx = -INFINITY;
        if (ok && !none) {
          tc_fence_after();
          tmem_ld32(s_col + (uint32_t)(32 * hf), sv);
          tmem_wait_ld();
          if (!all_in) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int key = kfirst + e;
              if (!(local ? key <= lim : key < w.M)) sv[e] = 0xFF800000u;
            }
          }
#pragma unroll
          for (int e = 0; e < 32; ++e) mx = fmaxf(mx, __uint_as_float(sv[e]));
        }
        xch[((g & 1) * kParts + hf) * kRows + r] = mx;
        pair_sync();  // (also: the row's four threads have read the score row before any writes P)
#pragma unroll
        for (int o = 1; o < kParts; ++o) mx = fmaxf(mx, xch[((g & 1) * kParts + ((hf + o) & 3)) * kRows + r]);
        if (!ok) continue;
        const bool need = mx > m_used + kHeadroom;  // (the same in the four threads of the row)
        const float m_old = m_used;
        if (need) m_used = mx;
        // key rows past the valid count, up to the keys summed: zero their V rows (this
        // tile's slot; all row threads)
        if (n_valid < n_keys) {
          // (once the tile's values have landed)
          if (ok && !__all_sync(0xffffffffu, mbar_wait(smem_u32(&full_v[g % kStages]), (uint32_t)((g / kStages) & 1),
                                                       abort_flag)))
            fail();
          const uint32_t vt = sbase + kOffRing + (g % kStages) * kTileBytes + 2 * kKVHalf;
          for (int idx = tid; idx < (n_keys - n_valid) * 16; idx += kRowWarps * 32) {
            const int row = n_valid + (idx >> 4), c16 = idx & 15;
            st_shared_v4(vt + (uint32_t)((c16 >> 3) * kKVHalf + row * 128 + (((c16 & 7) ^ (row & 7)) << 4)), 0u, 0u,
                         0u, 0u);
          }
          fence_async_smem();
        }
        const bool rescale = __any_sync(0xffffffffu, need);
        if (i > 0 && rescale) {  // O must be stable: PV_{g-1} done before it is rescaled
          wait_pv(g - 1);
          if (!ok) continue;
          const float alpha = need ? exp2f(m_old - m_used) : 1.0f;
#pragma unroll 1
          for (int hh = 0; hh < 2; ++hh) {  // this thread's 32 of the 128 output columns
            uint32_t o[16];
            const uint32_t col = kColO + (uint32_t)(32 * hf + 16 * hh);
            tmem_ld16(tmem_base + lane_addr + col, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st16(tmem_base + lane_addr + col, o);
          }
          if (need) l_sum *= alpha;
        }
        // the weights rounded to bf16 (the PV's A operand); the row sum adds the rounded values
        uint32_t pw[16];
        float psum = 0.f;
        if (!none) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const __nv_bfloat162 pb = __floats2bfloat162_rn(ex2_ftz(__uint_as_float(sv[2 * e]) - m_used),
                                                            ex2_ftz(__uint_as_float(sv[2 * e + 1]) - m_used));
            const float2 pr = __bfloat1622float2(pb);
            psum += pr.x + pr.y;
            pw[e] = *reinterpret_cast<const uint32_t*>(&pb);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) pw[e] = 0u;
        }
        // P_g over the scores it came from: columns 16 hf .. 16 hf + 15 of the tile's buffer
        tmem_st16(s_col + (uint32_t)(16 * hf), pw);
        tmem_wait_st();
        l_sum += psum;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bar_p[g % kSBufs]));
        // (no wait for PV_{g-1} here: the rows wait for a PV only before a rescale of O and
        // before the output; PV_t's barrier cannot complete its next phase, PV_{t+2}, before
        // the rows have released P_{t+2}, so skipping the phases in between is safe)
      }
    };

    // a unit's output: its last PV (tile g_end - 1), the row sums, O / sum as bf16 into the
    // output box's space in the layout of the query box (once the previous unit's store has
    // read it), then one TMA store per 64-dim half (rows past the block's last token fall
    // outside the tensor and are not written)
    auto output = [&](int64_t obl, int oh, int otok0, int g_end, float sum) {
      wait_pv(g_end - 1);
      // the row's sum of weights: all four parts (the exchange slot of tile g_end is free)
      xch[((g_end & 1) * kParts + hf) * kRows + r] = sum;
      pair_sync();
#pragma unroll
      for (int o = 1; o < kParts; ++o) sum += xch[((g_end & 1) * kParts + ((hf + o) & 3)) * kRows + r];
      ok = __all_sync(0xffffffffu, ok);
      if (tid == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");  // the previous store
      rows_sync();
      const uint32_t stage_o = sbase + kOffOut;
      if (ok) {
        const float inv = 1.0f / sum;
        uint32_t o[32];
        tmem_ld32(tmem_base + lane_addr + kColO + (uint32_t)(32 * hf), o);
        tmem_wait_ld();
        const uint32_t half = stage_o + (uint32_t)((hf >> 1) * kQBoxHalf) + (uint32_t)(r * 128);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          uint32_t wd[4];
#pragma unroll
          for (int v = 0; v < 4; ++v)
            wd[v] = pack2(__uint_as_float(o[8 * e + 2 * v]) * inv, __uint_as_float(o[8 * e + 2 * v + 1]) * inv);
          const int c = 4 * (hf & 1) + e;
          st_shared_v4(half + (uint32_t)((c ^ (r & 7)) << 4), wd[0], wd[1], wd[2], wd[3]);
        }
        fence_async_smem();
      } else {
        *abort_flag = 1;
        if (lane == 0) msa::set_err(dev_err, MSA_DEVERR_TIMEOUT);
      }
      // (O is read: from here the next unit's first PV may overwrite it)
      tc_fence_before();
      rows_sync();
      if (tid == 0 && !*abort_flag) {
        tma_store_4d(&tm_out, stage_o, 0, oh * G, otok0, (int)obl);
        tma_store_4d(&tm_out, stage_o + kQBoxHalf, kHalf, oh * G, otok0, (int)obl);
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      }
    };

    bool have_prev = false;
    int64_t prev_bl = 0;
    int prev_h = 0, prev_tok0 = 0, g = 0, vu = 0;
    for (bool more = walk.first(); more; more = walk.next(), ++vu) {
      stage_q(walk, vu);
      if (have_prev) output(prev_bl, prev_h, prev_tok0, g, l_sum);
      run_tiles(walk, g);
      g += walk.nt;
      have_prev = true;
      prev_bl = walk.bl;
      prev_h = walk.h;
      prev_tok0 = walk.tok0;
    }
    if (have_prev) output(prev_bl, prev_h, prev_tok0, g, l_sum);
    if (tid == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");  // the last box is read out
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

// bf16 [B*L][T][Hq][128] (queries or outputs), box [128 / G tokens][G heads][64 dims],
// 128-byte swizzle; coordinates (dim, head, token, b*L + l)
bool make_rows_map(CUtensorMap* m, const void* base, int Hq, int T, int BL, int G) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)Hq, (cuuint64_t)T, (cuuint64_t)BL};
  const cuuint64_t strides[3] = {(cuuint64_t)kD * 2, (cuuint64_t)Hq * kD * 2, (cuuint64_t)T * Hq * kD * 2};
  const cuuint32_t box[4] = {(cuuint32_t)kHalf, (cuuint32_t)G, (cuuint32_t)(kRows / G), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int G>
int launch_g(const Args& a, cudaStream_t s, const char** why) {
  CUtensorMap tm_mem, tm_lk, tm_lv, tm_q, tm_out;
  const uint64_t mem_rows = (uint64_t)a.B * a.L * 2 * a.H * a.M_max;
  const uint64_t loc_rows = (uint64_t)a.B * a.L * a.H * a.cap;
  if (!make_map(&tm_mem, a.mem_kv, mem_rows) || !make_map(&tm_lk, a.local_k, loc_rows) ||
      !make_map(&tm_lv, a.local_v, loc_rows) || !make_rows_map(&tm_q, a.q, a.H * G, a.T, a.B * a.L, G) ||
      !make_rows_map(&tm_out, a.out, a.H * G, a.T, a.B * a.L, G)) {
    *why = "cuTensorMapEncodeTiled failed";
    return 1;
  }
  constexpr int kSmem = Lay<G>::kSmem;
  if (cudaFuncSetAttribute(prefill_tc_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) != cudaSuccess) {
    *why = "cudaFuncSetAttribute (shared memory)";
    return 1;
  }
  const int tiles = (a.T + kRows / G - 1) / (kRows / G);
  // persistent: at most one CTA per SM, each walking its share of the (tile pair, key head,
  // query x layer) list
  const int64_t pairs = (int64_t)(tiles + 1) / 2 * a.H * a.B * a.L;
  const int ctas = (int)std::min<int64_t>(pairs, std::max(1, msa::sm_count()));
  RopeW rw;
  for (int j = 0; j < kHalf; ++j) {
    const long double turns = exp2l(-2.0L * j / kD * (long double)a.log2_theta) / (2.0L * 3.14159265358979323846264338L);
    rw.step[j] = (unsigned long long)llroundl(ldexpl(turns, 64));
  }
  prefill_tc_kernel<G><<<dim3(ctas, 1, 1), kThreads, kSmem, s>>>(
      tm_mem, tm_lk, tm_lv, tm_q, tm_out, a.T, a.L, a.H, a.local_len, a.cap, a.mem_len, a.M_max, a.pos_off, rw,
      a.qscale, a.B * a.L, a.dev_err);
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
  return mem_rows + kTile < (1ull << 31) && loc_rows + kTile < (1ull << 31);
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
