// Router query projection on the tensor cores, fused with the routing query's
// normalisation and group sum.
//
// Follows "【MSA】突破100M Token 上下文：记忆稀疏注意力架构深度解析", section 5.1 (the routing
// layers' decoupled projector router_q_proj: hidden -> query heads x 128, no bias) and
// section 5.2 with "MSA端到端可训练记忆模型完整开源，支持亿级Token上下文", section 架构 (the
// routing score is the mean over the query heads of the cosine with the block key).  For
// token t and layer l the projection is P = h_t W_l^T; query head q is P[q*128 .. q*128+127].
// The routing operand of key head g is (1/Hq) * sum over the G query heads q of group g of
// P_q / max(||P_q||, 1e-8): the same operand the query-prep kernel builds from a given Q_r.
//
// One unit = (layer l, key head g, 128 tokens): a GEMM tile M = 128 tokens x N = 128 G
// features (the G heads of the group) over K = hidden_size, bf16 operands, fp32 in TMEM.
// The whole group's heads are in one accumulator, so the epilogue can normalise each head
// and sum the group before anything leaves the SM; P itself is never stored.  With more
// than 128 tokens, units of 256 tokens run on pairs of SMs (a 2-CTA cluster, tcgen05
// cta_group::2, M = 256): each CTA loads its 128 token rows and half of every MMA's weight
// rows, both CTAs' copies complete on the leader's barrier, the leader issues the MMAs and
// its commits reach both CTAs, and each CTA's epilogue handles its own 128 tokens.  No load
// uses cluster multicast.
// Warp roles (192 threads, persistent, one CTA per SM):
//   warp 0      TMA producer: A = 128 tokens x 128 B of h, B = 128 G features x 128 B of
//               W (boxes of at most 256 rows), 128-byte swizzle, into a ring of stages
//   warp 1      one thread issues tcgen05.mma (kind::f16, M = 128, N = min(128 G, 256);
//               two MMAs per K step for G = 4) and commits stage / accumulator completion
//   warps 2..5  epilogue, thread = token row (TMEM lane): pass 1 the G head norms, pass 2
//               the normalised group sum in 32-column slices, written as the operand rows
//               (fp32, bf16 + bf16 residual, E4M3 x 2^11 as requested)
// Every wait is bounded (2 s); on a timeout the kernel sets MSA_DEVERR_TIMEOUT, drains its
// own copies and MMAs and frees TMEM.
#include <cuda.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "route_bound.cuh"
#include "route_proj.cuh"
#include "tc_common.cuh"

namespace route_proj {
namespace {
using namespace tc;

constexpr int kD = 128;
constexpr int kBM = 128;
constexpr int kRowBytes = 128;  // one swizzled row per K-block: 64 bf16
constexpr int kBK = 64;
constexpr int kABytes = kBM * kRowBytes;
constexpr int kThreads = 192;

template <int G, bool PAIR>
struct Cfg {
  static constexpr int kN = kD * G;                    // features per unit
  static constexpr int kMmaN = kN < 256 ? kN : 256;    // N of one MMA
  static constexpr int kMmas = kN / kMmaN;             // MMAs per K step
  static constexpr int kRows = PAIR ? 2 * kBM : kBM;   // tokens per unit (M of the MMA)
  static constexpr int kBox = PAIR ? kMmaN / 2 : kMmaN;  // W rows per TMA box held by this CTA
  static constexpr int kBBytes = kMmas * kBox * kRowBytes;
  static constexpr int kStage = kABytes + kBBytes;
  static constexpr int kStages = (200 * 1024) / kStage > 4 ? 4 : (200 * 1024) / kStage;
  static constexpr int kTmemCols = kN;                 // 128, 256 or 512: one accumulator
  static constexpr int kSmem = kStages * kStage + 1024 + 256;
};

template <int G, bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
    proj_kernel(const __grid_constant__ CUtensorMap tm_h, const __grid_constant__ CUtensorMap tm_w, int T, int kblocks,
                int L, int Hq, int H, int m_tiles, int n_rows, const __grid_constant__ Layout lay,
                float* __restrict__ qt_f32, __nv_bfloat16* __restrict__ qt_bf16, __nv_bfloat16* __restrict__ qt_lo,
                uint8_t* __restrict__ qt_f8, float* __restrict__ etok, int32_t* dev_err) {
  using K = Cfg<G, PAIR>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + K::kStages * K::kStage);
  uint64_t* full = bars;
  uint64_t* empty = bars + K::kStages;
  uint64_t* accf = empty + K::kStages;
  uint64_t* acce = accf + 1;
  uint64_t* drain = acce + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int units = L * H * m_tiles;
  const uint32_t rank = PAIR ? cluster_rank() : 0u;
  const bool leader = rank == 0;
  const int first_unit = PAIR ? (int)(blockIdx.x / 2) : (int)blockIdx.x;
  const int unit_stride = PAIR ? (int)(gridDim.x / 2) : (int)gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < K::kStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(accf), 1);
    mbar_init(smem_u32(acce), PAIR ? 8 : 4);
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0) {
    tmem_alloc<PAIR>(smem_u32(tmem_slot), K::kTmemCols);
    tmem_relinquish<PAIR>();
  }
  tc_fence_before();
  if (PAIR) cluster_sync_all();  // both CTAs' barriers initialised before any remote use
  else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_h)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_w)) : "memory");
      const uint64_t pol_h = policy_evict_last(), pol_w = policy_evict_first();
      int armed[K::kStages];
#pragma unroll
      for (int s = 0; s < K::kStages; ++s) armed[s] = -1;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int u = first_unit; u < units && ok; u += unit_stride) {
        const int mt = u % m_tiles, g = (u / m_tiles) % H, l = u / (m_tiles * H);
        const int row_h = mt * K::kRows + (int)rank * kBM;
        const int row_w = (l * Hq + g * G) * kD + (int)rank * K::kBox;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&full[stage]);
          const uint32_t sa = smem_u32(smem + stage * K::kStage);
          if (PAIR) {
            const uint32_t fb_lead = map_to_rank(fb, 0);  // both CTAs' bytes land on the leader's barrier
            if (leader) mbar_arrive_expect_tx(fb, 2 * K::kStage);
            tma_load_2d_pair(sa, &tm_h, fb_lead, kb * kBK, row_h, pol_h);
#pragma unroll
            for (int i = 0; i < K::kMmas; ++i)
              tma_load_2d_pair(sa + kABytes + i * K::kBox * kRowBytes, &tm_w, fb_lead, kb * kBK,
                               row_w + i * K::kMmaN, pol_w);
          } else {
            mbar_arrive_expect_tx(fb, K::kStage);
            tma_load_2d(sa, &tm_h, fb, kb * kBK, row_h, pol_h);
#pragma unroll
            for (int i = 0; i < K::kMmas; ++i)
              tma_load_2d(sa + kABytes + i * K::kBox * kRowBytes, &tm_w, fb, kb * kBK, row_w + i * K::kMmaN, pol_w);
          }
          armed[stage] = (int)phase;
          if (++stage == K::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        msa::set_err(dev_err, MSA_DEVERR_TIMEOUT);
        // let the copies this CTA issued land (the leader's barriers see both CTAs' bytes)
        if (leader)
          for (int s = 0; s < K::kStages; ++s)
            if (armed[s] >= 0) mbar_drain(smem_u32(&full[s]), (uint32_t)armed[s]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer (the leader of a pair issues for both CTAs)
      constexpr uint32_t idesc = idesc_make(K::kRows, K::kMmaN, false);
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true, issued = false;
      for (int u = first_unit; u < units && ok; u += unit_stride) {
        if (!mbar_wait(smem_u32(acce), acc_phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(smem_u32(&full[stage]), phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * K::kStage);
          const uint64_t da = sw128_desc(sa);
#pragma unroll
          for (int k = 0; k < kRowBytes / 32; ++k)  // 16 bf16 of K per MMA
#pragma unroll
            for (int i = 0; i < K::kMmas; ++i)
              umma<PAIR, false>(tmem_base + (uint32_t)(i * K::kMmaN), da + (uint64_t)(2 * k),
                                sw128_desc(sa + kABytes + i * K::kBox * kRowBytes) + (uint64_t)(2 * k), idesc,
                                (kb | k) != 0 ? 1u : 0u);
          issued = true;
          umma_commit<PAIR>(smem_u32(&empty[stage]));
          if (++stage == K::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit<PAIR>(smem_u32(accf));
        acc_phase ^= 1u;
      }
      if (!ok) {
        *abort_flag = 1;
        msa::set_err(dev_err, MSA_DEVERR_TIMEOUT);
        if (issued) {
          umma_commit<PAIR>(smem_u32(drain));  // arrives once every MMA issued so far has finished
          mbar_drain(smem_u32(drain), 0u);
        }
      }
    }
  } else {
    // ---------------- epilogue (warps 2..5 -> TMEM lane quarters 2, 3, 0, 1)
    const int quarter = warp & 3;
    const int hd = H * kD;
    const float inv_hq = 1.0f / (float)Hq;
    const uint32_t acce_lead = PAIR ? map_to_rank(smem_u32(acce), 0) : smem_u32(acce);
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int u = first_unit; u < units && ok; u += unit_stride) {
      const int mt = u % m_tiles, g = (u / m_tiles) % H, l = u / (m_tiles * H);
      const int t = mt * K::kRows + (int)rank * kBM + quarter * 32 + lane;
      int orow = -1;
      if (t < T) {
        int lo = 0, hi = lay.n_queries;  // largest b with off[b] <= t
        while (hi - lo > 1) {
          const int mid = (lo + hi) >> 1;
          if (lay.off[mid] <= t) lo = mid; else hi = mid;
        }
        orow = lay.row0[lo] + (t - lay.off[lo]);
      }
      if (!mbar_wait(smem_u32(accf), acc_phase, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16);
      // pass 1: the norm of each of the group's heads
      float inv[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float ss = 0.f;
#pragma unroll 1
        for (int c = 0; c < kD / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tbase + (uint32_t)(h * kD + c * 32), r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) ss = fmaf(__uint_as_float(r[i]), __uint_as_float(r[i]), ss);
        }
        inv[h] = 1.0f / fmaxf(sqrtf(ss), 1e-8f);
      }
      // pass 2: (1/Hq) * sum of the unit heads, 32 columns at a time (and the norms of
      // the filter error bounds: q, its bf16 rounding and residual, its E4M3 operand and residual)
      float bsum[6] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
      for (int c = 0; c < kD / 32; ++c) {
        float acc[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) acc[i] = 0.f;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          uint32_t r[32];
          tmem_ld32(tbase + (uint32_t)(h * kD + c * 32), r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[i] += __uint_as_float(r[i]) * inv[h];
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) acc[i] *= inv_hq;
        if (orow < 0) continue;
        if (etok != nullptr) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float hf = __bfloat162float(__float2bfloat16_rn(acc[i])), db = hf - acc[i];
            const float a = acc[i] * route_tc::kF8QueryScale, ah = route_bound::e4m3_round(a);
            const float as = ah * (1.0f / route_tc::kF8QueryScale), da = (ah - a) * (1.0f / route_tc::kF8QueryScale);
            bsum[0] = fmaf(acc[i], acc[i], bsum[0]);
            bsum[1] = fmaf(db, db, bsum[1]);
            bsum[2] = fmaf(hf, hf, bsum[2]);
            bsum[3] = fmaf(as, as, bsum[3]);
            bsum[4] = fmaf(da, da, bsum[4]);
            bsum[5] += fabsf(as);
          }
        }
        const int e0 = g * kD + c * 32;
        if (qt_f32 != nullptr) {
          float4* dst = reinterpret_cast<float4*>(qt_f32 + ((int64_t)l * T + t) * hd + e0);
#pragma unroll
          for (int i = 0; i < 8; ++i) dst[i] = make_float4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2], acc[4 * i + 3]);
        }
        const int64_t oi = ((int64_t)l * n_rows + orow) * hd + e0;
        if (qt_bf16 != nullptr) {
          uint32_t hw[16], lw[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const __nv_bfloat162 hv = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
            hw[i] = *reinterpret_cast<const uint32_t*>(&hv);
            const float r0 = acc[2 * i] - __uint_as_float(hw[i] << 16);
            const float r1 = acc[2 * i + 1] - __uint_as_float(hw[i] & 0xFFFF0000u);
            const __nv_bfloat162 lv = __floats2bfloat162_rn(r0, r1);
            lw[i] = *reinterpret_cast<const uint32_t*>(&lv);
          }
          uint4* dh = reinterpret_cast<uint4*>(qt_bf16 + oi);
          uint4* dl = reinterpret_cast<uint4*>(qt_lo + oi);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            dh[i] = make_uint4(hw[4 * i], hw[4 * i + 1], hw[4 * i + 2], hw[4 * i + 3]);
            dl[i] = make_uint4(lw[4 * i], lw[4 * i + 1], lw[4 * i + 2], lw[4 * i + 3]);
          }
        }
        if (qt_f8 != nullptr) {
          uint32_t fw[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint32_t a = __nv_cvt_float2_to_fp8x2(
                make_float2(acc[4 * i] * route_tc::kF8QueryScale, acc[4 * i + 1] * route_tc::kF8QueryScale),
                __NV_SATFINITE, __NV_E4M3);
            const uint32_t b = __nv_cvt_float2_to_fp8x2(
                make_float2(acc[4 * i + 2] * route_tc::kF8QueryScale, acc[4 * i + 3] * route_tc::kF8QueryScale),
                __NV_SATFINITE, __NV_E4M3);
            fw[i] = a | (b << 16);
          }
          uint4* df = reinterpret_cast<uint4*>(qt_f8 + oi);
          df[0] = make_uint4(fw[0], fw[1], fw[2], fw[3]);
          df[1] = make_uint4(fw[4], fw[5], fw[6], fw[7]);
        }
      }
      if (etok != nullptr && orow >= 0) {
        // this key head's share of the token's bounds
        const float2 eb = route_bound::head_bounds(sqrtf(bsum[0]), sqrtf(bsum[1]), sqrtf(bsum[2]), sqrtf(bsum[3]),
                                                   sqrtf(bsum[4]), bsum[5]);
        atomicAdd(etok + ((int64_t)route_bound::kBoundF8 * L + l) * T + t,
                  eb.x * route_bound::kBoundSlack + route_bound::kBoundFloor);
        atomicAdd(etok + ((int64_t)route_bound::kBoundBf16 * L + l) * T + t,
                  eb.y * route_bound::kBoundSlack + route_bound::kBoundFloor);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (PAIR) mbar_arrive_cluster(acce_lead);
        else mbar_arrive(acce_lead);
      }
      acc_phase ^= 1u;
    }
    if (!ok && lane == 0) {
      *abort_flag = 1;
      msa::set_err(dev_err, MSA_DEVERR_TIMEOUT);
    }
  }

  tc_fence_before();
  if (PAIR) cluster_sync_all();  // no CTA exits while its peer may still signal its barriers
  else __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc<PAIR>(tmem_base, K::kTmemCols);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// bf16 [rows][cols] row-major, box [box_rows][64 elements], 128-byte swizzle; rows past
// the end read as zero.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kBK, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int G, bool PAIR>
int launch_g(const Args& a, cudaStream_t s, const char** why) {
  using K = Cfg<G, PAIR>;
  CUtensorMap mh, mw;
  if (!make_map(&mh, a.hidden, (uint64_t)a.T, (uint64_t)a.hidden_size, kBM) ||
      !make_map(&mw, a.w, (uint64_t)a.L * a.Hq * kD, (uint64_t)a.hidden_size, K::kBox)) {
    *why = "cuTensorMapEncodeTiled failed";
    return 1;
  }
  const int m_tiles = (a.T + K::kRows - 1) / K::kRows;
  const long long units = (long long)a.L * a.H * m_tiles;
  const int per_unit = PAIR ? 2 : 1;
  int grid = msa::sm_count() / per_unit * per_unit;
  if (units * per_unit < grid) grid = (int)(units * per_unit);
  if (cudaFuncSetAttribute(proj_kernel<G, PAIR>, cudaFuncAttributeMaxDynamicSharedMemorySize, K::kSmem) !=
      cudaSuccess) {
    *why = "cudaFuncSetAttribute (shared memory)";
    return 1;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = K::kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = per_unit;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, proj_kernel<G, PAIR>, mh, mw, a.T, a.hidden_size / kBK, a.L, a.Hq, a.H, m_tiles,
                         a.n_rows, a.lay, a.qt_f32, a.qt_bf16, a.qt_lo, a.qt_f8, a.etok, a.dev_err) != cudaSuccess) {
    *why = "kernel launch";
    return 1;
  }
  return 0;
}

}  // namespace

bool supported(int Hq, int H, int hidden_size) {
  if (H < 1 || Hq % H != 0) return false;
  const int G = Hq / H;
  return (G == 1 || G == 2 || G == 4) && hidden_size >= kBK && hidden_size % kBK == 0;
}

int launch(const Args& a, cudaStream_t s, const char** why) {
  if (!supported(a.Hq, a.H, a.hidden_size)) {
    *why = "unsupported sizes";
    return 1;
  }
  if ((long long)a.L * a.Hq * kD >= (1ll << 31) || (long long)a.L * a.H * ((a.T + kBM - 1) / kBM) >= (1ll << 31)) {
    *why = "sizes beyond 32-bit TMA coordinates";
    return 1;
  }
  // paired M = 256 tiles (two SMs per tile, each streaming half of the weight rows) once
  // the tokens fill more than one 128-row tile
  const bool pair = a.T > kBM;
  switch (a.Hq / a.H) {
    case 1: return pair ? launch_g<1, true>(a, s, why) : launch_g<1, false>(a, s, why);
    case 2: return pair ? launch_g<2, true>(a, s, why) : launch_g<2, false>(a, s, why);
    default: return pair ? launch_g<4, true>(a, s, why) : launch_g<4, false>(a, s, why);
  }
}

}  // namespace route_proj
