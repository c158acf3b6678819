// Tensor-core (tcgen05) routing scores with a fused token-max epilogue.
//
// Per layer l the scores of every memory block c against every query token t are
//   D[c][t] = < kr_hat[l][c][:], qt[l][t][:] >      (K = 8 heads x 128 = 1024)
// a dense GEMM with fp32 accumulation (M = blocks, N = query tokens) on bf16 operands
// (kind::f16) or on E4M3 operands (kind::f8f6f4; keys stored x 2^8, queries x 2^11, the
// product rescaled by 2^-19 in the epilogue).  One 128-byte shared-memory row holds 64
// bf16 or 128 E4M3 elements and one MMA consumes 32 bytes of K either way, so both
// forms share the tiling, swizzle and descriptors; E4M3 halves the K-blocks per tile.
// The epilogue reduces each row over the columns of every query, then over the rows of
// the same document within the warp (runs of consecutive blocks), and folds the result
// into the document's score with one atomicMax per run; D itself never leaves TMEM.  These low-precision scores are a filter: the caller rescores the
// pairs that can hold the maximum exactly.
//
// Warp roles of the persistent kernel (192 threads, one CTA per SM):
//   warp 0      TMA producer: A tile [128 blocks x 128 B] + B tile [tokens x 128 B] per
//               K-block into a ring of shared-memory stages (128-byte swizzle)
//   warp 1      one thread issues tcgen05.mma (fp32 accumulate, 32 bytes of K each) into one of
//               two TMEM accumulators and commits stage / accumulator completion to mbarriers
//   warps 2..5  epilogue: tcgen05.ld 32 columns at a time, max over each query's columns
//               and over each document's rows, atomicMax per document; then release the
//               accumulator
// Paired mode (PAIR, for N tiles of 128 and 256): a cluster of two CTAs on two SMs runs
// M=256 tiles with tcgen05.mma.cta_group::2.  Each CTA loads its 128 key rows and half of
// the query tile, so each SM streams half the query bytes per key byte of the single-CTA
// form.  The leader (rank 0) issues the MMAs; both CTAs' loads complete on the leader's
// stage barrier; commits are multicast to both CTAs; the peer's epilogue releases the
// accumulator on the leader's barrier.  No load uses cluster multicast.
// Every wait is bounded (2 s on the global timer); on a timeout the kernel sets
// MSA_DEVERR_TIMEOUT, drains its own copies and MMAs (bounded) and frees TMEM.
#include <cuda.h>

#include "common.cuh"
#include "route_tc.cuh"
#include "tc_common.cuh"

namespace route_tc {
namespace {

constexpr int kBM = 128;
constexpr int kRowBytes = 128;           // one swizzled shared-memory row per K-block
constexpr int kKDim = 1024;              // 8 key heads x 128
constexpr int kABytes = kBM * kRowBytes; // 16 KB
constexpr int kThreads = 192;
constexpr int kMaskLayers = 64;          // layer-mask entries kept in shared memory

template <int BN, bool PAIR, bool F8>
struct Cfg {
  static constexpr int kElem = F8 ? 1 : 2;                 // operand bytes
  static constexpr int kBK = kRowBytes / kElem;            // elements per K-block
  static constexpr int kKBlocks = kKDim / kBK;             // 16 (bf16) or 8 (E4M3)
  static constexpr int kBRows = PAIR ? BN / 2 : BN;  // query rows of the B tile held per CTA
  static constexpr int kBBytes = kBRows * kRowBytes;
  static constexpr int kStage = kABytes + kBBytes;
  static constexpr int kStages = (196 * 1024) / kStage > 8 ? 8 : (196 * 1024) / kStage;
  static constexpr int kTmemCols = 2 * BN;  // two accumulators: 128, 256 or 512 columns
  static constexpr int kRows = PAIR ? 2 * kBM : kBM;  // key rows per unit (M of the MMA)
  static constexpr int kBarBytes = 256;
  static constexpr int kSmem = kStages * kStage + 1024 + kBarBytes;
};

using namespace tc;

// ------------------------------------------------------------------ kernel
template <int BN, bool PAIR, bool F8>
__global__ void __launch_bounds__(kThreads, 1)
    route_tc_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b, int L,
                    long long C, int n_rows, int m_tiles, const __grid_constant__ QueryLayout ql,
                    const int32_t* __restrict__ block_doc, uint32_t* __restrict__ doc_score, int n_docs,
                    int32_t* dev_err,
                    const int32_t* __restrict__ layer_only) {
  using K = Cfg<BN, PAIR, F8>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + K::kStages * K::kStage);
  uint64_t* full = bars;
  uint64_t* empty = bars + K::kStages;
  uint64_t* accf = empty + K::kStages;
  uint64_t* acce = accf + 2;
  uint64_t* drain = acce + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_tiles = n_rows / BN;
  const int units = L * m_tiles;
  const uint32_t rank = PAIR ? cluster_rank() : 0u;
  const bool leader = rank == 0;
  const int first_unit = PAIR ? (int)(blockIdx.x / 2) : (int)blockIdx.x;
  const int unit_stride = PAIR ? (int)(gridDim.x / 2) : (int)gridDim.x;
  // with a layer mask: nothing to do returns before any set-up (every CTA of a pair reads
  // the same mask); otherwise whole masked layers are stepped over, the same way by every role
  __shared__ int s_active[kMaskLayers];
  if (layer_only != nullptr) {
    int any = 0;
    for (int i = threadIdx.x; i < L; i += blockDim.x) {
      const int a = layer_only[i] != 0;
      if (i < kMaskLayers) s_active[i] = a;
      any |= a;
    }
    if (!__syncthreads_or(any)) return;
  }
  auto active = [&](int l) -> bool {
    return layer_only == nullptr || (l < kMaskLayers ? s_active[l] != 0 : layer_only[l] != 0);
  };
  // the first unit >= u of this CTA's sequence (first_unit + i * unit_stride) in an active layer
  auto next_active = [&](int u) -> int {
    while (u < units && !active(u / m_tiles)) {
      const int nxt = (u / m_tiles + 1) * m_tiles;
      u = nxt + ((first_unit - nxt) % unit_stride + unit_stride) % unit_stride;
    }
    return u;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < K::kStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&accf[b]), 1);
      mbar_init(smem_u32(&acce[b]), PAIR ? 8 : 4);
    }
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
  if (PAIR) cluster_sync_all();  // barriers of both CTAs initialised before any remote use
  else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs of a pair)
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_a)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_b)) : "memory");
      const uint64_t pol_a = policy_evict_first(), pol_b = policy_evict_last();
      int armed[K::kStages];
#pragma unroll
      for (int s = 0; s < K::kStages; ++s) armed[s] = -1;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int u = next_active(first_unit); u < units && ok; u = next_active(u + unit_stride)) {
        const int l = u / m_tiles, mt = u % m_tiles;
        const int row_a = (int)((long long)l * C) + mt * K::kRows + (int)rank * kBM;
        for (int nt = 0; nt < n_tiles && ok; ++nt) {
          const int row_b = l * n_rows + nt * BN + (int)rank * K::kBRows;
          for (int kb = 0; kb < K::kKBlocks; ++kb) {
            if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, abort_flag)) {
              ok = false;
              break;
            }
            const uint32_t fb = smem_u32(&full[stage]);
            const uint32_t sa = smem_u32(smem + stage * K::kStage);
            if (PAIR) {
              const uint32_t fb_lead = map_to_rank(fb, 0);  // both CTAs' bytes land on the leader's barrier
              if (leader) mbar_arrive_expect_tx(fb, 2 * K::kStage);
              tma_load_2d_pair(sa, &tm_a, fb_lead, kb * K::kBK, row_a, pol_a);
              tma_load_2d_pair(sa + kABytes, &tm_b, fb_lead, kb * K::kBK, row_b, pol_b);
            } else {
              mbar_arrive_expect_tx(fb, K::kStage);
              tma_load_2d(sa, &tm_a, fb, kb * K::kBK, row_a, pol_a);
              tma_load_2d(sa + kABytes, &tm_b, fb, kb * K::kBK, row_b, pol_b);
            }
            armed[stage] = (int)phase;
            if (++stage == K::kStages) {
              stage = 0;
              phase ^= 1u;
            }
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
      constexpr uint32_t idesc = idesc_make(K::kRows, BN, F8);
      int stage = 0, buf = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true, issued = false;
      for (int u = next_active(first_unit); u < units && ok; u = next_active(u + unit_stride)) {
        for (int nt = 0; nt < n_tiles && ok; ++nt) {
          if (!mbar_wait(smem_u32(&acce[buf]), acc_phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN);
          for (int kb = 0; kb < K::kKBlocks; ++kb) {
            if (!mbar_wait(smem_u32(&full[stage]), phase, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sa = smem_u32(smem + stage * K::kStage);
            const uint64_t da = sw128_desc(sa), db = sw128_desc(sa + kABytes);
#pragma unroll
            for (int k = 0; k < kRowBytes / 32; ++k)  // 32 bytes of K per MMA
              umma<PAIR, F8>(d_tmem, da + (uint64_t)(2 * k), db + (uint64_t)(2 * k), idesc, (kb | k) != 0 ? 1u : 0u);
            issued = true;
            umma_commit<PAIR>(smem_u32(&empty[stage]));
            if (++stage == K::kStages) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (!ok) break;
          umma_commit<PAIR>(smem_u32(&accf[buf]));
          if (++buf == 2) {
            buf = 0;
            acc_phase ^= 1u;
          }
        }
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
    const int row_in_tile = quarter * 32 + lane;
    const uint32_t acce_lead0 = PAIR ? map_to_rank(smem_u32(&acce[0]), 0) : smem_u32(&acce[0]);
    int buf = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int u = next_active(first_unit); u < units && ok; u = next_active(u + unit_stride)) {
      const int l = u / m_tiles, mt = u % m_tiles;
      const long long row = (long long)mt * K::kRows + (long long)rank * kBM + row_in_tile;
      const bool row_ok = row < C;
      const int my_doc = row_ok ? __ldg(block_doc + row) : -1;
      int carry_b = -1;           // query whose columns continue into the next N tile
      float carry_m = -INFINITY;
      for (int nt = 0; nt < n_tiles; ++nt) {
        if (!mbar_wait(smem_u32(&accf[buf]), acc_phase, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * BN);
        // two 32-column slices per TMEM round trip
#pragma unroll 1
        for (int c64 = 0; c64 < BN / 64; ++c64) {
          const int colA = nt * BN + c64 * 64;
          if (colA >= ql.row0[ql.n_queries]) break;  // trailing padding columns
          uint32_t ra[32], rb[32];
          tmem_ld32(tbase + (uint32_t)(c64 * 64), ra);
          tmem_ld32(tbase + (uint32_t)(c64 * 64 + 32), rb);
          tmem_wait_ld();
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const int col0 = colA + 32 * half;
            if (col0 >= ql.row0[ql.n_queries]) break;
            int lo = 0, hi = ql.n_queries;  // owner: largest b with row0[b] <= col0
            while (hi - lo > 1) {
              const int mid = (lo + hi) >> 1;
              if (ql.row0[mid] <= col0) lo = mid; else hi = mid;
            }
            const int b = lo;
            const int t0 = col0 - ql.row0[b];  // token index of column col0 in query b
            const int valid = min(32, ql.len[b] - t0);
            const uint32_t* r = half ? rb : ra;
            float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
            if (valid == 32) {  // (the same for every lane: a slice spans all the rows)
#pragma unroll
              for (int i = 0; i < 32; ++i) mx[i & 3] = fmaxf(mx[i & 3], __uint_as_float(r[i]));
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (i < valid) mx[i & 3] = fmaxf(mx[i & 3], __uint_as_float(r[i]));
            }
            float m1 = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
            if (b == carry_b) m1 = fmaxf(m1, carry_m);
            if (t0 + 32 >= ql.len[b]) {  // (the same for every lane)
              // the rows of one document are consecutive: max over each run of equal
              // documents in the warp, one atomic per run
              float v = F8 ? m1 * kF8ScoreScale : m1;
#pragma unroll
              for (int off = 1; off < 32; off <<= 1) {
                const float vo = __shfl_down_sync(0xffffffffu, v, off);
                const int dd = __shfl_down_sync(0xffffffffu, my_doc, off);
                if (lane + off < 32 && dd == my_doc) v = fmaxf(v, vo);
              }
              const int dprev = __shfl_up_sync(0xffffffffu, my_doc, 1);
              if (my_doc >= 0 && (lane == 0 || dprev != my_doc)) {
                const uint32_t ub = __float_as_uint(v);
                atomicMax(doc_score + ((long long)b * L + l) * n_docs + my_doc,
                          (ub & 0x80000000u) ? ~ub : (ub | 0x80000000u));
              }
              carry_b = -1;
            } else {
              carry_b = b;
              carry_m = m1;
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (PAIR) mbar_arrive_cluster(acce_lead0 + (uint32_t)(buf * 8));
          else mbar_arrive(smem_u32(&acce[buf]));
        }
        if (++buf == 2) {
          buf = 0;
          acc_phase ^= 1u;
        }
      }
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

// ------------------------------------------------------------------ host side
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

// 2D row-major [rows][1024] map (bf16 or bytes) with a box of [box_rows][128 bytes] and
// the 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows, bool f8) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const int elem = f8 ? 1 : 2;
  const cuuint64_t dims[2] = {(cuuint64_t)kKDim, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)kKDim * elem};
  const cuuint32_t box[2] = {(cuuint32_t)(kRowBytes / elem), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, f8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, bool PAIR, bool F8>
int launch_bn(const LaunchArgs& a, cudaStream_t s, const char** why) {
  using K = Cfg<BN, PAIR, F8>;
  CUtensorMap ma, mb;
  const uint64_t rows_a = (uint64_t)a.L * (uint64_t)a.C;
  if (!make_map(&ma, a.kr_hat, rows_a, kBM, F8) || !make_map(&mb, a.qt, (uint64_t)a.L * a.n_rows, K::kBRows, F8)) {
    *why = "cuTensorMapEncodeTiled failed";
    return 1;
  }
  const int m_tiles = (int)((a.C + K::kRows - 1) / K::kRows);
  const long long units = (long long)a.L * m_tiles;
  const int per_unit = PAIR ? 2 : 1;
  int grid = msa::sm_count() / per_unit * per_unit;
  if (units * per_unit < grid) grid = (int)(units * per_unit);
  if (cudaFuncSetAttribute(route_tc_kernel<BN, PAIR, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize, K::kSmem) !=
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
  if (cudaLaunchKernelEx(&cfg, route_tc_kernel<BN, PAIR, F8>, ma, mb, a.L, (long long)a.C, a.n_rows, m_tiles, a.ql,
                         a.block_doc, a.doc_score, a.n_docs, a.dev_err, a.layer_only) != cudaSuccess) {
    *why = "kernel launch";
    return 1;
  }
  return 0;
}

}  // namespace

bool supported(int n_kv_heads) { return n_kv_heads == 8; }

int launch(const LaunchArgs& a, cudaStream_t s, int* launches, const char** why) {
  *launches = 0;
  if ((long long)a.L * a.C >= (1ll << 31) || (long long)a.L * a.n_rows >= (1ll << 31)) {
    *why = "bank too large for 32-bit TMA row coordinates";
    return 1;
  }
  const int bn = tile_n(a.n_rows);
  if (a.n_rows % bn != 0) {
    *why = "operand rows not a multiple of the N tile";
    return 1;
  }
  int r;
  if (a.f8) {
    if (bn == 64) r = launch_bn<64, false, true>(a, s, why);
    else if (a.pair && bn == 128) r = launch_bn<128, true, true>(a, s, why);
    else if (bn == 128) r = launch_bn<128, false, true>(a, s, why);
    else if (a.pair) r = launch_bn<256, true, true>(a, s, why);
    else r = launch_bn<256, false, true>(a, s, why);
  } else {
    if (bn == 64) r = launch_bn<64, false, false>(a, s, why);
    else if (a.pair && bn == 128) r = launch_bn<128, true, false>(a, s, why);
    else if (bn == 128) r = launch_bn<128, false, false>(a, s, why);
    else if (a.pair) r = launch_bn<256, true, false>(a, s, why);
    else r = launch_bn<256, false, false>(a, s, why);
  }
  if (r == 0) *launches = 1;
  return r;
}

namespace {
// One CTA of 64 threads, the set-up and exit path of the tensor-core kernels on their
// own: warp 0 takes 32 columns of tensor memory, thread 0 waits on a barrier of count 1
// that nothing arrives on (unless release_first), bounded by limit_ns on the global timer;
// on expiry it sets MSA_DEVERR_TIMEOUT, and the tensor memory is freed before the kernel
// returns.
__global__ void __launch_bounds__(64) wait_selftest_kernel(unsigned long long limit_ns, int release_first,
                                                           int32_t* dev_err) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const int warp = threadIdx.x / 32;
  if (threadIdx.x == 0) {
    tc::mbar_init(tc::smem_u32(&bar), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    tc::tmem_alloc<false>(tc::smem_u32(&tmem_slot), 32);
    tc::tmem_relinquish<false>();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (threadIdx.x == 0) {
    if (release_first) tc::mbar_arrive(tc::smem_u32(&bar));
    if (!tc::mbar_wait(tc::smem_u32(&bar), 0, &abort_flag, limit_ns)) {
      abort_flag = 1;
      msa::set_err(dev_err, MSA_DEVERR_TIMEOUT);
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 0) tc::tmem_dealloc<false>(tmem_slot, 32);
}
}  // namespace

int launch_wait_selftest(unsigned long long limit_ns, int release_first, int32_t* dev_err, cudaStream_t s) {
  wait_selftest_kernel<<<1, 64, 0, s>>>(limit_ns, release_first, dev_err);
  return cudaGetLastError() == cudaSuccess ? 0 : 1;
}

}  // namespace route_tc
