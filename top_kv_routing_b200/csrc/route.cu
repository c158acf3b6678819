// Step 2: routing scores + fused top-k document selection.
//
// Follows "MSA端到端可训练记忆模型完整开源，支持亿级Token上下文", section 架构 (cosine routing,
// mean over heads then max over tokens, Top-k documents) and the MSA paper reading notes,
// section 路由投影器 + Top-k 稀疏注意力 (Top-16 against every document's pooled K_r).
//
// Launch sequence of one call:
//   1. qprep    Q_r -> qt[l][t][g][:] = (1/Hq) sum_{h: h/G = g} Q_r[t][h] / max(||Q_r[t][h]||,1e-8)
//               (fp32 for the exact kernels, bf16 rows padded per query for the GEMM)
//   2. score    m[b][l][c] = max_{t in b} cos-score(t, c)
//               scan path (few tokens): exact fp32 on CUDA cores, keys normalised per head
//               tensor path: tcgen05 GEMM on bf16 operands, or on the E4M3 filter copy of
//               the keys (a filter)
//   3. docmax   scan path: S[doc] = max of m over the document's blocks; per-CTA best
//               candidates.  Tensor path: the GEMM epilogue folds every block's maximum
//               into its document's score directly (atomicMax), no block scores stored
//   4. merge    scan path: the per-CTA candidates -> top_k.  Tensor path: radix selection
//               of the K2 filter candidates from the document scores
//   tensor path only:
//   5. rescore  exact scores of the K2 candidates: every block of the document against
//               every token of the query, on the tensor cores with ~fp32 operands
//   6. final    top_k of the exact scores; certification of the selection (E4M3: layers
//               that fail go through steps 2-6 again with the bf16 filter)
// The score matrix s[t][c] only ever lives in registers / TMEM.
#include <cuda_fp8.h>

#include "common.cuh"
#include "msa_route.h"
#include "route_proj.cuh"
#include "route_bound.cuh"
#include "route_tc.cuh"
#include "tc_common.cuh"

MSA_DEFINE_LAST_ERROR(msa_route_last_error)

namespace {
using namespace route_bound;

constexpr int kD = 128;
constexpr int kMaxQueries = 256;
constexpr int kMaxTopK = 64;
constexpr int kMaxCandidates = 128;  // documents rescored exactly after the tensor-core filter
constexpr int kTopkThreads = 512;
constexpr int kMaxDocs = 1 << 20;    // documents per bank
constexpr int kMaxBlocks = 64;       // docmax CTAs per (query, layer)
constexpr int kMaxWide = 1024;       // candidates of the widened rescoring

// Candidates rescored exactly on the tensor-core path.
int rescore_count(int32_t n_docs, int32_t k) {
  int k2 = 2 * k > k + 32 ? 2 * k : k + 32;
  if (k2 > kMaxCandidates) k2 = kMaxCandidates;
  return n_docs < k2 ? n_docs : k2;
}
// Candidates of the widened rescoring (layers whose selection the bf16 filter could not
// certify).
int wide_count(int32_t n_docs) { return n_docs < kMaxWide ? n_docs : kMaxWide; }

static thread_local int32_t g_launches = 0;
static thread_local cudaEvent_t g_prof_start = nullptr, g_prof_stop = nullptr;
static thread_local cudaEvent_t g_qprof_start = nullptr, g_qprof_stop = nullptr;
static thread_local bool g_pair_mode = true;

struct QueryOffsets {
  int32_t n;
  int32_t off[kMaxQueries + 1];   // token offsets of the queries in qr
  int32_t row0[kMaxQueries + 1];  // first row of each query in the padded bf16 operand
};

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

int topk_blocks(int32_t n_docs) {
  int nb = (n_docs + 511) / 512;
  if (nb < 1) nb = 1;
  if (nb > kMaxBlocks) nb = kMaxBlocks;
  return nb;
}

int pow2_at_least(int n) {
  int p = 1;
  while (p < n) p <<= 1;
  return p;
}

struct WsLayout {
  size_t qt_f32, qt_bf16, qt_lo, qt_f8, m, cand, apx, exact, redo, doc_score, block_doc, agg, apx_agg, exact_agg,
      etok, apx_w, exact_w, apx_agg_w, exact_agg_w, total;
  int n_pad;
  int nblk;
  int k2;
  int kw;
};

// Upper bound of the padded operand rows for B queries of T_total tokens in all.
int operand_rows_bound(int32_t T_total, int32_t B) {
  const int r = T_total + (route_tc::kQueryAlign - 1) * B;
  return (r + route_tc::kMaxTileN - 1) / route_tc::kMaxTileN * route_tc::kMaxTileN;
}

WsLayout ws_layout(int32_t L, int32_t B, int32_t T_total, int32_t H, int64_t C, int32_t n_docs, int32_t k) {
  WsLayout w;
  w.n_pad = operand_rows_bound(T_total, B);
  w.nblk = topk_blocks(n_docs);
  w.k2 = rescore_count(n_docs, k);
  w.kw = wide_count(n_docs);
  const int ksel = w.k2 > k ? w.k2 : k;
  const size_t k2s = (size_t)(ksel > 0 ? ksel : 1), kws = (size_t)(w.kw > 0 ? w.kw : 1);
  size_t o = 0;
  w.qt_f32 = o;
  o += align256((size_t)L * T_total * H * kD * sizeof(float));
  w.qt_bf16 = o;
  o += align256((size_t)L * w.n_pad * H * kD * 2);
  w.qt_lo = o;
  o += align256((size_t)L * w.n_pad * H * kD * 2);
  w.qt_f8 = o;
  o += align256((size_t)L * w.n_pad * H * kD);
  w.m = o;
  o += align256((size_t)B * L * (size_t)C * sizeof(float));
  w.cand = o;
  o += align256((size_t)B * L * w.nblk * ksel * sizeof(unsigned long long));
  w.apx = o;
  o += align256((size_t)B * L * k2s * sizeof(unsigned long long));
  w.exact = o;
  o += align256((size_t)B * L * k2s * sizeof(float));
  w.redo = o;  // three layer masks: E4M3 pass failed, bf16 pass failed, widened pass failed
  o += align256((size_t)3 * L * sizeof(int32_t));
  w.doc_score = o;
  o += align256((size_t)B * L * (size_t)(n_docs > 0 ? n_docs : 1) * sizeof(uint32_t));
  w.block_doc = o;
  o += align256((size_t)(C > 0 ? C : 1) * sizeof(int32_t));
  // layer-aggregated selection: mean document scores and their candidates per query
  w.agg = o;
  o += align256((size_t)B * (size_t)(n_docs > 0 ? n_docs : 1) * sizeof(uint32_t));
  w.apx_agg = o;
  o += align256((size_t)B * k2s * sizeof(unsigned long long));
  w.exact_agg = o;
  o += align256((size_t)B * k2s * sizeof(uint32_t));
  // per (bound kind, layer, token) filter error bounds
  w.etok = o;
  o += align256((size_t)2 * L * T_total * sizeof(float));
  // the widened rescoring's candidates
  w.apx_w = o;
  o += align256((size_t)B * L * kws * sizeof(unsigned long long));
  w.exact_w = o;
  o += align256((size_t)B * L * kws * sizeof(uint32_t));
  w.apx_agg_w = o;
  o += align256((size_t)B * kws * sizeof(unsigned long long));
  w.exact_agg_w = o;
  o += align256((size_t)B * kws * sizeof(uint32_t));
  w.total = o;
  return w;
}

// ---------------------------------------------------------------------------- 1. q prep
// grid (T_total, L); block 128 threads.  Hq <= 64.  The bf16 copy of token t of query b
// goes to operand row row0[b] + (t - off[b]) of layer l (n_rows rows per layer).
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__global__ void __launch_bounds__(128) qprep_kernel(const void* __restrict__ qr, int q_is_bf16, int T_total,
                                                    int Hq, int H, int n_rows, QueryOffsets qo,
                                                    float* __restrict__ qt_f32, __nv_bfloat16* __restrict__ qt_bf16,
                                                    __nv_bfloat16* __restrict__ qt_lo, uint8_t* __restrict__ qt_f8,
                                                    float* __restrict__ etok, int n_layers) {
  __shared__ float qhat[64][kD];
  __shared__ float red[16][4][6];  // per key head, per warp: the six sums of the bounds
  const int t = blockIdx.x, l = blockIdx.y;
  int qb = 0;
  {
    int lo = 0, hi = qo.n;  // largest b with off[b] <= t
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (qo.off[mid] <= t) lo = mid; else hi = mid;
    }
    qb = lo;
  }
  const int orow = qo.row0[qb] + (t - qo.off[qb]);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t row0 = ((int64_t)l * T_total + t) * Hq * kD;
  for (int h = warp; h < Hq; h += 4) {
    float x[4];
    if (q_is_bf16) {
      const uint2 w = *reinterpret_cast<const uint2*>(reinterpret_cast<const __nv_bfloat16*>(qr) + row0 +
                                                      (int64_t)h * kD + 4 * lane);
      const float2 a = msa::bf16x2_to_float2(w.x), b = msa::bf16x2_to_float2(w.y);
      x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
    } else {
      const float4 a = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(qr) + row0 +
                                                        (int64_t)h * kD + 4 * lane);
      x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    }
    float ss = x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = 1.0f / fmaxf(sqrtf(ss), 1e-8f);
#pragma unroll
    for (int u = 0; u < 4; ++u) qhat[h][4 * lane + u] = x[u] * inv;
  }
  __syncthreads();
  const int G = Hq / H;
  const float inv_hq = 1.0f / (float)Hq;
  // (every thread runs the same number of iterations: H * 128 is a multiple of 128)
  for (int e = threadIdx.x; e < H * kD; e += blockDim.x) {
    const int g = e / kD, j = e % kD;
    float acc = 0.f;
    for (int u = 0; u < G; ++u) acc += qhat[g * G + u][j];
    acc *= inv_hq;
    if (qt_f32 != nullptr) qt_f32[((int64_t)l * T_total + t) * H * kD + e] = acc;
    const int64_t oi = ((int64_t)l * n_rows + orow) * H * kD + e;
    const __nv_bfloat16 hi = __float2bfloat16_rn(acc);
    if (qt_bf16 != nullptr) {
      qt_bf16[oi] = hi;
      if (qt_lo != nullptr) qt_lo[oi] = __float2bfloat16_rn(acc - __bfloat162float(hi));
    }
    if (qt_f8 != nullptr) qt_f8[oi] = __nv_cvt_float_to_fp8(acc * route_tc::kF8QueryScale, __NV_SATFINITE, __NV_E4M3);
    if (etok != nullptr && g < 16) {
      const float hf = __bfloat162float(hi), db = hf - acc;
      const float a = acc * route_tc::kF8QueryScale, ah = e4m3_round(a), da = (ah - a) * (1.0f / route_tc::kF8QueryScale);
      const float as = ah * (1.0f / route_tc::kF8QueryScale);
      float v[6] = {acc * acc, db * db, hf * hf, as * as, da * da, fabsf(as)};
#pragma unroll
      for (int i = 0; i < 6; ++i) v[i] = warp_sum(v[i]);
      if ((threadIdx.x & 31) == 0)
#pragma unroll
        for (int i = 0; i < 6; ++i) red[g][threadIdx.x >> 5][i] = v[i];
    }
  }
  if (etok == nullptr) return;
  __syncthreads();
  // thread g < H: the bounds of key head g; then their sums over the heads
  float2 eb = make_float2(0.f, 0.f);
  if (threadIdx.x < H && threadIdx.x < 16) {
    float v[6];
#pragma unroll
    for (int i = 0; i < 6; ++i) v[i] = red[threadIdx.x][0][i] + red[threadIdx.x][1][i] + red[threadIdx.x][2][i] +
                                     red[threadIdx.x][3][i];
    eb = head_bounds(sqrtf(v[0]), sqrtf(v[1]), sqrtf(v[2]), sqrtf(v[3]), sqrtf(v[4]), v[5]);
  }
  if (threadIdx.x < 32) {
    eb.x = warp_sum(eb.x);
    eb.y = warp_sum(eb.y);
    if (threadIdx.x == 0) {
      etok[((int64_t)kBoundF8 * n_layers + l) * T_total + t] = eb.x * kBoundSlack + kBoundFloor;
      etok[((int64_t)kBoundBf16 * n_layers + l) * T_total + t] = eb.y * kBoundSlack + kBoundFloor;
    }
  }
}

// Document scores are kept as the ordered bits of make_key's high word (monotonic as
// unsigned ints, so atomicMax works on them); this is -inf, a document with no block.
constexpr uint32_t kOrdNegInf = 0x007FFFFFu;

// Zero every operand row that holds no query token (per-query alignment gaps and the
// tail up to n_rows), in 16-byte words, in up to three operand buffers; on the tensor
// path also write the block -> document map and set every (query, layer, document)
// score to -inf.
struct PadTargets {
  uint4* buf[3];
  int words_per_row[3];
};

__global__ void route_prep_kernel(PadTargets pt, int n_rows, int L, QueryOffsets qo,
                                  const int64_t* __restrict__ doc_chunk_off, int n_docs,
                                  int32_t* __restrict__ block_doc, uint32_t* __restrict__ doc_score,
                                  int64_t n_scores, float* __restrict__ etok, int64_t n_etok,
                                  int32_t* __restrict__ redo, int n_redo) {
  const int64_t i0 = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int k = 0; k < 3; ++k) {
    if (pt.buf[k] == nullptr) continue;
    const int wpr = pt.words_per_row[k];
    const int64_t total = (int64_t)L * n_rows * wpr;
    for (int64_t i = i0; i < total; i += stride) {
      const int r = (int)((i / wpr) % n_rows);
      int lo = 0, hi = qo.n;
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (qo.row0[mid] <= r) lo = mid; else hi = mid;
      }
      const bool token_row = r < qo.row0[qo.n] && (r - qo.row0[lo]) < (qo.off[lo + 1] - qo.off[lo]);
      if (!token_row) pt.buf[k][i] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  if (block_doc != nullptr)
    for (int64_t d = i0; d < n_docs; d += stride)
      for (int64_t c = doc_chunk_off[d]; c < doc_chunk_off[d + 1]; ++c) block_doc[c] = (int32_t)d;
  if (doc_score != nullptr)
    for (int64_t i = i0; i < n_scores; i += stride) doc_score[i] = kOrdNegInf;
  for (int64_t i = i0; i < n_etok; i += stride) etok[i] = 0.f;  // (the projection adds into it)
  for (int64_t i = i0; i < n_redo; i += stride) redo[i] = 0;
}

// grid (L, B): the document scores of the layers `only` marks back to -inf
__global__ void doc_reset_kernel(uint32_t* __restrict__ doc_score, int L, int n_docs,
                                 const int32_t* __restrict__ only) {
  const int l = blockIdx.x, b = blockIdx.y;
  if (only[l] == 0) return;
  uint32_t* sc = doc_score + ((int64_t)b * L + l) * n_docs;
  for (int d = threadIdx.x; d < n_docs; d += blockDim.x) sc[d] = kOrdNegInf;
}

// ---------------------------------------------------------------------------- E4M3 keys
// 8 threads per (row, head): 16 bf16 each; the head is renormalised in fp32 (the same
// 1 / max(||k||, 1e-8) as the exact kernels) and stored x kF8KeyScale as E4M3.  The loop
// runs per warp (4 heads a pass) so every lane takes part in the shuffles.
__global__ void __launch_bounds__(256) filter_keys_kernel(const __nv_bfloat16* __restrict__ kr, int64_t n_heads,
                                                          uint8_t* __restrict__ out) {
  const int lane = threadIdx.x & 31, sub = lane & 7;
  const int64_t warp0 = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t n_warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t base = warp0 * 4; base < n_heads; base += n_warps * 4) {
    const int64_t hh = base + (lane >> 3);
    const bool ok = hh < n_heads;
    float x[16];
    float ss = 0.f;
    if (ok) {
      const uint4* src = reinterpret_cast<const uint4*>(kr + hh * kD) + 2 * sub;
      const uint4 w0 = __ldcs(src), w1 = __ldcs(src + 1);
      const uint32_t w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float2 f = msa::bf16x2_to_float2(w[i]);
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) ss = fmaf(x[i], x[i], ss);
    }
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
    ss += __shfl_xor_sync(0xffffffffu, ss, 4);
    if (ok) {
      const float sc = route_tc::kF8KeyScale / fmaxf(sqrtf(ss), 1e-8f);
      uint32_t o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(x[4 * i] * sc, x[4 * i + 1] * sc), __NV_SATFINITE,
                                                     __NV_E4M3);
        const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(x[4 * i + 2] * sc, x[4 * i + 3] * sc),
                                                     __NV_SATFINITE, __NV_E4M3);
        o[i] = lo | (hi << 16);
      }
      __stcs(reinterpret_cast<uint4*>(out + hh * kD) + sub, make_uint4(o[0], o[1], o[2], o[3]));
    }
  }
}

// ---------------------------------------------------------------------------- key rows
// A warp holds one key row of R = 2*NV*128 elements: lane owns the 8-element vectors
// v = lane + 32 i (i < NV), i.e. head (v >> 4) = 2 i + (lane >> 4).  The row is widened
// to fp32 and every head is scaled by 1 / max(||k_head||, 1e-8) computed from the stored
// bf16 values, so dots with the unit query sums are exact cosines (fp32).
template <int NV>
__device__ __forceinline__ void load_unit_row(const __nv_bfloat16* __restrict__ row, int lane, float (&kx)[NV][8]) {
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(row) + lane + 32 * i);
    float2 f;
    f = msa::bf16x2_to_float2(w.x); kx[i][0] = f.x; kx[i][1] = f.y;
    f = msa::bf16x2_to_float2(w.y); kx[i][2] = f.x; kx[i][3] = f.y;
    f = msa::bf16x2_to_float2(w.z); kx[i][4] = f.x; kx[i][5] = f.y;
    f = msa::bf16x2_to_float2(w.w); kx[i][6] = f.x; kx[i][7] = f.y;
  }
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) ss = fmaf(kx[i][u], kx[i][u], ss);
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);   // the 16 lanes of a head half-warp
    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
    ss += __shfl_xor_sync(0xffffffffu, ss, 4);
    ss += __shfl_xor_sync(0xffffffffu, ss, 8);
    const float rho = 1.0f / fmaxf(sqrtf(ss), 1e-8f);
#pragma unroll
    for (int u = 0; u < 8; ++u) kx[i][u] *= rho;
  }
}

// <qt[t], unit row> for the lane's slice (before the warp reduction).
template <int NV>
__device__ __forceinline__ float lane_dot(const float4* __restrict__ qv, int lane, const float (&kx)[NV][8]) {
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const float4 a = __ldg(qv + 2 * (lane + 32 * i));
    const float4 b = __ldg(qv + 2 * (lane + 32 * i) + 1);
    acc = fmaf(kx[i][0], a.x, acc);
    acc = fmaf(kx[i][1], a.y, acc);
    acc = fmaf(kx[i][2], a.z, acc);
    acc = fmaf(kx[i][3], a.w, acc);
    acc = fmaf(kx[i][4], b.x, acc);
    acc = fmaf(kx[i][5], b.y, acc);
    acc = fmaf(kx[i][6], b.z, acc);
    acc = fmaf(kx[i][7], b.w, acc);
  }
  return acc;
}

// ---------------------------------------------------------------------------- 2a. scan
// One warp per (layer, block) task: exact cosine scores of the block against every
// query token, running max per query.
template <int NV>
__global__ void __launch_bounds__(256) scan_kernel(const __nv_bfloat16* __restrict__ kr_hat,
                                                   const float* __restrict__ qt, int L, int64_t C,
                                                   int T_total, QueryOffsets qo, float* __restrict__ m) {
  constexpr int R = NV * 256;
  const int lane = threadIdx.x % 32;
  const int64_t warp_global = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) / 32;
  const int64_t n_warps = (int64_t)gridDim.x * blockDim.x / 32;
  const int64_t tasks = (int64_t)L * C;
  for (int64_t task = warp_global; task < tasks; task += n_warps) {
    const int l = (int)(task / C);
    const int64_t c = task % C;
    float kx[NV][8];
    load_unit_row<NV>(kr_hat + ((int64_t)l * C + c) * R, lane, kx);
    const float* qbase = qt + (int64_t)l * T_total * R;
    for (int b = 0; b < qo.n; ++b) {
      float best = -INFINITY;
      for (int t = qo.off[b]; t < qo.off[b + 1]; ++t)
        best = fmaxf(best, warp_sum(lane_dot<NV>(reinterpret_cast<const float4*>(qbase + (int64_t)t * R), lane, kx)));
      if (lane == 0) m[((int64_t)b * L + l) * C + c] = best;
    }
  }
}

__device__ __forceinline__ void rs_ldsm_x4(uint32_t addr, uint32_t (&a)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
               : "r"(addr));
}
__device__ __forceinline__ void rs_mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------------------- 2a. scan (streaming, tensor cores)
// The streaming scan of few-token queries (T_total <= 4 tokens, all queries of the call;
// H <= 8 key heads).  Persistent, one CTA per SM, thirteen warps.  Warp 12 streams tiles
// of 16 consecutive blocks of one layer into 6 shared-memory stages, one cp.async.bulk per
// block row issued by lanes 0..15 (rows padded by 16 bytes, so that ldmatrix reads them
// without bank conflicts; completion on mbarriers, every wait bounded).  Warps 0..11 are
// six pairs; pair p takes the tiles p, p + 6, ..., always in the stage only it reads (so
// no warp waits on a stage's next fill before the previous one), each warp of the pair
// half of the key heads.  Per key head, on the tensor cores (mma.sync m16n8k16, fp32
// accumulation, even and odd k-steps in two chains): A = 16 key rows x 16 dims (the stored
// bf16 keys, exact); B = the query sums of up to 4 tokens as 8 columns, the bf16 value of
// each token in columns 0..3 and its bf16 residual in 4..7 (about 16 mantissa bits).  The
// rows' squared norms are summed in fp32 from the same A fragments; each head's dot is
// scaled by 1 / max(||k||, 1e-8) and the heads summed, the second warp's half through
// shared memory; the maximum over each query's tokens goes to m.  On a timeout the kernel
// sets MSA_DEVERR_TIMEOUT, waits (bounded) for its own copies in flight and returns.
constexpr int kScanPairs = 6;
constexpr int kScanConsumers = 2 * kScanPairs;
constexpr int kScanThreads = 32 * (kScanConsumers + 1);
constexpr int kScanTile = 16;
constexpr int kScanStages = kScanPairs;
constexpr int kScanMmaTokens = 4;

__device__ __forceinline__ void scan_bulk_copy(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

template <int H>
struct ScanCfg {
  static constexpr int kHW = H / 2;                       // key heads per warp
  static constexpr int kRowBytes = H * kD * 2;
  static constexpr int kStride = kRowBytes + 16;          // padded row in shared memory
  static constexpr int kStageBytes = kScanTile * kStride;
  static constexpr int kSmem = kScanStages * kStageBytes + kScanPairs * 2 * 32 * 16;  // + the pairs' exchange
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo_elem, float hi_elem) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo_elem, hi_elem);
  return *reinterpret_cast<const uint32_t*>(&v);
}

template <int H>
__global__ void __launch_bounds__(kScanThreads, 1) scan_mma_kernel(const __nv_bfloat16* __restrict__ kr_hat,
                                                                   const float* __restrict__ qt, int L, int64_t C,
                                                                   int T_total,
                                                                   const __grid_constant__ QueryOffsets qo,
                                                                   float* __restrict__ m, int32_t* dev_err) {
  using K = ScanCfg<H>;
  constexpr int R = H * kD;
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ __align__(8) uint64_t full[kScanStages], empty[kScanStages];
  __shared__ int abort_flag;
  __shared__ int pair_ok[kScanPairs][2][2];  // per pair, tile parity, warp: its wait succeeded
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t tpl = (C + kScanTile - 1) / kScanTile;  // tiles per layer
  const int64_t tiles = (int64_t)L * tpl;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kScanStages; ++i) {
      tc::mbar_init(tc::smem_u32(&full[i]), 1);
      tc::mbar_init(tc::smem_u32(&empty[i]), 2);
    }
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  const uint32_t ring_base = tc::smem_u32(ring);

  if (warp == kScanConsumers) {
    // ------------------------------------------------------------ producer: lane 0 waits for
    // a free stage and arms its barrier, then lanes 0..15 issue one row copy each
    uint32_t armed = 0u, armed_phase = 0u;  // stages with copies issued, and their phase bit
    bool ok = true;
    int64_t i = 0;
    for (int64_t u = blockIdx.x; u < tiles; u += gridDim.x, ++i) {
      const int st = (int)(i % kScanStages);
      const uint32_t ph = (uint32_t)((i / kScanStages) & 1);
      bool got = true;
      if (lane == 0) got = tc::mbar_wait(tc::smem_u32(&empty[st]), ph ^ 1u, &abort_flag);
      if (!__shfl_sync(0xffffffffu, got, 0)) {
        ok = false;
        break;
      }
      const int l = (int)(u / tpl);
      const int64_t c0 = (u % tpl) * kScanTile;
      const int n = (int)min((int64_t)kScanTile, C - c0);
      const uint32_t fb = tc::smem_u32(&full[st]);
      if (lane == 0) tc::mbar_arrive_expect_tx(fb, (uint32_t)n * K::kRowBytes);
      __syncwarp();  // armed before any copy can complete on it
      if (lane < n)
        scan_bulk_copy(ring_base + st * K::kStageBytes + lane * K::kStride,
                       kr_hat + ((int64_t)l * C + c0 + lane) * R, K::kRowBytes, fb);
      armed |= 1u << st;
      armed_phase = (armed_phase & ~(1u << st)) | (ph << st);
    }
    if (lane == 0) {
      if (!ok) {
        abort_flag = 1;
        msa::set_err(dev_err, MSA_DEVERR_TIMEOUT);
      }
      // no copy may still be writing this CTA's shared memory when it exits
      for (int k = 0; k < kScanStages; ++k)
        if ((armed >> k) & 1u) tc::mbar_drain(tc::smem_u32(&full[k]), (armed_phase >> k) & 1u);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int pair = warp >> 1, sub = warp & 1;
  const int g = lane >> 2, t = lane & 3;
  const int lrow = (lane & 7) + 8 * ((lane >> 3) & 1), lhalf = lane >> 4;
  float4* xch = reinterpret_cast<float4*>(ring + kScanStages * K::kStageBytes) + pair * 2 * 32;
  uint32_t bq[K::kHW][8][2];  // B fragments of this warp's heads (values in columns 0..3, residuals 4..7)
  int cur_l = -1;
  int64_t i = pair;  // this CTA's tile index
  for (int64_t u = blockIdx.x + (int64_t)pair * gridDim.x, k = 0; u < tiles;
       u += (int64_t)kScanPairs * gridDim.x, i += kScanPairs, ++k) {
    const int l = (int)(u / tpl);
    const int64_t c0 = (u % tpl) * kScanTile;
    const int n = (int)min((int64_t)kScanTile, C - c0);
    if (l != cur_l) {
      // column g of B: token g & 3, its bf16 value (g < 4) or residual (g >= 4); rows
      // k = 2t, 2t+1 (b0) and 2t+8, 2t+9 (b1) of each 16-dim slice
      const int tok = g & 3;
      const bool lo = g >= 4;
      const float* qrow = qt + ((int64_t)l * T_total + tok) * R;
#pragma unroll
      for (int j = 0; j < K::kHW; ++j)
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          float x[4] = {0.f, 0.f, 0.f, 0.f};
          if (tok < T_total) {
            const int d0 = (sub * K::kHW + j) * kD + 16 * ks + 2 * t;
            const float2 p = __ldg(reinterpret_cast<const float2*>(qrow + d0));
            const float2 p8 = __ldg(reinterpret_cast<const float2*>(qrow + d0 + 8));
            x[0] = p.x; x[1] = p.y; x[2] = p8.x; x[3] = p8.y;
          }
          float v[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float hi = __bfloat162float(__float2bfloat16_rn(x[e]));
            v[e] = lo ? x[e] - hi : x[e];
          }
          bq[j][ks][0] = pack_bf16x2(v[0], v[1]);
          bq[j][ks][1] = pack_bf16x2(v[2], v[3]);
        }
      cur_l = l;
    }
    const int st = (int)(i % kScanStages);
    const uint32_t ph = (uint32_t)((i / kScanStages) & 1);
    // (warp-uniform; a failed wait raises the abort flag, the pair still meets at its
    // barrier below, and both warps leave on the flags they exchange there)
    const bool ok = __all_sync(0xffffffffu, tc::mbar_wait(tc::smem_u32(&full[st]), ph, &abort_flag));
    if (!ok) abort_flag = 1;
    float tot[4] = {0.f, 0.f, 0.f, 0.f};  // rows g, g (tokens 2(t&1), +1), rows g+8, g+8
    if (ok) {
      const uint32_t arow = ring_base + st * K::kStageBytes + lrow * K::kStride + lhalf * 16;
#pragma unroll
      for (int j = 0; j < K::kHW; ++j) {
        const int hh = sub * K::kHW + j;
        float acc[4] = {0.f, 0.f, 0.f, 0.f}, acc2[4] = {0.f, 0.f, 0.f, 0.f};  // even / odd k-steps
        float ss0 = 0.f, ss1 = 0.f;  // squared norms of rows g, g + 8 (this lane's elements)
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          uint32_t a[4];
          rs_ldsm_x4(arow + (uint32_t)((hh * kD + 16 * ks) * 2), a);
          if (ks & 1) rs_mma(acc2, a, bq[j][ks][0], bq[j][ks][1]);
          else rs_mma(acc, a, bq[j][ks][0], bq[j][ks][1]);
          const float2 f0 = msa::bf16x2_to_float2(a[0]), f1 = msa::bf16x2_to_float2(a[1]);
          const float2 f2 = msa::bf16x2_to_float2(a[2]), f3 = msa::bf16x2_to_float2(a[3]);
          ss0 = fmaf(f0.x, f0.x, ss0); ss0 = fmaf(f0.y, f0.y, ss0); ss0 = fmaf(f2.x, f2.x, ss0); ss0 = fmaf(f2.y, f2.y, ss0);
          ss1 = fmaf(f1.x, f1.x, ss1); ss1 = fmaf(f1.y, f1.y, ss1); ss1 = fmaf(f3.x, f3.x, ss1); ss1 = fmaf(f3.y, f3.y, ss1);
        }
        ss0 += __shfl_xor_sync(0xffffffffu, ss0, 1);  // the row's 4 lanes t
        ss0 += __shfl_xor_sync(0xffffffffu, ss0, 2);
        ss1 += __shfl_xor_sync(0xffffffffu, ss1, 1);
        ss1 += __shfl_xor_sync(0xffffffffu, ss1, 2);
        const float r0 = 1.0f / fmaxf(sqrtf(ss0), 1e-8f), r1 = 1.0f / fmaxf(sqrtf(ss1), 1e-8f);
        // columns 2t, 2t+1: lanes t < 2 hold the values, lanes t >= 2 the residuals of the
        // same tokens; the pair sum is the ~16-bit dot
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc[e] += acc2[e];
          acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 2);
        }
        tot[0] = fmaf(r0, acc[0], tot[0]);
        tot[1] = fmaf(r0, acc[1], tot[1]);
        tot[2] = fmaf(r1, acc[2], tot[2]);
        tot[3] = fmaf(r1, acc[3], tot[3]);
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(tc::smem_u32(&empty[st]));  // done with the stage
    }
    // the second warp's half of the heads, through shared memory (double-buffered by the
    // pair's tile count, so one barrier per tile orders writes and reads)
    if (sub == 1) xch[(k & 1) * 32 + lane] = make_float4(tot[0], tot[1], tot[2], tot[3]);
    if (lane == 0) pair_ok[pair][k & 1][sub] = ok ? 1 : 0;
    asm volatile("bar.sync %0, 64;" ::"r"(1 + pair) : "memory");
    if (!(pair_ok[pair][k & 1][0] && pair_ok[pair][k & 1][1])) break;  // (the same in both warps)
    if (sub == 1) continue;
    const float4 o = xch[(k & 1) * 32 + lane];
    tot[0] += o.x;
    tot[1] += o.y;
    tot[2] += o.z;
    tot[3] += o.w;
    // lane (g, t): tokens 2(t&1), 2(t&1)+1 of rows g, g+8; the other pair from lane t ^ 1
    float oth[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) oth[e] = __shfl_xor_sync(0xffffffffu, tot[e], 1);
    if (t == 0) {
      const float s0[4] = {tot[0], tot[1], oth[0], oth[1]};  // row g, tokens 0..3
      const float s1[4] = {tot[2], tot[3], oth[2], oth[3]};  // row g + 8
      for (int b = 0; b < qo.n; ++b) {
        float b0 = -INFINITY, b1 = -INFINITY;
#pragma unroll
        for (int q = 0; q < kScanMmaTokens; ++q)
          if (q >= qo.off[b] && q < qo.off[b + 1]) {
            b0 = fmaxf(b0, s0[q]);
            b1 = fmaxf(b1, s1[q]);
          }
        float* mrow = m + ((int64_t)b * L + l) * C + c0;
        if (g < n) mrow[g] = b0;
        if (g + 8 < n) mrow[g + 8] = b1;
      }
    }
  }
  if (lane == 0 && abort_flag) msa::set_err(dev_err, MSA_DEVERR_TIMEOUT);
}

// ---------------------------------------------------------------------------- 2a'. exact fallback
// The scan of the layers `only` marks (tensor path, 8 key heads), for every query: the
// last resort when no filter could certify a layer's selection.  A token's query sum is
// read as its bf16 operand row plus the bf16 residual row (about 16 mantissa bits; the
// tensor path keeps no fp32 copy).  Returns at once when no layer is marked.
__global__ void __launch_bounds__(256) scan_fallback_kernel(const __nv_bfloat16* __restrict__ kr_hat,
                                                            const __nv_bfloat16* __restrict__ q_hi,
                                                            const __nv_bfloat16* __restrict__ q_lo, int L, int64_t C,
                                                            int n_rows, QueryOffsets qo, float* __restrict__ m,
                                                            const int32_t* __restrict__ only) {
  constexpr int NV = 4, R = NV * 256;
  int any = 0;
  for (int i = threadIdx.x; i < L; i += blockDim.x) any |= only[i] != 0;
  if (!__syncthreads_or(any)) return;
  const int lane = threadIdx.x % 32;
  const int64_t warp_global = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) / 32;
  const int64_t n_warps = (int64_t)gridDim.x * blockDim.x / 32;
  for (int64_t task = warp_global; task < (int64_t)L * C; task += n_warps) {
    const int l = (int)(task / C);
    if (only[l] == 0) continue;
    const int64_t c = task % C;
    float kx[NV][8];
    load_unit_row<NV>(kr_hat + ((int64_t)l * C + c) * R, lane, kx);
    for (int b = 0; b < qo.n; ++b) {
      float best = -INFINITY;
      const int T = qo.off[b + 1] - qo.off[b];
      for (int t = 0; t < T; ++t) {
        const int64_t row = (int64_t)l * n_rows + qo.row0[b] + t;
        const uint4* hv = reinterpret_cast<const uint4*>(q_hi + row * R);
        const uint4* lv = reinterpret_cast<const uint4*>(q_lo + row * R);
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
          const uint4 wh = __ldg(hv + lane + 32 * i), wl = __ldg(lv + lane + 32 * i);
          const uint32_t h4[4] = {wh.x, wh.y, wh.z, wh.w}, l4[4] = {wl.x, wl.y, wl.z, wl.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float2 fh = msa::bf16x2_to_float2(h4[u]), fl = msa::bf16x2_to_float2(l4[u]);
            acc = fmaf(kx[i][2 * u], fh.x + fl.x, acc);
            acc = fmaf(kx[i][2 * u + 1], fh.y + fl.y, acc);
          }
        }
        best = fmaxf(best, warp_sum(acc));
      }
      if (lane == 0) m[((int64_t)b * L + l) * C + c] = best;
    }
  }
}

// ---------------------------------------------------------------------------- 3/4. top-k
// Candidate keys order (score desc, id asc) as unsigned integers; 0 = empty slot.
__device__ __forceinline__ unsigned long long make_key(float s, int doc) {
  uint32_t u = __float_as_uint(s);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((unsigned long long)u << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)doc);
}

__device__ __forceinline__ void split_key(unsigned long long key, int* doc, float* s) {
  if (key == 0ull) {
    *doc = -1;
    *s = -INFINITY;
    return;
  }
  uint32_t u = (uint32_t)(key >> 32);
  u = (u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u;
  *s = __uint_as_float(u);
  *doc = (int)(0xFFFFFFFFu - (uint32_t)(key & 0xFFFFFFFFull));
}

// Sorts keys[0..n) (smem, n a power of two) in descending order (bitonic network).
__device__ void block_sort_desc(unsigned long long* keys, int n) {
  for (int k = 2; k <= n; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const unsigned long long a = keys[i], b = keys[ixj];
          const bool desc = (i & k) == 0;
          if (desc ? (a < b) : (a > b)) {
            keys[i] = b;
            keys[ixj] = a;
          }
        }
      }
      __syncthreads();
    }
  }
}

// grid (nblk, L, B): documents [blk*per, (blk+1)*per) of (b, l); writes its k_sel best keys.
__global__ void __launch_bounds__(kTopkThreads) docmax_topk_kernel(const float* __restrict__ m,
                                                                   const int64_t* __restrict__ doc_chunk_off,
                                                                   int n_docs, int64_t C, int L, int k_sel,
                                                                   int n_pow2, unsigned long long* __restrict__ cand,
                                                                   const int32_t* __restrict__ only) {
  extern __shared__ unsigned long long tk_smem[];
  const int blk = blockIdx.x, l = blockIdx.y, b = blockIdx.z;
  if (only != nullptr && only[l] == 0) return;
  const int nblk = gridDim.x;
  const int per = (n_docs + nblk - 1) / nblk;
  const int d0 = blk * per;
  const int d1 = min(n_docs, d0 + per);
  const int n = max(0, d1 - d0);
  const float* mb = m + ((int64_t)b * L + l) * C;
  for (int i = threadIdx.x; i < n_pow2; i += blockDim.x) {
    unsigned long long key = 0ull;
    if (i < n) {
      const int doc = d0 + i;
      const int64_t c0 = __ldg(doc_chunk_off + doc), c1 = __ldg(doc_chunk_off + doc + 1);
      float s0 = -INFINITY, s1 = -INFINITY, s2 = -INFINITY, s3 = -INFINITY;
      int64_t c = c0;
      for (; c + 4 <= c1; c += 4) {
        s0 = fmaxf(s0, __ldg(mb + c));
        s1 = fmaxf(s1, __ldg(mb + c + 1));
        s2 = fmaxf(s2, __ldg(mb + c + 2));
        s3 = fmaxf(s3, __ldg(mb + c + 3));
      }
      for (; c < c1; ++c) s0 = fmaxf(s0, __ldg(mb + c));
      key = make_key(fmaxf(fmaxf(s0, s1), fmaxf(s2, s3)), doc);
    }
    tk_smem[i] = key;
  }
  __syncthreads();
  block_sort_desc(tk_smem, n_pow2);
  unsigned long long* out = cand + (((int64_t)b * L + l) * nblk + blk) * k_sel;
  for (int r = threadIdx.x; r < k_sel; r += blockDim.x) out[r] = r < n_pow2 ? tk_smem[r] : 0ull;
}

// grid (L, B): merges nblk * k_sel candidates into the k_sel best.  Writes keys_out
// [B][L][k_sel] when given, else ids / scores [B][L][k_sel].
__global__ void __launch_bounds__(kTopkThreads) merge_topk_kernel(const unsigned long long* __restrict__ cand,
                                                                  int nblk, int L, int k_sel, int n_pow2,
                                                                  unsigned long long* __restrict__ keys_out,
                                                                  int32_t* __restrict__ out_ids,
                                                                  float* __restrict__ out_scores,
                                                                  const int32_t* __restrict__ only) {
  extern __shared__ unsigned long long tk_smem[];
  const int l = blockIdx.x, b = blockIdx.y;
  if (only != nullptr && only[l] == 0) return;
  const int n = nblk * k_sel;
  const unsigned long long* src = cand + ((int64_t)b * L + l) * n;
  for (int i = threadIdx.x; i < n_pow2; i += blockDim.x) tk_smem[i] = i < n ? src[i] : 0ull;
  __syncthreads();
  block_sort_desc(tk_smem, n_pow2);
  for (int r = threadIdx.x; r < k_sel; r += blockDim.x) {
    const int64_t o = ((int64_t)b * L + l) * k_sel + r;
    const unsigned long long key = r < n_pow2 ? tk_smem[r] : 0ull;
    if (keys_out != nullptr) {
      keys_out[o] = key;
    } else {
      int doc;
      float s;
      split_key(key, &doc, &s);
      out_ids[o] = doc;
      out_scores[o] = s;
    }
  }
}

// grid (L, B), 1024 threads: the k_sel best documents of (b, l) by score (equal scores:
// smaller id first), as keys in descending order (key 0: no document).  Radix selection
// on the ordered score bits, 8 bits a pass (histograms with warp-aggregated shared
// atomics, kSelBatch independent loads per thread in flight), then one pass collecting
// the documents above the threshold value and those at it; the lowest ids at it are
// taken (an ordered scan only when more than kSelEqCap documents share that value).
constexpr int kSelThreads = 1024;
constexpr int kSelBatch = 16;
constexpr int kSelEqCap = 1024;

template <int MAXC>
__global__ void __launch_bounds__(kSelThreads) topk_docs_kernel(const uint32_t* __restrict__ doc_score, int L,
                                                                int n_docs, int k_sel,
                                                                unsigned long long* __restrict__ out,
                                                                uint32_t* __restrict__ exact_bits,
                                                                const int32_t* __restrict__ only) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_prefix, s_mask;
  __shared__ int s_need, s_gt, s_eq, s_taken;
  __shared__ int wsum[kSelThreads / 32];
  __shared__ unsigned long long keys[MAXC];
  __shared__ int eq_docs[kSelEqCap];
  const int l = blockIdx.x, b = blockIdx.y;
  if (only != nullptr && only[l] == 0) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t* sc = doc_score + ((int64_t)b * L + l) * n_docs;
  unsigned long long* o = out + ((int64_t)b * L + l) * k_sel;
  const int K = min(k_sel, n_docs);
  constexpr int kSpan = kSelThreads * kSelBatch;
  if (tid == 0) {
    s_prefix = 0u;
    s_mask = 0u;
    s_need = K;
    s_gt = 0;
    s_eq = 0;
    s_taken = 0;
  }
  if (K > 0) {
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0u;
      __syncthreads();
      const uint32_t prefix = s_prefix, mask = s_mask;
      for (int d0 = 0; d0 < n_docs; d0 += kSpan) {  // (uniform trip count for the match)
        uint32_t u[kSelBatch];
#pragma unroll
        for (int j = 0; j < kSelBatch; ++j) {
          const int d = d0 + j * kSelThreads + tid;
          u[j] = d < n_docs ? __ldcg(sc + d) : 0u;
        }
#pragma unroll
        for (int j = 0; j < kSelBatch; ++j) {
          const int d = d0 + j * kSelThreads + tid;
          const bool in = d < n_docs && (u[j] & mask) == prefix;
          const uint32_t bin = in ? (u[j] >> shift) & 255u : 256u;
          const uint32_t same = __match_any_sync(0xffffffffu, bin);
          if (in && lane == __ffs(same) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(same));
        }
      }
      __syncthreads();
      if (warp == 0) {
        // lane i owns bins 8i .. 8i+7; sfx = documents in bins >= 8i
        int c = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) c += (int)hist[8 * lane + j];
        int sfx = c;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int t = __shfl_down_sync(0xffffffffu, sfx, off);
          if (lane + off < 32) sfx += t;
        }
        int nxt = __shfl_down_sync(0xffffffffu, sfx, 1);
        if (lane == 31) nxt = 0;
        const int need = s_need;
        if (sfx >= need && nxt < need) {
          int cum = nxt;
          for (int j = 7; j >= 0; --j) {
            const int bin = 8 * lane + j;
            if (cum + (int)hist[bin] >= need) {
              s_need = need - cum;
              s_prefix = prefix | ((uint32_t)bin << shift);
              s_mask = mask | (255u << shift);
              break;
            }
            cum += (int)hist[bin];
          }
        }
      }
      __syncthreads();
    }
    // the documents above the threshold value, and those at it
    const uint32_t thr = s_prefix;
    const int need = s_need;
    for (int d0 = 0; d0 < n_docs; d0 += kSpan) {
      uint32_t u[kSelBatch];
#pragma unroll
      for (int j = 0; j < kSelBatch; ++j) {
        const int d = d0 + j * kSelThreads + tid;
        u[j] = d < n_docs ? __ldcg(sc + d) : 0u;
      }
#pragma unroll
      for (int j = 0; j < kSelBatch; ++j) {
        const int d = d0 + j * kSelThreads + tid;
        if (d >= n_docs) continue;
        if (u[j] > thr) {
          keys[atomicAdd(&s_gt, 1)] = ((unsigned long long)u[j] << 32) | (0xFFFFFFFFull - (uint32_t)d);
        } else if (u[j] == thr) {
          const int slot = atomicAdd(&s_eq, 1);
          if (slot < kSelEqCap) eq_docs[slot] = d;
        }
      }
    }
    __syncthreads();
    const int n_gt = s_gt;  // = K - need
    const int n_eq = s_eq;
    if (n_eq <= kSelEqCap) {
      // the need lowest ids among the documents at the threshold value
      int n_pow = 1;
      while (n_pow < n_eq) n_pow <<= 1;
      for (int i = n_eq + tid; i < n_pow; i += kSelThreads) eq_docs[i] = 0x7FFFFFFF;
      __syncthreads();
      for (int kk = 2; kk <= n_pow; kk <<= 1) {  // ascending bitonic sort
        for (int jj = kk >> 1; jj > 0; jj >>= 1) {
          for (int i = tid; i < n_pow; i += kSelThreads) {
            const int ixj = i ^ jj;
            if (ixj > i) {
              const int x = eq_docs[i], y = eq_docs[ixj];
              const bool up = (i & kk) == 0;
              if (up ? (x > y) : (x < y)) {
                eq_docs[i] = y;
                eq_docs[ixj] = x;
              }
            }
          }
          __syncthreads();
        }
      }
      for (int i = tid; i < need; i += kSelThreads)
        keys[n_gt + i] = ((unsigned long long)thr << 32) | (0xFFFFFFFFull - (uint32_t)eq_docs[i]);
    } else {
      // very many documents share the threshold value: take the lowest ids in order
      for (int d0 = 0; d0 < n_docs; d0 += kSelThreads) {
        const int taken = s_taken;
        if (taken >= need) break;  // (uniform: read after the barrier below)
        const int d = d0 + tid;
        const bool eq = d < n_docs && sc[d] == thr;
        const uint32_t bal = __ballot_sync(0xffffffffu, eq);
        if (lane == 0) wsum[warp] = __popc(bal);
        __syncthreads();
        int before = 0;
        for (int w = 0; w < warp; ++w) before += wsum[w];
        const int rank = taken + before + __popc(bal & ((1u << lane) - 1u));
        if (eq && rank < need) keys[n_gt + rank] = ((unsigned long long)thr << 32) | (0xFFFFFFFFull - (uint32_t)d);
        __syncthreads();
        if (tid == 0) {
          int tot = 0;
          for (int w = 0; w < kSelThreads / 32; ++w) tot += wsum[w];
          s_taken = taken + tot;
        }
        __syncthreads();
      }
    }
    __syncthreads();
    const int n_pow2 = K <= 1 ? 1 : (1 << (32 - __clz(K - 1)));
    for (int i = K + tid; i < n_pow2; i += kSelThreads) keys[i] = 0ull;
    __syncthreads();
    block_sort_desc(keys, n_pow2);
  }
  for (int r = tid; r < k_sel; r += kSelThreads) {
    o[r] = r < K ? keys[r] : 0ull;
    exact_bits[((int64_t)b * L + l) * k_sel + r] = kOrdNegInf;  // the rescoring max-accumulates here
  }
}

// ---------------------------------------------------------------------------- 2c. exact rescoring
// The exact score of filter candidate r of (b, l) is the maximum over all of the
// document's blocks and all of the query's tokens of
//   s[t][c] = sum_h rho[c][h] * < qt[t][h], k[c][h] >,  rho = 1 / max(||k[c][h]||, 1e-8)
// with k the stored bf16 keys.  The dots run on the tensor cores (mma.sync m16n8k16,
// fp32 accumulate): A = 16 blocks of keys (exact in bf16), B = 8 query tokens carried as
// bf16(qt) plus its bf16 residual (two MMAs, ~16 mantissa bits of qt); each head's dot is
// scaled by rho in fp32 and summed over the heads.
//
// K-dimension order: MMA k-step ks covers head h = ks / 8, and within it thread t's four
// k-indices {2t, 2t+1, 2t+8, 2t+9} are the memory dims 128h + 32t + 4(ks % 8) + {0..3},
// so every thread reads each query token with 16-byte loads; the key tile is written to
// shared memory in the same order (rows of 64 k-steps x 32 bytes, 16-byte chunks XOR-
// swizzled by row for conflict-free ldmatrix).

// grid (x, L, B), 256 threads: the blocks of all K2 candidates of (b, l), laid end to
// end, are cut into tiles of kRsTile blocks; CTA x takes tiles x, x + gridDim.x, ...
// Each tile is staged once (64 KB of keys = 4 MMA row tiles), and every warp reads the
// query rows of its tokens once per head for all four row tiles.  The maximum of every
// (block, token) pair goes to its candidate through shared atomics on ordered bits, then
// one global atomicMax per candidate into exact_bits (set to -inf by the selection).
constexpr int kRsTile = 64;
constexpr int kRsWarps = 8;
constexpr size_t kRsSmem = (size_t)kRsTile * 8 * kD * 2;  // the staged keys

template <int MAXC>
__global__ void __launch_bounds__(kRsWarps * 32) rescore_mma_kernel(
    const __nv_bfloat16* __restrict__ kr_hat, const __nv_bfloat16* __restrict__ q_hi,
    const __nv_bfloat16* __restrict__ q_lo, int L, int64_t C, int n_rows, QueryOffsets qo,
    const int64_t* __restrict__ doc_chunk_off, const unsigned long long* __restrict__ apx, int K2,
    uint32_t* __restrict__ exact_bits, const int32_t* __restrict__ only) {
  constexpr int kRowBytes = 8 * kD * 2;  // 2048
  extern __shared__ __align__(128) uint8_t ktile[];
  __shared__ float rho[kRsTile][8];
  __shared__ int64_t cand_c0[MAXC];
  __shared__ int cand_start[MAXC + 1];
  __shared__ int row_rank[kRsTile];
  __shared__ uint32_t row_best[kRsTile];
  __shared__ uint32_t best[MAXC];
  const int l = blockIdx.y, b = blockIdx.z;
  if (only != nullptr && only[l] == 0) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int64_t o = ((int64_t)b * L + l) * K2;
  // the candidates' block ranges, end to end
  if (warp == 0) {
    int run = 0;
#pragma unroll 4
    for (int i = 0; i < MAXC / 32; ++i) {
      if (32 * i >= K2) break;  // (uniform over the warp)
      const int r = 32 * i + lane;
      int n = 0;
      int64_t c0 = 0;
      if (r < K2) {
        int doc;
        float sc;
        split_key(apx[o + r], &doc, &sc);
        if (doc >= 0) {
          c0 = doc_chunk_off[doc];
          n = (int)(doc_chunk_off[doc + 1] - c0);
        }
        cand_c0[r] = c0;
      }
      int incl = n;  // inclusive prefix over the 32 lanes
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      if (r < K2) cand_start[r] = run + incl - n;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) cand_start[K2] = run;
  }
  for (int r = tid; r < K2; r += blockDim.x) best[r] = 0x007FFFFFu;  // -inf
  __syncthreads();
  const int n_blocks = cand_start[K2];
  const int T = qo.off[b + 1] - qo.off[b];
  const int n_tiles = (T + 7) / 8;
  const int64_t qrow0 = (int64_t)l * n_rows + qo.row0[b];
  const uint32_t kt_base = static_cast<uint32_t>(__cvta_generic_to_shared(ktile));
  const int lrow = (lane & 7) + 8 * ((lane >> 3) & 1), lhalf = lane >> 4;
  for (int f0 = blockIdx.x * kRsTile; f0 < n_blocks; f0 += gridDim.x * kRsTile) {
    if (tid < kRsTile) {
      const int f = f0 + tid;
      int rr = -1;
      if (f < n_blocks) {  // candidate holding flat block f: the last start <= f
        int lo = 0, hi = K2;
        while (hi - lo > 1) {
          const int mid = (lo + hi) >> 1;
          if (cand_start[mid] <= f) lo = mid; else hi = mid;
        }
        rr = lo;
      }
      row_rank[tid] = rr;
      row_best[tid] = 0x007FFFFFu;
    }
    __syncthreads();
    // stage the tile in MMA k order (see above); rows past the end are zero
    for (int i = tid; i < kRsTile * 128; i += blockDim.x) {
      const int row = i >> 7, mp = i & 127;
      const int rr = row_rank[row];
      uint4 w = make_uint4(0u, 0u, 0u, 0u);
      if (rr >= 0) {
        const int64_t c = cand_c0[rr] + (f0 + row - cand_start[rr]);
        w = __ldg(reinterpret_cast<const uint4*>(kr_hat + ((int64_t)l * C + c) * 8 * kD) + mp);
      }
      const int h = mp >> 4, tp = (mp >> 2) & 3, m = mp & 3;
      const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int ks = 8 * h + 2 * m + (j >> 1), half = j & 1;
        const int chunk = (2 * ks + half) ^ (row & 7);
        *reinterpret_cast<uint32_t*>(ktile + row * kRowBytes + chunk * 16 + tp * 4) = wv[j];
      }
    }
    __syncthreads();
    for (int i = tid; i < kRsTile * 8; i += blockDim.x) {  // 1 / ||k|| per (row, head)
      // (summed in the head's logical chunk order, so the value does not depend on the
      // row's place in the tile)
      const int row = i >> 3, h = i & 7;
      const uint4* src = reinterpret_cast<const uint4*>(ktile + row * kRowBytes);
      float ss = 0.f;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const uint4 w = src[(16 * h + j) ^ (row & 7)];
        const float2 f0v = msa::bf16x2_to_float2(w.x), f1 = msa::bf16x2_to_float2(w.y);
        const float2 f2 = msa::bf16x2_to_float2(w.z), f3 = msa::bf16x2_to_float2(w.w);
        ss = fmaf(f0v.x, f0v.x, ss); ss = fmaf(f0v.y, f0v.y, ss); ss = fmaf(f1.x, f1.x, ss); ss = fmaf(f1.y, f1.y, ss);
        ss = fmaf(f2.x, f2.x, ss); ss = fmaf(f2.y, f2.y, ss); ss = fmaf(f3.x, f3.x, ss); ss = fmaf(f3.y, f3.y, ss);
      }
      rho[row][h] = 1.0f / fmaxf(sqrtf(ss), 1e-8f);
    }
    __syncthreads();
    for (int nt = warp; nt < n_tiles; nt += kRsWarps) {
      const int tok = 8 * nt + g;  // this lane's B column (token); padded rows are zero
      const uint4* qh = reinterpret_cast<const uint4*>(q_hi + (qrow0 + tok) * 8 * kD) + 4 * t;
      const uint4* ql = reinterpret_cast<const uint4*>(q_lo + (qrow0 + tok) * 8 * kD) + 4 * t;
      float tot[kRsTile / 16][4];
#pragma unroll
      for (int mt = 0; mt < kRsTile / 16; ++mt) tot[mt][0] = tot[mt][1] = tot[mt][2] = tot[mt][3] = 0.f;
#pragma unroll 1
      for (int h = 0; h < 8; ++h) {
        uint4 xh[4], xl[4];  // dims 128h + 32t .. +32 of token tok
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          xh[m] = __ldg(qh + 16 * h + m);
          xl[m] = __ldg(ql + 16 * h + m);
        }
#pragma unroll
        for (int mt = 0; mt < kRsTile / 16; ++mt) {
          const uint32_t arow = kt_base + (16 * mt + lrow) * kRowBytes;
          float acc_h[4] = {0.f, 0.f, 0.f, 0.f}, acc_l[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const int ks = 8 * h + kk;
            uint32_t a4[4];
            rs_ldsm_x4(arow + (((2 * ks + lhalf) ^ (lrow & 7)) << 4), a4);
            const uint4& vh = xh[kk >> 1];
            const uint4& vl = xl[kk >> 1];
            if (kk & 1) {
              rs_mma(acc_h, a4, vh.z, vh.w);
              rs_mma(acc_l, a4, vl.z, vl.w);
            } else {
              rs_mma(acc_h, a4, vh.x, vh.y);
              rs_mma(acc_l, a4, vl.x, vl.y);
            }
          }
          const float ra = rho[16 * mt + g][h], rb = rho[16 * mt + g + 8][h];
          tot[mt][0] = fmaf(ra, acc_h[0] + acc_l[0], tot[mt][0]);
          tot[mt][1] = fmaf(ra, acc_h[1] + acc_l[1], tot[mt][1]);
          tot[mt][2] = fmaf(rb, acc_h[2] + acc_l[2], tot[mt][2]);
          tot[mt][3] = fmaf(rb, acc_h[3] + acc_l[3], tot[mt][3]);
        }
      }
      // C: rows g / g+8 of each row tile, tokens 8nt + 2t + {0, 1}; the row's maximum
      // over this warp's 8 tokens, then into the row's shared maximum
      const int t0 = 8 * nt + 2 * t;
#pragma unroll
      for (int mt = 0; mt < kRsTile / 16; ++mt) {
        float va = -INFINITY, vb = -INFINITY;
        if (t0 < T) { va = tot[mt][0]; vb = tot[mt][2]; }
        if (t0 + 1 < T) { va = fmaxf(va, tot[mt][1]); vb = fmaxf(vb, tot[mt][3]); }
        va = fmaxf(va, __shfl_xor_sync(0xffffffffu, va, 1));
        va = fmaxf(va, __shfl_xor_sync(0xffffffffu, va, 2));
        vb = fmaxf(vb, __shfl_xor_sync(0xffffffffu, vb, 1));
        vb = fmaxf(vb, __shfl_xor_sync(0xffffffffu, vb, 2));
        if (t == 0) {
          const uint32_t ua = __float_as_uint(va), ub = __float_as_uint(vb);
          atomicMax(&row_best[16 * mt + g], (ua & 0x80000000u) ? ~ua : (ua | 0x80000000u));
          atomicMax(&row_best[16 * mt + g + 8], (ub & 0x80000000u) ? ~ub : (ub | 0x80000000u));
        }
      }
    }
    __syncthreads();
    if (tid < kRsTile && row_rank[tid] >= 0) atomicMax(&best[row_rank[tid]], row_best[tid]);
    __syncthreads();  // before the tile is restaged
  }
  for (int r = tid; r < K2; r += blockDim.x)
    if (best[r] != 0x007FFFFFu) atomicMax(&exact_bits[o + r], best[r]);
}

// The filter error bound of query b in layer l: the largest token bound of the query
// (etok: one bound kind, [L][T_total]); 128-thread reduction, every thread gets it.
__device__ float query_bound(const float* __restrict__ etok, int l, int T_total, const QueryOffsets& qo, int b,
                             float* red) {
  float e = 0.f;
  for (int t = qo.off[b] + threadIdx.x; t < qo.off[b + 1]; t += blockDim.x) e = fmaxf(e, etok[(int64_t)l * T_total + t]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) e = fmaxf(e, __shfl_xor_sync(0xffffffffu, e, o));
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = e;
  __syncthreads();
  e = 0.f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) e = fmaxf(e, red[w]);
  return e;
}

// grid (L, B), 128 threads: final top-k of the K2 exactly rescored candidates.  The
// selection is certified when the k-th exact score beats the best filter score left out
// (the K2-th) by more than the (query, layer)'s filter error bound (query_bound).  An
// uncertified layer is marked in redo_out for the next stage (MSA_DEVERR_UNCERTIFIED when
// there is none).  With only given, layers it does not mark are left as they are.
template <int MAXC>
__global__ void __launch_bounds__(128) select_final_kernel(const unsigned long long* __restrict__ apx,
                                                           const uint32_t* __restrict__ exact_bits, int K2, int k,
                                                           int n_docs, int L, const float* __restrict__ etok,
                                                           int T_total, QueryOffsets qo,
                                                           int32_t* __restrict__ out_ids,
                                                           float* __restrict__ out_scores, int32_t* dev_err,
                                                           int32_t* __restrict__ redo_out,
                                                           const int32_t* __restrict__ only) {
  __shared__ unsigned long long keys[MAXC];
  __shared__ float red[4];
  const int l = blockIdx.x, b = blockIdx.y;
  if (only != nullptr && only[l] == 0) return;
  const int64_t base = ((int64_t)b * L + l) * K2;
  const int n_pow2 = K2 <= 1 ? 1 : (1 << (32 - __clz(K2 - 1)));
  for (int i = threadIdx.x; i < n_pow2; i += blockDim.x) {
    unsigned long long key = 0ull;
    if (i < K2) {
      int doc;
      float s;
      split_key(apx[base + i], &doc, &s);
      if (doc >= 0) key = ((unsigned long long)exact_bits[base + i] << 32) | (0xFFFFFFFFull - (uint32_t)doc);
    }
    keys[i] = key;
  }
  const float err = query_bound(etok, l, T_total, qo, b, red);  // (its barriers order the stores above)
  block_sort_desc(keys, n_pow2);
  for (int r = threadIdx.x; r < k; r += blockDim.x) {
    int doc;
    float s;
    split_key(r < n_pow2 ? keys[r] : 0ull, &doc, &s);
    out_ids[((int64_t)b * L + l) * k + r] = doc;
    out_scores[((int64_t)b * L + l) * k + r] = s;
  }
  if (threadIdx.x == 0 && n_docs > K2 && K2 >= k) {
    int d_left, d_kth;
    float s_left, s_kth;
    split_key(apx[base + K2 - 1], &d_left, &s_left);
    split_key(keys[k - 1], &d_kth, &s_kth);
    if (!(s_kth > s_left + err)) {
      if (redo_out != nullptr) redo_out[l] = 1;
      else msa::set_err(dev_err, MSA_DEVERR_UNCERTIFIED);
    }
  }
}

// ---------------------------------------------------------------------------- layer-aggregated selection
// One selection shared by every layer: documents ranked by the mean over layers of their
// scores.  Scores travel as ordered bits (make_key's high word).
__device__ __forceinline__ float ord_to_float(uint32_t u) {
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u);
}
__device__ __forceinline__ uint32_t float_to_ord(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// agg[b][d] = mean over layers of doc_score[b][l][d] (in layer order; -inf stays -inf).
// gate: run only when gate[0] != 0 (the second pass), or always when null.
__global__ void layer_mean_kernel(const uint32_t* __restrict__ doc_score, int B, int L, int n_docs,
                                  uint32_t* __restrict__ agg, const int32_t* __restrict__ gate) {
  if (gate != nullptr && gate[0] == 0) return;
  const float inv_l = 1.0f / (float)L;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < (int64_t)B * n_docs;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t b = i / n_docs, d = i % n_docs;
    float acc = 0.f;
    for (int l = 0; l < L; ++l) acc += ord_to_float(doc_score[(b * L + l) * n_docs + d]);
    agg[i] = float_to_ord(acc * inv_l);
  }
}

// Every layer of query b takes the shared candidates; their exact scores restart at -inf.
__global__ void replicate_candidates_kernel(const unsigned long long* __restrict__ apx_agg, int B, int L, int K2,
                                            unsigned long long* __restrict__ apx, uint32_t* __restrict__ exact_bits,
                                            const int32_t* __restrict__ gate) {
  if (gate != nullptr && gate[0] == 0) return;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < (int64_t)B * L * K2;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t b = i / ((int64_t)L * K2), r = i % K2;
    apx[i] = apx_agg[b * K2 + r];
    exact_bits[i] = kOrdNegInf;
  }
}

// grid (B): the final top-k of the shared candidates by the mean over layers of their
// exact scores, written to every layer; certified when the k-th exact mean beats the best
// mean filter score left out by more than the mean over layers of the query's bounds plus
// the fp32 rounding of the two means (else the mark on every layer in redo_out, or
// MSA_DEVERR_UNCERTIFIED).
template <int MAXC>
__global__ void __launch_bounds__(128) select_final_mean_kernel(
    const unsigned long long* __restrict__ apx_agg, const uint32_t* __restrict__ exact_bits, int K2, int k, int n_docs,
    int L, const float* __restrict__ etok, int T_total, QueryOffsets qo, int32_t* __restrict__ out_ids,
    float* __restrict__ out_scores, int32_t* dev_err, int32_t* __restrict__ redo_out, const int32_t* __restrict__ gate) {
  __shared__ unsigned long long keys[MAXC];
  __shared__ float red[4];
  if (gate != nullptr && gate[0] == 0) return;
  const int b = blockIdx.x;
  const int n_pow2 = K2 <= 1 ? 1 : (1 << (32 - __clz(K2 - 1)));
  const float inv_l = 1.0f / (float)L;
  for (int i = threadIdx.x; i < n_pow2; i += blockDim.x) {
    unsigned long long key = 0ull;
    if (i < K2) {
      int doc;
      float s;
      split_key(apx_agg[(int64_t)b * K2 + i], &doc, &s);
      if (doc >= 0) {
        float acc = 0.f;
        for (int l = 0; l < L; ++l) acc += ord_to_float(exact_bits[((int64_t)b * L + l) * K2 + i]);
        key = make_key(acc * inv_l, doc);
      }
    }
    keys[i] = key;
  }
  float err = 0.f;
  for (int l = 0; l < L; ++l) err += query_bound(etok, l, T_total, qo, b, red);
  err = err * inv_l * kBoundSlack + (float)(L + 1) * (1.0f / 4194304);  // + (L + 1) 2^-22
  block_sort_desc(keys, n_pow2);
  for (int e = threadIdx.x; e < L * k; e += blockDim.x) {
    const int l = e / k, r = e % k;
    int doc;
    float s;
    split_key(r < n_pow2 ? keys[r] : 0ull, &doc, &s);
    out_ids[((int64_t)b * L + l) * k + r] = doc;
    out_scores[((int64_t)b * L + l) * k + r] = s;
  }
  if (threadIdx.x == 0 && n_docs > K2 && K2 >= k) {
    int d_left, d_kth;
    float s_left, s_kth;
    split_key(apx_agg[(int64_t)b * K2 + K2 - 1], &d_left, &s_left);
    split_key(keys[k - 1], &d_kth, &s_kth);
    if (!(s_kth > s_left + err)) {
      if (redo_out != nullptr)
        for (int l = 0; l < L; ++l) redo_out[l] = 1;
      else
        msa::set_err(dev_err, MSA_DEVERR_UNCERTIFIED);
    }
  }
}

// grid (L, B): exact document scores from the fallback scan's block scores m, as ordered
// bits into doc_score (layers `only` marks).
__global__ void doc_exact_kernel(const float* __restrict__ m, const int64_t* __restrict__ doc_chunk_off, int n_docs,
                                 int64_t C, int L, uint32_t* __restrict__ doc_score, const int32_t* __restrict__ only) {
  const int l = blockIdx.x, b = blockIdx.y;
  if (only[l] == 0) return;
  const float* mb = m + ((int64_t)b * L + l) * C;
  uint32_t* out = doc_score + ((int64_t)b * L + l) * n_docs;
  for (int d = threadIdx.x; d < n_docs; d += blockDim.x) {
    float s = -INFINITY;
    for (int64_t c = doc_chunk_off[d]; c < doc_chunk_off[d + 1]; ++c) s = fmaxf(s, mb[c]);
    out[d] = float_to_ord(s);
  }
}

// grid (B): the keys of query b's final selection (best first) written as ids / scores to
// every layer (gate: only when gate[0] != 0).
__global__ void keys_to_layers_kernel(const unsigned long long* __restrict__ keys, int k, int L,
                                      int32_t* __restrict__ out_ids, float* __restrict__ out_scores,
                                      const int32_t* __restrict__ gate) {
  if (gate != nullptr && gate[0] == 0) return;
  const int b = blockIdx.x;
  for (int e = threadIdx.x; e < L * k; e += blockDim.x) {
    const int l = e / k, r = e % k;
    int doc;
    float s;
    split_key(keys[(int64_t)b * k + r], &doc, &s);
    out_ids[((int64_t)b * L + l) * k + r] = doc;
    out_scores[((int64_t)b * L + l) * k + r] = s;
  }
}

// grid (L, B): keys [B][L][k] (best first) split into ids / scores.
__global__ void keys_to_out_kernel(const unsigned long long* __restrict__ keys, int k, int L,
                                   int32_t* __restrict__ out_ids, float* __restrict__ out_scores) {
  const int64_t o = ((int64_t)blockIdx.y * L + blockIdx.x) * k;
  for (int r = threadIdx.x; r < k; r += blockDim.x) {
    int doc;
    float s;
    split_key(keys[o + r], &doc, &s);
    out_ids[o + r] = doc;
    out_scores[o + r] = s;
  }
}

// Query tokens (all queries of a call) the tensor-core streaming scan takes: up to 4 (its
// B operand holds each token's bf16 value and residual in 8 columns), for 2, 4 or 8 key
// heads (each warp of a pair keeps half of the heads' B fragments in registers).
int scan_mma_tokens(int H) { return (H == 2 || H == 4 || H == 8) ? kScanMmaTokens : 0; }

template <int H>
msa_status launch_scan_mma_h(const __nv_bfloat16* kr, const float* qt, int L, int64_t C, int T_total,
                             const QueryOffsets& qo, float* m, int32_t* dev_err, cudaStream_t s) {
  using K = ScanCfg<H>;
  MSA_CUDA_TRY(cudaFuncSetAttribute(scan_mma_kernel<H>, cudaFuncAttributeMaxDynamicSharedMemorySize, K::kSmem));
  const int64_t tiles = (int64_t)L * ((C + kScanTile - 1) / kScanTile);
  const int grid = (int)(tiles < msa::sm_count() ? tiles : msa::sm_count());
  scan_mma_kernel<H><<<grid, kScanThreads, K::kSmem, s>>>(kr, qt, L, C, T_total, qo, m, dev_err);
  MSA_CUDA_TRY(cudaGetLastError());
  return msa_ok();
}

// The tensor-core streaming scan for H <= 8 key heads and T_total <= scan_mma_tokens(H).
msa_status launch_scan_mma(int H, int T_total, const __nv_bfloat16* kr, const float* qt, int L, int64_t C,
                           const QueryOffsets& qo, float* m, int32_t* dev_err, cudaStream_t s) {
  switch (H) {
    case 2: return launch_scan_mma_h<2>(kr, qt, L, C, T_total, qo, m, dev_err, s);
    case 4: return launch_scan_mma_h<4>(kr, qt, L, C, T_total, qo, m, dev_err, s);
    default: return launch_scan_mma_h<8>(kr, qt, L, C, T_total, qo, m, dev_err, s);
  }
}

}  // namespace

extern "C" msa_status msa_route_topk_workspace_size(int32_t n_layers, int32_t n_queries, int32_t total_q_tokens,
                                                    int32_t n_kv_heads, int64_t n_chunks, int32_t n_docs,
                                                    int32_t top_k, size_t* bytes) {
  if (!bytes || n_layers < 1 || n_queries < 1 || total_q_tokens < n_queries || n_chunks < 0 || n_docs < 0 ||
      top_k < 1 || top_k > kMaxTopK || n_kv_heads < 1 || n_kv_heads > 16)
    return msa_fail(MSA_ERR_INVALID_ARG, "bad sizes");
  *bytes = ws_layout(n_layers, n_queries, total_q_tokens, n_kv_heads, n_chunks, n_docs, top_k).total;
  return msa_ok();
}

extern "C" int32_t msa_route_last_launch_count(void) { return g_launches; }

extern "C" msa_status msa_route_wait_selftest(int64_t wait_ns, int32_t release_first, int32_t* dev_err,
                                              msa_stream_t stream) {
  if (!dev_err) return msa_fail(MSA_ERR_INVALID_ARG, "null pointer");
  if (wait_ns < 1 || wait_ns > 10000000000ll) return msa_fail(MSA_ERR_INVALID_ARG, "wait_ns in [1, 1e10]");
  const int arch = msa::current_device_is_sm100(nullptr);
  if (arch < 0) return msa_fail(MSA_ERR_CUDA, "no CUDA device");
  if (arch == 0) return msa_fail(MSA_ERR_UNSUPPORTED, "device is not sm_100");
  if (route_tc::launch_wait_selftest((unsigned long long)wait_ns, release_first, dev_err,
                                     reinterpret_cast<cudaStream_t>(stream)) != 0)
    return msa_fail(MSA_ERR_CUDA, "self-test launch");
  return msa_ok();
}

extern "C" msa_status msa_route_set_pair_mode(int32_t enabled) {
  g_pair_mode = enabled != 0;
  return msa_ok();
}

extern "C" msa_status msa_route_set_query_profile_events(void* start_event, void* stop_event) {
  g_qprof_start = (start_event && stop_event) ? reinterpret_cast<cudaEvent_t>(start_event) : nullptr;
  g_qprof_stop = (start_event && stop_event) ? reinterpret_cast<cudaEvent_t>(stop_event) : nullptr;
  return msa_ok();
}

extern "C" msa_status msa_route_set_profile_events(void* start_event, void* stop_event) {
  g_prof_start = (start_event && stop_event) ? reinterpret_cast<cudaEvent_t>(start_event) : nullptr;
  g_prof_stop = (start_event && stop_event) ? reinterpret_cast<cudaEvent_t>(stop_event) : nullptr;
  return msa_ok();
}

extern "C" msa_status msa_route_filter_keys(const void* kr_hat, int32_t n_layers, int64_t n_chunks,
                                            int32_t n_kv_heads, int32_t head_dim, void* kr_f8, msa_stream_t stream) {
  if (!kr_hat || !kr_f8) return msa_fail(MSA_ERR_INVALID_ARG, "null pointer");
  if (head_dim != kD) return msa_fail(MSA_ERR_INVALID_ARG, "head_dim must be 128");
  if (n_layers < 1 || n_chunks < 0 || n_kv_heads < 1 || n_kv_heads > 16)
    return msa_fail(MSA_ERR_INVALID_ARG, "bad sizes");
  if (!msa::aligned16(kr_hat) || !msa::aligned16(kr_f8)) return msa_fail(MSA_ERR_INVALID_ARG, "16-byte alignment");
  const int arch = msa::current_device_is_sm100(nullptr);
  if (arch < 0) return msa_fail(MSA_ERR_CUDA, "no CUDA device");
  if (arch == 0) return msa_fail(MSA_ERR_UNSUPPORTED, "device is not sm_100");
  const int64_t n_heads = (int64_t)n_layers * n_chunks * n_kv_heads;
  if (n_heads == 0) return msa_ok();
  int64_t blocks = (n_heads + 31) / 32;  // 256 threads = 32 heads a pass
  const int64_t cap = (int64_t)msa::sm_count() * 16;
  if (blocks > cap) blocks = cap;
  filter_keys_kernel<<<(unsigned)blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const __nv_bfloat16*>(kr_hat), n_heads, reinterpret_cast<uint8_t*>(kr_f8));
  MSA_CUDA_TRY(cudaGetLastError());
  return msa_ok();
}

namespace {
// Where the routing query comes from: a given Q_r (qr), or hidden states projected by the
// router's query weights inside the call (hidden, w).
struct QuerySrc {
  const void* qr;
  msa_dtype q_dtype;
  const void* hidden;
  const void* w;
  int32_t hidden_size;
};

msa_status route_impl(const QuerySrc& src, const int32_t* q_offsets_host, int32_t n_queries, const void* kr_hat,
                      const void* kr_f8, const int64_t* doc_chunk_offsets, int32_t n_docs, int64_t n_chunks,
                      int32_t n_layers, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, int32_t top_k,
                      int32_t* out_ids, float* out_scores, void* workspace, size_t workspace_bytes, int32_t flags,
                      int32_t* dev_err, msa_stream_t stream) {
  g_launches = 0;
  const void* qr = src.qr;
  const msa_dtype q_dtype = src.q_dtype;
  const bool project = src.hidden != nullptr;
  if (!(qr || (project && src.w)) || !q_offsets_host || !kr_hat || !doc_chunk_offsets || !out_ids || !out_scores ||
      !workspace)
    return msa_fail(MSA_ERR_INVALID_ARG, "null pointer");
  if (project && !route_proj::supported(n_q_heads, n_kv_heads, src.hidden_size))
    return msa_fail(MSA_ERR_INVALID_ARG, "projection: hidden_size a multiple of 64, n_q_heads / n_kv_heads in {1,2,4}");
  if (head_dim != kD) return msa_fail(MSA_ERR_INVALID_ARG, "head_dim must be 128");
  if (n_kv_heads != 2 && n_kv_heads != 4 && n_kv_heads != 8 && n_kv_heads != 16)
    return msa_fail(MSA_ERR_INVALID_ARG, "n_kv_heads must be 2, 4, 8 or 16");
  if (n_q_heads < n_kv_heads || n_q_heads % n_kv_heads != 0 || n_q_heads > 64)
    return msa_fail(MSA_ERR_INVALID_ARG, "n_q_heads must be a multiple of n_kv_heads, <= 64");
  if (n_queries < 1 || n_queries > kMaxQueries) return msa_fail(MSA_ERR_INVALID_ARG, "n_queries in [1,256]");
  if (top_k < 1 || top_k > kMaxTopK) return msa_fail(MSA_ERR_INVALID_ARG, "top_k in [1,64]");
  if (n_layers < 1 || n_chunks < 0 || n_docs < 0 || n_docs > kMaxDocs)
    return msa_fail(MSA_ERR_INVALID_ARG, "bad counts (n_docs <= 2^20)");
  if (!project && q_dtype != MSA_F32 && q_dtype != MSA_BF16) return msa_fail(MSA_ERR_UNSUPPORTED, "q_dtype");
  const bool layer_mean = (flags & MSA_ROUTE_LAYER_MEAN) != 0;
  const bool filter_only = (flags & MSA_ROUTE_FILTER_SCORES) != 0;
  flags &= ~(MSA_ROUTE_LAYER_MEAN | MSA_ROUTE_FILTER_SCORES);
  if (flags < MSA_ROUTE_AUTO || flags > MSA_ROUTE_TENSOR_F8) return msa_fail(MSA_ERR_INVALID_ARG, "flags");
  if (layer_mean && flags == MSA_ROUTE_SCAN)
    return msa_fail(MSA_ERR_INVALID_ARG, "MSA_ROUTE_LAYER_MEAN runs on the tensor path, not MSA_ROUTE_SCAN");
  if (filter_only && (layer_mean || (flags != MSA_ROUTE_TENSOR && flags != MSA_ROUTE_TENSOR_F8)))
    return msa_fail(MSA_ERR_INVALID_ARG, "MSA_ROUTE_FILTER_SCORES takes MSA_ROUTE_TENSOR or _TENSOR_F8 alone");
  if (flags == MSA_ROUTE_TENSOR_F8 && !kr_f8)
    return msa_fail(MSA_ERR_INVALID_ARG, "MSA_ROUTE_TENSOR_F8 needs the E4M3 keys (msa_route_filter_keys)");
  if (!msa::aligned16(qr) || !msa::aligned16(kr_hat) || !msa::aligned16(kr_f8) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) || !msa::aligned16(src.hidden) || !msa::aligned16(src.w))
    return msa_fail(MSA_ERR_INVALID_ARG, "alignment: qr/hidden/w/kr_hat/kr_f8 16 B, workspace 256 B");
  QueryOffsets qo;
  qo.n = n_queries;
  if (q_offsets_host[0] != 0) return msa_fail(MSA_ERR_INVALID_ARG, "q_offsets[0] must be 0");
  for (int b = 0; b <= n_queries; ++b) {
    qo.off[b] = q_offsets_host[b];
    if (b > 0 && qo.off[b] <= qo.off[b - 1]) return msa_fail(MSA_ERR_INVALID_ARG, "every query needs >= 1 token");
  }
  const int T_total = qo.off[n_queries];
  route_tc::padded_rows(qo.off, n_queries, qo.row0);
  const int n_rows = route_tc::operand_rows(qo.off, n_queries);
  const WsLayout w = ws_layout(n_layers, n_queries, T_total, n_kv_heads, n_chunks, n_docs, top_k);
  if (workspace_bytes < w.total) return msa_fail(MSA_ERR_CAPACITY, "workspace too small (%zu < %zu)",
                                                 workspace_bytes, w.total);
  if (n_rows > w.n_pad) return msa_fail(MSA_ERR_INVALID_ARG, "internal: operand rows exceed bound");
  const int arch = msa::current_device_is_sm100(nullptr);
  if (arch < 0) return msa_fail(MSA_ERR_CUDA, "no CUDA device");
  if (arch == 0) return msa_fail(MSA_ERR_UNSUPPORTED, "device is not sm_100");

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char* ws = reinterpret_cast<char*>(workspace);
  float* qt_f32 = reinterpret_cast<float*>(ws + w.qt_f32);
  __nv_bfloat16* qt_bf16 = reinterpret_cast<__nv_bfloat16*>(ws + w.qt_bf16);
  float* m = reinterpret_cast<float*>(ws + w.m);
  unsigned long long* cand = reinterpret_cast<unsigned long long*>(ws + w.cand);
  const int H = n_kv_heads;

  // Path: the streaming scan while the query is a handful of tokens (those its tensor-core
  // form takes), the tcgen05 filter GEMM beyond: on the E4M3 keys when the caller has them
  // and the queries average at least kF8MinTokens tokens (below that the E4M3 bound leaves
  // most layers to the bf16 second pass, which then costs more than the bf16 filter alone).
  constexpr int32_t kF8MinTokens = 16;
  int path = flags;
  if (path == MSA_ROUTE_AUTO)
    path = (T_total <= scan_mma_tokens(n_kv_heads) && !layer_mean)
               ? MSA_ROUTE_SCAN
               : (kr_f8 && T_total >= kF8MinTokens * n_queries ? MSA_ROUTE_TENSOR_F8 : MSA_ROUTE_TENSOR);
  if ((path == MSA_ROUTE_TENSOR || path == MSA_ROUTE_TENSOR_F8) && !route_tc::supported(H)) {
    if (flags != MSA_ROUTE_AUTO || layer_mean)
      return msa_fail(MSA_ERR_UNSUPPORTED, "tensor path needs n_kv_heads = 8");
    path = MSA_ROUTE_SCAN;
  }
  const bool tensor = (path == MSA_ROUTE_TENSOR || path == MSA_ROUTE_TENSOR_F8) && n_chunks > 0;
  const bool f8 = tensor && path == MSA_ROUTE_TENSOR_F8;

  uint8_t* qt_f8 = reinterpret_cast<uint8_t*>(ws + w.qt_f8);
  uint32_t* doc_score = reinterpret_cast<uint32_t*>(ws + w.doc_score);
  int32_t* block_doc = reinterpret_cast<int32_t*>(ws + w.block_doc);
  __nv_bfloat16* qt_lo = reinterpret_cast<__nv_bfloat16*>(ws + w.qt_lo);
  // layer masks: redo1 = the E4M3 pass could not certify, redo2 = nor the bf16 pass,
  // redo3 = nor the widened rescoring (exact scan); etok = the per-token filter bounds
  int32_t* redo1 = reinterpret_cast<int32_t*>(ws + w.redo);
  int32_t* redo2 = redo1 + n_layers;
  int32_t* redo3 = redo2 + n_layers;
  float* etok = reinterpret_cast<float*>(ws + w.etok);
  const float* etok_f8 = etok + (size_t)kBoundF8 * n_layers * T_total;
  const float* etok_bf16 = etok + (size_t)kBoundBf16 * n_layers * T_total;
  if (tensor) {
    // operand rows: bf16 (GEMM, and the high half of the exact rescoring), its residual
    // (the low half) and, on the E4M3 path, E4M3
    PadTargets pt;
    pt.buf[0] = reinterpret_cast<uint4*>(qt_bf16);
    pt.words_per_row[0] = H * kD * 2 / 16;
    pt.buf[1] = reinterpret_cast<uint4*>(qt_lo);
    pt.words_per_row[1] = H * kD * 2 / 16;
    pt.buf[2] = f8 ? reinterpret_cast<uint4*>(qt_f8) : nullptr;
    pt.words_per_row[2] = H * kD / 16;
    route_prep_kernel<<<msa::sm_count() * 4, 256, 0, s>>>(pt, n_rows, n_layers, qo, doc_chunk_offsets, n_docs,
                                                           block_doc, doc_score,
                                                           (int64_t)n_queries * n_layers * n_docs, etok,
                                                           (int64_t)2 * n_layers * T_total, redo1, 3 * n_layers);
    ++g_launches;
    MSA_CUDA_TRY(cudaGetLastError());
  }
  if (g_qprof_start) MSA_CUDA_TRY(cudaEventRecord(g_qprof_start, s));
  if (project) {
    // Q_r = hidden W^T on the tensor cores, normalised and group-summed in the epilogue
    route_proj::Args pa;
    pa.hidden = src.hidden;
    pa.w = src.w;
    pa.T = T_total;
    pa.hidden_size = src.hidden_size;
    pa.L = n_layers;
    pa.Hq = n_q_heads;
    pa.H = H;
    pa.n_rows = n_rows;
    pa.lay.n_queries = n_queries;
    for (int b = 0; b <= n_queries; ++b) {
      pa.lay.off[b] = qo.off[b];
      pa.lay.row0[b] = qo.row0[b];
    }
    pa.qt_f32 = tensor ? nullptr : qt_f32;
    pa.qt_bf16 = tensor ? qt_bf16 : nullptr;
    pa.qt_lo = tensor ? qt_lo : nullptr;
    pa.qt_f8 = f8 ? qt_f8 : nullptr;
    pa.etok = tensor ? etok : nullptr;
    pa.dev_err = dev_err;
    const char* why = nullptr;
    if (route_proj::launch(pa, s, &why) != 0)
      return msa_fail(MSA_ERR_CUDA, "router projection: %s", why ? why : "launch failed");
  } else {
    qprep_kernel<<<dim3(T_total, n_layers), 128, 0, s>>>(qr, q_dtype == MSA_BF16, T_total, n_q_heads, H, n_rows, qo,
                                                        tensor ? nullptr : qt_f32, tensor ? qt_bf16 : nullptr,
                                                        tensor ? qt_lo : nullptr, f8 ? qt_f8 : nullptr,
                                                        tensor ? etok : nullptr, n_layers);
  }
  ++g_launches;
  MSA_CUDA_TRY(cudaGetLastError());
  if (g_qprof_stop) MSA_CUDA_TRY(cudaEventRecord(g_qprof_stop, s));

  // tcgen05 filter GEMM over all blocks of the layers `only` marks (all when null)
  auto gemm = [&](bool e4m3, const int32_t* only) -> msa_status {
    route_tc::LaunchArgs a;
    a.kr_hat = e4m3 ? kr_f8 : kr_hat;
    a.qt = e4m3 ? static_cast<const void*>(qt_f8) : static_cast<const void*>(qt_bf16);
    a.f8 = e4m3;
    a.layer_only = only;
    a.L = n_layers;
    a.C = n_chunks;
    a.n_rows = n_rows;
    a.ql.n_queries = n_queries;
    for (int b = 0; b <= n_queries; ++b) a.ql.row0[b] = qo.row0[b];
    for (int b = 0; b < n_queries; ++b) a.ql.len[b] = qo.off[b + 1] - qo.off[b];
    a.block_doc = block_doc;
    a.doc_score = doc_score;
    a.n_docs = n_docs;
    a.dev_err = dev_err;
    a.pair = g_pair_mode;
    int launches = 0;
    const char* why = nullptr;
    if (route_tc::launch(a, s, &launches, &why) != 0)
      return msa_fail(MSA_ERR_CUDA, "tensor-core route: %s", why ? why : "launch failed");
    g_launches += launches;
    return msa_ok();
  };

  if (n_chunks > 0) {
    if (g_prof_start) MSA_CUDA_TRY(cudaEventRecord(g_prof_start, s));
    if (!tensor && T_total <= scan_mma_tokens(H)) {
      const msa_status st = launch_scan_mma(H, T_total, (const __nv_bfloat16*)kr_hat, qt_f32, n_layers, n_chunks,
                                            qo, m, dev_err, s);
      if (st != MSA_OK) return st;
      ++g_launches;
    } else if (!tensor) {
      int64_t warps = (int64_t)n_layers * n_chunks;
      int64_t blocks = (warps + 7) / 8;
      const int64_t cap = (int64_t)msa::sm_count() * 8;
      if (blocks > cap) blocks = cap;
      switch (H) {
        case 2: scan_kernel<1><<<(unsigned)blocks, 256, 0, s>>>((const __nv_bfloat16*)kr_hat, qt_f32, n_layers, n_chunks, T_total, qo, m); break;
        case 4: scan_kernel<2><<<(unsigned)blocks, 256, 0, s>>>((const __nv_bfloat16*)kr_hat, qt_f32, n_layers, n_chunks, T_total, qo, m); break;
        case 8: scan_kernel<4><<<(unsigned)blocks, 256, 0, s>>>((const __nv_bfloat16*)kr_hat, qt_f32, n_layers, n_chunks, T_total, qo, m); break;
        default: scan_kernel<8><<<(unsigned)blocks, 256, 0, s>>>((const __nv_bfloat16*)kr_hat, qt_f32, n_layers, n_chunks, T_total, qo, m); break;
      }
      ++g_launches;
      MSA_CUDA_TRY(cudaGetLastError());
    } else {
      const msa_status st = gemm(f8, nullptr);
      if (st != MSA_OK) return st;
    }
    if (g_prof_stop) MSA_CUDA_TRY(cudaEventRecord(g_prof_stop, s));
  }
  const int per = (n_docs + w.nblk - 1) / w.nblk;
  const int doc_pow2 = pow2_at_least(per > 0 ? per : 1);
  const size_t tk_smem = (size_t)doc_pow2 * sizeof(unsigned long long);
  if (tk_smem > 48 * 1024)
    MSA_CUDA_TRY(cudaFuncSetAttribute(docmax_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tk_smem));
  const int mg_pow2 = pow2_at_least(w.nblk * top_k);
  const size_t mg_smem = (size_t)mg_pow2 * sizeof(unsigned long long);
  if (mg_smem > 48 * 1024)
    MSA_CUDA_TRY(cudaFuncSetAttribute(merge_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)mg_smem));
  // exact per-block scores m -> per-CTA best documents -> top_k (only: the layers marked)
  auto docmax_merge = [&](const int32_t* only) -> msa_status {
    docmax_topk_kernel<<<dim3(w.nblk, n_layers, n_queries), kTopkThreads, tk_smem, s>>>(
        m, doc_chunk_offsets, n_docs, n_chunks, n_layers, top_k, doc_pow2, cand, only);
    ++g_launches;
    MSA_CUDA_TRY(cudaGetLastError());
    merge_topk_kernel<<<dim3(n_layers, n_queries), kTopkThreads, mg_smem, s>>>(cand, w.nblk, n_layers, top_k, mg_pow2,
                                                                            nullptr, out_ids, out_scores, only);
    ++g_launches;
    MSA_CUDA_TRY(cudaGetLastError());
    return msa_ok();
  };
  if (!tensor || n_docs == 0) return docmax_merge(nullptr);  // scan path: exact scores

  unsigned long long* apx = reinterpret_cast<unsigned long long*>(ws + w.apx);
  uint32_t* exact = reinterpret_cast<uint32_t*>(ws + w.exact);
  if (filter_only) {
    // the documents' filter scores themselves (no rescoring): for measuring the filter
    topk_docs_kernel<kMaxCandidates><<<dim3(n_layers, n_queries), kSelThreads, 0, s>>>(doc_score, n_layers, n_docs,
                                                                                      top_k, apx, exact, nullptr);
    ++g_launches;
    MSA_CUDA_TRY(cudaGetLastError());
    keys_to_out_kernel<<<dim3(n_layers, n_queries), 64, 0, s>>>(apx, top_k, n_layers, out_ids, out_scores);
    ++g_launches;
    MSA_CUDA_TRY(cudaGetLastError());
    return msa_ok();
  }

  // tensor path: the GEMM scores are a filter; the K2 best documents by those scores are
  // rescored exactly (fp32 cosines) and the final top-k is taken from the exact scores
  const int K2 = w.k2, KW = w.kw;
  unsigned long long* apx_w = reinterpret_cast<unsigned long long*>(ws + w.apx_w);
  uint32_t* exact_w = reinterpret_cast<uint32_t*>(ws + w.exact_w);
  MSA_CUDA_TRY(cudaFuncSetAttribute(rescore_mma_kernel<kMaxCandidates>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)kRsSmem));
  MSA_CUDA_TRY(cudaFuncSetAttribute(rescore_mma_kernel<kMaxWide>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)kRsSmem));
  // CTAs per (query, layer) of the rescoring: about two per SM in all, at most 8; the
  // widened rescoring (rarely more than a few layers) up to 32
  const int lb = n_layers * n_queries;
  int rs_x = (2 * msa::sm_count() + lb - 1) / lb;
  rs_x = rs_x < 1 ? 1 : (rs_x > 8 ? 8 : rs_x);
  int rs_xw = (4 * msa::sm_count() + lb - 1) / lb;
  rs_xw = rs_xw < 1 ? 1 : (rs_xw > 32 ? 32 : rs_xw);
  // K best documents by filter score -> exact rescoring -> final top-k + certification,
  // on the layers `only` marks; uncertified layers go to redo_out
  auto select = [&](bool wide, const float* eb, int32_t* redo_out, const int32_t* only) -> msa_status {
    if (!wide) {
      topk_docs_kernel<kMaxCandidates><<<dim3(n_layers, n_queries), kSelThreads, 0, s>>>(doc_score, n_layers, n_docs,
                                                                                        K2, apx, exact, only);
      ++g_launches;
      MSA_CUDA_TRY(cudaGetLastError());
      rescore_mma_kernel<kMaxCandidates><<<dim3(rs_x, n_layers, n_queries), kRsWarps * 32, kRsSmem, s>>>(
          (const __nv_bfloat16*)kr_hat, qt_bf16, qt_lo, n_layers, n_chunks, n_rows, qo, doc_chunk_offsets, apx, K2,
          exact, only);
      ++g_launches;
      MSA_CUDA_TRY(cudaGetLastError());
      select_final_kernel<kMaxCandidates><<<dim3(n_layers, n_queries), 128, 0, s>>>(
          apx, exact, K2, top_k, n_docs, n_layers, eb, T_total, qo, out_ids, out_scores, dev_err, redo_out, only);
    } else {
      topk_docs_kernel<kMaxWide><<<dim3(n_layers, n_queries), kSelThreads, 0, s>>>(doc_score, n_layers, n_docs, KW,
                                                                                  apx_w, exact_w, only);
      ++g_launches;
      MSA_CUDA_TRY(cudaGetLastError());
      rescore_mma_kernel<kMaxWide><<<dim3(rs_xw, n_layers, n_queries), kRsWarps * 32, kRsSmem, s>>>(
          (const __nv_bfloat16*)kr_hat, qt_bf16, qt_lo, n_layers, n_chunks, n_rows, qo, doc_chunk_offsets, apx_w, KW,
          exact_w, only);
      ++g_launches;
      MSA_CUDA_TRY(cudaGetLastError());
      select_final_kernel<kMaxWide><<<dim3(n_layers, n_queries), 128, 0, s>>>(
          apx_w, exact_w, KW, top_k, n_docs, n_layers, eb, T_total, qo, out_ids, out_scores, dev_err, redo_out, only);
    }
    ++g_launches;
    MSA_CUDA_TRY(cudaGetLastError());
    return msa_ok();
  };
  // the exact scan of the layers `only` marks, for every query (block scores into m)
  int64_t fb_blocks = ((int64_t)n_layers * n_chunks + 7) / 8;
  if (fb_blocks > (int64_t)msa::sm_count() * 8) fb_blocks = (int64_t)msa::sm_count() * 8;
  if (fb_blocks < 1) fb_blocks = 1;
  auto exact_scan = [&](const int32_t* only) -> msa_status {
    scan_fallback_kernel<<<(unsigned)fb_blocks, 256, 0, s>>>((const __nv_bfloat16*)kr_hat, qt_bf16, qt_lo, n_layers,
                                                             n_chunks, n_rows, qo, m, only);
    ++g_launches;
    MSA_CUDA_TRY(cudaGetLastError());
    return msa_ok();
  };
  msa_status st;
  if (!layer_mean) {
    // E4M3 pass -> (its uncertified layers) bf16 pass -> (uncertified) widened rescoring
    // -> (uncertified) exact scan; each stage's kernels return at once when no layer is
    // marked for them
    if (f8) {
      if ((st = select(false, etok_f8, redo1, nullptr)) != MSA_OK) return st;
      doc_reset_kernel<<<dim3(n_layers, n_queries), 256, 0, s>>>(doc_score, n_layers, n_docs, redo1);
      ++g_launches;
      MSA_CUDA_TRY(cudaGetLastError());
      if ((st = gemm(false, redo1)) != MSA_OK) return st;
      if ((st = select(false, etok_bf16, redo2, redo1)) != MSA_OK) return st;
    } else {
      if ((st = select(false, etok_bf16, redo2, nullptr)) != MSA_OK) return st;
    }
    if (n_docs <= K2) return msa_ok();  // every document was rescored: nothing left to certify
    if ((st = select(true, etok_bf16, redo3, redo2)) != MSA_OK) return st;
    if (n_docs <= KW) return msa_ok();
    if ((st = exact_scan(redo3)) != MSA_OK) return st;
    return docmax_merge(redo3);
  }

  // the layer-aggregated variant: shared candidates from the mean filter scores, exact
  // rescoring in every layer, final top-k on the mean exact scores (gate: the later
  // stages run only when the earlier one marked the layers; every layer is marked alike)
  unsigned long long* apx_agg = reinterpret_cast<unsigned long long*>(ws + w.apx_agg);
  uint32_t* agg = reinterpret_cast<uint32_t*>(ws + w.agg);
  uint32_t* exact_agg = reinterpret_cast<uint32_t*>(ws + w.exact_agg);
  unsigned long long* apx_agg_w = reinterpret_cast<unsigned long long*>(ws + w.apx_agg_w);
  uint32_t* exact_agg_w = reinterpret_cast<uint32_t*>(ws + w.exact_agg_w);
  const int64_t n_agg = (int64_t)n_queries * n_docs;
  const int mean_blocks =
      (int)((n_agg + 255) / 256 < msa::sm_count() * 4 ? (n_agg + 255) / 256 : msa::sm_count() * 4);
  auto layer_mean_scores = [&](const int32_t* gate) -> msa_status {
    layer_mean_kernel<<<mean_blocks > 0 ? mean_blocks : 1, 256, 0, s>>>(doc_score, n_queries, n_layers, n_docs, agg,
                                                                        gate);
    ++g_launches;
    MSA_CUDA_TRY(cudaGetLastError());
    return msa_ok();
  };
  auto select_mean = [&](bool wide, const float* eb, int32_t* redo_out, const int32_t* gate) -> msa_status {
    msa_status r = layer_mean_scores(gate);
    if (r != MSA_OK) return r;
    const int K = wide ? KW : K2;
    unsigned long long* aa = wide ? apx_agg_w : apx_agg;
    unsigned long long* ap = wide ? apx_w : apx;
    uint32_t* ex = wide ? exact_w : exact;
    if (wide)
      topk_docs_kernel<kMaxWide><<<dim3(1, n_queries), kSelThreads, 0, s>>>(agg, 1, n_docs, K, aa, exact_agg_w, gate);
    else
      topk_docs_kernel<kMaxCandidates><<<dim3(1, n_queries), kSelThreads, 0, s>>>(agg, 1, n_docs, K, aa, exact_agg,
                                                                                 gate);
    ++g_launches;
    MSA_CUDA_TRY(cudaGetLastError());
    const int64_t n_rep = (int64_t)n_queries * n_layers * K;
    replicate_candidates_kernel<<<(int)((n_rep + 255) / 256), 256, 0, s>>>(aa, n_queries, n_layers, K, ap, ex, gate);
    ++g_launches;
    MSA_CUDA_TRY(cudaGetLastError());
    if (wide) {
      rescore_mma_kernel<kMaxWide><<<dim3(rs_xw, n_layers, n_queries), kRsWarps * 32, kRsSmem, s>>>(
          (const __nv_bfloat16*)kr_hat, qt_bf16, qt_lo, n_layers, n_chunks, n_rows, qo, doc_chunk_offsets, ap, K, ex,
          gate);
      ++g_launches;
      MSA_CUDA_TRY(cudaGetLastError());
      select_final_mean_kernel<kMaxWide><<<n_queries, 128, 0, s>>>(aa, ex, K, top_k, n_docs, n_layers, eb, T_total, qo,
                                                                  out_ids, out_scores, dev_err, redo_out, gate);
    } else {
      rescore_mma_kernel<kMaxCandidates><<<dim3(rs_x, n_layers, n_queries), kRsWarps * 32, kRsSmem, s>>>(
          (const __nv_bfloat16*)kr_hat, qt_bf16, qt_lo, n_layers, n_chunks, n_rows, qo, doc_chunk_offsets, ap, K, ex,
          gate);
      ++g_launches;
      MSA_CUDA_TRY(cudaGetLastError());
      select_final_mean_kernel<kMaxCandidates><<<n_queries, 128, 0, s>>>(aa, ex, K, top_k, n_docs, n_layers, eb,
                                                                        T_total, qo, out_ids, out_scores, dev_err,
                                                                        redo_out, gate);
    }
    ++g_launches;
    MSA_CUDA_TRY(cudaGetLastError());
    return msa_ok();
  };
  if (f8) {
    if ((st = select_mean(false, etok_f8, redo1, nullptr)) != MSA_OK) return st;
    doc_reset_kernel<<<dim3(n_layers, n_queries), 256, 0, s>>>(doc_score, n_layers, n_docs, redo1);
    ++g_launches;
    MSA_CUDA_TRY(cudaGetLastError());
    if ((st = gemm(false, redo1)) != MSA_OK) return st;
    if ((st = select_mean(false, etok_bf16, redo2, redo1)) != MSA_OK) return st;
  } else {
    if ((st = select_mean(false, etok_bf16, redo2, nullptr)) != MSA_OK) return st;
  }
  if (n_docs <= K2) return msa_ok();
  if ((st = select_mean(true, etok_bf16, redo3, redo2)) != MSA_OK) return st;
  if (n_docs <= KW) return msa_ok();
  // exact scan of every layer, exact document scores, their mean, top_k to every layer
  if ((st = exact_scan(redo3)) != MSA_OK) return st;
  doc_exact_kernel<<<dim3(n_layers, n_queries), 256, 0, s>>>(m, doc_chunk_offsets, n_docs, n_chunks, n_layers,
                                                            doc_score, redo3);
  ++g_launches;
  MSA_CUDA_TRY(cudaGetLastError());
  if ((st = layer_mean_scores(redo3)) != MSA_OK) return st;
  topk_docs_kernel<kMaxCandidates><<<dim3(1, n_queries), kSelThreads, 0, s>>>(agg, 1, n_docs, top_k, apx_agg,
                                                                             exact_agg, redo3);
  ++g_launches;
  MSA_CUDA_TRY(cudaGetLastError());
  keys_to_layers_kernel<<<n_queries, 128, 0, s>>>(apx_agg, top_k, n_layers, out_ids, out_scores, redo3);
  ++g_launches;
  MSA_CUDA_TRY(cudaGetLastError());
  return msa_ok();
}

}  // namespace

extern "C" msa_status msa_route_topk(const void* qr, msa_dtype q_dtype, const int32_t* q_offsets_host,
                                     int32_t n_queries, const void* kr_hat, const void* kr_f8,
                                     const int64_t* doc_chunk_offsets,
                                     int32_t n_docs, int64_t n_chunks, int32_t n_layers, int32_t n_q_heads,
                                     int32_t n_kv_heads, int32_t head_dim, int32_t top_k, int32_t* out_ids,
                                     float* out_scores, void* workspace, size_t workspace_bytes, int32_t flags,
                                     int32_t* dev_err, msa_stream_t stream) {
  const QuerySrc src{qr, q_dtype, nullptr, nullptr, 0};
  return route_impl(src, q_offsets_host, n_queries, kr_hat, kr_f8, doc_chunk_offsets, n_docs, n_chunks, n_layers,
                    n_q_heads, n_kv_heads, head_dim, top_k, out_ids, out_scores, workspace, workspace_bytes, flags,
                    dev_err, stream);
}

extern "C" msa_status msa_route_topk_hidden(const void* hidden, const void* w_router_q, int32_t hidden_size,
                                            const int32_t* q_offsets_host, int32_t n_queries, const void* kr_hat,
                                            const void* kr_f8, const int64_t* doc_chunk_offsets, int32_t n_docs,
                                            int64_t n_chunks, int32_t n_layers, int32_t n_q_heads,
                                            int32_t n_kv_heads, int32_t head_dim, int32_t top_k, int32_t* out_ids,
                                            float* out_scores, void* workspace, size_t workspace_bytes,
                                            int32_t flags, int32_t* dev_err, msa_stream_t stream) {
  if (!hidden || !w_router_q) return msa_fail(MSA_ERR_INVALID_ARG, "null pointer");
  const QuerySrc src{nullptr, MSA_BF16, hidden, w_router_q, hidden_size};
  return route_impl(src, q_offsets_host, n_queries, kr_hat, kr_f8, doc_chunk_offsets, n_docs, n_chunks, n_layers,
                    n_q_heads, n_kv_heads, head_dim, top_k, out_ids, out_scores, workspace, workspace_bytes, flags,
                    dev_err, stream);
}
