// Step 2: routing scores + fused top-k document selection.
//
// Follows "MSA端到端可训练记忆模型完整开源，支持亿级Token上下文", section 架构 (cosine routing,
// mean over heads then max over tokens, Top-k documents) and the MSA paper reading notes,
// section 路由投影器 + Top-k 稀疏注意力 (Top-16 against every document's pooled K_r).
//
// Launch sequence of one call:
//   1. qprep    Q_r -> qt[l][t][g][:] = (1/Hq) sum_{h: h/G = g} Q_r[t][h] / max(||Q_r[t][h]||,1e-8)
//               (fp32 for the scan, bf16 rows padded to the tile for the tensor-core path)
//   2. score    m[b][l][c] = max_{t in b} <qt[l][t], kr_hat[l][c]>   (scan or tcgen05 GEMM)
//   3. docmax   S[doc] = max of m over the document's blocks; per-CTA top-k candidates
//   4. merge    one CTA per (b, l) merges the candidates into the final top-k
// The score matrix s[t][c] only ever lives in registers / TMEM.
#include "common.cuh"
#include "msa_route.h"
#include "route_tc.cuh"

MSA_DEFINE_LAST_ERROR(msa_route_last_error)

namespace {

constexpr int kD = 128;
constexpr int kMaxQueries = 256;
constexpr int kMaxTopK = 64;
constexpr int kTopkThreads = 256;

static thread_local int32_t g_launches = 0;

struct QueryOffsets {
  int32_t n;
  int32_t off[kMaxQueries + 1];
};

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

int topk_blocks(int32_t n_docs) {
  int nb = (n_docs + 511) / 512;
  if (nb < 1) nb = 1;
  if (nb > 256) nb = 256;
  return nb;
}

struct WsLayout {
  size_t qt_f32, qt_bf16, m, cand, total;
  int n_pad;
  int nblk;
};

WsLayout ws_layout(int32_t L, int32_t B, int32_t T_total, int32_t H, int64_t C, int32_t n_docs, int32_t k) {
  WsLayout w;
  w.n_pad = route_tc::padded_tokens(T_total);
  w.nblk = topk_blocks(n_docs);
  size_t o = 0;
  w.qt_f32 = o;
  o += align256((size_t)L * T_total * H * kD * sizeof(float));
  w.qt_bf16 = o;
  o += align256((size_t)L * w.n_pad * H * kD * 2);
  w.m = o;
  o += align256((size_t)B * L * (size_t)C * sizeof(float));
  w.cand = o;
  o += align256((size_t)B * L * w.nblk * k * sizeof(unsigned long long));
  w.total = o;
  return w;
}

// ---------------------------------------------------------------------------- 1. q prep
// grid (T_total, L); block 128 threads.  Hq <= 64.
__global__ void __launch_bounds__(128) qprep_kernel(const void* __restrict__ qr, int q_is_bf16, int T_total,
                                                    int Hq, int H, int n_pad, float* __restrict__ qt_f32,
                                                    __nv_bfloat16* __restrict__ qt_bf16) {
  __shared__ float qhat[64][kD];
  const int t = blockIdx.x, l = blockIdx.y;
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
  for (int e = threadIdx.x; e < H * kD; e += blockDim.x) {
    const int g = e / kD, j = e % kD;
    float acc = 0.f;
    for (int u = 0; u < G; ++u) acc += qhat[g * G + u][j];
    acc *= inv_hq;
    qt_f32[((int64_t)l * T_total + t) * H * kD + e] = acc;
    qt_bf16[((int64_t)l * n_pad + t) * H * kD + e] = __float2bfloat16_rn(acc);
  }
}

// Zero the padding rows [T_total, n_pad) of the bf16 operand of every layer.
__global__ void zero_pad_kernel(__nv_bfloat16* __restrict__ qt_bf16, int T_total, int n_pad, int row, int L) {
  const int64_t per_layer = (int64_t)(n_pad - T_total) * row;
  const int64_t total = per_layer * L;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t l = i / per_layer, r = i % per_layer;
    qt_bf16[(l * n_pad + T_total) * row + r] = __float2bfloat16_rn(0.f);
  }
}

// ---------------------------------------------------------------------------- 2a. scan
// One warp per (layer, block) task.  Lane holds NV 8-element vectors of the key row
// (vectors lane, lane+32, ...), dots them against every query token, reduces across the
// warp and keeps the running max per query.
template <int NV>
__global__ void __launch_bounds__(256) scan_kernel(const __nv_bfloat16* __restrict__ kr_hat,
                                                   const float* __restrict__ qt, int L, int64_t C,
                                                   int T_total, QueryOffsets qo, float* __restrict__ m) {
  constexpr int R = NV * 256;  // elements per key row = H * 128
  const int lane = threadIdx.x % 32;
  const int64_t warp_global = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) / 32;
  const int64_t n_warps = (int64_t)gridDim.x * blockDim.x / 32;
  const int64_t tasks = (int64_t)L * C;
  for (int64_t task = warp_global; task < tasks; task += n_warps) {
    const int l = (int)(task / C);
    const int64_t c = task % C;
    const __nv_bfloat16* row = kr_hat + ((int64_t)l * C + c) * R;
    float kx[NV][8];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(row) + lane + 32 * i);
      float2 f;
      f = msa::bf16x2_to_float2(w.x); kx[i][0] = f.x; kx[i][1] = f.y;
      f = msa::bf16x2_to_float2(w.y); kx[i][2] = f.x; kx[i][3] = f.y;
      f = msa::bf16x2_to_float2(w.z); kx[i][4] = f.x; kx[i][5] = f.y;
      f = msa::bf16x2_to_float2(w.w); kx[i][6] = f.x; kx[i][7] = f.y;
    }
    const float* qbase = qt + (int64_t)l * T_total * R;
    for (int b = 0; b < qo.n; ++b) {
      float best = -INFINITY;
      for (int t = qo.off[b]; t < qo.off[b + 1]; ++t) {
        const float4* qv = reinterpret_cast<const float4*>(qbase + (int64_t)t * R);
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
          const float4 a = __ldg(qv + 2 * (lane + 32 * i));
          const float4 bq = __ldg(qv + 2 * (lane + 32 * i) + 1);
          acc = fmaf(kx[i][0], a.x, acc);
          acc = fmaf(kx[i][1], a.y, acc);
          acc = fmaf(kx[i][2], a.z, acc);
          acc = fmaf(kx[i][3], a.w, acc);
          acc = fmaf(kx[i][4], bq.x, acc);
          acc = fmaf(kx[i][5], bq.y, acc);
          acc = fmaf(kx[i][6], bq.z, acc);
          acc = fmaf(kx[i][7], bq.w, acc);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        best = fmaxf(best, acc);
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

__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long w = __shfl_xor_sync(0xffffffffu, v, o);
    v = w > v ? w : v;
  }
  return v;
}

// Block-wide max of v (all threads get it).
__device__ unsigned long long block_max_u64(unsigned long long v, unsigned long long* red) {
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  v = warp_max_u64(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  unsigned long long r = 0ull;
  for (int i = 0; i < (int)(blockDim.x / 32); ++i) r = red[i] > r ? red[i] : r;
  return r;
}

// Selects the k largest keys of keys[0..n) (smem, destroyed) into out[0..k).
__device__ void block_select_topk(unsigned long long* keys, int n, int k, unsigned long long* out,
                                  unsigned long long* red) {
  for (int r = 0; r < k; ++r) {
    unsigned long long mine = 0ull;
    for (int i = threadIdx.x; i < n; i += blockDim.x) mine = keys[i] > mine ? keys[i] : mine;
    const unsigned long long best = block_max_u64(mine, red);
    if (threadIdx.x == 0) out[r] = best;
    if (best != 0ull)
      for (int i = threadIdx.x; i < n; i += blockDim.x)
        if (keys[i] == best) keys[i] = 0ull;
    __syncthreads();
  }
}

// grid (nblk, L, B): documents [blk*per, (blk+1)*per) of (b, l).
__global__ void __launch_bounds__(kTopkThreads) docmax_topk_kernel(const float* __restrict__ m,
                                                                   const int64_t* __restrict__ doc_chunk_off,
                                                                   int n_docs, int64_t C, int L, int k,
                                                                   unsigned long long* __restrict__ cand) {
  extern __shared__ unsigned long long tk_smem[];
  __shared__ unsigned long long red[kTopkThreads / 32];
  const int blk = blockIdx.x, l = blockIdx.y, b = blockIdx.z;
  const int nblk = gridDim.x;
  const int per = (n_docs + nblk - 1) / nblk;
  const int d0 = blk * per;
  const int d1 = min(n_docs, d0 + per);
  const int n = max(0, d1 - d0);
  const float* mb = m + ((int64_t)b * L + l) * C;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int doc = d0 + i;
    const int64_t c0 = __ldg(doc_chunk_off + doc), c1 = __ldg(doc_chunk_off + doc + 1);
    float s = -INFINITY;
    for (int64_t c = c0; c < c1; ++c) s = fmaxf(s, __ldg(mb + c));
    tk_smem[i] = make_key(s, doc);
  }
  __syncthreads();
  unsigned long long* out = cand + (((int64_t)b * L + l) * nblk + blk) * k;
  block_select_topk(tk_smem, n, k, out, red);
}

// grid (L, B): merges nblk * k candidates.
__global__ void __launch_bounds__(kTopkThreads) merge_topk_kernel(const unsigned long long* __restrict__ cand,
                                                                  int nblk, int L, int k,
                                                                  int32_t* __restrict__ out_ids,
                                                                  float* __restrict__ out_scores) {
  extern __shared__ unsigned long long tk_smem[];
  __shared__ unsigned long long red[kTopkThreads / 32];
  __shared__ unsigned long long best[kMaxTopK];
  const int l = blockIdx.x, b = blockIdx.y;
  const int n = nblk * k;
  const unsigned long long* src = cand + ((int64_t)b * L + l) * n;
  for (int i = threadIdx.x; i < n; i += blockDim.x) tk_smem[i] = src[i];
  __syncthreads();
  block_select_topk(tk_smem, n, k, best, red);
  for (int r = threadIdx.x; r < k; r += blockDim.x) {
    int doc;
    float s;
    split_key(best[r], &doc, &s);
    out_ids[((int64_t)b * L + l) * k + r] = doc;
    out_scores[((int64_t)b * L + l) * k + r] = s;
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

extern "C" msa_status msa_route_topk(const void* qr, msa_dtype q_dtype, const int32_t* q_offsets_host,
                                     int32_t n_queries, const void* kr_hat, const int64_t* doc_chunk_offsets,
                                     int32_t n_docs, int64_t n_chunks, int32_t n_layers, int32_t n_q_heads,
                                     int32_t n_kv_heads, int32_t head_dim, int32_t top_k, int32_t* out_ids,
                                     float* out_scores, void* workspace, size_t workspace_bytes, int32_t flags,
                                     int32_t* dev_err, msa_stream_t stream) {
  g_launches = 0;
  if (!qr || !q_offsets_host || !kr_hat || !doc_chunk_offsets || !out_ids || !out_scores || !workspace)
    return msa_fail(MSA_ERR_INVALID_ARG, "null pointer");
  if (head_dim != kD) return msa_fail(MSA_ERR_INVALID_ARG, "head_dim must be 128");
  if (n_kv_heads != 2 && n_kv_heads != 4 && n_kv_heads != 8 && n_kv_heads != 16)
    return msa_fail(MSA_ERR_INVALID_ARG, "n_kv_heads must be 2, 4, 8 or 16");
  if (n_q_heads < n_kv_heads || n_q_heads % n_kv_heads != 0 || n_q_heads > 64)
    return msa_fail(MSA_ERR_INVALID_ARG, "n_q_heads must be a multiple of n_kv_heads, <= 64");
  if (n_queries < 1 || n_queries > kMaxQueries) return msa_fail(MSA_ERR_INVALID_ARG, "n_queries in [1,256]");
  if (top_k < 1 || top_k > kMaxTopK) return msa_fail(MSA_ERR_INVALID_ARG, "top_k in [1,64]");
  if (n_layers < 1 || n_chunks < 0 || n_docs < 0) return msa_fail(MSA_ERR_INVALID_ARG, "bad counts");
  if (q_dtype != MSA_F32 && q_dtype != MSA_BF16) return msa_fail(MSA_ERR_UNSUPPORTED, "q_dtype");
  if (flags < MSA_ROUTE_AUTO || flags > MSA_ROUTE_TENSOR) return msa_fail(MSA_ERR_INVALID_ARG, "flags");
  if (!msa::aligned16(qr) || !msa::aligned16(kr_hat) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return msa_fail(MSA_ERR_INVALID_ARG, "alignment: qr/kr_hat 16 B, workspace 256 B");
  QueryOffsets qo;
  qo.n = n_queries;
  if (q_offsets_host[0] != 0) return msa_fail(MSA_ERR_INVALID_ARG, "q_offsets[0] must be 0");
  for (int b = 0; b <= n_queries; ++b) {
    qo.off[b] = q_offsets_host[b];
    if (b > 0 && qo.off[b] <= qo.off[b - 1]) return msa_fail(MSA_ERR_INVALID_ARG, "every query needs >= 1 token");
  }
  const int T_total = qo.off[n_queries];
  const WsLayout w = ws_layout(n_layers, n_queries, T_total, n_kv_heads, n_chunks, n_docs, top_k);
  if (workspace_bytes < w.total) return msa_fail(MSA_ERR_CAPACITY, "workspace too small (%zu < %zu)",
                                                 workspace_bytes, w.total);
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

  // Path: the CUDA-core scan while the query is a handful of tokens, tensor cores beyond.
  int path = flags;
  if (path == MSA_ROUTE_AUTO) path = (T_total <= route_tc::kScanMaxTokens) ? MSA_ROUTE_SCAN : MSA_ROUTE_TENSOR;
  if (path == MSA_ROUTE_TENSOR && !route_tc::supported(H)) {
    if (flags == MSA_ROUTE_TENSOR) return msa_fail(MSA_ERR_UNSUPPORTED, "tensor path needs n_kv_heads = 8");
    path = MSA_ROUTE_SCAN;
  }

  qprep_kernel<<<dim3(T_total, n_layers), 128, 0, s>>>(qr, q_dtype == MSA_BF16, T_total, n_q_heads, H, w.n_pad,
                                                      qt_f32, qt_bf16);
  ++g_launches;
  MSA_CUDA_TRY(cudaGetLastError());
  if (n_chunks > 0) {
    if (path == MSA_ROUTE_SCAN) {
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
      if (w.n_pad > T_total) {
        zero_pad_kernel<<<64, 256, 0, s>>>(qt_bf16, T_total, w.n_pad, H * kD, n_layers);
        ++g_launches;
        MSA_CUDA_TRY(cudaGetLastError());
      }
      route_tc::LaunchArgs a;
      a.kr_hat = kr_hat;
      a.qt = qt_bf16;
      a.L = n_layers;
      a.C = n_chunks;
      a.n_pad = w.n_pad;
      a.n_queries = n_queries;
      for (int b = 0; b <= n_queries; ++b) a.q_off[b] = qo.off[b];
      a.m = m;
      int launches = 0;
      const char* why = nullptr;
      if (route_tc::launch(a, s, &launches, &why) != 0)
        return msa_fail(MSA_ERR_CUDA, "tensor-core route: %s", why ? why : "launch failed");
      g_launches += launches;
    }
  }
  const size_t tk_smem = (size_t)((n_docs + w.nblk - 1) / w.nblk) * sizeof(unsigned long long);
  const size_t mg_smem = (size_t)w.nblk * top_k * sizeof(unsigned long long);
  if (tk_smem > 48 * 1024) {
    MSA_CUDA_TRY(cudaFuncSetAttribute(docmax_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tk_smem));
  }
  if (mg_smem > 48 * 1024) {
    MSA_CUDA_TRY(cudaFuncSetAttribute(merge_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)mg_smem));
  }
  docmax_topk_kernel<<<dim3(w.nblk, n_layers, n_queries), kTopkThreads, tk_smem, s>>>(m, doc_chunk_offsets, n_docs,
                                                                                   n_chunks, n_layers, top_k, cand);
  ++g_launches;
  MSA_CUDA_TRY(cudaGetLastError());
  merge_topk_kernel<<<dim3(n_layers, n_queries), kTopkThreads, mg_smem, s>>>(cand, w.nblk, n_layers, top_k, out_ids,
                                                                          out_scores);
  ++g_launches;
  MSA_CUDA_TRY(cudaGetLastError());
  (void)dev_err;
  return msa_ok();
}
