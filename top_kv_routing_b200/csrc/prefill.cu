// Prefill: a block of new tokens per query (the query's own tokens) through sparse
// attention over [gathered memory blocks ; the local cache up to each token].
//
// Follows "MSA端到端可训练记忆模型完整开源，支持亿级Token上下文", section 推理流水线 (the query is
// processed over the selected documents' compressed K/V joined to its local context;
// 全局 RoPE offset by k) and the MSA paper reading notes, section 推理全流程.  Token i of a
// block is the decode step at local index local_len + i: it sees the whole memory and the
// local keys 0 .. local_len + i.
//
// Three launches: (1) the new keys are rotated (RoPE at position offset + local index),
// rounded to the cache's bf16 and appended with the new values; (2) attention, one
// 128-thread CTA per (query, layer, key head, block of 64/G tokens): warp w owns the MMA
// row tile of (token, query head) rows 16w .. 16w+15 (row r = token r / G, head r % G), so
// every K/V tile serves all G query heads of the key head; K/V tiles of 16 keys stream
// through a 3-stage cp.async ring shared by the CTA; S = QK^T and O += PV on mma.sync
// m16n8k16 bf16 with the rotated query and the softmax weights each split into bf16 +
// bf16 residual (two MMAs, about 16 mantissa bits), online softmax per row in the log2
// domain with the causal limit of each row; (3) local_len += n_new.
#include "attn_common.cuh"
#include "common.cuh"
#include "msa_prefill.h"

MSA_DEFINE_LAST_ERROR(msa_prefill_last_error)

namespace {
using namespace attn;

constexpr int kD = 128;
constexpr int kHalf = 64;
constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kRows = 16 * kWarps;  // (token, head) rows per CTA
constexpr int kTileKeys = 16;
constexpr int kStages = 3;
constexpr int kRowBytes = kD * 2;
constexpr int kStageBytes = 2 * kTileKeys * kRowBytes;  // 16 K rows then 16 V rows
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ void angle_cs(double pos, int j, double log2_theta, float* c, float* s) {
  double u = pos * (exp2(-2.0 * (double)j / (double)kD * log2_theta) * 0.31830988618379067154);  // angle / pi
  u -= 2.0 * rint(0.5 * u);                                                                   // in [-1, 1]
  sincospif((float)u, s, c);
}

// (1) grid (n_new, H, B * L), 128 threads: rotate, round and append token i's key and value.
__global__ void __launch_bounds__(kThreads) prefill_append_kernel(
    const __nv_bfloat16* __restrict__ k_new, const __nv_bfloat16* __restrict__ v_new, int T, int L, int H,
    __nv_bfloat16* __restrict__ local_k, __nv_bfloat16* __restrict__ local_v, const int32_t* __restrict__ local_len,
    int cap, const int32_t* __restrict__ mem_len, int M_max, int pos_off, double log2_theta, int32_t* dev_err) {
  const int i = blockIdx.x, h = blockIdx.y;
  const int64_t bl = blockIdx.z;
  const int b = (int)(bl / L);
  const int tid = threadIdx.x;
  const int len = local_len[b];
  if (len < 0 || len + T > cap) {
    if (i == 0 && h == 0 && (bl % L) == 0 && tid == 0) msa::set_err(dev_err, MSA_DEVERR_LOCAL_FULL);
    return;
  }
  if (i == 0 && h == 0 && tid == 0 && mem_len[bl] > M_max) msa::set_err(dev_err, MSA_DEVERR_CAPACITY);
  const int64_t src = ((bl * T + i) * H + h) * kD;
  const int64_t dst = ((bl * H + h) * (int64_t)cap + len + i) * kD;
  if (tid < kHalf) {
    float c, s;
    angle_cs((double)pos_off + (double)(len + i), tid, log2_theta, &c, &s);
    const float a = __bfloat162float(k_new[src + tid]), bb = __bfloat162float(k_new[src + tid + kHalf]);
    local_k[dst + tid] = __float2bfloat16_rn(a * c - bb * s);
    local_k[dst + tid + kHalf] = __float2bfloat16_rn(bb * c + a * s);
  }
  local_v[dst + tid] = v_new[src + tid];
}

// (3) one thread per query: the length advances by the block (unless the cache was full).
__global__ void prefill_advance_kernel(int32_t* local_len, int B, int T, int cap) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B && local_len[b] >= 0 && local_len[b] + T <= cap) local_len[b] += T;
}

// (2) attention
template <int G>
__global__ void __launch_bounds__(kThreads, 3) prefill_attn_kernel(
    const __nv_bfloat16* __restrict__ q, int T, int L, int H, const __nv_bfloat16* __restrict__ local_k,
    const __nv_bfloat16* __restrict__ local_v, const int32_t* __restrict__ local_len, int cap,
    const __nv_bfloat16* __restrict__ mem_kv, const int32_t* __restrict__ mem_len, int M_max, int pos_off,
    double log2_theta, float qscale, __nv_bfloat16* __restrict__ out) {
  constexpr int kTok = kRows / G;  // tokens per CTA
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* ring = smem;                                                      // kStages x 8 KB
  float (*qs)[kD] = reinterpret_cast<float (*)[kD]>(smem + kStages * kStageBytes);  // [kRows][128]
  float2 (*tcs)[kHalf] = reinterpret_cast<float2 (*)[kHalf]>(smem + kStages * kStageBytes + kRows * kD * 4);
  const int h = blockIdx.y;
  const int64_t bl = blockIdx.z;
  const int b = (int)(bl / L);
  const int tok0 = blockIdx.x * kTok;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int Hq = H * G;
  const int len = local_len[b];
  if (len < 0 || len + T > cap) return;  // (the append kernel has set MSA_DEVERR_LOCAL_FULL)
  int M = mem_len[bl];
  M = M < 0 ? 0 : (M > M_max ? M_max : M);
  const int tok_last = min(T, tok0 + kTok) - 1;

  // ---- key tiles: memory, then local rows 0 .. len + tok_last (the new rows included)
  const int nt_mem = (M + kTileKeys - 1) / kTileKeys;
  const int n_local = len + tok_last + 1;
  const int nt = nt_mem + (n_local + kTileKeys - 1) / kTileKeys;
  const __nv_bfloat16* memk = mem_kv + ((bl * 2 + 0) * H + h) * (int64_t)M_max * kD;
  const __nv_bfloat16* memv = mem_kv + ((bl * 2 + 1) * H + h) * (int64_t)M_max * kD;
  const __nv_bfloat16* lock = local_k + (bl * H + h) * (int64_t)cap * kD;
  const __nv_bfloat16* locv = local_v + (bl * H + h) * (int64_t)cap * kD;
  const uint32_t ring_u32 = smem_u32(ring);
  auto issue = [&](int i) {
    const __nv_bfloat16 *kp, *vp;
    int n_copy;
    if (i < nt_mem) {
      kp = memk + (int64_t)i * kTileKeys * kD;
      vp = memv + (int64_t)i * kTileKeys * kD;
      n_copy = min(kTileKeys, M - i * kTileKeys);
    } else {
      const int r0 = (i - nt_mem) * kTileKeys;
      kp = lock + (int64_t)r0 * kD;
      vp = locv + (int64_t)r0 * kD;
      n_copy = min(kTileKeys, n_local - r0);
    }
    const uint32_t st = ring_u32 + (i % kStages) * kStageBytes;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = tid + kThreads * j;  // 512 chunks of 16 bytes
      const int row = c >> 4, chunk = c & 15;  // rows 0..15 K, 16..31 V
      const int key = row & 15;
      const bool ok = key < n_copy;
      const __nv_bfloat16* src = (row < kTileKeys ? kp : vp) + (ok ? key * kD + chunk * 8 : 0);
      cp_async16(st + row * kRowBytes + ((chunk ^ (row & 7)) << 4), src, ok ? 16u : 0u);
    }
  };
  issue(0);
  cp_async_commit();
  if (nt > 1) issue(1);
  cp_async_commit();

  // ---- rotated, scaled queries of the CTA's rows (rows past the block are zero)
  for (int e = tid; e < kTok * kHalf; e += kThreads) {
    const int tl = e / kHalf, j = e % kHalf;
    float c = 1.f, s = 0.f;
    if (tok0 + tl < T) angle_cs((double)pos_off + (double)(len + tok0 + tl), j, log2_theta, &c, &s);
    tcs[tl][j] = make_float2(c, s);
  }
  __syncthreads();
  for (int e = tid; e < kRows * kHalf; e += kThreads) {
    const int r = e / kHalf, j = e % kHalf;
    const int tl = r / G, hd = r % G;
    float r0 = 0.f, r1 = 0.f;
    if (tok0 + tl < T) {
      const __nv_bfloat16* qp = q + ((bl * T + tok0 + tl) * Hq + (int64_t)h * G + hd) * kD;
      const float a = __bfloat162float(qp[j]), bb = __bfloat162float(qp[j + kHalf]);
      const float2 cs = tcs[tl][j];
      r0 = (a * cs.x - bb * cs.y) * qscale;
      r1 = (bb * cs.x + a * cs.y) * qscale;
    }
    qs[r][j] = r0;
    qs[r][j + kHalf] = r1;
  }
  __syncthreads();
  // this warp's rows: ra = 16 warp + g, rb = ra + 8; fragments of bf16(q') and its residual
  const int ra = 16 * warp + g, rb = ra + 8;
  uint32_t qh[8][4], ql[8][4];
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const float2 x0 = *reinterpret_cast<const float2*>(&qs[ra][16 * ks + 2 * t]);
    const float2 x1 = *reinterpret_cast<const float2*>(&qs[rb][16 * ks + 2 * t]);
    const float2 x2 = *reinterpret_cast<const float2*>(&qs[ra][16 * ks + 8 + 2 * t]);
    const float2 x3 = *reinterpret_cast<const float2*>(&qs[rb][16 * ks + 8 + 2 * t]);
    split_pair(x0.x, x0.y, qh[ks][0], ql[ks][0]);
    split_pair(x1.x, x1.y, qh[ks][1], ql[ks][1]);
    split_pair(x2.x, x2.y, qh[ks][2], ql[ks][2]);
    split_pair(x3.x, x3.y, qh[ks][3], ql[ks][3]);
  }
  // causal limits (local index) of the two rows; rows past the block see every key
  const int pa_lim = len + min(tok0 + ra / G, T - 1);
  const int pb_lim = len + min(tok0 + rb / G, T - 1);

  float o[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float ma = -INFINITY, mb = -INFINITY, la = 0.f, lb = 0.f;
  for (int i = 0; i < nt; ++i) {
    cp_async_wait<1>();  // tile i has landed (only tile i + 1 may still be in flight)
    __syncthreads();     // ... for every thread; and tile i - 1's stage is free again
    if (i + 2 < nt) issue(i + 2);
    cp_async_commit();
    const uint32_t st = ring_u32 + (i % kStages) * kStageBytes;
    const bool local = i >= nt_mem;
    const int k0 = local ? (i - nt_mem) * kTileKeys : i * kTileKeys;  // first key of the tile

    float s[2][2][4];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
#pragma unroll
      for (int u = 0; u < 2; ++u) s[j][u][0] = s[j][u][1] = s[j][u][2] = s[j][u][3] = 0.f;
    }
    // s[j][0] accumulates the bf16(q') products of key group j, s[j][1] the residual's;
    // dependent MMAs are issued four apart
#pragma unroll
    for (int ks2 = 0; ks2 < 4; ++ks2) {
      uint32_t b[2][4];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int row = 8 * j + (lane & 7);
        const int chunk = 4 * ks2 + (lane >> 3);
        ldsm_x4(st + row * kRowBytes + ((chunk ^ (row & 7)) << 4), b[j][0], b[j][1], b[j][2], b[j][3]);
      }
#pragma unroll
      for (int e = 0; e < 2; ++e) {
#pragma unroll
        for (int j = 0; j < 2; ++j) mma_bf16(s[j][0], qh[2 * ks2 + e], b[j][2 * e], b[j][2 * e + 1]);
#pragma unroll
        for (int j = 0; j < 2; ++j) mma_bf16(s[j][1], ql[2 * ks2 + e], b[j][2 * e], b[j][2 * e + 1]);
      }
    }
    // scores of rows ra (c0, c1) and rb (c2, c3) for keys 8j + 2t + e
    float sa[4], sb[4];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int key = k0 + 8 * j + 2 * t + e;
        const bool ok_a = local ? key <= pa_lim : key < M;
        const bool ok_b = local ? key <= pb_lim : key < M;
        sa[2 * j + e] = ok_a ? s[j][0][e] + s[j][1][e] : -INFINITY;
        sb[2 * j + e] = ok_b ? s[j][0][2 + e] + s[j][1][2 + e] : -INFINITY;
      }
    }
    float xa = fmaxf(fmaxf(sa[0], sa[1]), fmaxf(sa[2], sa[3]));
    float xb = fmaxf(fmaxf(sb[0], sb[1]), fmaxf(sb[2], sb[3]));
    xa = fmaxf(xa, __shfl_xor_sync(0xffffffffu, xa, 1));
    xa = fmaxf(xa, __shfl_xor_sync(0xffffffffu, xa, 2));
    xb = fmaxf(xb, __shfl_xor_sync(0xffffffffu, xb, 1));
    xb = fmaxf(xb, __shfl_xor_sync(0xffffffffu, xb, 2));
    // (every row has a valid key in the first tile it sees, so the maxima stay finite)
    const float na = fmaxf(ma, xa), nb = fmaxf(mb, xb);
    const float aa = exp2f(ma - na), ab = exp2f(mb - nb);  // 0 while the maximum is still -inf
    float pa[4], pb[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      pa[u] = exp2f(sa[u] - na);
      pb[u] = exp2f(sb[u] - nb);
    }
    la = fmaf(la, aa, (pa[0] + pa[1]) + (pa[2] + pa[3]));
    lb = fmaf(lb, ab, (pb[0] + pb[1]) + (pb[2] + pb[3]));
    ma = na;
    mb = nb;
    if (__any_sync(0xffffffffu, aa != 1.f || ab != 1.f)) {
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        o[n][0] *= aa; o[n][1] *= aa; o[n][2] *= ab; o[n][3] *= ab;
      }
    }
    // P as A fragments (row ra: a0 keys 2t.., a2 keys 8+2t..; row rb: a1, a3), bf16 + residual
    uint32_t ph[4], pl[4];
    split_pair(pa[0], pa[1], ph[0], pl[0]);
    split_pair(pb[0], pb[1], ph[1], pl[1]);
    split_pair(pa[2], pa[3], ph[2], pl[2]);
    split_pair(pb[2], pb[3], ph[3], pl[3]);
    const int vkey = (lane & 7) + 8 * ((lane >> 3) & 1);
    const int vrow = kTileKeys + vkey;
#pragma unroll
    for (int i4 = 0; i4 < 4; ++i4) {  // 32 output dims per round, dependent MMAs four apart
      uint32_t v[2][4];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int chunk = 4 * i4 + 2 * u + (lane >> 4);
        ldsm_x4_t(st + vrow * kRowBytes + ((chunk ^ (vrow & 7)) << 4), v[u][0], v[u][1], v[u][2], v[u][3]);
      }
#pragma unroll
      for (int n = 0; n < 4; ++n) mma_bf16(o[4 * i4 + n], ph, v[n >> 1][2 * (n & 1)], v[n >> 1][2 * (n & 1) + 1]);
#pragma unroll
      for (int n = 0; n < 4; ++n) mma_bf16(o[4 * i4 + n], pl, v[n >> 1][2 * (n & 1)], v[n >> 1][2 * (n & 1) + 1]);
    }
  }
  cp_async_wait<0>();
  la += __shfl_xor_sync(0xffffffffu, la, 1);
  la += __shfl_xor_sync(0xffffffffu, la, 2);
  lb += __shfl_xor_sync(0xffffffffu, lb, 1);
  lb += __shfl_xor_sync(0xffffffffu, lb, 2);
  const float inv_a = 1.0f / la, inv_b = 1.0f / lb;
  const int ta = tok0 + ra / G, tb = tok0 + rb / G;
  __nv_bfloat16* oa = out + ((bl * T + ta) * Hq + (int64_t)h * G + ra % G) * kD;
  __nv_bfloat16* ob = out + ((bl * T + tb) * Hq + (int64_t)h * G + rb % G) * kD;
#pragma unroll
  for (int n = 0; n < 16; ++n) {
    const int d = 8 * n + 2 * t;
    if (ta < T)
      *reinterpret_cast<uint32_t*>(oa + d) =
          pack_bf16(__float2bfloat16_rn(o[n][0] * inv_a), __float2bfloat16_rn(o[n][1] * inv_a));
    if (tb < T)
      *reinterpret_cast<uint32_t*>(ob + d) =
          pack_bf16(__float2bfloat16_rn(o[n][2] * inv_b), __float2bfloat16_rn(o[n][3] * inv_b));
  }
}

template <int G>
size_t attn_smem() {
  return (size_t)kStages * kStageBytes + (size_t)kRows * kD * 4 + (size_t)(kRows / G) * kHalf * sizeof(float2);
}

}  // namespace

extern "C" msa_status msa_sparse_prefill(const void* q, const void* k_new, const void* v_new, int32_t n_new,
                                         int32_t n_queries, int32_t n_layers, int32_t n_q_heads, int32_t n_kv_heads,
                                         int32_t head_dim, void* local_k, void* local_v, int32_t* local_len,
                                         int32_t local_cap, const void* mem_kv, const int32_t* mem_len,
                                         int32_t max_mem_chunks, int32_t rope_pos_offset, float rope_theta,
                                         float softmax_scale, void* out, int32_t* dev_err, msa_stream_t stream) {
  if (!q || !k_new || !v_new || !local_k || !local_v || !local_len || !mem_kv || !mem_len || !out)
    return msa_fail(MSA_ERR_INVALID_ARG, "null pointer");
  if (head_dim != kD) return msa_fail(MSA_ERR_INVALID_ARG, "head_dim must be 128");
  if (n_kv_heads < 1 || n_kv_heads > 16 || n_q_heads % n_kv_heads != 0)
    return msa_fail(MSA_ERR_INVALID_ARG, "n_q_heads must be a multiple of n_kv_heads (<= 16)");
  const int G = n_q_heads / n_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return msa_fail(MSA_ERR_INVALID_ARG, "n_q_heads / n_kv_heads in {1,2,4,8}");
  if (n_new < 1 || n_queries < 1 || n_layers < 1 || (int64_t)n_queries * n_layers > 65535 || local_cap < 1 ||
      max_mem_chunks < 1)
    return msa_fail(MSA_ERR_INVALID_ARG, "bad counts (n_queries * n_layers <= 65535)");
  if (!(rope_theta > 1.0f)) return msa_fail(MSA_ERR_INVALID_ARG, "rope_theta must be > 1");
  if (!msa::aligned16(q) || !msa::aligned16(mem_kv) || !msa::aligned16(local_k) || !msa::aligned16(local_v) ||
      !msa::aligned16(out))
    return msa_fail(MSA_ERR_INVALID_ARG, "16-byte alignment (q, mem_kv, local_k, local_v, out)");
  const int arch = msa::current_device_is_sm100(nullptr);
  if (arch < 0) return msa_fail(MSA_ERR_CUDA, "no CUDA device");
  if (arch == 0) return msa_fail(MSA_ERR_UNSUPPORTED, "device is not sm_100");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const double log2_theta = log2((double)rope_theta);
  const float qscale = softmax_scale * kLog2e;
  const int BL = n_queries * n_layers;
  prefill_append_kernel<<<dim3(n_new, n_kv_heads, BL), kThreads, 0, s>>>(
      (const __nv_bfloat16*)k_new, (const __nv_bfloat16*)v_new, n_new, n_layers, n_kv_heads, (__nv_bfloat16*)local_k,
      (__nv_bfloat16*)local_v, local_len, local_cap, mem_len, max_mem_chunks, rope_pos_offset, log2_theta, dev_err);
  MSA_CUDA_TRY(cudaGetLastError());
#define MSA_PREFILL_LAUNCH(GG)                                                                                    \
  {                                                                                                               \
    const size_t smem = attn_smem<GG>();                                                                          \
    MSA_CUDA_TRY(cudaFuncSetAttribute(prefill_attn_kernel<GG>, cudaFuncAttributeMaxDynamicSharedMemorySize,      \
                                      (int)smem));                                                                \
    const int blocks = (n_new + kRows / GG - 1) / (kRows / GG);                                                   \
    prefill_attn_kernel<GG><<<dim3(blocks, n_kv_heads, BL), kThreads, smem, s>>>(                                 \
        (const __nv_bfloat16*)q, n_new, n_layers, n_kv_heads, (const __nv_bfloat16*)local_k,                     \
        (const __nv_bfloat16*)local_v, local_len, local_cap, (const __nv_bfloat16*)mem_kv, mem_len,              \
        max_mem_chunks, rope_pos_offset, log2_theta, qscale, (__nv_bfloat16*)out);                               \
  }
  switch (G) {
    case 1: MSA_PREFILL_LAUNCH(1); break;
    case 2: MSA_PREFILL_LAUNCH(2); break;
    case 4: MSA_PREFILL_LAUNCH(4); break;
    default: MSA_PREFILL_LAUNCH(8); break;
  }
#undef MSA_PREFILL_LAUNCH
  MSA_CUDA_TRY(cudaGetLastError());
  prefill_advance_kernel<<<(n_queries + 127) / 128, 128, 0, s>>>(local_len, n_queries, n_new, local_cap);
  MSA_CUDA_TRY(cudaGetLastError());
  return msa_ok();
}
