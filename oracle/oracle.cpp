// CPU oracle for the Memory Sparse Attention (MSA) hot path.
//
// TEST INFRASTRUCTURE ONLY.  Plain, slow, single-threaded C++ in double precision that
// states what each step computes.  Only the tests, the package smoke check and the
// benchmark's CPU-baseline leg may load it; the product path never does.  It shares no
// code, header, table or constant with the CUDA path.
//
// Sources (page title, section):
//  [README]  "MSA端到端可训练记忆模型完整开源，支持亿级Token上下文", sections 架构 and 推理流水线
//  [NOTES]   "MSA paper reading notes" (xiaohongrsx.github.io), sections 路由投影器 + Top-k 稀疏注意力,
//            文档级 RoPE, KV 缓存压缩 + Memory Parallel, 推理全流程
//  [DEEP]    "【MSA】突破100M Token 上下文：记忆稀疏注意力架构深度解析", sections 3.3.1, 3.3.2,
//            5.1 (router projectors), 5.2 (forward), 5.3 (map_tensor_to_group_ids)
//
// Readings where the pages are silent or garbled are listed beside each function.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <limits>
#include <utility>
#include <vector>

namespace {

const double kNegInf = -std::numeric_limits<double>::infinity();

// Rotate-half RoPE of one head vector at position pos.  Dimension j < d/2 pairs with
// j + d/2, rotating by angle pos * theta^(-2j/d) ([DEEP] 5.2: apply_rotary_pos_emb with
// cos/sin tables; the pairing is the rotate_half convention of that function).
void rope(const double* x, int32_t d, int64_t pos, double theta, double* out) {
  const int32_t half = d / 2;
  for (int32_t j = 0; j < half; ++j) {
    const double inv_freq = pow(theta, -2.0 * (double)j / (double)d);
    const double ang = (double)pos * inv_freq;
    const double c = cos(ang), s = sin(ang);
    const double a = x[j], b = x[j + half];
    out[j] = a * c - b * s;
    out[j + half] = b * c + a * s;
  }
}

double dot(const double* a, const double* b, int32_t n) {
  double s = 0.0;
  for (int32_t i = 0; i < n; ++i) s += a[i] * b[i];
  return s;
}

double norm2(const double* a, int32_t n) { return sqrt(dot(a, a, n)); }

// Cosine similarity with each vector's norm clamped below at 1e-8, as the eps of
// torch.nn.functional.cosine_similarity ([DEEP] 5.2 uses F.cosine_similarity).
double cosine(const double* a, const double* b, int32_t n) {
  const double na = std::max(norm2(a, n), 1e-8), nb = std::max(norm2(b, n), 1e-8);
  return dot(a, b, n) / (na * nb);
}

}  // namespace

extern "C" {

// RoPE of a single vector (exposed so the tests can pin the convention directly).
void oracle_rope(const double* x, int32_t d, int64_t pos, double theta, double* out) {
  rope(x, d, pos, theta, out);
}

// Number of memory blocks: each document is cut into blocks of `chunk` consecutive
// tokens that never cross a document boundary; a trailing partial block counts
// ([NOTES] 路由投影器: fixed-length blocks of 64; [DEEP] 3.3.2: 64 tokens -> 1 block).
// Writes the per-document block offsets (n_docs + 1 entries) when out is non-NULL.
int64_t oracle_count_chunks(const int64_t* doc_tok_off, int32_t n_docs, int32_t chunk,
                            int64_t* doc_chunk_off) {
  int64_t total = 0;
  if (doc_chunk_off) doc_chunk_off[0] = 0;
  for (int32_t doc = 0; doc < n_docs; ++doc) {
    const int64_t n = doc_tok_off[doc + 1] - doc_tok_off[doc];
    int64_t blocks = 0;
    for (int64_t start = 0; start < n; start += chunk) ++blocks;
    total += blocks;
    if (doc_chunk_off) doc_chunk_off[doc + 1] = total;
  }
  return total;
}

// Step 1, offline block compression ([README] 架构: K/V/K_r compressed by block mean
// pooling; 并行 RoPE: positions restart at 0 in every document; [NOTES] 文档级 RoPE).
// For every document and token i: K'_i = RoPE(K_i, i - doc_start) when rope_k != 0;
// V and K_r are not rotated (reading: RoPE acts on attention keys only, [DEEP] 5.2
// rotates q/k, and the router projections are taken without it).  Every block of the
// document averages its real tokens.  Outputs are [n_chunks][H][d] in double; kr_norm
// is ||mean K_r|| per (block, head) and kr_unit = mean K_r / max(norm, 1e-8).
// Any input or output pointer may be NULL (that stream is skipped).  Returns the block
// count, or -1 if it exceeds cap_chunks.
int64_t oracle_pool(const float* k, const float* v, const float* kr, const int64_t* doc_tok_off,
                    int32_t n_docs, int32_t H, int32_t d, int32_t chunk, double theta, int32_t rope_k,
                    double* k_bar, double* v_bar, double* kr_bar, double* kr_unit, double* kr_norm,
                    int64_t cap_chunks) {
  const int64_t n_chunks = oracle_count_chunks(doc_tok_off, n_docs, chunk, nullptr);
  if (n_chunks > cap_chunks) return -1;
  const int64_t row = (int64_t)H * d;
  std::vector<double> tok(d), rot(d);
  int64_t c = 0;
  for (int32_t doc = 0; doc < n_docs; ++doc) {
    const int64_t t0 = doc_tok_off[doc], t1 = doc_tok_off[doc + 1];
    for (int64_t start = t0; start < t1; start += chunk, ++c) {
      const int64_t end = std::min(start + (int64_t)chunk, t1);
      const double count = (double)(end - start);
      for (int32_t h = 0; h < H; ++h) {
        std::vector<double> sk(d, 0.0), sv(d, 0.0), sr(d, 0.0);
        for (int64_t t = start; t < end; ++t) {
          const int64_t off = t * row + (int64_t)h * d;
          if (k) {
            for (int32_t j = 0; j < d; ++j) tok[j] = k[off + j];
            if (rope_k) {
              rope(tok.data(), d, t - t0, theta, rot.data());
            } else {
              rot = tok;
            }
            for (int32_t j = 0; j < d; ++j) sk[j] += rot[j];
          }
          if (v)
            for (int32_t j = 0; j < d; ++j) sv[j] += v[off + j];
          if (kr)
            for (int32_t j = 0; j < d; ++j) sr[j] += kr[off + j];
        }
        const int64_t o = c * row + (int64_t)h * d;
        for (int32_t j = 0; j < d; ++j) {
          if (k && k_bar) k_bar[o + j] = sk[j] / count;
          if (v && v_bar) v_bar[o + j] = sv[j] / count;
          if (kr && kr_bar) kr_bar[o + j] = sr[j] / count;
        }
        if (kr) {
          std::vector<double> mean(d);
          for (int32_t j = 0; j < d; ++j) mean[j] = sr[j] / count;
          const double nr = norm2(mean.data(), d);
          if (kr_norm) kr_norm[c * H + h] = nr;
          if (kr_unit)
            for (int32_t j = 0; j < d; ++j) kr_unit[o + j] = mean[j] / std::max(nr, 1e-8);
        }
      }
    }
  }
  return n_chunks;
}

// Top-k documents by score, descending; equal scores keep the smaller id first.  With
// fewer than k documents the tail is padded with id -1 and score -inf.
void oracle_topk(const double* doc_score, int32_t n_docs, int32_t k, int32_t* ids, double* scores) {
  std::vector<std::pair<double, int32_t>> all;
  all.reserve(n_docs);
  for (int32_t i = 0; i < n_docs; ++i) all.push_back({doc_score[i], i});
  std::sort(all.begin(), all.end(), [](const std::pair<double, int32_t>& a,
                                       const std::pair<double, int32_t>& b) {
    if (a.first != b.first) return a.first > b.first;
    return a.second < b.second;
  });
  for (int32_t i = 0; i < k; ++i) {
    if (i < n_docs) {
      ids[i] = all[i].second;
      scores[i] = all[i].first;
    } else {
      ids[i] = -1;
      scores[i] = kNegInf;
    }
  }
}

// Step 2, online routing, explicit form, for one routing layer and one query
// ([README] 架构: cosine similarity between router query and pooled router keys, mean
// over attention heads first, then max over query tokens, Top-k documents; [NOTES]
// 路由投影器 + Top-k 稀疏注意力: cosine against every document's pooled K_r, Top-16).
//   s[t][c] = (1/Hq) sum_h cos(Q_r[t][h], Kbar_r[c][h / (Hq/H)])   (GQA pairing)
//   m[c]    = max_t s[t][c]
//   S[doc]  = max over the document's blocks of m[c]   (documents with no block: -inf)
// qr is [T][Hq][d], kr is [C][H][d].  doc_score gets S, chunk_score (optional) gets m.
// Returns 0, or -1 when Hq is not a multiple of H.
int32_t oracle_route_explicit(const float* qr, int32_t T, int32_t Hq, const float* kr, int64_t C,
                              int32_t H, int32_t d, const int64_t* doc_chunk_off, int32_t n_docs,
                              int32_t top_k, double* doc_score, double* chunk_score, int32_t* ids,
                              double* scores) {
  if (H <= 0 || Hq % H != 0) return -1;
  const int32_t G = Hq / H;
  std::vector<double> q((size_t)T * Hq * d), kv((size_t)C * H * d);
  for (size_t i = 0; i < q.size(); ++i) q[i] = qr[i];
  for (size_t i = 0; i < kv.size(); ++i) kv[i] = kr[i];
  std::vector<double> m(C, kNegInf);
  for (int64_t c = 0; c < C; ++c) {
    for (int32_t t = 0; t < T; ++t) {
      double head_sum = 0.0;
      for (int32_t h = 0; h < Hq; ++h) {
        const double* qv = &q[((size_t)t * Hq + h) * d];
        const double* kvv = &kv[((size_t)c * H + h / G) * d];
        head_sum += cosine(qv, kvv, d);
      }
      const double s = head_sum / (double)Hq;
      if (s > m[c]) m[c] = s;
    }
  }
  for (int32_t doc = 0; doc < n_docs; ++doc) {
    double best = kNegInf;
    for (int64_t c = doc_chunk_off[doc]; c < doc_chunk_off[doc + 1]; ++c) best = std::max(best, m[c]);
    doc_score[doc] = best;
  }
  if (chunk_score)
    for (int64_t c = 0; c < C; ++c) chunk_score[c] = m[c];
  oracle_topk(doc_score, n_docs, top_k, ids, scores);
  return 0;
}

// The per-key-head query operand of the grouped form below, on its own:
//   qt[t][g] = (1/Hq) sum over the G query heads h with h / G == g of
//              Q_r[t][h] / max(||Q_r[t][h]||, 1e-8)
// so that s[t][c] = sum_g <qt[t][g], Kbar_r[c][g]> / max(||Kbar_r[c][g]||, 1e-8).  The head
// pairing h -> h / G is [DEEP] 5.1 (router_q: Hq heads, router_k: H heads, GQA).
int32_t oracle_query_sums(const float* qr, int32_t T, int32_t Hq, int32_t H, int32_t d, double* qt) {
  if (H <= 0 || Hq % H != 0) return -1;
  const int32_t G = Hq / H;
  for (size_t i = 0; i < (size_t)T * H * d; ++i) qt[i] = 0.0;
  for (int32_t t = 0; t < T; ++t)
    for (int32_t h = 0; h < Hq; ++h) {
      double n = 0.0;
      for (int32_t j = 0; j < d; ++j) {
        const double x = qr[((size_t)t * Hq + h) * d + j];
        n += x * x;
      }
      const double inv = 1.0 / std::max(sqrt(n), 1e-8);
      for (int32_t j = 0; j < d; ++j)
        qt[((size_t)t * H + h / G) * d + j] += qr[((size_t)t * Hq + h) * d + j] * inv / (double)Hq;
    }
  return 0;
}

// Step 2, grouped form of the same score, written separately (4x fewer products):
//   qhat[t][h] = Q_r[t][h] / max(||Q_r[t][h]||, 1e-8)
//   qsum[t][g] = sum over the G query heads h with h / G == g of qhat[t][h]
//   s[t][c]    = (1/Hq) sum_g <qsum[t][g], Kbar_r[c][g]> / max(||Kbar_r[c][g]||, 1e-8)
// which is the explicit mean of cosines regrouped by key head.  Same outputs.
int32_t oracle_route_grouped(const float* qr, int32_t T, int32_t Hq, const float* kr, int64_t C,
                             int32_t H, int32_t d, const int64_t* doc_chunk_off, int32_t n_docs,
                             int32_t top_k, double* doc_score, double* chunk_score, int32_t* ids,
                             double* scores) {
  if (H <= 0 || Hq % H != 0) return -1;
  const int32_t G = Hq / H;
  std::vector<double> qsum((size_t)T * H * d, 0.0);
  for (int32_t t = 0; t < T; ++t)
    for (int32_t h = 0; h < Hq; ++h) {
      double n = 0.0;
      for (int32_t j = 0; j < d; ++j) {
        const double x = qr[((size_t)t * Hq + h) * d + j];
        n += x * x;
      }
      const double inv = 1.0 / std::max(sqrt(n), 1e-8);
      for (int32_t j = 0; j < d; ++j)
        qsum[((size_t)t * H + h / G) * d + j] += qr[((size_t)t * Hq + h) * d + j] * inv;
    }
  std::vector<double> m(C, kNegInf), key(d);
  for (int64_t c = 0; c < C; ++c) {
    std::vector<double> scaled((size_t)H * d);
    for (int32_t g = 0; g < H; ++g) {
      double n = 0.0;
      for (int32_t j = 0; j < d; ++j) {
        key[j] = kr[((size_t)c * H + g) * d + j];
        n += key[j] * key[j];
      }
      const double inv = 1.0 / std::max(sqrt(n), 1e-8);
      for (int32_t j = 0; j < d; ++j) scaled[(size_t)g * d + j] = key[j] * inv;
    }
    for (int32_t t = 0; t < T; ++t) {
      double acc = 0.0;
      for (int32_t g = 0; g < H; ++g) acc += dot(&qsum[((size_t)t * H + g) * d], &scaled[(size_t)g * d], d);
      const double s = acc / (double)Hq;
      if (s > m[c]) m[c] = s;
    }
  }
  for (int32_t doc = 0; doc < n_docs; ++doc) {
    double best = kNegInf;
    for (int64_t c = doc_chunk_off[doc]; c < doc_chunk_off[doc + 1]; ++c) best = std::max(best, m[c]);
    doc_score[doc] = best;
  }
  if (chunk_score)
    for (int64_t c = 0; c < C; ++c) chunk_score[c] = m[c];
  oracle_topk(doc_score, n_docs, top_k, ids, scores);
  return 0;
}

// Step 3, load only the selected documents' compressed K/V ([README] 推理流水线 step 2
// and 记忆并行: content K/V live in host memory and only the selected documents are
// fetched; [NOTES] KV 缓存压缩: ~19 MB per query for the Top-16).
// host_kv is [L][C][2][H][d] (bf16 bit patterns, K then V per block); ids is
// [B][L][k] (layer l uses its own selection; -1 = empty slot).  For each (b, l) the
// selected documents' blocks are packed in rank order into out [B][L][2][H][M_max][d];
// mem_len[b][l] gets the packed block count.  Rows past mem_len are left untouched.
// Returns 0, -1 on a bad document id, -2 if a selection exceeds M_max blocks.
int32_t oracle_gather(const uint16_t* host_kv, int32_t L, int64_t C, int32_t H, int32_t d,
                      const int64_t* doc_chunk_off, int32_t n_docs, const int32_t* ids, int32_t B,
                      int32_t k, int32_t M_max, uint16_t* out, int32_t* mem_len) {
  const int64_t hd = (int64_t)H * d;
  for (int32_t b = 0; b < B; ++b)
    for (int32_t l = 0; l < L; ++l) {
      int64_t m = 0;
      for (int32_t r = 0; r < k; ++r) {
        const int32_t doc = ids[((int64_t)b * L + l) * k + r];
        if (doc < 0) continue;
        if (doc >= n_docs) return -1;
        for (int64_t c = doc_chunk_off[doc]; c < doc_chunk_off[doc + 1]; ++c, ++m) {
          if (m >= M_max) return -2;
          for (int32_t kvsel = 0; kvsel < 2; ++kvsel)
            for (int32_t h = 0; h < H; ++h) {
              const uint16_t* src = host_kv + (((int64_t)l * C + c) * 2 + kvsel) * hd + (int64_t)h * d;
              uint16_t* dst = out + (((((int64_t)b * L + l) * 2 + kvsel) * H + h) * (int64_t)M_max + m) * d;
              memcpy(dst, src, sizeof(uint16_t) * (size_t)d);
            }
        }
      }
      mem_len[(int64_t)b * L + l] = (int32_t)m;
    }
  return 0;
}

// Step 4, one decode token for one (sequence, layer) ([README] 架构: the selected
// documents' compressed K/V are concatenated with the query's local K/V for
// autoregressive decoding; 全局 RoPE: the query's start index is offset by k so the
// order is background -> query -> generation; [NOTES] 推理全流程: memory KV stays fixed
// while the local KV grows per token).
//   q, k_new get RoPE at position pos (= k offset + local index); v_new does not.
//   The rotated k_new and v_new are appended at local index local_len.
//   Keys = [memory blocks (already rotated document-wise at encode time) ;
//           local keys 0 .. local_len inclusive]; no mask (memory precedes the query).
//   out[h] = softmax(scale * <q_h, K_j>) . V_j over those keys, KV head h / (Hq/H).
// mem_kv is [2][H][M_stride][d] with M valid blocks; local_k/local_v are [H][Lcap][d]
// and are updated.  Returns 0, or -2 when local_len >= Lcap.
int32_t oracle_decode(const float* q, const float* k_new, const float* v_new, const float* mem_kv,
                      int32_t M, int32_t M_stride, double* local_k, double* local_v, int32_t local_len,
                      int32_t Lcap, int64_t pos, double theta, double scale, int32_t Hq, int32_t H,
                      int32_t d, double* out) {
  if (local_len >= Lcap) return -2;
  const int32_t G = Hq / H;
  std::vector<double> x(d), r(d);
  for (int32_t h = 0; h < H; ++h) {
    for (int32_t j = 0; j < d; ++j) x[j] = k_new[(size_t)h * d + j];
    rope(x.data(), d, pos, theta, r.data());
    for (int32_t j = 0; j < d; ++j) {
      local_k[((size_t)h * Lcap + local_len) * d + j] = r[j];
      local_v[((size_t)h * Lcap + local_len) * d + j] = v_new[(size_t)h * d + j];
    }
  }
  const int32_t n_keys = M + local_len + 1;
  std::vector<double> qr(d), logits(n_keys), kj(d);
  for (int32_t hq = 0; hq < Hq; ++hq) {
    const int32_t h = hq / G;
    for (int32_t j = 0; j < d; ++j) x[j] = q[(size_t)hq * d + j];
    rope(x.data(), d, pos, theta, qr.data());
    double mx = kNegInf;
    for (int32_t i = 0; i < n_keys; ++i) {
      if (i < M) {
        for (int32_t j = 0; j < d; ++j) kj[j] = mem_kv[(((size_t)0 * H + h) * M_stride + i) * d + j];
      } else {
        const int32_t li = i - M;
        for (int32_t j = 0; j < d; ++j) kj[j] = local_k[((size_t)h * Lcap + li) * d + j];
      }
      logits[i] = scale * dot(qr.data(), kj.data(), d);
      mx = std::max(mx, logits[i]);
    }
    double denom = 0.0;
    for (int32_t i = 0; i < n_keys; ++i) {
      logits[i] = exp(logits[i] - mx);
      denom += logits[i];
    }
    for (int32_t j = 0; j < d; ++j) {
      double acc = 0.0;
      for (int32_t i = 0; i < n_keys; ++i) {
        const double vj = i < M ? (double)mem_kv[(((size_t)1 * H + h) * M_stride + i) * d + j]
                                : local_v[((size_t)h * Lcap + (i - M)) * d + j];
        acc += logits[i] * vj;
      }
      out[(size_t)hq * d + j] = acc / denom;
    }
  }
  return 0;
}

// Prefill of n_new tokens (a query's own tokens): token i is the decode step at local
// index local_len + i and position pos + i, so it sees the memory and every local key up
// to and including its own.  [README] 推理流水线 step 3 / [NOTES] 推理全流程: the query is
// processed over [selected memory ; local context] before generation continues.
int32_t oracle_prefill(const float* q, const float* k_new, const float* v_new, int32_t n_new, const float* mem_kv,
                       int32_t M, int32_t M_stride, double* local_k, double* local_v, int32_t local_len,
                       int32_t Lcap, int64_t pos, double theta, double scale, int32_t Hq, int32_t H, int32_t d,
                       double* out) {
  for (int32_t i = 0; i < n_new; ++i) {
    const int32_t r = oracle_decode(q + (size_t)i * Hq * d, k_new + (size_t)i * H * d, v_new + (size_t)i * H * d,
                                    mem_kv, M, M_stride, local_k, local_v, local_len + i, Lcap, pos + i, theta,
                                    scale, Hq, H, d, out + (size_t)i * Hq * d);
    if (r != 0) return r;
  }
  return 0;
}

// Router query projection of one routing layer ([DEEP] 5.1: the decoupled router_q_proj
// is a bias-free linear map hidden -> n_q_heads * head_dim; 5.2: it is applied to the
// layer's input hidden states).  out[t][j] = sum_k h[t][k] * w[j][k], in double.
void oracle_router_project(const float* h, int32_t T, int32_t hidden, const float* w, int32_t F, double* out) {
  for (int32_t t = 0; t < T; ++t)
    for (int32_t j = 0; j < F; ++j) {
      double acc = 0.0;
      for (int32_t k = 0; k < hidden; ++k) acc += (double)h[(size_t)t * hidden + k] * (double)w[(size_t)j * hidden + k];
      out[(size_t)t * F + j] = acc;
    }
}

}  // extern "C"
