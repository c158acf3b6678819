// Tensor-core (tcgen05) routing score path: interface used by route.cu.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace route_tc {

constexpr int kMaxQueries = 256;
// Query lengths up to this many tokens (all queries of a call together) use the scan.
constexpr int kScanMaxTokens = 8;
// Every query's tokens start on a multiple of this many operand rows, so that each
// 32-column slice of the accumulator belongs to a single query.
constexpr int kQueryAlign = 32;
// N tile of the MMA (columns = query tokens); the padded token count is a multiple.
constexpr int kMaxTileN = 256;

// Padded operand row of every query: row0[b] = sum over b' < b of round_up(T_b', 32).
inline int padded_rows(const int* q_off, int n_queries, int* row0) {
  int r = 0;
  for (int b = 0; b < n_queries; ++b) {
    if (row0) row0[b] = r;
    const int t = q_off[b + 1] - q_off[b];
    r += (t + kQueryAlign - 1) / kQueryAlign * kQueryAlign;
  }
  if (row0) row0[n_queries] = r;
  return r;
}

// N tile for a padded token count: the smallest of 64/128/256 covering it, else 256.
inline int tile_n(int rows) { return rows <= 64 ? 64 : (rows <= 128 ? 128 : 256); }

// Rows of the bf16 query operand per layer: padded rows rounded up to the N tile.
inline int operand_rows(const int* q_off, int n_queries) {
  const int r = padded_rows(q_off, n_queries, nullptr);
  const int bn = tile_n(r);
  return (r + bn - 1) / bn * bn;
}

bool supported(int n_kv_heads);

// E4M3 operand scales: unit keys are stored x 2^8 (|x| <= 256), the query operand rows
// (each element at most 1 / n_kv_heads = 1/8 in magnitude) x 2^11 (|x| <= 256); both stay
// inside the E4M3 range (448) and the GEMM result is rescaled by 2^-19.
constexpr float kF8KeyScale = 256.0f;
constexpr float kF8QueryScale = 2048.0f;
constexpr float kF8ScoreScale = 1.0f / (256.0f * 2048.0f);

struct QueryLayout {
  int n_queries;
  int row0[kMaxQueries + 1];   // first operand row of each query (aligned to 32)
  int len[kMaxQueries];        // tokens of each query
};

struct LaunchArgs {
  const void* kr_hat;  // bf16 [L][C][8][128], or E4M3 x kF8KeyScale when f8
  const void* qt;      // bf16 [L][n_rows][8][128] (E4M3 x kF8QueryScale when f8), padding rows zero
  int L;
  int64_t C;
  int n_rows;          // operand rows per layer (multiple of the N tile)
  QueryLayout ql;
  const int32_t* block_doc;  // [C] document of each block
  uint32_t* doc_score;       // [B][L][n_docs] ordered bits of the filter score, max-accumulated
  int n_docs;
  int32_t* dev_err;
  bool pair;           // M=256 tiles on CTA pairs (cta_group::2) for N tiles of 128 / 256
  bool f8;             // E4M3 operands (kind::f8f6f4)
  const int32_t* layer_only = nullptr;  // DEVICE [L]: when given, layers marked 0 are skipped
};

// Enqueues the score kernel; returns 0 on success (launches += kernels enqueued).
int launch(const LaunchArgs& a, cudaStream_t s, int* launches, const char** why);

// Enqueues the bounded-wait self test (see msa_route_wait_selftest); 0 on success.
int launch_wait_selftest(unsigned long long limit_ns, int release_first, int32_t* dev_err, cudaStream_t s);

}  // namespace route_tc
