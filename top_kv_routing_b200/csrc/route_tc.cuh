// Tensor-core (tcgen05) routing score path: interface used by route.cu.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace route_tc {

constexpr int kMaxQueries = 256;
// Query lengths up to this many tokens (all queries of a call together) use the scan.
constexpr int kScanMaxTokens = 8;

// Rows of the bf16 query operand: padded to the tensor-core N tile.
inline int padded_tokens(int t) { return (t + 63) / 64 * 64; }

bool supported(int n_kv_heads);

struct LaunchArgs {
  const void* kr_hat;  // bf16 [L][C][8][128]
  const void* qt;      // bf16 [L][n_pad][8][128], rows >= total tokens are zero
  int L;
  int64_t C;
  int n_pad;
  int n_queries;
  int q_off[kMaxQueries + 1];
  float* m;            // [B][L][C]
};

// Enqueues the score kernel(s); returns 0 on success (launches += kernels enqueued).
int launch(const LaunchArgs& a, cudaStream_t s, int* launches, const char** why);

}  // namespace route_tc
