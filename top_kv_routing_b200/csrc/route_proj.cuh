// Router query projection fused with the query normalisation and group sum (host-side
// interface used by route.cu; not part of the ABI).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "route_tc.cuh"

namespace route_proj {

struct Layout {
  int n_queries;
  int off[route_tc::kMaxQueries + 1];   // token offsets of the queries in `hidden`
  int row0[route_tc::kMaxQueries + 1];  // first operand row of each query
};

struct Args {
  const void* hidden;  // bf16 [T][hidden_size]
  const void* w;       // bf16 [L][Hq * 128][hidden_size]
  int T, hidden_size, L, Hq, H, n_rows;
  Layout lay;
  float* qt_f32;               // [L][T][H * 128] or null
  __nv_bfloat16* qt_bf16;      // [L][n_rows][H * 128] or null (with qt_lo)
  __nv_bfloat16* qt_lo;
  uint8_t* qt_f8;              // [L][n_rows][H * 128] or null
  float* etok;                 // [2][L][T] filter error bounds per token (zeroed by the
                               // caller; each key head's share is added), or null
  int32_t* dev_err;
};

// Sizes the fused kernel takes: hidden_size a multiple of 64, Hq / H in {1, 2, 4}, T >= 1.
bool supported(int Hq, int H, int hidden_size);
int launch(const Args& a, cudaStream_t s, const char** why);

}  // namespace route_proj
