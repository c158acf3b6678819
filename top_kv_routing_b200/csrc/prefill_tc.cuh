// tcgen05 prefill attention (host-side interface used by prefill.cu; not part of the ABI).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace prefill_tc {

// RoPE frequencies of one call in fixed point, computed on the host: step[j] =
// round(2^64 * theta^(-2j/128) / (2 pi)), the rotation of frequency j per position in units
// of 2^-64 turns.  The angle of position p is then p * step[j] mod 2^64 turns (exact integer
// arithmetic, no range reduction needed).
struct RopeW {
  unsigned long long step[64];
};

struct Args {
  const __nv_bfloat16* q;       // [B][L][T][H*G][128]
  __nv_bfloat16* out;           // [B][L][T][H*G][128]
  const __nv_bfloat16* local_k; // [B][L][H][cap][128] (the block's rows already appended)
  const __nv_bfloat16* local_v;
  const int32_t* local_len;     // [B] (before the block)
  const __nv_bfloat16* mem_kv;  // [B][L][2][H][M_max][128]
  const int32_t* mem_len;       // [B][L]
  int T, B, L, H, G, cap, M_max, pos_off;
  double log2_theta;
  float qscale;                 // softmax scale x log2(e)
  int32_t* dev_err;
};

// Sizes within the kernel's 32-bit tensor-map row coordinates.
bool supported(const Args& a);
int launch(const Args& a, cudaStream_t s, const char** why);

}  // namespace prefill_tc
