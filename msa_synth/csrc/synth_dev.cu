// Device fill of seeded synthetic tensors; bit-identical to msa_synth.fill on the host.
// Used to materialise large synthetic banks directly in HBM.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "synth.h"

namespace {

template <bool BF16>
__global__ void synth_fill_kernel(void* __restrict__ dst, uint64_t key, int64_t row0, int64_t n_rows,
                                  int32_t row_len, float sigma, int apply_sigma,
                                  const float* __restrict__ topic, int32_t topic_len,
                                  const int32_t* __restrict__ row_topic) {
  const float ih_scale = __uint_as_float(SYNTH_IH_SCALE_BITS);
  const int64_t n_vec = n_rows * (int64_t)row_len / 8;
  for (int64_t v = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; v < n_vec;
       v += (int64_t)gridDim.x * blockDim.x) {
    const int64_t e0 = v * 8;
    const int64_t r = e0 / row_len;
    const int32_t c0 = (int32_t)(e0 - r * row_len);
    const uint64_t base = (uint64_t)(row0 + r) * (uint64_t)row_len + (uint64_t)c0;
    int32_t tr = -1;
    if (topic != nullptr && row_topic != nullptr) tr = row_topic[r];
    float x[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float f = __fmul_rn((float)synth_ih_centered(synth_hash(key, base + i)), ih_scale);
      if (apply_sigma) f = __fmul_rn(f, sigma);
      if (tr >= 0) f = __fadd_rn(f, topic[(int64_t)tr * topic_len + (c0 + i) % topic_len]);
      x[i] = f;
    }
    if (BF16) {
      uint4 out;
      __nv_bfloat162* p = reinterpret_cast<__nv_bfloat162*>(&out);
#pragma unroll
      for (int i = 0; i < 4; ++i) p[i] = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
      reinterpret_cast<uint4*>(dst)[v] = out;
    } else {
      float4* d = reinterpret_cast<float4*>(dst) + 2 * v;
      d[0] = make_float4(x[0], x[1], x[2], x[3]);
      d[1] = make_float4(x[4], x[5], x[6], x[7]);
    }
  }
}

}  // namespace

extern "C" {

// Fill rows [row0, row0 + n_rows) of a [rows][row_len] tensor into dst (device memory,
// 16-byte aligned, row 0 of dst = row row0).  dtype 0 = fp32, 1 = bf16.  topic is a
// device [n_topics][topic_len] fp32 table and row_topic a device [n_rows] int32 table
// (either NULL to skip).  Returns 0, or 1 for bad arguments, 2 for a launch error.
int msa_synth_fill(void* dst, int32_t dtype, uint64_t seed, uint32_t stream, uint32_t layer,
                   uint32_t sub, int64_t row0, int64_t n_rows, int32_t row_len, float sigma,
                   const float* topic, int32_t topic_len, const int32_t* row_topic,
                   cudaStream_t s) {
  if (dst == nullptr || n_rows < 0 || row0 < 0 || row_len <= 0 || (row_len % 8) != 0 ||
      (dtype != 0 && dtype != 1) || (topic != nullptr && topic_len <= 0) ||
      (reinterpret_cast<uintptr_t>(dst) & 15u) != 0)
    return 1;
  if (n_rows == 0) return 0;
  const uint64_t key = synth_tensor_key(seed, stream, layer, sub);
  const int64_t n_vec = n_rows * (int64_t)row_len / 8;
  int64_t blocks = (n_vec + 255) / 256;
  if (blocks > 148 * 64) blocks = 148 * 64;
  const int apply_sigma = sigma != 1.0f;
  if (dtype == 1)
    synth_fill_kernel<true><<<(unsigned)blocks, 256, 0, s>>>(dst, key, row0, n_rows, row_len, sigma,
                                                             apply_sigma, topic, topic_len, row_topic);
  else
    synth_fill_kernel<false><<<(unsigned)blocks, 256, 0, s>>>(dst, key, row0, n_rows, row_len, sigma,
                                                              apply_sigma, topic, topic_len, row_topic);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

}  // extern "C"
