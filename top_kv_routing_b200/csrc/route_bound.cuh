// Error bounds of the tensor-core routing filter (shared by the query preparation and the
// fused router projection, which compute them per query token, and by the selection,
// which certifies with them).  Not part of the ABI.
#pragma once
#include <cuda_fp8.h>

namespace route_bound {

// The tensor-core scores are a filter.  A selection made from them is certified only
// with a bound on |filter - exact| that follows from the operands' rounding, computed per
// query token from the query's own operand rows (the key side enters through its format
// alone).  Notation, per token t and key head g: q = the fp32 query sum (1/Hq) sum of the
// group's unit query heads, k = the stored bf16 key head, exact score
// s = sum_g <q_g, k_g> / ||k_g||.
//  bf16 filter  f = sum_g <bf16(q_g), k_g>, fp32 accumulation.  Per head:
//    |<bf16(q) - q, k>|           <= ||bf16(q) - q|| (1 + dK)          (Cauchy-Schwarz)
//    |<q, k> (1 - 1/||k||)|       <= dK ||q||
//    accumulation                 <= kAcc (1 + dK) ||bf16(q)||
//  with dK the key-norm precondition: every stored key head is the bf16 rounding
//  (nearest) of a unit vector, so | ||k|| - 1 | <= 2^-8 (+ the fp32 normalisation's error).
//  E4M3 filter  f8 = 2^-19 sum_g <e4m3(2^11 q_g), e4m3(2^8 k_g / ||k_g||)>.  With a = 2^11 q,
//  a^ its E4M3 value and b = 2^8 k / ||k|| (fp32, |b_i - 2^8 k^_i| <= 2^-17 |2^8 k^_i|), each
//  E4M3 rounding obeys |x^ - x| <= u8 |x| + eta (u8 = 2^-4; eta = 2^-10, half the smallest
//  subnormal).  Per head (scaled back by 2^-19):
//    (||a^ - a|| + u8 ||a^||) 2^-11 (1 + 2^-15) + 2^-18 ||a^||_1 / 2^11 + 2^-16 ||q||
//    + kAcc 1.07 ||a^|| / 2^11
//  The exact rescoring itself (bf16 query plus bf16 residual, fp32 accumulation, fp32 key
//  norms) is within kRescore ||q_g|| per head.  A document's score is a maximum over the
//  query's tokens and blocks, so the bound of a (query, layer) is the largest over its
//  tokens.  Accumulation model (an assumption about the tensor cores, checked by the GPU
//  tests on adversarial rows): every addition is an fp32 operation rounded to nearest or
//  toward zero, so 1,023 additions are within 1023 * 2^-23 < 2^-13 of the sum of |products|.
constexpr float kU8 = 0.0625f;                          // E4M3 unit roundoff
constexpr float kKeyDev = 1.0f / 256 + 1.0f / 524288;   // dK
constexpr float kAcc = 1.0f / 8192;                     // 2^-13
constexpr float kRescore = 1.0f / 8192;                 // rescoring error per unit of ||q_g||
constexpr float kBoundSlack = 1.0f + 1.0f / 1024;       // covers the fp32 arithmetic of the bound
constexpr float kBoundFloor = 1.0f / 16777216;          // 2^-24 absolute

// Kinds of bound kept per (layer, token): [kind][L][T].
enum { kBoundF8 = 0, kBoundBf16 = 1 };

// E4M3 value of x (OCP FP8 E4M3, nearest even, saturating) as fp32.
__device__ __forceinline__ float e4m3_round(float x) {
  const __nv_fp8_storage_t v = __nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
  return __half2float(__half(__nv_cvt_fp8_to_halfraw(v, __NV_E4M3)));
}

// Filter error bounds of one key head of one token from its norms (derivation above):
// nq = ||q_g||, ndb = ||bf16(q_g) - q_g||, nhb = ||bf16(q_g)||, na = ||a^_g|| / 2^11,
// nda = ||a^_g - a_g|| / 2^11, l1a = ||a^_g||_1 / 2^11.  Returns the E4M3 and bf16 bounds of
// the head, each with the rescoring's share.
__device__ __forceinline__ float2 head_bounds(float nq, float ndb, float nhb, float na, float nda, float l1a) {
  const float e_r = kRescore * nq;
  const float e_bf16 = ndb * (1.0f + kKeyDev) + kKeyDev * nq + kAcc * (1.0f + kKeyDev) * nhb;
  const float e_f8 = (nda + kU8 * na) * (1.0f + 1.0f / 32768) + (1.0f / 262144) * l1a + (1.0f / 65536) * nq +
                     kAcc * 1.07f * na;
  return make_float2(e_f8 + e_r, e_bf16 + e_r);
}

}  // namespace route_bound
