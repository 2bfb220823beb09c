// elmo_common.cuh -- device helpers shared by the ELMO head kernels (sm_100a).
//
// Counter-based random numbers (Philox4x32-10, Salmon, Moraes, Dror, Shaw,
// "Parallel Random Numbers: As Easy as 1, 2, 3", SC'11) and the exact
// stochastic rounding that replaces FP32 master weights in ELMO ("ELMO:
// Efficiency via Low-precision and Peak Memory Optimization in Large Output
// Spaces", abstract; atlas summary "Approach").
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/elmo.h"

namespace elmo {

// ---------------------------------------------------------------- Philox
// Ten rounds of the Philox-4x32 bijection.  Round r maps counter words
// (c0, c1, c2, c3) to (hi(B*c2) ^ c1 ^ k0, lo(B*c2), hi(A*c0) ^ c3 ^ k1,
// lo(A*c0)) with the key advanced by the Weyl increments after every round;
// A, B, and the increments are the constants published for Philox4x32.
struct u32x4 { uint32_t x, y, z, w; };

__device__ __forceinline__ u32x4 philox10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                           uint32_t k0, uint32_t k1) {
  constexpr uint32_t kMulA = 0xD2511F53u, kMulB = 0xCD9E8D57u;
  constexpr uint32_t kWeyl0 = 0x9E3779B9u, kWeyl1 = 0xBB67AE85u;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t hiA = __umulhi(kMulA, c0), loA = kMulA * c0;
    const uint32_t hiB = __umulhi(kMulB, c2), loB = kMulB * c2;
    const uint32_t n0 = hiB ^ c1 ^ k0, n2 = hiA ^ c3 ^ k1;
    c0 = n0; c1 = loB; c2 = n2; c3 = loA;
    k0 += kWeyl0; k1 += kWeyl1;
  }
  return {c0, c1, c2, c3};
}

// The Philox block that serves elements 8*blk .. 8*blk+7 of SR stream
// (seed, step): counter (blk, step), key = seed.  Element idx takes the
// 16-bit half (idx & 1) of word ((idx >> 1) & 3), low half first.
__device__ __forceinline__ u32x4 sr_block(uint64_t seed, uint64_t step, uint64_t blk) {
  return philox10((uint32_t)blk, (uint32_t)(blk >> 32), (uint32_t)step, (uint32_t)(step >> 32),
                  (uint32_t)seed, (uint32_t)(seed >> 32));
}

__device__ __forceinline__ uint32_t sr_word(const u32x4& r, int w) {
  return w == 0 ? r.x : w == 1 ? r.y : w == 2 ? r.z : r.w;
}

__device__ __forceinline__ uint32_t sr_draw(uint64_t seed, uint64_t step, uint64_t idx) {
  const u32x4 r = sr_block(seed, step, idx >> 3);
  const uint32_t word = sr_word(r, (int)((idx >> 1) & 3));
  return (idx & 1) ? (word >> 16) : (word & 0xFFFFu);
}

// ---------------------------------------------------------------- formats
__device__ __forceinline__ float bf16_to_f32(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }

// E4M3FN code -> value: exponent field 0 is subnormal (m * 2^-9); S.1111.111 is NaN.
__device__ __forceinline__ float e4m3_to_f32(uint8_t c) {
  const uint32_t e = (c >> 3) & 15u, m = c & 7u;
  float mag;
  if (e == 0) mag = (float)m * 0.001953125f;  // m * 2^-9
  else mag = __uint_as_float(((e + 120u) << 23) | (m << 20));
  if (e == 15 && m == 7) mag = __int_as_float(0x7FC00000);
  return (c & 0x80) ? -mag : mag;
}

// Round to nearest even onto the bf16 grid (hardware conversion).
__device__ __forceinline__ uint16_t f32_to_bf16_rn(float v) {
  uint16_t r;
  asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(v));
  return r;
}

// Round to nearest even onto the E4M3 grid, saturating (hardware conversion).
__device__ __forceinline__ uint8_t f32_to_e4m3_rn(float v) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
  return (uint8_t)(r & 0xFF);
}

// ---------------------------------------------------------------- SR
// Stochastic rounding of fp32 v with a 16-bit draw k (u = k / 2^16): v on
// the grid is kept; otherwise with neighbours lo < |v| < hi it returns hi iff
// u < f = (|v| - lo) / (hi - lo), sign restored.
//
// bf16: the bf16 magnitude just below |v| is the top half of |v|'s bit
// pattern and f * 2^16 is exactly the bottom half (the grid is uniform in the
// pattern within a binade and across fp32 subnormals), so u < f is k < frac.
__device__ __forceinline__ uint16_t sr_bf16(float v, uint32_t k) {
  const uint32_t b = __float_as_uint(v);
  const uint32_t mag = b & 0x7FFFFFFFu;
  const uint32_t sign = (b >> 16) & 0x8000u;
  if (mag > 0x7F800000u) return 0x7FC0;            // NaN
  uint32_t r = mag >> 16;
  if (mag < 0x7F800000u) {
    r += (k < (mag & 0xFFFFu)) ? 1u : 0u;
    r = min(r, 0x7F7Fu);                            // never round a finite value to inf
  }
  return (uint16_t)(sign | r);
}

// E4M3: with e' = max(floor(log2 |v|), -6) the grid spacing near |v| is
// 2^(e'-3), so t = |v| * 2^(3-e') is exact, lo = floor(t) and f = t - lo are
// exact, and the code is (e' + 6) * 8 + lo + [u < f] (lo runs 8..15 in a
// normal binade, 0..7 below 2^-6; a carry to 16 moves to the next binade).
__device__ __forceinline__ uint8_t sr_e4m3(float v, uint32_t k) {
  const uint32_t b = __float_as_uint(v);
  const uint32_t mag = b & 0x7FFFFFFFu;
  const uint8_t sign = (uint8_t)((b >> 24) & 0x80u);
  if (mag > 0x7F800000u) return 0x7F;              // NaN
  const float a = __uint_as_float(mag);
  if (a >= 448.0f) return sign | 0x7E;              // saturate (inf included)
  const int eb = (int)(mag >> 23);                  // biased exponent (0 for fp32 subnormals)
  const int e = max(eb - 127, -6);
  const float scale = __uint_as_float((uint32_t)(130 - e) << 23);  // 2^(3 - e)
  const float t = __fmul_rn(a, scale);
  const float lo = truncf(t);
  const float f = __fsub_rn(t, lo);
  const float u = __fmul_rn((float)k, 1.52587890625e-05f);          // k * 2^-16, exact
  const int code = (e + 6) * 8 + (int)lo + (u < f ? 1 : 0);
  return sign | (uint8_t)code;
}

}  // namespace elmo
