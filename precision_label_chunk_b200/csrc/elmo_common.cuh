// elmo_common.cuh -- device helpers shared by the ELMO head kernels (sm_100a).
//
// Counter-based random numbers (Philox4x32-10, Salmon, Moraes, Dror, Shaw,
// "Parallel Random Numbers: As Easy as 1, 2, 3", SC'11) and the exact
// stochastic rounding that replaces FP32 master weights in ELMO ("ELMO:
// Efficiency via Low-precision and Peak Memory Optimization in Large Output
// Spaces", abstract; atlas summary "Approach").
#pragma once

#include <cuda_fp16.h>
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
    // separate high and low 32-bit products: measured ~30% fewer instructions
    // per block on sm_100a than forming the 64-bit product
    const uint32_t hiA = __umulhi(kMulA, c0), loA = kMulA * c0;
    const uint32_t hiB = __umulhi(kMulB, c2), loB = kMulB * c2;
    const uint32_t n0 = hiB ^ c1 ^ k0, n2 = hiA ^ c3 ^ k1;
    c0 = n0; c1 = loB; c2 = n2; c3 = loA;
    k0 += kWeyl0; k1 += kWeyl1;
  }
  return {c0, c1, c2, c3};
}

// The round keys of one seed: round r uses (k0[r], k1[r]) = the seed's low
// and high words plus r times the Weyl increments (mod 2^32), the schedule of
// philox10 above.  Formed once on the host and passed by value as a kernel
// parameter, so each round's XOR reads its key from the constant bank.
struct PhiloxKeys { uint32_t k0[10], k1[10]; };

inline PhiloxKeys philox_keys(uint64_t seed) {
  PhiloxKeys K;
  uint32_t a = (uint32_t)seed, b = (uint32_t)(seed >> 32);
  for (int r = 0; r < 10; ++r) {
    K.k0[r] = a;
    K.k1[r] = b;
    a += 0x9E3779B9u;
    b += 0xBB67AE85u;
  }
  return K;
}

// 32 x 32 -> 64-bit product as (lo, hi) from one wide multiply
__device__ __forceinline__ void mul_wide_u32(uint32_t a, uint32_t b, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b64 t;\n\tmul.wide.u32 t, %2, %3;\n\tmov.b64 {%0, %1}, t;\n\t}"
      : "=r"(lo), "=r"(hi) : "r"(a), "r"(b));
}

__device__ __forceinline__ u32x4 philox10_rk(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                              const PhiloxKeys& K) {
  constexpr uint32_t kMulA = 0xD2511F53u, kMulB = 0xCD9E8D57u;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    uint32_t loA, hiA, loB, hiB;
    mul_wide_u32(c0, kMulA, loA, hiA);
    mul_wide_u32(c2, kMulB, loB, hiB);
    const uint32_t n0 = hiB ^ c1 ^ K.k0[r], n2 = hiA ^ c3 ^ K.k1[r];
    c0 = n0; c1 = loB; c2 = n2; c3 = loA;
  }
  return {c0, c1, c2, c3};
}

__device__ __forceinline__ u32x4 sr_block_rk(const PhiloxKeys& K, uint64_t step, uint64_t blk) {
  return philox10_rk((uint32_t)blk, (uint32_t)(blk >> 32), (uint32_t)step, (uint32_t)(step >> 32), K);
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
// Stochastic rounding of fp32 v with a 16-bit draw k: v on the grid is kept;
// otherwise, with neighbours lo < |v| < hi and f = (|v| - lo) / (hi - lo), it
// returns hi iff k < floor(2^16 f), sign restored: the complemented draw is
// added to the first 16 discarded bits and the sum truncated.
//
// On the fp32 bit pattern: if the bits below the target precision hold the
// fraction F (n bits: 16 for bf16, 20 for E4M3, 21 for E5M2), then
// floor(2^16 f) = floor(F / 2^(n-16)), and adding (2^16 - 1 - k) 2^(n-16)
// carries into the first kept bit exactly when k < floor(F / 2^(n-16)).
// Below the smallest normal value of E4M3 (2^-6; the subnormal spacing is
// 2^-9) |v| is first moved into the binade [2^-6, 2^-5), which has the same
// spacing, by adding 2^-6 rounded toward zero: that keeps floor(F) of the
// exact fraction, and floor(floor(F) / 16) = floor(F / 16), so the carry test
// stays exact; 2^-6 is subtracted again exactly afterwards.
//
// The sm_100a stochastic conversions (cvt.rs.satfinite.e4m3x4.f32 and
// .e5m2x4.f32) apply this rule with the 16-bit field 2^16 - 1 - k of their
// random operand, subnormal range and saturation included; an element in
// byte 0 or 2 of the result takes the low or high half of the operand (bytes
// 1 and 3 take a bit-reversed copy of the same halves, so each conversion
// here rounds two values, in bytes 0 and 2, with independent draws).
__device__ __forceinline__ uint16_t sr_bf16(float v, uint32_t k) {
  const uint32_t b = __float_as_uint(v);
  const uint32_t mag = b & 0x7FFFFFFFu;
  const uint32_t sign = (b >> 16) & 0x8000u;
  uint32_t r = min((mag + 0xFFFFu - k) >> 16, 0x7F7Fu);   // never round a finite value to inf
  r = (mag >= 0x7F800000u) ? ((mag == 0x7F800000u) ? 0x7F80u : 0x7FC0u) : r;
  return (uint16_t)((mag > 0x7F800000u) ? r : (sign | r));
}

// The SR result as an fp32 value on the E4M3 grid (|v| >= 448 and inf are
// left above 448 for the saturating conversion; NaN becomes +NaN).
__device__ __forceinline__ float sr_e4m3_value(float v, uint32_t k) {
  const uint32_t b = __float_as_uint(v);
  const uint32_t mag = b & 0x7FFFFFFFu;
  const float a = __uint_as_float(mag);
  const float c = (a < 0.015625f) ? 0.015625f : 0.0f;       // 2^-6 below the normal range
  const float s = __fadd_rz(a, c);
  const uint32_t t = (__float_as_uint(s) + ((0xFFFFu - k) << 4)) & 0xFFF00000u;
  const float r = __fsub_rn(__uint_as_float(t), c);
  const float out = __uint_as_float(__float_as_uint(r) | (b & 0x80000000u));
  return (mag > 0x7F800000u) ? __uint_as_float(0x7FC00000u) : out;
}

// The SR result of a finite v as an fp32 value on the E5M2 grid (magnitudes
// above 57344 are left there for the saturating conversion).  As for E4M3,
// with the subnormal range below 2^-14 (spacing 2^-16) moved up one binade.
__device__ __forceinline__ float sr_e5m2_finite_value(float v, uint32_t k) {
  const uint32_t b = __float_as_uint(v);
  const float a = __uint_as_float(b & 0x7FFFFFFFu);
  const float c = (a < 0x1p-14f) ? 0x1p-14f : 0.0f;
  const float s = __fadd_rz(a, c);
  const uint32_t t = (__float_as_uint(s) + ((0xFFFFu - k) << 5)) & 0xFFE00000u;
  const float r = __fsub_rn(__uint_as_float(t), c);
  return __uint_as_float(__float_as_uint(r) | (b & 0x80000000u));
}

// Two fp32 values -> two E4M3 codes (hi in the upper byte), RNE + saturating.
__device__ __forceinline__ uint32_t pack_e4m3x2(float hi, float lo) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two fp32 values -> two E5M2 codes (hi in the upper byte), RNE + saturating.
__device__ __forceinline__ uint32_t pack_e5m2x2(float hi, float lo) {
  uint16_t r;
  asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// E5M2 code -> value: an E5M2 code is the upper byte of the binary16 value.
__device__ __forceinline__ float e5m2_to_f32(uint8_t c) {
  float f;
  const uint16_t h = (uint16_t)((uint16_t)c << 8);
  asm("cvt.f32.f16 %0, %1;" : "=f"(f) : "h"(h));
  return f;
}

// Two fp32 values -> two bf16 (hi in the upper half), RNE.
__device__ __forceinline__ uint32_t pack_bf16x2(float hi, float lo) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ uint8_t sr_e4m3(float v, uint32_t k) {
  return (uint8_t)(pack_e4m3x2(0.0f, sr_e4m3_value(v, k)) & 0xFF);
}

// Four fp32 values -> four codes (byte i = value i) by the stochastic
// conversions: values 0 and 1 take the low and high 16-bit draws of w01,
// values 2 and 3 those of w23.  Saturating: E4M3 maps NaN of either sign to
// 0x7F and +-inf to +-448, +-0 and fp32 denormals to +-0 (checked on B200
// against the rounding's definition); E5M2's infinities must stay infinite,
// so E5M2 callers send NaN and infinities to sr_e5m2_code.
__device__ __forceinline__ uint32_t sr_e4m3x4_hw(float v0, float v1, float v2, float v3, uint32_t w01,
                                                 uint32_t w23) {
  uint32_t a, b;
  asm("cvt.rs.satfinite.e4m3x4.f32 %0, {%1, %2, %3, %4}, %5;"
      : "=r"(a) : "f"(0.0f), "f"(v1), "f"(0.0f), "f"(v0), "r"(~w01));
  asm("cvt.rs.satfinite.e4m3x4.f32 %0, {%1, %2, %3, %4}, %5;"
      : "=r"(b) : "f"(0.0f), "f"(v3), "f"(0.0f), "f"(v2), "r"(~w23));
  return __byte_perm(a, b, 0x6420);
}

__device__ __forceinline__ uint32_t sr_e5m2x4_hw(float v0, float v1, float v2, float v3, uint32_t w01,
                                                 uint32_t w23) {
  uint32_t a, b;
  asm("cvt.rs.satfinite.e5m2x4.f32 %0, {%1, %2, %3, %4}, %5;"
      : "=r"(a) : "f"(0.0f), "f"(v1), "f"(0.0f), "f"(v0), "r"(~w01));
  asm("cvt.rs.satfinite.e5m2x4.f32 %0, {%1, %2, %3, %4}, %5;"
      : "=r"(b) : "f"(0.0f), "f"(v3), "f"(0.0f), "f"(v2), "r"(~w23));
  return __byte_perm(a, b, 0x6420);
}

// Eight values rounded with the eight 16-bit draws of one Philox block (draw
// e is half e & 1 of word e >> 1).  bf16: add-and-truncate on the fp32 bit
// pattern (adding 2^16 - 1 - k carries into the first kept bit exactly when
// k < F, F the 16 discarded bits); E4M3: the stochastic conversion.  A bf16
// group holding a NaN, an infinity or a magnitude of 2^127 or more (where the
// carry could reach the exponent's top) takes the per-element path.
__device__ __forceinline__ uint4 sr8_bf16(const float (&v)[8], const u32x4& r) {
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
  float probe = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) probe = __fmaf_rn(__fmul_rn(v[i], 2.0f), 0.0f, probe);
  uint32_t o[4];
  if (probe == 0.0f) {
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const uint32_t t0 = __float_as_uint(v[2 * p]) + (0xFFFFu - (w[p] & 0xFFFFu));
      const uint32_t t1 = __float_as_uint(v[2 * p + 1]) + (0xFFFFu - (w[p] >> 16));
      o[p] = __byte_perm(t0, t1, 0x7632);
    }
  } else {
#pragma unroll
    for (int p = 0; p < 4; ++p)
      o[p] = (uint32_t)sr_bf16(v[2 * p], w[p] & 0xFFFFu) | ((uint32_t)sr_bf16(v[2 * p + 1], w[p] >> 16) << 16);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// E4M3: the stochastic conversion for every value, NaN (0x7F), +-inf
// (+-448), +-0 and fp32 denormals included (the rounding's own results there).
__device__ __forceinline__ uint2 sr8_e4m3(const float (&v)[8], const u32x4& r) {
  return make_uint2(sr_e4m3x4_hw(v[0], v[1], v[2], v[3], r.x, r.y), sr_e4m3x4_hw(v[4], v[5], v[6], v[7], r.z, r.w));
}

// Stochastic rounding of v onto the OCP E5M2 grid with a 16-bit draw k, as
// an E5M2 code: NaN -> 0x7F, +-inf kept, magnitudes at or above the largest
// finite 57344 saturate to it.  From 2^-14 up E5M2 keeps 2 of fp32's 23
// mantissa bits (add-and-truncate at 21 bits); below, its subnormal grid is
// the multiples of 2^-16, and with t = |v| 2^16 (exact) and q = floor(t),
// t - q are exact in fp32, and the result is
// (q + [k < floor(2^16 (t - q))]) 2^-16.
__device__ __forceinline__ uint32_t sr_e5m2_code(float v, uint32_t k) {
  const uint32_t b = __float_as_uint(v);
  const uint32_t sign = (b >> 24) & 0x80u;
  const uint32_t mag = b & 0x7FFFFFFFu;
  if (mag > 0x7F800000u) return 0x7Fu;                    // NaN
  if (mag == 0x7F800000u) return sign | 0x7Cu;            // +-inf
  if (mag >= 0x47600000u) return sign | 0x7Bu;            // |v| >= 57344: the largest finite value
  float o;
  if (mag >= 0x38800000u) {                               // |v| >= 2^-14
    o = __uint_as_float((mag + ((0xFFFFu - k) << 5)) & ~0x1FFFFFu);
  } else {
    const float t = __fmul_rn(__uint_as_float(mag), 65536.0f);
    const float q = floorf(t);
    const float up = (float)k < floorf(__fmul_rn(__fsub_rn(t, q), 65536.0f)) ? 1.0f : 0.0f;
    o = __fmul_rn(__fadd_rn(q, up), 0x1p-16f);
  }
  uint16_t r;
  asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(o));
  return sign | (r & 0x7Fu);                              // o is on the grid: the conversion is exact
}

// Four E5M2 codes (byte i = element i) -> fp32 values, exact (an E5M2 code is
// the upper byte of the binary16 value).
__device__ __forceinline__ void e5m2x4_to_f32(uint32_t w, float (&o)[4]) {
  uint32_t h01, h23;
  asm("cvt.rn.f16x2.e5m2x2 %0, %1;" : "=r"(h01) : "h"((uint16_t)(w & 0xFFFF)));
  asm("cvt.rn.f16x2.e5m2x2 %0, %1;" : "=r"(h23) : "h"((uint16_t)(w >> 16)));
  o[0] = __half2float(__ushort_as_half((unsigned short)(h01 & 0xFFFF)));
  o[1] = __half2float(__ushort_as_half((unsigned short)(h01 >> 16)));
  o[2] = __half2float(__ushort_as_half((unsigned short)(h23 & 0xFFFF)));
  o[3] = __half2float(__ushort_as_half((unsigned short)(h23 >> 16)));
}

// Four E4M3 codes (byte i = element i) -> fp32 values, exact.
__device__ __forceinline__ void e4m3x4_to_f32(uint32_t w, float (&o)[4]) {
  uint32_t h01, h23;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h01) : "h"((uint16_t)(w & 0xFFFF)));
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h23) : "h"((uint16_t)(w >> 16)));
  o[0] = __half2float(__ushort_as_half((unsigned short)(h01 & 0xFFFF)));
  o[1] = __half2float(__ushort_as_half((unsigned short)(h01 >> 16)));
  o[2] = __half2float(__ushort_as_half((unsigned short)(h23 & 0xFFFF)));
  o[3] = __half2float(__ushort_as_half((unsigned short)(h23 >> 16)));
}

}  // namespace elmo
