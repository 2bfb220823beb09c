// step_common.cuh -- device pieces shared by the kernels of the training step:
// bounded-wait bookkeeping, the gradient operand G = sigmoid(Z) - Y with its
// certified rounding, and the stochastic-rounding SGD update of 16 weights.
//
// "ELMO: Efficiency via Low-precision and Peak Memory Optimization in Large
// Output Spaces", atlas summary "Approach": the classifier's gradient is fused
// with a momentum-free SGD update applied by stochastic rounding onto the BF16
// or E4M3 grid, without FP32 master weights.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "elmo_common.cuh"
#include "elmo_internal.h"
#include "tc_ptx.cuh"

namespace elmo {
namespace {

using namespace tc;

constexpr int kThreads = 576;                    // 18 warps: TMA, MMA, 16 epilogue
constexpr int kEpiWarps = 16;
constexpr long long kWaitCycles = 4000000000LL;   // ~2 s at 2 GHz: only a broken pipeline waits this long
constexpr uint32_t kBox = 16384;                  // one 128-row x 128-byte TMA box

__device__ __forceinline__ void record_timeout(int32_t* status, volatile int* abort, int site) {
  *abort = 1;
  if (atomicCAS(status, 0, (int)ELMO_ETIMEOUT) == 0) status[1] = site;
}

// Positives of label `l` among the sorted keys (label << 8 | sample) in
// [k0, k1): a 256-bit sample mask.
__device__ __forceinline__ void label_mask(const uint32_t* __restrict__ keys, int k0, int k1, int64_t l,
                                           uint32_t (&m)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = 0;
  for (int i = k0; i < k1; ++i) {
    const uint32_t key = __ldg(keys + i);
    if ((int64_t)(key >> 8) == l) {
      const uint32_t b = key & 0xFFu;
#pragma unroll
      for (int w = 0; w < 8; ++w)
        if ((b >> 5) == (uint32_t)w) m[w] |= 1u << (b & 31);
    }
  }
}


__device__ __forceinline__ float exp2f_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcpf_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float tanhf_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// fp32 multiply that keeps denormal inputs and results whatever -ftz says
__device__ __forceinline__ float mul_rn_denorm(float a, float b) {
  float y;
  asm("mul.rn.f32 %0, %1, %2;" : "=f"(y) : "f"(a), "f"(b));
  return y;
}

// ---------------------------------------------------------------- epilogue pieces
// The gradient operand of the next two contractions for 16 elements:
// G = sigmoid(z) - y rounded to nearest even onto bf16 (kG = 0), or 2^8 G onto
// E4M3 (kG = 1) or E5M2 (kG = 2), z = acc * inv_sx; y = 1 at the positives.
// The code is the one that sigmoid(z) = 1 / (1 + e^-z) correctly rounded to
// fp32 gives.
//
// Fast path (y = 0): x = 2^8 sigmoid(z) (or sigmoid(z) for bf16) from one ex2
// and one rcp of the special-function unit, x = 1 / (2^-8 (1 + 2^t)) with
// t = acc * (-log2(e) inv_sx) (inv_sx is a power of two, so the one rounding
// of t is relative 2^-24 and the fp32 log2(e) is within 2^-26 of log2(e)).
// For z >= -kZlim the distance of x from 2^8 fl32(sigmoid(z)) is below kT
// units in the last place of x: the rounding of t moves 2^t by at most
// |z| 1.22 2^-24, ex2 and rcp add their own relative errors (measured on the
// device: below 2^-22 and 2^-23 over the range used) and 1 + 2^t and sigmoid's
// own fp32 rounding one ulp each.  Within one binade the grid's midpoints are
// the fp32 values whose bits below the grid's last mantissa bit read
// 100...0 (kMid), so x rounds like 2^8 fl32(sigmoid(z)) unless those bits lie
// within kT of kMid.  Elements where they do (about 2 kT 2^-16 of them for
// bf16, 2 kT 2^-20 for E4M3), positives, logits below -kZlim, NaN logits and
// padding take the per-element exact path: sigmoid in double precision,
// rounded to fp32, then the format's rounding.  ybits: positives; vbits: valid
// elements (the others, batch padding and labels past the range, get code 0);
// out: 4 words of 8-bit codes or 8 words of bf16, element 0 in the low bits.
template <int kG>
__device__ __forceinline__ uint32_t grad_pack2(float hi, float lo) {
  return kG == 0 ? pack_bf16x2(hi, lo) : kG == 1 ? pack_e4m3x2(hi, lo) : pack_e5m2x2(hi, lo);
}

template <int kG>
__device__ __noinline__ uint32_t grad_code_exact(float acc, float inv_sx, bool pos) {
  constexpr float sc = kG ? 256.0f : 1.0f;
  const float z = __fmul_rn(acc, inv_sx);
  const float s = (float)(1.0 / (1.0 + exp(-(double)z)));
  const float x = __fmaf_rn(s, sc, pos ? -sc : 0.0f);     // sc (s - y): the scale is exact
  return grad_pack2<kG>(0.0f, x) & (kG ? 0xFFu : 0xFFFFu);
}

template <int kG>
struct GradWindow {
  // fp32 bits below the grid's last mantissa bit, the pattern of a midpoint,
  // the half-width of the window in ulps of x, the lowest logit of the fast path
  static constexpr uint32_t kMask = kG == 0 ? 0xFFFFu : (kG == 1 ? 0xFFFFFu : 0x1FFFFFu);
  static constexpr uint32_t kMid = (kMask >> 1) + 1u;
  static constexpr uint32_t kT = kG == 0 ? 14u : 24u;
  static constexpr float kZlim = kG == 0 ? 4.0f : 8.0f;
};

// the lowest accumulator value of the fast path: -kZlim / inv_sx
template <int kG>
__device__ __forceinline__ float grad_acc_floor(float inv_sx) {
  return __fdiv_rn(-GradWindow<kG>::kZlim, inv_sx);
}

template <int kG>
__device__ __forceinline__ void grad_codes16(const uint32_t* acc, float inv_sx, float acc_lo, uint32_t ybits,
                                             uint32_t vbits, uint32_t* out) {
  using Wd = GradWindow<kG>;
  constexpr float isc = kG ? 0.00390625f : 1.0f;
  const float zmul = -1.4426950408889634f * inv_sx;
  float x[16];
  bool slow = (ybits != 0u) | (vbits != 0xFFFFu);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float a = __uint_as_float(acc[i]);
    x[i] = rcpf_approx(__fmaf_rn(exp2f_approx(__fmul_rn(a, zmul)), isc, isc));
    const uint32_t off = (__float_as_uint(x[i]) - (Wd::kMid - Wd::kT)) & Wd::kMask;
    slow |= (off <= 2u * Wd::kT) | !(a >= acc_lo);
  }
#pragma unroll
  for (int q = 0; q < (kG ? 4 : 8); ++q)
    out[q] = kG ? grad_pack2<kG>(x[4 * q + 1], x[4 * q]) | (grad_pack2<kG>(x[4 * q + 3], x[4 * q + 2]) << 16)
                : grad_pack2<kG>(x[2 * q + 1], x[2 * q]);
  if (slow) {                                  // rare: positives, padding, near-midpoint or low logits
    constexpr int kPer = kG ? 4 : 2;
    constexpr int kBits = 32 / kPer;
#pragma unroll
    for (int i = 0; i < 16; ++i) {             // unrolled: x and acc stay in registers
      const float a = __uint_as_float(acc[i]);
      const uint32_t off = (__float_as_uint(x[i]) - (Wd::kMid - Wd::kT)) & Wd::kMask;
      const bool v = (vbits >> i) & 1u, y = (ybits >> i) & 1u;
      if (!v || y || off <= 2u * Wd::kT || !(a >= acc_lo)) {
        const uint32_t c = v ? grad_code_exact<kG>(a, inv_sx, y) : 0u;
        const int q = i / kPer, sh = (i % kPer) * kBits;
        const uint32_t m = (kG ? 0xFFu : 0xFFFFu) << sh;
        out[q] = (out[q] & ~m) | (c << sh);
      }
    }
  }
}

// The operand value of code `c` (G, with 2^-8 undone for the 8-bit formats).
template <int kG>
__device__ __forceinline__ float grad_value(uint32_t c) {
  return kG == 0 ? bf16_to_f32((uint16_t)c)
                 : (kG == 1 ? e4m3_to_f32((uint8_t)c) : e5m2_to_f32((uint8_t)c)) * 0.00390625f;
}

// G for 16 samples b0 .. b0+15 of one label row, stored label-major as the
// next contraction's operand (the resident-X and streamed-X kernels A).
template <int kFp8, int kG5 = 0>
__device__ __forceinline__ void grad16(const uint32_t* r, float inv_sx, float acc_lo, uint32_t ybits, int b0, int B,
                                       uint8_t* __restrict__ gtile, int row, bool row_invalid,
                                       float* __restrict__ Zrow, float* __restrict__ Grow) {
  constexpr int kG = kFp8 ? (kG5 ? 2 : 1) : 0;
  uint32_t vbits = 0;
  if (!row_invalid) vbits = b0 + 16 <= B ? 0xFFFFu : (B > b0 ? (1u << (B - b0)) - 1u : 0u);
  uint32_t packed[8];
  grad_codes16<kG>(r, inv_sx, acc_lo, ybits, vbits, packed);
  if (kFp8) {
    const int j = b0 >> 4;                                   // 16-byte chunk of samples
    *reinterpret_cast<uint4*>(gtile + ((j * 16 + (row >> 3)) << 7) + ((row & 7) << 4)) =
        make_uint4(packed[0], packed[1], packed[2], packed[3]);
  } else {
    const int j = b0 >> 3;                                   // first of two 16-byte chunks
    *reinterpret_cast<uint4*>(gtile + ((j * 16 + (row >> 3)) << 7) + ((row & 7) << 4)) =
        make_uint4(packed[0], packed[1], packed[2], packed[3]);
    *reinterpret_cast<uint4*>(gtile + (((j + 1) * 16 + (row >> 3)) << 7) + ((row & 7) << 4)) =
        make_uint4(packed[4], packed[5], packed[6], packed[7]);
  }
  if (Grow && !row_invalid) {
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (b0 + i < B)
        Grow[i] = grad_value<kG>(kFp8 ? (packed[i >> 2] >> (8 * (i & 3))) & 0xFFu
                                      : (packed[i >> 1] >> (16 * (i & 1))) & 0xFFFFu);
  }
  if (Zrow && !row_invalid) {
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (b0 + i < B) Zrow[i] = __fmul_rn(__uint_as_float(r[i]), inv_sx);
  }
}

// Positive-label bits of samples b0 .. b0+15 from the 256-bit mask.
__device__ __forceinline__ uint32_t mask16(const uint32_t (&m)[8], int b0) {
  uint32_t w = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) w = ((b0 >> 5) == i) ? m[i] : w;
  return (w >> (b0 & 16)) & 0xFFFFu;
}

// ---------------------------------------------------------------- the SR update
// The 16 draws of elements l*d + j0 .. +15 (two Philox blocks of the stream
// of the seed whose round keys are rk; blk_base more
// blocks in when this head holds the rows of a larger head from label_base on:
// blk_base = label_base * d / 8).  Independent of the gradient, so the update
// can form them while the MMAs of its tile are still running.
__device__ __forceinline__ void sr_draws16(const PhiloxKeys& rk, uint64_t step, uint64_t blk_base, int64_t l,
                                           int32_t d, int j0, uint32_t (&rw)[8]) {
  const uint64_t blk = blk_base + (((uint64_t)l * (uint64_t)d + (uint64_t)j0) >> 3);
  const u32x4 r0 = sr_block_rk(rk, step, blk), r1 = sr_block_rk(rk, step, blk + 1);
  rw[0] = r0.x; rw[1] = r0.y; rw[2] = r0.z; rw[3] = r0.w;
  rw[4] = r1.x; rw[5] = r1.y; rw[6] = r1.z; rw[7] = r1.w;
}

// W[l, j0 .. j0+15] = SR(W - lrs * acc) for one label row: old weights from the
// 128B-swizzled W tile in shared memory (row `row`, tile column jl), draws rw
// from sr_draws16.
//
// v = fl(w - fl(lrs dW)) (two roundings, denormals kept), then stochastic
// rounding with the element's 16-bit draw k: round away from the lower
// neighbour iff k < floor(2^16 f), f the position of |v| between its grid
// neighbours.  bf16: cvt.rs.bf16x2.f32 adds its 16 random bits to the 16
// discarded bits of each value and truncates, so passing 2^16 - 1 - k (the
// complemented draw) gives exactly this rounding; E4M3 and E5M2: the
// stochastic conversions to the 8-bit formats apply the same rule to a 16-bit
// field (sr_e4m3x4_hw / sr_e5m2x4_hw).  A group holding a NaN or an infinity
// takes the exact per-element path.
// kW: the weight grid, 0 bf16, 1 E4M3, 2 E5M2.  kInPlace: the new codes go
// back into the shared-memory tile where the old ones were read (for a bulk
// store of the whole tile), else to Wglob[l, j0 ..].
template <int kW, bool kInPlace = false>
__device__ __forceinline__ void update16(const uint32_t (&r)[16], const uint32_t (&rw)[8],
                                         const uint8_t* __restrict__ wtile, int row, int jl, int64_t l, int32_t d,
                                         int j0, float lrs, void* __restrict__ Wglob) {
  float wv[16];
  if (kW) {
    const uint4 x = *reinterpret_cast<const uint4*>(wtile + row * 128 + (((jl >> 4) ^ (row & 7)) << 4));
    const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float f4[4];
      if (kW == 1) e4m3x4_to_f32(xw[e], f4);
      else e5m2x4_to_f32(xw[e], f4);
#pragma unroll
      for (int i = 0; i < 4; ++i) wv[4 * e + i] = f4[i];
    }
  } else {
#pragma unroll
    for (int v = 0; v < 2; ++v) {
      const int c16 = ((jl & 63) >> 3) + v;
      const uint4 x = *reinterpret_cast<const uint4*>(wtile + (jl >> 6) * kBox + row * 128 + ((c16 ^ (row & 7)) << 4));
      const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        wv[8 * v + 2 * e] = __uint_as_float(xw[e] << 16);
        wv[8 * v + 2 * e + 1] = __uint_as_float(xw[e] & 0xFFFF0000u);
      }
    }
  }
  float vv[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) vv[i] = __fsub_rn(wv[i], __fmul_rn(lrs, __uint_as_float(r[i])));
  uint32_t wnew[8];
  // E4M3: the stochastic conversion also gives the rounding's results for
  // NaN (0x7F, either sign), +-inf (+-448), +-0 and fp32 denormals (+-0), as
  // checked on B200, so every group takes it.  bf16 and E5M2: a probe that is
  // not finite when some v is NaN or infinite (E5M2: the sum of 0 v, whose
  // infinities must stay infinite; bf16: the sum of 2 v, which also overflows
  // once some |v| >= 2^127, where rounding could pass the largest finite
  // value) sends the group to the exact per-element path.
  float probe = 0.0f;
  if (kW != 1) {
#pragma unroll
    for (int i = 0; i < 16; ++i) probe = __fmaf_rn(vv[i], kW ? 0.0f : 2.0f, probe);
  }
  if (kW == 1 || fabsf(probe) < INFINITY) {
    if (kW) {
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4)
        wnew[q4] = kW == 1 ? sr_e4m3x4_hw(vv[4 * q4], vv[4 * q4 + 1], vv[4 * q4 + 2], vv[4 * q4 + 3], rw[2 * q4],
                                          rw[2 * q4 + 1])
                           : sr_e5m2x4_hw(vv[4 * q4], vv[4 * q4 + 1], vv[4 * q4 + 2], vv[4 * q4 + 3], rw[2 * q4],
                                          rw[2 * q4 + 1]);
    } else {
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        uint32_t o;   // element 2p (low half) takes the low 16 random bits, 2p + 1 the high
        asm("cvt.rs.bf16x2.f32 %0, %1, %2, %3;" : "=r"(o) : "f"(vv[2 * p + 1]), "f"(vv[2 * p]), "r"(~rw[p]));
        wnew[p] = o;
      }
    }
  } else {
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      if (kW == 1) {
        if (p < 4) {
          const uint32_t w0 = rw[2 * p], w1 = rw[2 * p + 1];
          const float o0 = sr_e4m3_value(vv[4 * p], w0 & 0xFFFFu), o1 = sr_e4m3_value(vv[4 * p + 1], w0 >> 16);
          const float o2 = sr_e4m3_value(vv[4 * p + 2], w1 & 0xFFFFu), o3 = sr_e4m3_value(vv[4 * p + 3], w1 >> 16);
          wnew[p] = pack_e4m3x2(o1, o0) | (pack_e4m3x2(o3, o2) << 16);
        }
      } else if (kW == 2) {
        if (p < 4) {
          const uint32_t w0 = rw[2 * p], w1 = rw[2 * p + 1];
          wnew[p] = sr_e5m2_code(vv[4 * p], w0 & 0xFFFFu) | (sr_e5m2_code(vv[4 * p + 1], w0 >> 16) << 8) |
                    (sr_e5m2_code(vv[4 * p + 2], w1 & 0xFFFFu) << 16) |
                    (sr_e5m2_code(vv[4 * p + 3], w1 >> 16) << 24);
        }
      } else {
        wnew[p] = (uint32_t)sr_bf16(vv[2 * p], rw[p] & 0xFFFFu) | ((uint32_t)sr_bf16(vv[2 * p + 1], rw[p] >> 16) << 16);
      }
    }
  }
  if (kInPlace) {
    uint8_t* wt = const_cast<uint8_t*>(wtile);
    if (kW) {
      *reinterpret_cast<uint4*>(wt + row * 128 + (((jl >> 4) ^ (row & 7)) << 4)) =
          make_uint4(wnew[0], wnew[1], wnew[2], wnew[3]);
    } else {
#pragma unroll
      for (int v = 0; v < 2; ++v) {
        const int c16 = ((jl & 63) >> 3) + v;
        *reinterpret_cast<uint4*>(wt + (jl >> 6) * kBox + row * 128 + ((c16 ^ (row & 7)) << 4)) =
            make_uint4(wnew[4 * v], wnew[4 * v + 1], wnew[4 * v + 2], wnew[4 * v + 3]);
      }
    }
  } else {
    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(Wglob) + ((size_t)l * d + j0) * (kW ? 1 : 2));
    dst[0] = make_uint4(wnew[0], wnew[1], wnew[2], wnew[3]);
    if (!kW) dst[1] = make_uint4(wnew[4], wnew[5], wnew[6], wnew[7]);
  }
}

}  // namespace
}  // namespace elmo
