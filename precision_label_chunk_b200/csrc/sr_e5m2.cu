// sr_e5m2.cu -- standalone stochastic rounding onto the OCP E5M2 grid.
//
// The same rounding as the other grids ("ELMO: Efficiency via Low-precision
// and Peak Memory Optimization in Large Output Spaces", abstract: stochastic
// rounding in place of FP32 master weights): with grid neighbours
// lo < |v| < hi, round to hi iff u < f = (|v| - lo) / (hi - lo), u = k / 2^16,
// sign restored.  E5M2 has infinities, so +-inf stays +-inf, a finite |v| at
// or above the largest finite value 57344 saturates to it, NaN -> 0x7F.
//
// The decision is exact.  Normal range (|v| >= 2^-14): E5M2 keeps 2 of fp32's
// 23 mantissa bits, so with F the 21 discarded bits, u < f <=> 32 k < F, and
// adding 2^21 - 1 - 32 k to the bit pattern carries into the first kept bit
// exactly then (into the exponent where the mantissa is full).  Below 2^-14
// the grid spacing is 2^-16: t = |v| 2^16, its integer part q and fraction
// t - q are exact in fp32, and the result is (q + [k < 2^16 (t - q)]) 2^-16.
#include "elmo_common.cuh"
#include "elmo_internal.h"

namespace elmo {
namespace {

__global__ void __launch_bounds__(256) sr_e5m2_kernel(const float* __restrict__ in, uint8_t* __restrict__ out,
                                                      int64_t n, uint64_t seed, uint64_t step, uint64_t base) {
  const uint64_t first_blk = base >> 3;
  const uint64_t last_blk = (base + (uint64_t)n - 1) >> 3;
  for (uint64_t q = first_blk + blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; q <= last_blk;
       q += (uint64_t)gridDim.x * blockDim.x) {
    const u32x4 r = sr_block(seed, step, q);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint64_t idx = q * 8 + e;
      if (idx < base || idx >= base + (uint64_t)n) continue;
      const uint32_t word = sr_word(r, e >> 1);
      out[idx - base] = (uint8_t)sr_e5m2_code(in[idx - base], (e & 1) ? (word >> 16) : (word & 0xFFFFu));
    }
  }
}

// Eight values with the eight draws of one Philox block, without a branch
// per value.  Below 2^-14 a value is first moved into [2^-14, 2^-13), whose
// spacing is also 2^-16, by adding 2^-14 rounded toward +inf: in units of the
// 21 discarded bits that keeps ceil(F), and for an integer 32 k,
// 32 k < F <=> 32 k < ceil(F), so the carry test stays exact; the 2^-14 is
// taken off again exactly.  Values at or above 57344 round to at least 57344
// and the saturating conversion brings them to 57344.  A group holding a NaN
// or an infinity takes the per-value path.
__device__ __forceinline__ uint2 sr8_e5m2(const float (&v)[8], const u32x4& r) {
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
  float probe = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) probe = __fmaf_rn(v[i], 0.0f, probe);
  if (probe != 0.0f) {
    uint32_t c[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) c[e] = sr_e5m2_code(v[e], (e & 1) ? (w[e >> 1] >> 16) : (w[e >> 1] & 0xFFFFu));
    return make_uint2(c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24), c[4] | (c[5] << 8) | (c[6] << 16) | (c[7] << 24));
  }
  float o[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const uint32_t k = (e & 1) ? (w[e >> 1] >> 16) : (w[e >> 1] & 0xFFFFu);
    const float a = fabsf(v[e]);
    // sub = 1 when |v| < 2^-14: (2^-14 - |v|) 2^100 is then >= 2^62, else <= 0
    const float sub = __saturatef(__fmaf_rn(-a, 0x1p100f, 0x1p86f));
    const float sh = __fmaf_ru(sub, 0x1p-14f, a);
    const uint32_t t = (__float_as_uint(sh) + (0x1FFFFFu - (k << 5))) & 0xFFE00000u;
    o[e] = copysignf(__fmaf_rn(sub, -0x1p-14f, __uint_as_float(t)), v[e]);
  }
  return make_uint2(pack_e5m2x2(o[1], o[0]) | (pack_e5m2x2(o[3], o[2]) << 16),
                    pack_e5m2x2(o[5], o[4]) | (pack_e5m2x2(o[7], o[6]) << 16));
}

// Whole Philox blocks: thread t rounds the 8 values of block q0 + t (two
// 16-byte streaming loads, one 8-byte streaming store).
__global__ void __launch_bounds__(256) sr_e5m2_vec_kernel(const float4* __restrict__ in, uint2* __restrict__ out,
                                                          int64_t nblk, uint64_t seed, uint64_t step, uint64_t q0) {
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < nblk; t += (int64_t)gridDim.x * blockDim.x) {
    const float4 a = __ldcs(in + 2 * t), b = __ldcs(in + 2 * t + 1);
    const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    __stcs(out + t, sr8_e5m2(v, sr_block(seed, step, q0 + (uint64_t)t)));
  }
}

int grid_of(uint64_t work) {
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  uint64_t g = (work + 255) / 256;
  const uint64_t cap = (uint64_t)nsm * 8;
  if (g > cap) g = cap;
  return (int)(g > 0 ? g : 1);
}

}  // namespace

cudaError_t launch_sr_e5m2(const float* in, uint8_t* out, int64_t n, uint64_t seed, uint64_t step, uint64_t base,
                           cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  int64_t done = 0;
  if ((base & 7) == 0 && (reinterpret_cast<uintptr_t>(in) & 15) == 0 && (reinterpret_cast<uintptr_t>(out) & 7) == 0 &&
      n >= 8) {
    const int64_t nblk = n / 8;
    sr_e5m2_vec_kernel<<<grid_of((uint64_t)nblk), 256, 0, s>>>(reinterpret_cast<const float4*>(in),
                                                               reinterpret_cast<uint2*>(out), nblk, seed, step,
                                                               base >> 3);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    done = nblk * 8;
    if (done == n) return cudaSuccess;
  }
  const int64_t m = n - done;
  const uint64_t b0 = base + (uint64_t)done;
  const uint64_t blocks = (((b0 + m - 1) >> 3) - (b0 >> 3)) + 1;
  sr_e5m2_kernel<<<grid_of(blocks), 256, 0, s>>>(in + done, out + done, m, seed, step, b0);
  return cudaGetLastError();
}

}  // namespace elmo
