// sr_e5m2.cu -- standalone stochastic rounding onto the OCP E5M2 grid.
//
// The same rounding as the other grids ("ELMO: Efficiency via Low-precision
// and Peak Memory Optimization in Large Output Spaces", abstract: stochastic
// rounding in place of FP32 master weights): with grid neighbours
// lo < |v| < hi and f = (|v| - lo) / (hi - lo), round to hi iff
// k < floor(2^16 f) for the element's 16-bit draw k, sign restored.  E5M2 has
// infinities, so +-inf stays +-inf, a finite |v| at or above the largest
// finite value 57344 saturates to it, NaN -> 0x7F.
//
// Finite values go through the stochastic conversion cvt.rs.satfinite
// .e5m2x4.f32, which applies exactly this rule; the per-value path
// (sr_e5m2_code) handles NaN and infinities and the unaligned edges.
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

// Eight values with the eight draws of one Philox block: the stochastic
// conversion when all are finite, else the per-value path.
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
  return make_uint2(sr_e5m2x4_hw(v[0], v[1], v[2], v[3], w[0], w[1]), sr_e5m2x4_hw(v[4], v[5], v[6], v[7], w[2], w[3]));
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
