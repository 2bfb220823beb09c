// sr.cu -- standalone stochastic rounding, its random draws, and the head fill.
//
// Stochastic rounding replaces FP32 master weights for the ELMO classifier
// ("ELMO: Efficiency via Low-precision and Peak Memory Optimization in Large
// Output Spaces", abstract; atlas summary "Approach").  One thread serves one
// Philox block, i.e. 8 consecutive elements of the stream.
#include "elmo_common.cuh"
#include "elmo_internal.h"

namespace elmo {
namespace {

__global__ void __launch_bounds__(256) sr_round_kernel(const float* __restrict__ in, void* __restrict__ out,
                                                       int64_t n, int dt, uint64_t seed, uint64_t step,
                                                       uint64_t base) {
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
      const uint32_t k = (e & 1) ? (word >> 16) : (word & 0xFFFFu);
      const int64_t i = (int64_t)(idx - base);
      const float v = in[i];
      if (dt == ELMO_BF16) static_cast<uint16_t*>(out)[i] = sr_bf16(v, k);
      else static_cast<uint8_t*>(out)[i] = sr_e4m3(v, k);
    }
  }
}

// Whole Philox blocks: thread t rounds the 8 values of block q0 + t, read as
// two 16-byte loads and written as one 8-byte (E4M3) or 16-byte (bf16) store,
// all streaming (the data are touched once).
template <int kFp8>
__global__ void __launch_bounds__(256) sr_round_vec_kernel(const float4* __restrict__ in, void* __restrict__ out,
                                                           int64_t nblk, uint64_t seed, uint64_t step,
                                                           uint64_t q0) {
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < nblk; t += (int64_t)gridDim.x * blockDim.x) {
    const float4 a = __ldcs(in + 2 * t), b = __ldcs(in + 2 * t + 1);
    const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    const u32x4 r = sr_block(seed, step, q0 + (uint64_t)t);
    if (kFp8) __stcs(reinterpret_cast<uint2*>(out) + t, sr8_e4m3(v, r));
    else __stcs(reinterpret_cast<uint4*>(out) + t, sr8_bf16(v, r));
  }
}

__global__ void __launch_bounds__(256) sr_draws_kernel(uint16_t* __restrict__ out, int64_t n, uint64_t seed,
                                                       uint64_t step, uint64_t base) {
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
      out[idx - base] = (uint16_t)((e & 1) ? (word >> 16) : (word & 0xFFFFu));
    }
  }
}

// W[i] = SR(std * n_g): g = index_base + i the element's index in the whole
// head (index_base a multiple of 8), n_g standard normal by the Box-Muller
// transform of two 32-bit Philox words (block g >> 2 of step 2^64-2 serves
// elements 4q..4q+3), rounded with the SR draw of element g at step 2^64-1.
__global__ void __launch_bounds__(256) fill_kernel(void* __restrict__ W, int64_t n, int dt, float std,
                                                   uint64_t seed, uint64_t blk_base) {
  const uint64_t nblk = ((uint64_t)n + 7) >> 3;
  for (uint64_t q = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; q < nblk;
       q += (uint64_t)gridDim.x * blockDim.x) {
    float nv[8];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint64_t nb = (blk_base + q) * 2 + h;
      const u32x4 r = philox10((uint32_t)nb, (uint32_t)(nb >> 32), 0xFFFFFFFEu, 0xFFFFFFFFu,
                               (uint32_t)seed, (uint32_t)(seed >> 32));
      const uint32_t wd[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
      for (int p = 0; p < 2; ++p) {
        const float u1 = ((float)wd[2 * p] + 1.0f) * 2.3283064365386963e-10f;  // (0, 1]
        const float u2 = (float)wd[2 * p + 1] * 2.3283064365386963e-10f;
        const float rad = sqrtf(-2.0f * logf(fminf(u1, 1.0f)));
        float sn, cs;
        sincospif(2.0f * u2, &sn, &cs);
        nv[h * 4 + 2 * p] = rad * cs;
        nv[h * 4 + 2 * p + 1] = rad * sn;
      }
    }
    const u32x4 r = sr_block(seed, ~0ull, blk_base + q);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint64_t i = q * 8 + e;
      if (i >= (uint64_t)n) break;
      const uint32_t word = sr_word(r, e >> 1);
      const uint32_t k = (e & 1) ? (word >> 16) : (word & 0xFFFFu);
      const float v = std * nv[e];
      if (dt == ELMO_BF16) static_cast<uint16_t*>(W)[i] = sr_bf16(v, k);
      else if (dt == ELMO_FP8_E5M2) static_cast<uint8_t*>(W)[i] = (uint8_t)sr_e5m2_code(v, k);
      else static_cast<uint8_t*>(W)[i] = sr_e4m3(v, k);
    }
  }
}

int grid_for(uint64_t work, int per_block) {
  uint64_t g = (work + per_block - 1) / per_block;
  if (g > 148ull * 64) g = 148ull * 64;
  return (int)(g > 0 ? g : 1);
}

}  // namespace

cudaError_t launch_sr_round(const float* in, void* out, int64_t n, elmo_dtype dt, uint64_t seed,
                            uint64_t step, uint64_t base, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const size_t esz = dt == ELMO_BF16 ? 2 : 1;
  const bool aligned = (base & 7) == 0 && (reinterpret_cast<uintptr_t>(in) & 15) == 0 &&
                       (reinterpret_cast<uintptr_t>(out) & (8 * esz - 1)) == 0;
  int64_t done = 0;
  if (aligned && n >= 8) {
    const int64_t nblk = n / 8;
    static int per_sm[2] = {0, 0};                  // resident CTAs per SM of each instance
    const int which = dt == ELMO_BF16 ? 0 : 1;
    if (!per_sm[which]) {
      int m = 0;
      if (dt == ELMO_BF16) cudaOccupancyMaxActiveBlocksPerMultiprocessor(&m, sr_round_vec_kernel<0>, 256, 0);
      else cudaOccupancyMaxActiveBlocksPerMultiprocessor(&m, sr_round_vec_kernel<1>, 256, 0);
      per_sm[which] = m > 0 ? m : 4;
    }
    int dev = 0, nsm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    int64_t grid = (nblk + 255) / 256;
    if (grid > (int64_t)nsm * per_sm[which]) grid = (int64_t)nsm * per_sm[which];
    const float4* in4 = reinterpret_cast<const float4*>(in);
    if (dt == ELMO_BF16) sr_round_vec_kernel<0><<<(int)grid, 256, 0, s>>>(in4, out, nblk, seed, step, base >> 3);
    else sr_round_vec_kernel<1><<<(int)grid, 256, 0, s>>>(in4, out, nblk, seed, step, base >> 3);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    done = nblk * 8;
    if (done == n) return cudaSuccess;
  }
  // values not in whole aligned blocks: one thread per Philox block, element by element
  const int64_t m = n - done;
  const uint64_t b0 = base + (uint64_t)done;
  const uint64_t blocks = (((b0 + m - 1) >> 3) - (b0 >> 3)) + 1;
  sr_round_kernel<<<grid_for(blocks, 256), 256, 0, s>>>(in + done, static_cast<uint8_t*>(out) + done * esz, m,
                                                        (int)dt, seed, step, b0);
  return cudaGetLastError();
}

cudaError_t launch_sr_draws(uint16_t* out, int64_t n, uint64_t seed, uint64_t step, uint64_t base,
                            cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const uint64_t blocks = (((base + n - 1) >> 3) - (base >> 3)) + 1;
  sr_draws_kernel<<<grid_for(blocks, 256), 256, 0, s>>>(out, n, seed, step, base);
  return cudaGetLastError();
}

cudaError_t launch_fill(void* W, int64_t n, elmo_dtype dt, float std, uint64_t seed, uint64_t index_base,
                        cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  if (index_base & 7) return cudaErrorInvalidValue;
  fill_kernel<<<grid_for(((uint64_t)n + 7) >> 3, 256), 256, 0, s>>>(W, n, (int)dt, std, seed, index_base >> 3);
  return cudaGetLastError();
}

}  // namespace elmo
