// step_simt.cu -- the ELMO head step written with CUDA cores only, in the
// accumulation order of its definition.  Used as the first correct path and
// as the slow-but-simple comparison path of the tensor-core kernels.
//
// "ELMO: Efficiency via Low-precision and Peak Memory Optimization in Large
// Output Spaces", atlas summary "Approach": the classifier gradient
// G = sigmoid(Z) - Y with Z = X W_c^T, the input gradient dX += G W_c (old
// W_c), and the momentum-free update W_c <- SR(W_c - lr G^T X).
#include "elmo_common.cuh"
#include "elmo_internal.h"

namespace elmo {
namespace {

// Keys are grouped by 128-label tile (tile g at [tile_ptr[g], tile_ptr[g+1])).
__device__ __forceinline__ bool is_positive(const uint32_t* keys, const int32_t* tile_ptr, int64_t l, int b) {
  const uint32_t key = ((uint32_t)l << 8) | (uint32_t)b;
  const int64_t g = l >> 7;
  for (int i = tile_ptr[g]; i < tile_ptr[g + 1]; ++i)
    if (keys[i] == key) return true;
  return false;
}

__device__ __forceinline__ float w_at(const void* W, int dt, int64_t i) {
  return dt == ELMO_BF16 ? bf16_to_f32(static_cast<const uint16_t*>(W)[i])
                         : e4m3_to_f32(static_cast<const uint8_t*>(W)[i]);
}

// x operand of the contraction: bf16 mode X itself, fp8 mode the E4M3 code of X * s_X.
__device__ __forceinline__ float x_at(const uint16_t* X, const uint8_t* xq, int dt, int64_t i) {
  return dt == ELMO_BF16 ? bf16_to_f32(X[i]) : e4m3_to_f32(xq[i]);
}

__device__ __forceinline__ float g_at(const void* gbuf, int dt, int64_t i) {
  return dt == ELMO_BF16 ? bf16_to_f32(static_cast<const uint16_t*>(gbuf)[i])
                         : e4m3_to_f32(static_cast<const uint8_t*>(gbuf)[i]);
}

__global__ void grad_simt_kernel(const void* __restrict__ W, int dt, int32_t d, const uint16_t* __restrict__ X,
                                 const uint8_t* __restrict__ xq, const float* __restrict__ xscale, int32_t B,
                                 int64_t l0, int64_t l1, const uint32_t* __restrict__ keys,
                                 const int32_t* __restrict__ tile_ptr, void* __restrict__ gbuf,
                                 float* __restrict__ Zout, float* __restrict__ Gout) {
  const int64_t n = (l1 - l0) * B;
  const float inv_sx = dt == ELMO_BF16 ? 1.0f : xscale[1];
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < n; t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t l = l0 + t / B;
    const int b = (int)(t % B);
    float acc = 0.0f;
    for (int j = 0; j < d; ++j)
      acc = __fmaf_rn(x_at(X, xq, dt, (int64_t)b * d + j), w_at(W, dt, l * d + j), acc);
    const float z = __fmul_rn(acc, inv_sx);
    const float sig = 1.0f / (1.0f + expf(-z));
    const float g = sig - (is_positive(keys, tile_ptr, l, b) ? 1.0f : 0.0f);
    float gv;
    if (dt == ELMO_BF16) {
      const uint16_t c = f32_to_bf16_rn(g);
      static_cast<uint16_t*>(gbuf)[t] = c;
      gv = bf16_to_f32(c);
    } else {
      const uint8_t c = f32_to_e4m3_rn(g * 256.0f);
      static_cast<uint8_t*>(gbuf)[t] = c;
      gv = e4m3_to_f32(c) * 0.00390625f;
    }
    if (Zout) Zout[t] = z;
    if (Gout) Gout[t] = gv;
  }
}

__global__ void dx_simt_kernel(const void* __restrict__ W, int dt, int32_t d, int32_t B, int64_t l0,
                               int64_t l1, const void* __restrict__ gbuf, float* __restrict__ dX) {
  const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (t >= (int64_t)B * d) return;
  const int b = (int)(t / d), j = (int)(t % d);
  const int64_t span = l1 - l0;
  const int64_t a = l0 + span * blockIdx.y / gridDim.y, e = l0 + span * (blockIdx.y + 1) / gridDim.y;
  float acc = 0.0f;
  for (int64_t l = a; l < e; ++l)
    acc = __fmaf_rn(g_at(gbuf, dt, (l - l0) * B + b), w_at(W, dt, l * d + j), acc);
  atomicAdd(&dX[t], dt == ELMO_BF16 ? acc : acc * 0.00390625f);
}

__global__ void update_simt_kernel(void* __restrict__ W, int dt, int32_t d, const uint16_t* __restrict__ X,
                                   const uint8_t* __restrict__ xq, const float* __restrict__ xscale, int32_t B,
                                   int64_t l0, int64_t l1, const void* __restrict__ gbuf, float lr,
                                   uint64_t seed, uint64_t step, uint64_t idx_base) {
  const int64_t groups = (l1 - l0) * (d / 8);
  const float dw_scale = dt == ELMO_BF16 ? 1.0f : 0.00390625f * xscale[1];
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < groups;
       t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t l = l0 + t / (d / 8);
    const int j0 = (int)(t % (d / 8)) * 8;
    const uint64_t idx0 = idx_base + (uint64_t)l * d + j0;   // index in the whole head
    const u32x4 r = sr_block(seed, step, idx0 >> 3);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int j = j0 + e;
      float dw = 0.0f;
      for (int b = 0; b < B; ++b)
        dw = __fmaf_rn(g_at(gbuf, dt, (l - l0) * B + b), x_at(X, xq, dt, (int64_t)b * d + j), dw);
      dw = __fmul_rn(dw, dw_scale);
      const float w = w_at(W, dt, l * d + j);
      const float v = __fsub_rn(w, __fmul_rn(lr, dw));
      const uint32_t word = sr_word(r, e >> 1);
      const uint32_t k = (e & 1) ? (word >> 16) : (word & 0xFFFFu);
      if (dt == ELMO_BF16) static_cast<uint16_t*>(W)[l * d + j] = sr_bf16(v, k);
      else static_cast<uint8_t*>(W)[l * d + j] = sr_e4m3(v, k);
    }
  }
}

int grid_cap(int64_t work, int per_block) {
  int64_t g = (work + per_block - 1) / per_block;
  if (g > 148 * 32) g = 148 * 32;
  return (int)(g > 0 ? g : 1);
}

}  // namespace

cudaError_t launch_grad_simt(const elmo_head* h, const uint16_t* X, int32_t B, int64_t l0, int64_t l1,
                             void* gbuf, float* Zout, float* Gout, cudaStream_t s) {
  if (l1 <= l0) return cudaSuccess;
  grad_simt_kernel<<<grid_cap((l1 - l0) * B, 256), 256, 0, s>>>(h->W, (int)h->dt, h->d, X, h->xq, h->xscale, B,
                                                                 l0, l1, h->keys, h->tile_ptr, gbuf, Zout, Gout);
  return cudaGetLastError();
}

cudaError_t launch_dx_simt(const elmo_head* h, int32_t B, int64_t l0, int64_t l1, const void* gbuf, float* dX,
                           cudaStream_t s) {
  if (l1 <= l0) return cudaSuccess;
  const int64_t n = (int64_t)B * h->d;
  dim3 grid((unsigned)((n + 255) / 256), 1);
  int64_t splits = (148 * 16) / (int64_t)grid.x;
  splits = splits < 1 ? 1 : splits;
  if (splits > (l1 - l0)) splits = l1 - l0;
  grid.y = (unsigned)splits;
  dx_simt_kernel<<<grid, 256, 0, s>>>(h->W, (int)h->dt, h->d, B, l0, l1, gbuf, dX);
  return cudaGetLastError();
}

cudaError_t launch_update_simt(const elmo_head* h, const uint16_t* X, int32_t B, int64_t l0, int64_t l1,
                               const void* gbuf, float lr, uint64_t seed, uint64_t step, cudaStream_t s) {
  if (l1 <= l0) return cudaSuccess;
  update_simt_kernel<<<grid_cap((l1 - l0) * (h->d / 8), 128), 128, 0, s>>>(
      h->W, (int)h->dt, h->d, X, h->xq, h->xscale, B, l0, l1, gbuf, lr, seed, step,
      (uint64_t)h->label_base * (uint64_t)h->d);
  return cudaGetLastError();
}

}  // namespace elmo
