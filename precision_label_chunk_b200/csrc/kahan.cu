// kahan.cu -- the encoder side of a pure-BF16 model.
//
// "ELMO: Efficiency via Low-precision and Peak Memory Optimization in Large
// Output Spaces" (atlas summary "Approach"; abstract) trains the whole model
// in BF16 without FP32 master weights: the classifier with stochastic
// rounding, the encoder with Kahan summation.  The head hands dX to the
// encoder in BF16 (elmo_round_bf16), and a dense BF16 layer is updated by
// compensated SGD (elmo_kahan_sgd): parameters p and compensation c in bf16,
// gradient g in bf16, every operation one IEEE fp32 operation, the two stored
// results rounded to nearest-even:
//     u = -(lr g),  y = u + c,  p' = bf16(p + y),  c' = bf16(y - (p' - p)).
// Kahan's compensated summation applied to p + sum of the increments.
//
// Both passes stream their operands once: HBM-bound, 16-byte vector loads
// and evict-first stores, a grid of whole waves over the SMs.
#include "elmo_common.cuh"
#include "elmo_internal.h"

namespace elmo {
namespace {

// Round to nearest even onto bf16, NaN -> 0x7FC0.
__device__ __forceinline__ uint32_t bf16_bits_rn(float v) {
  return v != v ? 0x7FC0u : (uint32_t)f32_to_bf16_rn(v);
}

__device__ __forceinline__ void kahan1(uint32_t pb, uint32_t cb, uint32_t gb, float lr, uint32_t& po, uint32_t& co) {
  const float pv = __uint_as_float(pb << 16), cv = __uint_as_float(cb << 16), gv = __uint_as_float(gb << 16);
  const float u = -__fmul_rn(lr, gv);
  const float y = __fadd_rn(u, cv);
  po = bf16_bits_rn(__fadd_rn(pv, y));
  const float moved = __fsub_rn(__uint_as_float(po << 16), pv);
  co = bf16_bits_rn(__fsub_rn(y, moved));
}

// Two bf16 values per 32-bit word, low half first.
__device__ __forceinline__ void kahan2(uint32_t p, uint32_t c, uint32_t g, float lr, uint32_t& po, uint32_t& co) {
  uint32_t p0, c0, p1, c1;
  kahan1(p & 0xFFFFu, c & 0xFFFFu, g & 0xFFFFu, lr, p0, c0);
  kahan1(p >> 16, c >> 16, g >> 16, lr, p1, c1);
  po = p0 | (p1 << 16);
  co = c0 | (c1 << 16);
}

__global__ void __launch_bounds__(256) kahan_sgd_vec_kernel(uint4* __restrict__ P, uint4* __restrict__ C,
                                                            const uint4* __restrict__ G, int64_t n8, float lr) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
    const uint4 p = __ldcs(P + i), c = __ldcs(C + i), g = __ldcs(G + i);
    uint4 po, co;
    kahan2(p.x, c.x, g.x, lr, po.x, co.x);
    kahan2(p.y, c.y, g.y, lr, po.y, co.y);
    kahan2(p.z, c.z, g.z, lr, po.z, co.z);
    kahan2(p.w, c.w, g.w, lr, po.w, co.w);
    __stcs(P + i, po);
    __stcs(C + i, co);
  }
}

__global__ void __launch_bounds__(256) kahan_sgd_kernel(uint16_t* __restrict__ P, uint16_t* __restrict__ C,
                                                        const uint16_t* __restrict__ G, int64_t i0, int64_t n,
                                                        float lr) {
  for (int64_t i = i0 + blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    uint32_t po, co;
    kahan1(P[i], C[i], G[i], lr, po, co);
    P[i] = (uint16_t)po;
    C[i] = (uint16_t)co;
  }
}

__global__ void __launch_bounds__(256) round_bf16_vec_kernel(const float4* __restrict__ in, uint4* __restrict__ out,
                                                             int64_t n8) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
    const float4 a = __ldcs(in + 2 * i), b = __ldcs(in + 2 * i + 1);
    uint4 o;
    o.x = bf16_bits_rn(a.x) | (bf16_bits_rn(a.y) << 16);
    o.y = bf16_bits_rn(a.z) | (bf16_bits_rn(a.w) << 16);
    o.z = bf16_bits_rn(b.x) | (bf16_bits_rn(b.y) << 16);
    o.w = bf16_bits_rn(b.z) | (bf16_bits_rn(b.w) << 16);
    __stcs(out + i, o);
  }
}

__global__ void __launch_bounds__(256) round_bf16_kernel(const float* __restrict__ in, uint16_t* __restrict__ out,
                                                         int64_t i0, int64_t n) {
  for (int64_t i = i0 + blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = (uint16_t)bf16_bits_rn(in[i]);
}

int waves(int64_t work) {
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  int64_t g = (work + 255) / 256;
  const int64_t cap = (int64_t)nsm * 8;            // 8 resident CTAs of 256 threads per SM
  if (g > cap) g = cap;
  return (int)(g > 0 ? g : 1);
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

cudaError_t launch_kahan_sgd(void* p, void* c, const void* g, int64_t n, float lr, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  int64_t done = 0;
  if (al16(p) && al16(c) && al16(g) && n >= 8) {
    const int64_t n8 = n / 8;
    kahan_sgd_vec_kernel<<<waves(n8), 256, 0, s>>>(static_cast<uint4*>(p), static_cast<uint4*>(c),
                                                   static_cast<const uint4*>(g), n8, lr);
    done = n8 * 8;
  }
  if (done < n)
    kahan_sgd_kernel<<<waves(n - done), 256, 0, s>>>(static_cast<uint16_t*>(p), static_cast<uint16_t*>(c),
                                                     static_cast<const uint16_t*>(g), done, n, lr);
  return cudaGetLastError();
}

cudaError_t launch_round_bf16(const float* in, void* out, int64_t n, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  int64_t done = 0;
  if (al16(in) && al16(out) && n >= 8) {
    const int64_t n8 = n / 8;
    round_bf16_vec_kernel<<<waves(n8), 256, 0, s>>>(reinterpret_cast<const float4*>(in), static_cast<uint4*>(out), n8);
    done = n8 * 8;
  }
  if (done < n) round_bf16_kernel<<<waves(n - done), 256, 0, s>>>(in, static_cast<uint16_t*>(out), done, n);
  return cudaGetLastError();
}

}  // namespace elmo
