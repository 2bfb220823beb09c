// prep.cu -- per-step preparation of the sparse labels and of the X operand.
//
// Labels: the positives of a step arrive as CSR (rowptr, cols).  The kernels
// that form G = sigmoid(Z) - Y need them by label, so they are turned into
// sorted keys (label << 8 | sample) once per step; a label tile then finds its
// positives by binary search.  Malformed input (rowptr not monotone, rowptr[B]
// != nnz, a column outside [0, L)) is recorded in the head's status word as
// ELMO_EDATA and the offending entries are dropped.
//
// X in FP8 mode: the pages train the classifier in E4M3 without tensor
// scaling of the weights ("ELMO: Efficiency via Low-precision and Peak Memory
// Optimization in Large Output Spaces", atlas summary, "Surprising findings");
// the tensor-core operand X is brought into E4M3 range with one power-of-two
// scale per step, s_X = 2^e, e the largest integer with 2^e max|X| <= 448
// (clamped to [-126, 126]; 1 when max|X| is 0 or not finite), and rounded to
// nearest even.  The scale is undone exactly after the contraction.
#include "elmo_common.cuh"
#include "elmo_internal.h"

namespace elmo {
namespace {

__device__ __forceinline__ void set_status(int32_t* status, int code, int32_t detail) {
  if (atomicCAS(status, 0, code) == 0) status[1] = detail;
}

constexpr int kPrepThreads = 1024;

__global__ void __launch_bounds__(kPrepThreads) prep_labels_kernel(const int32_t* __restrict__ rowptr,
                                                                   const int32_t* __restrict__ cols, int32_t B,
                                                                   int32_t nnz, int64_t L, int32_t npow2,
                                                                   uint32_t* __restrict__ keys_out,
                                                                   int32_t* __restrict__ nkeys,
                                                                   int32_t* __restrict__ tile_ptr,
                                                                   int32_t* __restrict__ status) {
  extern __shared__ uint32_t sk[];
  __shared__ int bad_rows;
  __shared__ int nvalid;
  __shared__ int32_t rp[ELMO_MAX_BATCH + 1];
  const int tid = threadIdx.x;
  for (int b = tid; b <= B; b += blockDim.x) rp[b] = rowptr[b];
  if (tid == 0) nvalid = 0;
  __syncthreads();
  if (tid == 0) bad_rows = (rp[0] != 0 || rp[B] != nnz) ? 1 : 0;
  __syncthreads();
  for (int b = tid; b < B; b += blockDim.x)
    if (rp[b + 1] < rp[b]) bad_rows = 1;
  __syncthreads();
  const int ntg = (int)((L + 127) >> 7);     // 128-label tiles of the head
  if (bad_rows) {
    if (tid == 0) { set_status(status, ELMO_EDATA, -1); *nkeys = 0; }
    for (int g = tid; g <= ntg; g += blockDim.x) tile_ptr[g] = 0;
    return;
  }
  for (int i = tid; i < npow2; i += blockDim.x) {
    uint32_t key = 0xFFFFFFFFu;
    if (i < nnz) {
      int lo = 0, hi = B;                     // sample b with rowptr[b] <= i < rowptr[b+1]
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (rp[mid] <= i) lo = mid; else hi = mid;
      }
      const int32_t c = cols[i];
      if (c >= 0 && (int64_t)c < L) key = ((uint32_t)c << 8) | (uint32_t)lo;
      else set_status(status, ELMO_EDATA, i);
    }
    sk[i] = key;
  }
  __syncthreads();
  // bitonic sort, ascending
  for (int size = 2; size <= npow2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < npow2; i += blockDim.x) {
        const int j = i ^ stride;
        if (j > i) {
          const uint32_t a = sk[i], c = sk[j];
          const bool up = (i & size) == 0;
          if ((a > c) == up) { sk[i] = c; sk[j] = a; }
        }
      }
      __syncthreads();
    }
  }
  int cnt = 0;
  for (int i = tid; i < nnz; i += blockDim.x) {
    keys_out[i] = sk[i];
    cnt += sk[i] != 0xFFFFFFFFu;
  }
  atomicAdd(&nvalid, cnt);
  __syncthreads();
  const int nv = nvalid;
  if (tid == 0) *nkeys = nv;
  // tile_ptr[g] = first key whose label is in tile g or later (keys are label << 8 | sample)
  for (int g = tid; g <= ntg; g += blockDim.x) {
    int lo = 0, hi = nv;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if ((int)(sk[mid] >> 15) < g) lo = mid + 1; else hi = mid;
    }
    tile_ptr[g] = lo;
  }
}

// One CTA: max |X| with 16-byte loads, the power-of-two scale, then the E4M3
// codes of X * s_X (second pass mostly from L1/L2).  n is a multiple of 64.
__global__ void __launch_bounds__(kPrepThreads) prep_x_kernel(const uint16_t* __restrict__ X, int64_t n,
                                                              float* __restrict__ xscale,
                                                              uint8_t* __restrict__ xq) {
  __shared__ float red[kPrepThreads / 32];
  __shared__ int nonfinite;
  __shared__ float s_scale;
  const int tid = threadIdx.x;
  if (tid == 0) nonfinite = 0;
  __syncthreads();
  const uint4* X4 = reinterpret_cast<const uint4*>(X);
  const int64_t n8 = n / 8;
  uint32_t mbits = 0;       // max of |x| bit patterns (monotone for non-negative floats)
  for (int64_t i = tid; i < n8; i += blockDim.x) {
    const uint4 v = X4[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t lo = (w[e] << 16) & 0x7FFFFFFFu, hi = w[e] & 0x7FFF0000u;
      mbits = max(mbits, max(lo, hi));
    }
  }
  if (mbits >= 0x7F800000u) nonfinite = 1;
  for (int o = 16; o > 0; o >>= 1) mbits = max(mbits, __shfl_xor_sync(0xFFFFFFFFu, mbits, o));
  if ((tid & 31) == 0) red[tid >> 5] = __uint_as_float(mbits);
  __syncthreads();
  if (tid == 0) {
    float amax = 0.0f;
    for (int w = 0; w < kPrepThreads / 32; ++w) amax = fmaxf(amax, red[w]);
    float s = 1.0f;
    if (!nonfinite && amax > 0.0f) {
      // amax = mant * 2^E with mant in [0.5, 1); 448 = 0.875 * 2^9
      int E;
      const float mant = frexpf(amax, &E);
      int e = (mant <= 0.875f) ? 9 - E : 8 - E;
      e = max(-126, min(126, e));
      s = ldexpf(1.0f, e);
    }
    s_scale = s;
    xscale[0] = s;
    xscale[1] = 1.0f / s;
  }
  __syncthreads();
  const float s = s_scale;
  uint2* Q2 = reinterpret_cast<uint2*>(xq);
  for (int64_t i = tid; i < n8; i += blockDim.x) {
    const uint4 v = X4[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t q[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float x0 = __fmul_rn(__uint_as_float(w[2 * h] << 16), s), x1 = __fmul_rn(__uint_as_float(w[2 * h] & 0xFFFF0000u), s);
      const float x2 = __fmul_rn(__uint_as_float(w[2 * h + 1] << 16), s), x3 = __fmul_rn(__uint_as_float(w[2 * h + 1] & 0xFFFF0000u), s);
      q[h] = pack_e4m3x2(x1, x0) | (pack_e4m3x2(x3, x2) << 16);
    }
    Q2[i] = make_uint2(q[0], q[1]);
  }
}

}  // namespace

cudaError_t launch_prep_labels(elmo_head* h, const int32_t* rowptr, const int32_t* cols, int32_t B,
                               int32_t nnz, cudaStream_t s) {
  int32_t npow2 = 1;
  while (npow2 < nnz) npow2 <<= 1;
  const size_t smem = sizeof(uint32_t) * (size_t)npow2;
  cudaError_t e = cudaFuncSetAttribute(prep_labels_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)(sizeof(uint32_t) * ELMO_MAX_NNZ));
  if (e != cudaSuccess) return e;
  prep_labels_kernel<<<1, kPrepThreads, smem, s>>>(rowptr, cols, B, nnz, h->L, npow2, h->keys, h->nkeys,
                                                   h->tile_ptr, h->status);
  return cudaGetLastError();
}

cudaError_t launch_prep_x(elmo_head* h, const uint16_t* X, int32_t B, cudaStream_t s) {
  prep_x_kernel<<<1, kPrepThreads, 0, s>>>(X, (int64_t)B * h->d, h->xscale, h->xq);
  return cudaGetLastError();
}

}  // namespace elmo
