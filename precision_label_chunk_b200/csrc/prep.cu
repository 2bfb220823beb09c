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
                                                                   int32_t* __restrict__ status) {
  extern __shared__ uint32_t sk[];
  __shared__ int bad_rows;
  __shared__ int nvalid;
  const int tid = threadIdx.x;
  if (tid == 0) {
    bad_rows = (rowptr[0] != 0 || rowptr[B] != nnz) ? 1 : 0;
    nvalid = 0;
  }
  __syncthreads();
  for (int b = tid; b < B; b += blockDim.x)
    if (rowptr[b + 1] < rowptr[b]) bad_rows = 1;
  __syncthreads();
  if (bad_rows) {
    if (tid == 0) { set_status(status, ELMO_EDATA, -1); *nkeys = 0; }
    return;
  }
  for (int i = tid; i < npow2; i += blockDim.x) {
    uint32_t key = 0xFFFFFFFFu;
    if (i < nnz) {
      int lo = 0, hi = B;                     // sample b with rowptr[b] <= i < rowptr[b+1]
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (rowptr[mid] <= i) lo = mid; else hi = mid;
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
  if (tid == 0) *nkeys = nvalid;
}

__global__ void __launch_bounds__(kPrepThreads) prep_x_kernel(const uint16_t* __restrict__ X, int64_t n,
                                                              float* __restrict__ xscale,
                                                              uint8_t* __restrict__ xq) {
  __shared__ float red[kPrepThreads / 32];
  __shared__ int nonfinite;
  __shared__ float s_scale;
  const int tid = threadIdx.x;
  if (tid == 0) nonfinite = 0;
  __syncthreads();
  float m = 0.0f;
  for (int64_t i = tid; i < n; i += blockDim.x) {
    const float a = fabsf(bf16_to_f32(X[i]));
    if (!(a <= 3.4028234663852886e38f)) nonfinite = 1;
    else m = fmaxf(m, a);
  }
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((tid & 31) == 0) red[tid >> 5] = m;
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
  for (int64_t i = tid; i < n; i += blockDim.x) xq[i] = f32_to_e4m3_rn(__fmul_rn(bf16_to_f32(X[i]), s));
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
                                                   h->status);
  return cudaGetLastError();
}

cudaError_t launch_prep_x(elmo_head* h, const uint16_t* X, int32_t B, cudaStream_t s) {
  prep_x_kernel<<<1, kPrepThreads, 0, s>>>(X, (int64_t)B * h->d, h->xscale, h->xq);
  return cudaGetLastError();
}

}  // namespace elmo
