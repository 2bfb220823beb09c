// metrics.cu -- P@k of top-k predictions against the positive labels.
//
// "ELMO: Efficiency via Low-precision and Peak Memory Optimization in Large
// Output Spaces" (atlas summary, metrics) reports P@1/3/5: the fraction of a
// sample's first j predicted labels that are among its positives, averaged
// over samples.  Hit counts are integers, so the result does not depend on the
// order of accumulation: P@j = hits(j) / (j B) in double, then rounded to fp32.
#include "elmo_common.cuh"
#include "elmo_internal.h"

namespace elmo {
namespace {

constexpr int kMetThreads = 1024;

__global__ void __launch_bounds__(kMetThreads) precision_at_k_kernel(const int32_t* __restrict__ idx, int32_t B,
                                                                     int32_t k, const int32_t* __restrict__ rowptr,
                                                                     const int32_t* __restrict__ cols, int32_t nnz,
                                                                     float* __restrict__ p) {
  __shared__ unsigned int hits[ELMO_MAX_TOPK];   // hits among the first j + 1 predictions, over all rows
  for (int j = threadIdx.x; j < k; j += blockDim.x) hits[j] = 0;
  __syncthreads();
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    // positives of row b, clamped to the label list (a malformed rowptr reads nothing outside it)
    const int r0 = max(0, min(rowptr[b], nnz));
    const int r1 = max(r0, min(rowptr[b + 1], nnz));
    unsigned int h = 0;
    for (int i = 0; i < k; ++i) {
      const int32_t lab = idx[(size_t)b * k + i];
      bool hit = false;
      for (int q = r0; q < r1 && !hit; ++q) hit = cols[q] == lab;
      h += hit ? 1u : 0u;
      if (h) atomicAdd(&hits[i], h);
    }
  }
  __syncthreads();
  for (int j = threadIdx.x; j < k; j += blockDim.x) p[j] = (float)((double)hits[j] / ((double)(j + 1) * (double)B));
}

}  // namespace

cudaError_t launch_precision_at_k(const int32_t* idx, int32_t B, int32_t k, const int32_t* rowptr,
                                  const int32_t* cols, int32_t nnz, float* p, cudaStream_t s) {
  precision_at_k_kernel<<<1, kMetThreads, 0, s>>>(idx, B, k, rowptr, cols, nnz, p);
  return cudaGetLastError();
}

}  // namespace elmo
