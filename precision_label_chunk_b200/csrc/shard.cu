// shard.cu -- a head split by labels over several devices.
//
// The classifier head is the part of the model whose size grows with the label
// count, and with millions of labels it dominates the model's compute and
// memory ("ELMO: Efficiency via Low-precision and Peak Memory Optimization in
// Large Output Spaces", abstract).  Split by label rows, every device runs the
// same fused step on its rows: the step of a label depends only on that
// label's weights, X and whether the label is positive, so the only exchange
// is the sum of the per-device input gradients, and the stochastic rounding
// stays bit-identical because it draws by the element's index in the whole
// head.
//
// Prediction: every device ranks its own rows; the global top-k of a sample is
// the best k of the union of the per-device lists, merged here.
#include "elmo_common.cuh"
#include "elmo_internal.h"

namespace elmo {
namespace {

__global__ void __launch_bounds__(256) topk_offset_kernel(int32_t* __restrict__ idx, int64_t n, int32_t base) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    idx[i] += base;
}

// Does (sa, ia) rank before (sb, ib)?  Score descending, NaN after every
// number, equal scores by the lower label id.
__device__ __forceinline__ bool ranks_before(float sa, int32_t ia, float sb, int32_t ib) {
  const bool na = sa != sa, nb = sb != sb;
  if (na || nb) return na == nb ? ia < ib : nb;
  if (sa != sb) return sa > sb;
  return ia < ib;
}

// One thread per sample: a P-way merge of lists that are each sorted best
// first.  The label sets of the lists are disjoint (one list per device).
__global__ void __launch_bounds__(128) topk_merge_kernel(const int32_t* __restrict__ idx,
                                                         const float* __restrict__ score, int32_t P, int32_t B,
                                                         int32_t k, int32_t* __restrict__ idx_out,
                                                         float* __restrict__ score_out) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  uint8_t pos[ELMO_MAX_SHARDS];
  for (int p = 0; p < P; ++p) pos[p] = 0;
  for (int o = 0; o < k; ++o) {
    int best = -1;
    float bs = 0.0f;
    int32_t bi = 0;
    for (int p = 0; p < P; ++p) {
      if (pos[p] >= k) continue;
      const size_t at = ((size_t)p * B + b) * k + pos[p];
      const float s = score[at];
      const int32_t i = idx[at];
      if (best < 0 || ranks_before(s, i, bs, bi)) { best = p; bs = s; bi = i; }
    }
    ++pos[best];        // P lists of k entries hold at least k entries
    idx_out[(size_t)b * k + o] = bi;
    score_out[(size_t)b * k + o] = bs;
  }
}

}  // namespace

cudaError_t launch_topk_offset(int32_t* idx, int64_t n, int64_t label_base, cudaStream_t s) {
  if (n <= 0 || label_base == 0) return cudaSuccess;
  int64_t grid = (n + 255) / 256;
  if (grid > 148 * 8) grid = 148 * 8;
  topk_offset_kernel<<<(int)grid, 256, 0, s>>>(idx, n, (int32_t)label_base);
  return cudaGetLastError();
}

cudaError_t launch_topk_merge(const int32_t* idx, const float* score, int32_t P, int32_t B, int32_t k,
                              int32_t* idx_out, float* score_out, cudaStream_t s) {
  if (B <= 0) return cudaSuccess;
  topk_merge_kernel<<<(B + 127) / 128, 128, 0, s>>>(idx, score, P, B, k, idx_out, score_out);
  return cudaGetLastError();
}

}  // namespace elmo
