// topk_simt.cu -- exact chunked top-k with CUDA cores.
//
// Score of (b, l) is the fp32 fused multiply-add chain over j = 0..d-1 in
// order; ranking is score descending, ties to the lower label, NaN last.
// Labels are split into segments; every CTA (row, segment) keeps the
// segment's top-k, and a second kernel merges the segments of a row.  P@k
// evaluation in "ELMO: Efficiency via Low-precision and Peak Memory
// Optimization in Large Output Spaces" (atlas summary, metrics P@1/3/5)
// ranks labels this way.
#include <float.h>

#include "elmo_common.cuh"
#include "elmo_internal.h"

namespace elmo {
namespace {

constexpr int kSegLabels = 8192;
constexpr int kTopkThreads = 256;
constexpr int32_t kEmpty = 0x7FFFFFFF;

// true iff (sa, ia) ranks before (sb, ib)
__device__ __forceinline__ bool before(float sa, int32_t ia, float sb, int32_t ib) {
  if (ia == kEmpty) return false;
  if (ib == kEmpty) return true;
  const bool na = isnan(sa), nb = isnan(sb);
  if (na != nb) return nb;
  if (!na && sa != sb) return sa > sb;
  return ia < ib;
}

__device__ __forceinline__ float w_at(const void* W, int dt, int64_t i) {
  return dt == ELMO_BF16 ? bf16_to_f32(static_cast<const uint16_t*>(W)[i])
         : dt == ELMO_FP8_E5M2 ? e5m2_to_f32(static_cast<const uint8_t*>(W)[i])
                               : e4m3_to_f32(static_cast<const uint8_t*>(W)[i]);
}

// Work item w = (row r, segment seg) with r = w / nseg: the segment's top-k of
// query row b = rows[r] (rows == null: b = r), written at (r * nseg + seg) * k.
// The grid loops over the nr * nseg items, nr = *nrows (rows given) or B.
__global__ void __launch_bounds__(kTopkThreads) topk_segment_kernel(const void* __restrict__ W, int dt, int64_t L,
                                                                    int32_t d, const uint16_t* __restrict__ X,
                                                                    int32_t k, int32_t nseg, int32_t B,
                                                                    const int32_t* __restrict__ rows,
                                                                    const int32_t* __restrict__ nrows,
                                                                    float* __restrict__ cs,
                                                                    int32_t* __restrict__ ci) {
  extern __shared__ float sm[];          // x row [d], then k candidates per thread
  float* xs = sm;
  float* ls = sm + d;
  int32_t* li = reinterpret_cast<int32_t*>(ls + (size_t)kTopkThreads * k);
  __shared__ int head[kTopkThreads];
  __shared__ float rs[kTopkThreads];
  __shared__ int32_t ri[kTopkThreads];
  __shared__ int rt[kTopkThreads];
  const int tid = threadIdx.x;
  const int nr = rows ? *nrows : B;
  float* my_s = ls + (size_t)tid * k;
  int32_t* my_i = li + (size_t)tid * k;
  for (int64_t w = blockIdx.x; w < (int64_t)nr * nseg; w += gridDim.x) {
    const int r = (int)(w / nseg), seg = (int)(w % nseg);
    const int b = rows ? rows[r] : r;
    for (int j = tid; j < d; j += blockDim.x) xs[j] = bf16_to_f32(X[(int64_t)b * d + j]);
    for (int q = 0; q < k; ++q) { my_s[q] = -FLT_MAX; my_i[q] = kEmpty; }
    __syncthreads();
    const int64_t a = (int64_t)seg * kSegLabels;
    const int64_t e = min(L, a + kSegLabels);
    for (int64_t l = a + tid; l < e; l += blockDim.x) {
      float sc = 0.0f;
      for (int j = 0; j < d; ++j) sc = __fmaf_rn(xs[j], w_at(W, dt, l * d + j), sc);
      const int32_t li32 = (int32_t)l;
      if (!before(sc, li32, my_s[k - 1], my_i[k - 1])) continue;
      int p = k - 1;
      while (p > 0 && before(sc, li32, my_s[p - 1], my_i[p - 1])) {
        my_s[p] = my_s[p - 1]; my_i[p] = my_i[p - 1]; --p;
      }
      my_s[p] = sc; my_i[p] = li32;
    }
    __syncthreads();
    // merge the per-thread lists: k rounds of a block-wide arg-best over list heads
    head[tid] = 0;
    __syncthreads();
    for (int q = 0; q < k; ++q) {
      const int hp = head[tid];
      rs[tid] = hp < k ? my_s[hp] : -FLT_MAX;
      ri[tid] = hp < k ? my_i[hp] : kEmpty;
      rt[tid] = tid;
      __syncthreads();
      for (int off = kTopkThreads / 2; off > 0; off >>= 1) {
        if (tid < off && before(rs[tid + off], ri[tid + off], rs[tid], ri[tid])) {
          rs[tid] = rs[tid + off]; ri[tid] = ri[tid + off]; rt[tid] = rt[tid + off];
        }
        __syncthreads();
      }
      if (tid == 0) {
        const size_t o = ((size_t)r * nseg + seg) * k + q;
        cs[o] = rs[0];
        ci[o] = ri[0];
        if (ri[0] != kEmpty) head[rt[0]] += 1;
      }
      __syncthreads();
    }
  }
}

// Merge of the nseg segment lists of work row r into the top-k of query row
// b = rows[r] (rows == null: b = r); the grid loops over the rows.
__global__ void __launch_bounds__(kTopkThreads) topk_merge_kernel(const float* __restrict__ cs,
                                                                  const int32_t* __restrict__ ci, int32_t k,
                                                                  int32_t nseg, int32_t B,
                                                                  const int32_t* __restrict__ rows,
                                                                  const int32_t* __restrict__ nrows,
                                                                  int32_t* __restrict__ idx,
                                                                  float* __restrict__ score) {
  __shared__ float rs[kTopkThreads];
  __shared__ int32_t ri[kTopkThreads];
  __shared__ int32_t last_i;
  __shared__ float last_s;
  const int tid = threadIdx.x;
  const int nr = rows ? *nrows : B;
  const int64_t n = (int64_t)nseg * k;
  for (int r = blockIdx.x; r < nr; r += gridDim.x) {
    const int b = rows ? rows[r] : r;
    const float* sv = cs + (size_t)r * n;
    const int32_t* iv = ci + (size_t)r * n;
    if (tid == 0) { last_i = -1; last_s = 0.0f; }
    __syncthreads();
    for (int q = 0; q < k; ++q) {
      // best candidate strictly after the previously selected one
      float bs = -FLT_MAX;
      int32_t bi = kEmpty;
      const int32_t pi = last_i;
      const float ps = last_s;
      for (int64_t t = tid; t < n; t += blockDim.x) {
        const float cs_ = sv[t];
        const int32_t ci_ = iv[t];
        if (ci_ == kEmpty) continue;
        if (pi >= 0 && !before(ps, pi, cs_, ci_)) continue;
        if (before(cs_, ci_, bs, bi)) { bs = cs_; bi = ci_; }
      }
      rs[tid] = bs; ri[tid] = bi;
      __syncthreads();
      for (int off = kTopkThreads / 2; off > 0; off >>= 1) {
        if (tid < off && before(rs[tid + off], ri[tid + off], rs[tid], ri[tid])) {
          rs[tid] = rs[tid + off]; ri[tid] = ri[tid + off];
        }
        __syncthreads();
      }
      if (tid == 0) {
        idx[(size_t)b * k + q] = ri[0];
        score[(size_t)b * k + q] = rs[0];
        last_i = ri[0];
        last_s = rs[0];
      }
      __syncthreads();
    }
  }
}

}  // namespace

size_t topk_simt_workspace_bytes(const elmo_head* h, int32_t B, int32_t k) {
  const int64_t nseg = (h->L + kSegLabels - 1) / kSegLabels;
  return (size_t)B * nseg * k * (sizeof(float) + sizeof(int32_t));
}

cudaError_t launch_topk_simt_rows(const elmo_head* h, const uint16_t* X, int32_t B, int32_t k, const int32_t* rows,
                                  const int32_t* nrows, void* cand, int32_t* idx, float* score, cudaStream_t s) {
  const int32_t nseg = (int32_t)((h->L + kSegLabels - 1) / kSegLabels);
  float* cs = static_cast<float*>(cand);
  int32_t* ci = reinterpret_cast<int32_t*>(cs + (size_t)B * nseg * k);
  const size_t smem = sizeof(float) * (size_t)h->d + (size_t)kTopkThreads * k * (sizeof(float) + sizeof(int32_t));
  cudaError_t e = cudaFuncSetAttribute(topk_segment_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // a row list's length is known only on the device: a grid-stride grid of a few CTAs per SM
  const int64_t items = (int64_t)B * nseg;
  const int64_t cap = (int64_t)h->num_sms * 8;
  const int grid = (int)(rows ? cap : (items < cap ? items : cap));
  topk_segment_kernel<<<grid, kTopkThreads, smem, s>>>(h->W, w_format(h), h->L, h->d, X, k, nseg, B, rows, nrows, cs,
                                                       ci);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int mgrid = rows ? h->num_sms : B;
  topk_merge_kernel<<<mgrid, kTopkThreads, 0, s>>>(cs, ci, k, nseg, B, rows, nrows, idx, score);
  return cudaGetLastError();
}

}  // namespace elmo
