// prep.cu -- per-step preparation of the sparse labels and of the X operand.
//
// Labels: the positives of a step arrive as CSR (rowptr, cols).  The kernels
// that form G = sigmoid(Z) - Y need them by label tile, so they are bucketed
// once per step by a counting sort on the 128-label tile: keys
// (label << 8 | sample) grouped by tile, tile g's keys at
// [tile_ptr[g], tile_ptr[g+1]) in no particular order within the tile.
// Malformed input (rowptr not monotone, rowptr[B] != nnz, a column outside
// [0, labels_total)) is recorded in the head's status word as ELMO_EDATA and
// the offending entries are dropped.  A head that holds the label rows
// [label_base, label_base + L) of a larger head keeps the positives that fall
// in its rows, as local labels (label - label_base), and skips the others.
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

// One CTA.  Shared memory holds the keys and each key's slot in its tile
// (nnz <= 32768, so a slot fits 16 bits); the per-tile counters and their
// prefix sums live in tile_ptr itself ([ntg + 1] entries in global memory).
__device__ __forceinline__ void prep_labels_body(const int32_t* __restrict__ rowptr,
                                                                   const int32_t* __restrict__ cols, int32_t B,
                                                                   int32_t nnz, int64_t L,
                                                                   int64_t label_base, int64_t labels_total,
                                                                   uint32_t* __restrict__ keys_out,
                                                                   int32_t* __restrict__ nkeys,
                                                                   int32_t* __restrict__ tile_ptr,
                                                                   int32_t* __restrict__ status) {
  extern __shared__ uint32_t sk[];                                   // [nnz] keys
  uint16_t* slot = reinterpret_cast<uint16_t*>(sk + nnz);            // [nnz] slot within the tile
  __shared__ int bad_rows;
  __shared__ int nvalid;
  __shared__ int32_t rp[ELMO_MAX_BATCH + 1];
  __shared__ int32_t part[kPrepThreads];
  const int tid = threadIdx.x;
  const int ntg = (int)((L + 127) >> 7);     // 128-label tiles of the head
  for (int b = tid; b <= B; b += blockDim.x) rp[b] = rowptr[b];
  for (int g = tid; g <= ntg; g += blockDim.x) tile_ptr[g] = 0;
  if (tid == 0) nvalid = 0;
  __syncthreads();
  if (tid == 0) bad_rows = (rp[0] != 0 || rp[B] != nnz) ? 1 : 0;
  __syncthreads();
  for (int b = tid; b < B; b += blockDim.x)
    if (rp[b + 1] < rp[b]) bad_rows = 1;
  __syncthreads();
  if (bad_rows) {
    if (tid == 0) { set_status(status, ELMO_EDATA, -1); *nkeys = 0; }
    return;                                  // tile_ptr is all zero: no positives anywhere
  }
  // keys and per-tile counts (counts of tile g accumulate in tile_ptr[g + 1])
  int cnt = 0;
  for (int i = tid; i < nnz; i += blockDim.x) {
    int lo = 0, hi = B;                       // sample b with rowptr[b] <= i < rowptr[b+1]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (rp[mid] <= i) lo = mid; else hi = mid;
    }
    const int32_t c = cols[i];
    uint32_t key = 0xFFFFFFFFu;
    if (c >= 0 && (int64_t)c < labels_total) {
      const int64_t lc = (int64_t)c - label_base;   // label within this head's rows
      if (lc >= 0 && lc < L) {
        key = ((uint32_t)lc << 8) | (uint32_t)lo;
        slot[i] = (uint16_t)atomicAdd(&tile_ptr[(lc >> 7) + 1], 1);
        ++cnt;
      }
    } else {
      set_status(status, ELMO_EDATA, i);
    }
    sk[i] = key;
  }
  atomicAdd(&nvalid, cnt);
  __syncthreads();
  // inclusive scan of tile_ptr[1 .. ntg]: each thread a contiguous run, then the runs' totals
  const int n = ntg + 1;
  const int per = (n + kPrepThreads - 1) / kPrepThreads;
  const int g0 = tid * per, g1 = min(n, g0 + per);
  int32_t run = 0;
  for (int g = g0; g < g1; g += 8) {            // 8 independent loads in flight
    int32_t c[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) c[u] = g + u < g1 ? __ldcg(tile_ptr + g + u) : 0;   // formed by L2 atomics
#pragma unroll
    for (int u = 0; u < 8; ++u) run += c[u];
  }
  part[tid] = run;
  __syncthreads();
  for (int o = 1; o < kPrepThreads; o <<= 1) {   // Hillis-Steele scan of the run totals
    const int32_t v = tid >= o ? part[tid - o] : 0;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  int32_t acc = part[tid] - run;                 // exclusive prefix of this run
  for (int g = g0; g < g1; g += 8) {
    int32_t c[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) c[u] = g + u < g1 ? __ldcg(tile_ptr + g + u) : 0;
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (g + u < g1) { acc += c[u]; tile_ptr[g + u] = acc; }
  }
  __syncthreads();
  // scatter: tile g's keys land in [tile_ptr[g], tile_ptr[g + 1])
  for (int i = tid; i < nnz; i += blockDim.x) {
    const uint32_t key = sk[i];
    if (key != 0xFFFFFFFFu) keys_out[__ldcg(tile_ptr + (key >> 15)) + slot[i]] = key;
  }
  if (tid == 0) *nkeys = nvalid;
}

// One CTA: max |X| with 16-byte loads, the power-of-two scale, then the E4M3
// codes of X * s_X (second pass mostly from L1/L2).  n = B d, d a multiple
// of 64.  The codes go out twice: row-major (xq, [B x d]) and by 16-byte
// column chunk (xqt: chunk c of row b at byte (c * ELMO_MAX_BATCH + b) * 16),
// the layout in which a warp reads one chunk of 32 consecutive rows with
// 512 contiguous bytes when it copies X into tensor memory.
__device__ __forceinline__ void prep_x_body(const uint16_t* __restrict__ X, int64_t n, int32_t d,
                                            float* __restrict__ xscale, uint8_t* __restrict__ xq,
                                            uint8_t* __restrict__ xqt) {
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
    const int64_t b = (8 * i) / d, j = (8 * i) % d;           // 8 codes of row b from column j
    *reinterpret_cast<uint2*>(xqt + ((j >> 4) * ELMO_MAX_BATCH + b) * 16 + (j & 15)) = make_uint2(q[0], q[1]);
  }
}

__global__ void __launch_bounds__(kPrepThreads) prep_labels_kernel(const int32_t* __restrict__ rowptr,
                                                                   const int32_t* __restrict__ cols, int32_t B,
                                                                   int32_t nnz, int64_t L,
                                                                   int64_t label_base, int64_t labels_total,
                                                                   uint32_t* __restrict__ keys_out,
                                                                   int32_t* __restrict__ nkeys,
                                                                   int32_t* __restrict__ tile_ptr,
                                                                   int32_t* __restrict__ status) {
  prep_labels_body(rowptr, cols, B, nnz, L, label_base, labels_total, keys_out, nkeys, tile_ptr, status);
}

__global__ void __launch_bounds__(kPrepThreads) prep_x_kernel(const uint16_t* __restrict__ X, int64_t n, int32_t d,
                                                              float* __restrict__ xscale,
                                                              uint8_t* __restrict__ xq, uint8_t* __restrict__ xqt) {
  prep_x_body(X, n, d, xscale, xq, xqt);
}

// Both preparations of an E4M3 step in one launch: CTA 0 the labels, CTA 1 X.
__global__ void __launch_bounds__(kPrepThreads) prep_step_kernel(const int32_t* __restrict__ rowptr,
                                                                 const int32_t* __restrict__ cols, int32_t B,
                                                                 int32_t nnz, int64_t L,
                                                                 int64_t label_base, int64_t labels_total,
                                                                 uint32_t* __restrict__ keys_out,
                                                                 int32_t* __restrict__ nkeys,
                                                                 int32_t* __restrict__ tile_ptr,
                                                                 int32_t* __restrict__ status,
                                                                 const uint16_t* __restrict__ X, int64_t n,
                                                                 int32_t d, float* __restrict__ xscale,
                                                                 uint8_t* __restrict__ xq, uint8_t* __restrict__ xqt) {
  if (blockIdx.x == 0)
    prep_labels_body(rowptr, cols, B, nnz, L, label_base, labels_total, keys_out, nkeys, tile_ptr, status);
  else prep_x_body(X, n, d, xscale, xq, xqt);
}

}  // namespace

cudaError_t launch_prep_step(elmo_head* h, const int32_t* rowptr, const int32_t* cols, int32_t B, int32_t nnz,
                             const uint16_t* X, cudaStream_t s) {
  if (h->dt != ELMO_FP8_E4M3) return launch_prep_labels(h, rowptr, cols, B, nnz, s);
  const size_t smem = (sizeof(uint32_t) + sizeof(uint16_t)) * (size_t)(nnz > 0 ? nnz : 1);
  cudaError_t e = cudaFuncSetAttribute(prep_step_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)((sizeof(uint32_t) + sizeof(uint16_t)) * ELMO_MAX_NNZ));
  if (e != cudaSuccess) return e;
  prep_step_kernel<<<2, kPrepThreads, smem, s>>>(rowptr, cols, B, nnz, h->L, h->label_base, h->labels_total,
                                                 h->keys, h->nkeys, h->tile_ptr, h->status, X,
                                                 (int64_t)B * h->d, h->d, h->xscale, h->xq, h->xqt);
  return cudaGetLastError();
}

cudaError_t launch_prep_labels(elmo_head* h, const int32_t* rowptr, const int32_t* cols, int32_t B,
                               int32_t nnz, cudaStream_t s) {
  const size_t smem = (sizeof(uint32_t) + sizeof(uint16_t)) * (size_t)(nnz > 0 ? nnz : 1);
  cudaError_t e = cudaFuncSetAttribute(prep_labels_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)((sizeof(uint32_t) + sizeof(uint16_t)) * ELMO_MAX_NNZ));
  if (e != cudaSuccess) return e;
  prep_labels_kernel<<<1, kPrepThreads, smem, s>>>(rowptr, cols, B, nnz, h->L, h->label_base, h->labels_total,
                                                   h->keys, h->nkeys, h->tile_ptr, h->status);
  return cudaGetLastError();
}

cudaError_t launch_prep_x(elmo_head* h, const uint16_t* X, int32_t B, cudaStream_t s) {
  prep_x_kernel<<<1, kPrepThreads, 0, s>>>(X, (int64_t)B * h->d, h->d, h->xscale, h->xq, h->xqt);
  return cudaGetLastError();
}

}  // namespace elmo
