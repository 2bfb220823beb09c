// topk_tc.cu -- chunked top-k prediction with tensor-core screening.
//
// P@k evaluation in "ELMO: Efficiency via Low-precision and Peak Memory
// Optimization in Large Output Spaces" (atlas summary, metrics P@1/3/5) ranks
// every label of the head by its score x . w_l.  The reported score of (b, l)
// is the fp32 fused multiply-add chain over j = 0..d-1 in order (x as its bf16
// value, w as its stored value); the ranking is score descending, ties to the
// lower label, NaN last.  That chain cannot run on tensor cores, so the path
// has three stages:
//
//   1. screening (tcgen05): approximate scores S~ = X W^T for all labels, each
//      CTA keeping, per query, the kp best approximate scores of its label
//      range (kp >= k) and the smallest of them, which bounds every score of
//      the range it did not keep;
//   2. selection: per query, the kp best candidates over all ranges, their
//      exact chain scores, the top-k of those, and a certificate: if the k-th
//      exact score exceeds every non-candidate's approximate score by more
//      than the error bound delta, no label outside the candidates can enter
//      the top-k and the result equals the exact one;
//   3. the rows whose certificate fails (ties within delta, non-finite data)
//      are recomputed by the CUDA-core path over all labels.
//
// Operands.  bf16 heads: X (bf16) and W (bf16) go to kind::f16 MMAs as they
// are; every product is exact.  E4M3 heads: each query row is scaled by
// s_b = 2^e (the largest e with 2^e max|x_b| <= 448) and split into
// hi = x s_b truncated to the E4M3 grid and lo = RNE_e4m3(x s_b - hi); two
// kind::f8f6f4 MMAs accumulate hi W^T + lo W^T.  Because hi is a truncation,
// x s_b - hi holds the remaining 4 significant bits of the bf16 value and lo
// is exact unless those bits fall below E4M3's 2^-9 spacing; the residual
// r = x s_b - hi - lo is bounded per row.
//
// Error bound (per query b, any label l):
//   |S_chain(l) - S~(l)| <= (gamma (n1_b + r1_b) + r1_b) max|W|
// with n1_b = sum_j (|hi| + |lo|) / s_b, r1_b = sum_j |r| / s_b, max|W| the
// largest stored magnitude of the head (read each call), and
// gamma = nsteps 2^-20 + 1.01 d 2^-24: the first term allows each of the
// nsteps accumulating MMA instructions an error of 2^-20 of the sum of the
// magnitudes of its products (fp32 accumulation is about 2^-23), the second
// is the standard bound of a d-term fp32 fma chain (unit roundoff 2^-24).
//
// Layout.  The query panel (128 rows) sits in tensor memory as the MMA's A
// operand (columns 0..383: hi then lo, or bf16 X), so shared memory holds a
// 16-stage ring of W k-blocks (64 labels x 128 bytes) and the per-query
// candidate lists; accumulators D[128 queries x 64 labels] are double
// buffered in columns 384..511.  Lane r of D belongs to query r: each
// epilogue thread scans its own row, so the running selection needs no
// communication.  CTAs are (query panel, label range) with the panels of one
// range adjacent in the grid, so they stream the same W tiles together and
// the range crosses HBM about once.
#include <cuda.h>
#include <float.h>

#include "elmo_common.cuh"
#include "elmo_internal.h"
#include "tc_ptx.cuh"

namespace elmo {
namespace {

using namespace tc;

constexpr int kSThreads = 192;                   // warp 0 TMA, warp 1 MMA + TMEM, warps 2-5 epilogue
constexpr int kN = 64;                           // labels per tile (the MMA's N)
constexpr uint32_t kSBox = kN * 128;             // one W k-block: 64 labels x 128 bytes
constexpr int kSStages = 16;
constexpr int kNBuf = 2;                         // accumulator buffers
constexpr uint32_t kSAcc = 384;                  // first accumulator column (A operands below)
constexpr long long kSWait = 4000000000LL;       // ~2 s at 2 GHz
constexpr int32_t kEmpty = 0x7FFFFFFF;
constexpr int kPrepT = 128;
constexpr int kSelThreads = 512;

struct SmemS {
  uint64_t wfull[kSStages], wempty[kSStages], tfull[kNBuf], tempty[kNBuf];
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void record_timeout(int32_t* status, volatile int* abort, int site) {
  *abort = 1;
  if (atomicCAS(status, 0, (int)ELMO_ETIMEOUT) == 0) status[1] = site;
}

// true iff (sa, ia) ranks before (sb, ib): score descending, NaN last, ties to the lower label
__device__ __forceinline__ bool before(float sa, int32_t ia, float sb, int32_t ib) {
  if (ia == kEmpty) return false;
  if (ib == kEmpty) return true;
  const bool na = isnan(sa), nb = isnan(sb);
  if (na != nb) return nb;
  if (!na && sa != sb) return sa > sb;
  return ia < ib;
}

__device__ __forceinline__ float block_sum_ru(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v = __fadd_ru(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  const int w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float t = 0.0f;
  for (int i = 0; i < nw; ++i) t = __fadd_ru(t, red[i]);
  return t;
}

// ---------------------------------------------------------------- stage 0: operands and bounds
// One CTA per query row.  E4M3 heads: s_b, the hi / lo codes and the row's
// n1, r1; bf16 heads: n1 = sum |x| (r1 = 0, X is the operand).  Sums are
// rounded up so that they bound the exact ones.  Block 0 also clears the
// max|W| word and the failed-row count.
template <int kFp8>
__global__ void __launch_bounds__(kPrepT) topk_xprep_kernel(const uint16_t* __restrict__ X, int32_t d,
                                                            uint8_t* __restrict__ xa, uint8_t* __restrict__ xb,
                                                            float* __restrict__ xinv, float* __restrict__ n1,
                                                            float* __restrict__ r1, int32_t* __restrict__ rflag,
                                                            uint32_t* __restrict__ wmax, int32_t* __restrict__ nfail,
                                                            uint32_t* __restrict__ tshare) {
  __shared__ float red[kPrepT / 32];
  __shared__ uint32_t mx;
  const int b = blockIdx.x, tid = threadIdx.x;
  if (b == 0 && tid == 0) { *wmax = 0; *nfail = 0; }
  if (tid == 0) tshare[b] = 0;
  if (tid == 0) mx = 0;
  __syncthreads();
  const uint16_t* xr = X + (size_t)b * d;
  uint32_t m = 0;
  for (int j = tid; j < d; j += blockDim.x) m = max(m, (uint32_t)(xr[j] & 0x7FFFu));
  atomicMax(&mx, m);
  __syncthreads();
  const uint32_t amax_bits = mx;
  const bool nonfinite = amax_bits >= 0x7F80u;
  float s = 1.0f;
  if (kFp8 && !nonfinite && amax_bits != 0) {
    int E;
    const float mant = frexpf(__uint_as_float(amax_bits << 16), &E);   // amax = mant 2^E, mant in [0.5, 1)
    int e = (mant <= 0.875f) ? 9 - E : 8 - E;                          // 448 = 0.875 2^9
    e = max(-126, min(126, e));
    s = ldexpf(1.0f, e);
  }
  float sn = 0.0f, sr = 0.0f;
  for (int j = tid; j < d; j += blockDim.x) {
    const float x = __uint_as_float((uint32_t)xr[j] << 16);
    if (kFp8) {
      const float v = __fmul_rn(x, s);                                   // exact: power-of-two scale
      const float a = fabsf(v);
      // truncation toward zero onto the E4M3 grid: 3 mantissa bits from 2^-6 up, multiples of 2^-9 below
      const float t = a >= 0.015625f ? __uint_as_float(__float_as_uint(a) & 0xFFF00000u)
                                     : __fmul_rn(floorf(__fmul_rn(a, 512.0f)), 0.001953125f);
      const float hi = copysignf(t, v);
      const float lo = __fsub_rn(v, hi);                                 // exact
      const uint32_t ch = pack_e4m3x2(0.0f, hi) & 0xFFu;
      const uint32_t cl = pack_e4m3x2(0.0f, lo) & 0xFFu;
      const float lo_q = e4m3_to_f32((uint8_t)cl);
      xa[(size_t)b * d + j] = (uint8_t)ch;
      xb[(size_t)b * d + j] = (uint8_t)cl;
      sn = __fadd_ru(sn, __fadd_ru(fabsf(hi), fabsf(lo_q)));
      sr = __fadd_ru(sr, fabsf(__fsub_rn(lo, lo_q)));                  // exact difference of two floats near each other
    } else {
      sn = __fadd_ru(sn, fabsf(x));
    }
  }
  sn = block_sum_ru(sn, red);
  sr = block_sum_ru(sr, red);
  if (tid == 0) {
    const float inv = 1.0f / s;                                          // exact: s is a power of two
    xinv[b] = inv;
    n1[b] = __fmul_ru(sn, inv);
    r1[b] = __fmul_ru(sr, inv);
    rflag[b] = nonfinite || !(sn < FLT_MAX) ? 1 : 0;
  }
}

// max over the head of the stored magnitude code (E4M3: code & 0x7F, bf16:
// bits & 0x7FFF); both orders match the magnitudes, and the top codes mark
// NaN (E4M3 0x7F) or inf / NaN (bf16 >= 0x7F80).
template <int kFp8>
__global__ void __launch_bounds__(256) topk_wmax_kernel(const uint4* __restrict__ W, int64_t n16,
                                                        uint32_t* __restrict__ wmax) {
  uint32_t m = 0;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n16; i += (int64_t)gridDim.x * blockDim.x) {
    const uint4 v = W[i];
    if (kFp8) {
      m = __vmaxu4(m, v.x & 0x7F7F7F7Fu); m = __vmaxu4(m, v.y & 0x7F7F7F7Fu);
      m = __vmaxu4(m, v.z & 0x7F7F7F7Fu); m = __vmaxu4(m, v.w & 0x7F7F7F7Fu);
    } else {
      m = __vmaxu2(m, v.x & 0x7FFF7FFFu); m = __vmaxu2(m, v.y & 0x7FFF7FFFu);
      m = __vmaxu2(m, v.z & 0x7FFF7FFFu); m = __vmaxu2(m, v.w & 0x7FFF7FFFu);
    }
  }
  if (kFp8) m = max(max(m & 0xFFu, (m >> 8) & 0xFFu), max((m >> 16) & 0xFFu, m >> 24));
  else m = max(m & 0xFFFFu, m >> 16);
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((threadIdx.x & 31) == 0 && m) atomicMax(wmax, m);
}

// ---------------------------------------------------------------- stage 1: tensor-core screening
// Each epilogue thread keeps its query's best kp approximate scores of the
// CTA's label range as a binary min-heap in shared memory (element i of the
// thread in column r at [i * 128 + r]): the root is the admission threshold,
// and a new score above it replaces the root and sifts down (log2 kp steps).
__device__ __forceinline__ void heap_sift_down(float* hs, int32_t* hl, int r, int i, int kp) {
  const float v = hs[i * 128 + r];
  const int32_t vl = hl[i * 128 + r];
  while (true) {
    int c = 2 * i + 1;
    if (c >= kp) break;
    float cv = hs[c * 128 + r];
    if (c + 1 < kp) {
      const float c2 = hs[(c + 1) * 128 + r];
      if (c2 < cv) { cv = c2; ++c; }
    }
    if (!(cv < v)) break;
    hs[i * 128 + r] = cv;
    hl[i * 128 + r] = hl[c * 128 + r];
    i = c;
  }
  hs[i * 128 + r] = v;
  hl[i * 128 + r] = vl;
}

// Adds (z, lab) as the cnt-th kept score (cnt < kp: the heap is still being
// filled) or in place of the root; returns the new threshold: -inf until kp
// scores are kept, then the smallest kept score.
__device__ __forceinline__ float keep_candidate(float* hs, int32_t* hl, int r, int cnt, int kp, float z, int32_t lab) {
  if (cnt < kp) {
    hs[cnt * 128 + r] = z;
    hl[cnt * 128 + r] = lab;
    if (cnt + 1 < kp) return -INFINITY;
    for (int i = kp / 2 - 1; i >= 0; --i) heap_sift_down(hs, hl, r, i, kp);
    return hs[r];
  }
  hs[r] = z;
  hl[r] = lab;
  heap_sift_down(hs, hl, r, 0, kp);
  return hs[r];
}

// Float <-> unsigned key with the same order (for atomicMax on a threshold);
// key 0 stands for "no threshold yet" (-inf).
__device__ __forceinline__ uint32_t ord_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float ord_value(uint32_t k) {
  return k == 0 ? -INFINITY : __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Every label range of a query publishes its heap threshold (once its heap is
// full) to tshare[query]; all ranges reject scores at or below the largest
// published one.  That is sound for the certificate: a label not kept has an
// approximate score at most the threshold that was in force, and the output
// thr of a range is the largest threshold it used.
// Tiles of 64 labels (the MMA's N) with two accumulator buffers: the A
// operands take 384 of the 512 TMEM columns.
template <int kFp8, int kW5 = 0>
__global__ void __launch_bounds__(kSThreads, 1)
    topk_screen_tc(const __grid_constant__ CUtensorMap tmW, int64_t lbase, int64_t L, int32_t d, int32_t B, int32_t kp,
                   int32_t ngroups, const uint8_t* __restrict__ xa, const uint8_t* __restrict__ xb,
                   const float* __restrict__ xinv, float* __restrict__ cand_s, int32_t* __restrict__ cand_i,
                   float* __restrict__ thr, uint32_t* __restrict__ tshare, float* __restrict__ dump,
                   int32_t* __restrict__ status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = base;                                                   // kSStages W k-blocks
  float* zs = reinterpret_cast<float*>(base + kSStages * kSBox);          // [kN][128] a tile's scores
  float* ls = zs + kN * 128;                                              // [kp][128] kept scores (scaled)
  int32_t* li = reinterpret_cast<int32_t*>(ls + (size_t)kp * 128);        // [kp][128] their labels
  SmemS* S = reinterpret_cast<SmemS*>(li + (size_t)kp * 128);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int P = (B + 127) / 128;
  const int p = blockIdx.x % P, g = blockIdx.x / P;
  const int64_t T = (L + kN - 1) / kN;
  const int64_t t0 = T * g / ngroups, t1 = T * (g + 1) / ngroups;
  const int kbe = kFp8 ? 128 : 64;                  // elements of one 128-byte k-block
  const int nkb = (d + kbe - 1) / kbe;
  const int nops = kFp8 ? 2 : 1;
  const uint32_t opcols = (uint32_t)nkb * 32;       // TMEM columns of one A operand
  volatile int* abort = &S->abort;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSStages; ++s) { mbar_init(&S->wfull[s], 1); mbar_init(&S->wempty[s], 1); }
    for (int b2 = 0; b2 < kNBuf; ++b2) { mbar_init(&S->tfull[b2], 1); mbar_init(&S->tempty[b2], 4); }
    S->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) { tmem_alloc(&S->tmem_base, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S->tmem_base;

  // the query panel into TMEM as the A operand: row r of the panel in lane r
  if (warp >= 2) {
    const int q = warp & 3;
    const int row = p * 128 + q * 32 + lane;
    const size_t rowbytes = (size_t)d * (kFp8 ? 1 : 2);
    for (int op = 0; op < nops; ++op) {
      const uint8_t* src = (op == 0 ? xa : xb) + (size_t)row * rowbytes;
      for (uint32_t c0 = 0; c0 < opcols; c0 += 32) {
        uint32_t v[32];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const size_t off = (size_t)(c0 + 4 * u) * 4;
          uint4 w4 = make_uint4(0u, 0u, 0u, 0u);
          if (row < B && off < rowbytes) w4 = *reinterpret_cast<const uint4*>(src + off);
          v[4 * u] = w4.x; v[4 * u + 1] = w4.y; v[4 * u + 2] = w4.z; v[4 * u + 3] = w4.w;
        }
        tmem_st32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)op * opcols + c0, v);
      }
    }
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp == 0) {
    if (elect_one()) {
      tma_prefetch_desc(&tmW);
      uint32_t it = 0;
      for (int64_t t = t0; t < t1 && !*abort; ++t) {
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = (int)(it % kSStages);
          const uint32_t ph = (it / kSStages) & 1;
          if (!mbar_wait(&S->wempty[s], ph ^ 1, abort, kSWait)) { record_timeout(status, abort, 61); break; }
          mbar_arrive_expect_tx(&S->wfull[s], kSBox);
          tma_load_2d(ring + s * kSBox, &tmW, &S->wfull[s], kb * kbe, (int32_t)(lbase + t * kN));
        }
      }
    }
  } else if (warp == 1) {
    if (elect_one()) {
      const uint32_t idesc = kFp8 ? make_idesc(0, kW5, 0, 0, 128, kN) : make_idesc(1, 1, 0, 0, 128, kN);
      uint32_t it = 0, tc = 0;
      for (int64_t t = t0; t < t1 && !*abort; ++t, ++tc) {
        const uint32_t buf = tc % kNBuf, use = tc / kNBuf;
        if (!mbar_wait(&S->tempty[buf], (use & 1) ^ 1, abort, kSWait)) { record_timeout(status, abort, 62); break; }
        tc_fence_after();
        const uint32_t dcol = tmem + kSAcc + buf * kN;
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = (int)(it % kSStages);
          const uint32_t ph = (it / kSStages) & 1;
          if (!mbar_wait(&S->wfull[s], ph, abort, kSWait)) { record_timeout(status, abort, 63); break; }
          tc_fence_after();
          const uint32_t bsm = smem_u32(ring + s * kSBox);
          for (int op = 0; op < nops; ++op) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {   // 32 bytes of K per MMA: 32 E4M3 or 16 bf16 values
              const uint32_t a = tmem + (uint32_t)op * opcols + (uint32_t)kb * 32 + (uint32_t)k * 8;
              const uint64_t bd = sw128_desc(bsm + k * 32, 16, 1024);
              if (kFp8) mma_e4m3_ts(dcol, a, bd, idesc, (kb | op | k) != 0);
              else mma_bf16_ts(dcol, a, bd, idesc, (kb | op | k) != 0);
            }
          }
          mma_commit(&S->wempty[s]);
        }
        mma_commit(&S->tfull[buf]);
      }
    }
  } else {
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const int row = p * 128 + r;
    const bool live = row < B;
    for (int i = 0; i < kp; ++i) { ls[i * 128 + r] = -INFINITY; li[i * 128 + r] = -1; }
    float tau = -INFINITY;   // the smallest kept (scaled) score once kp are kept
    float tused = -INFINITY; // the largest rejection threshold used so far
    int cnt = 0;
    uint32_t tc = 0;
    for (int64_t t = t0; t < t1 && !*abort; ++t, ++tc) {
      const uint32_t buf = tc % kNBuf, use = tc / kNBuf;
      if (!mbar_wait(&S->tfull[buf], use & 1, abort, kSWait)) { record_timeout(status, abort, 64); break; }
      tc_fence_after();
      uint32_t v[kN / 32][32];
      const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + kSAcc + buf * kN;
#pragma unroll
      for (int h = 0; h < kN / 32; ++h) tmem_ld32(taddr + 32 * h, v[h]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S->tempty[buf]);
      if (!live) continue;
      const int64_t lb = t * kN;
      if (dump) {   // inspection: every screening score of the range, unscaled, no selection
        const float inv = xinv[row];
#pragma unroll
        for (int c = 0; c < kN; ++c)
          if (lb + c < L) dump[(size_t)row * L + lb + c] = __fmul_rn(__uint_as_float(v[c >> 5][c & 31]), inv);
        continue;
      }
      float teff = fmaxf(tau, ord_value(__ldcg(tshare + row)));
      // scores above the threshold, as a bit mask (the selection code below is
      // kept out of the unrolled scan so that it exists once in the binary)
      uint64_t mask = 0;
#pragma unroll
      for (int c = 0; c < kN; ++c)
        mask |= (uint64_t)(__uint_as_float(v[c >> 5][c & 31]) > teff) << c;
      if (lb + kN > L) mask &= L - lb >= 64 ? ~0ull : ((1ull << (L - lb)) - 1);
      if (mask) {
#pragma unroll
        for (int c = 0; c < kN; ++c) zs[c * 128 + r] = __uint_as_float(v[c >> 5][c & 31]);
        while (mask) {
          const int c = __ffsll((long long)mask) - 1;
          mask &= mask - 1;
          const float z = zs[c * 128 + r];
          if (z > teff) {   // labels arrive in order: equal scores never displace an earlier (lower) label
            tau = keep_candidate(ls, li, r, cnt, kp, z, (int32_t)(lb + c));
            if (cnt < kp) ++cnt;
            if (tau > teff) {
              teff = tau;
              atomicMax(tshare + row, ord_key(tau));
            }
          }
        }
      }
      tused = fmaxf(tused, teff);
    }
    if (live && !dump) {
      const float inv = xinv[row];
      const size_t o = ((size_t)row * ngroups + g) * kp;
      for (int i = 0; i < kp; ++i) {
        const int32_t id = li[i * 128 + r];
        cand_s[o + i] = id >= 0 ? __fmul_rn(ls[i * 128 + r], inv) : -INFINITY;
        cand_i[o + i] = id >= 0 ? id : kEmpty;
      }
      thr[(size_t)row * ngroups + g] = __fmul_rn(tused, inv);
    }
  }
  __syncthreads();
  if (*abort) __nanosleep(20000);
  if (warp == 1) { tc_fence_after(); tmem_dealloc(tmem, 512); }
}

// ---------------------------------------------------------------- stage 2: selection, exact rescoring, certificate
__device__ __forceinline__ float w_at(const void* W, int dt, int64_t i) {
  return dt == ELMO_BF16 ? bf16_to_f32(static_cast<const uint16_t*>(W)[i])
         : dt == ELMO_FP8_E5M2 ? e5m2_to_f32(static_cast<const uint8_t*>(W)[i])
                               : e4m3_to_f32(static_cast<const uint8_t*>(W)[i]);
}

// The certificate's bound on |exact chain score - screening score| of a query
// row (any label): (gamma (n1 + r1) + r1) max|W|, rounded up, plus 2^-126 for
// the rescaling of subnormal partial results.
__device__ __forceinline__ float screen_bound(float gamma, float n1, float r1, float maxw) {
  float dl = __fmul_ru(gamma, __fadd_ru(n1, r1));
  dl = __fmul_ru(__fadd_ru(dl, r1), maxw);
  return __fadd_ru(dl, 0x1p-126f);
}

__device__ __forceinline__ float maxw_value(uint32_t wc, int dt) {
  if (dt == ELMO_FP8_E5M2) return wc >= 0x7Cu ? NAN : e5m2_to_f32((uint8_t)wc);   // 0x7C inf, above NaN
  return dt == ELMO_FP8_E4M3 ? (wc >= 0x7Fu ? NAN : e4m3_to_f32((uint8_t)wc))
                             : (wc >= 0x7F80u ? NAN : bf16_to_f32((uint16_t)wc));
}

// Inspection: the bound of every query row (NaN where the row or the head
// holds non-finite values).
__global__ void topk_bound_kernel(int32_t B, float gamma, const float* __restrict__ n1, const float* __restrict__ r1,
                                  const int32_t* __restrict__ rflag, const uint32_t* __restrict__ wmax, int dt,
                                  float* __restrict__ out) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  out[b] = rflag[b] ? NAN : screen_bound(gamma, n1[b], r1[b], maxw_value(*wmax, dt));
}

__global__ void __launch_bounds__(kSelThreads) topk_select_kernel(
    const float* __restrict__ cand_s, const int32_t* __restrict__ cand_i, const float* __restrict__ thr,
    int32_t ngroups, int32_t kp, int32_t k, int32_t npow2, const uint16_t* __restrict__ X, const void* __restrict__ W,
    int dt, int32_t d, float gamma, const float* __restrict__ n1, const float* __restrict__ r1,
    const int32_t* __restrict__ rflag, const uint32_t* __restrict__ wmax, int32_t* __restrict__ idx,
    float* __restrict__ score, int32_t* __restrict__ fail_rows, int32_t* __restrict__ nfail) {
  extern __shared__ float sel[];
  float* ss = sel;                                            // [npow2] approximate scores
  int32_t* si = reinterpret_cast<int32_t*>(ss + npow2);       // [npow2] labels
  float* xs = reinterpret_cast<float*>(si + npow2);           // [d] the query row
  float* es = xs + d;                                         // [kp] exact scores
  int32_t* ei = reinterpret_cast<int32_t*>(es + kp);          // [kp] their labels
  float* rs = reinterpret_cast<float*>(ei + kp);              // [kp] ranked scores
  int32_t* ri = reinterpret_cast<int32_t*>(rs + kp);          // [kp] ranked labels
  __shared__ float umax[kSelThreads / 32];
  __shared__ int nzs[kSelThreads / 32];
  const int b = blockIdx.x, tid = threadIdx.x;
  const int n = ngroups * kp;
  for (int i = tid; i < npow2; i += blockDim.x) {
    float sv = -INFINITY;
    int32_t iv = kEmpty;
    if (i < n) {
      iv = cand_i[(size_t)b * n + i];
      if (iv != kEmpty) sv = cand_s[(size_t)b * n + i];
    }
    ss[i] = sv;
    si[i] = iv;
  }
  for (int j = tid; j < d; j += blockDim.x) xs[j] = bf16_to_f32(X[(size_t)b * d + j]);
  float u = -INFINITY;
  for (int gg = tid; gg < ngroups; gg += blockDim.x) u = fmaxf(u, thr[(size_t)b * ngroups + gg]);
  for (int o = 16; o > 0; o >>= 1) u = fmaxf(u, __shfl_xor_sync(0xFFFFFFFFu, u, o));
  if ((tid & 31) == 0) umax[tid >> 5] = u;
  __syncthreads();
  // bitonic sort of the candidates into ranking order (empty slots last)
  for (int size = 2; size <= npow2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < npow2; i += blockDim.x) {
        const int j = i ^ stride;
        if (j > i) {
          const float a = ss[i], c = ss[j];
          const int32_t ia = si[i], ic = si[j];
          const bool up = (i & size) == 0;
          if (before(c, ic, a, ia) == up) { ss[i] = c; ss[j] = a; si[i] = ic; si[j] = ia; }
        }
      }
      __syncthreads();
    }
  }
  int nz = 0;
  for (int i = tid; i < n; i += blockDim.x) nz += si[i] != kEmpty;
  for (int o = 16; o > 0; o >>= 1) nz += __shfl_xor_sync(0xFFFFFFFFu, nz, o);
  if ((tid & 31) == 0) nzs[tid >> 5] = nz;
  __syncthreads();
  nz = 0;
  u = -INFINITY;
  for (int w = 0; w < kSelThreads / 32; ++w) { nz += nzs[w]; u = fmaxf(u, umax[w]); }
  const int m = nz < kp ? nz : kp;                      // candidates rescored
  if (nz > kp) u = fmaxf(u, ss[kp]);                     // the best candidate left out
  // exact chain scores of the candidates
  if (tid < m) {
    const int64_t l = si[tid];
    float acc = 0.0f;
    if (dt == ELMO_FP8_E4M3 || dt == ELMO_FP8_E5M2) {
      const uint4* wr = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(W) + l * d);
      for (int j0 = 0; j0 < d; j0 += 16) {
        const uint4 q4 = wr[j0 >> 4];
        const uint32_t wq[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float f4[4];
          if (dt == ELMO_FP8_E5M2) e5m2x4_to_f32(wq[e], f4);
          else e4m3x4_to_f32(wq[e], f4);
#pragma unroll
          for (int i = 0; i < 4; ++i) acc = __fmaf_rn(xs[j0 + 4 * e + i], f4[i], acc);
        }
      }
    } else {
      for (int j = 0; j < d; ++j) acc = __fmaf_rn(xs[j], w_at(W, dt, l * d + j), acc);
    }
    es[tid] = acc;
    ei[tid] = (int32_t)l;
  }
  __syncthreads();
  if (tid < m) {
    int rank = 0;
    for (int o = 0; o < m; ++o) rank += (o != tid) && before(es[o], ei[o], es[tid], ei[tid]);
    rs[rank] = es[tid];
    ri[rank] = ei[tid];
  }
  __syncthreads();
  if (tid == 0) {
    const float maxw = maxw_value(*wmax, dt);
    bool ok = rflag[b] == 0 && m >= k && !isnan(maxw);
    if (ok) ok = !isnan(rs[k - 1]);
    if (ok && u != -INFINITY) ok = rs[k - 1] > __fadd_ru(u, screen_bound(gamma, n1[b], r1[b], maxw));
    if (ok) {
      for (int q = 0; q < k; ++q) {
        idx[(size_t)b * k + q] = ri[q];
        score[(size_t)b * k + q] = rs[q];
      }
    } else {
      fail_rows[atomicAdd(nfail, 1)] = b;
    }
  }
}

struct TopkLayout {
  int P, G, kp, npow2, N;
  size_t xa, xb, xinv, n1, r1, rflag, wmax, nfail, fail, cs, ci, thr, tshare, simt, total;
};

TopkLayout topk_layout(const elmo_head* h, int32_t B, int32_t k) {
  TopkLayout o{};
  const bool fp8 = h->dt == ELMO_FP8_E4M3;
  o.P = (B + 127) / 128;
  o.N = kN;
  const int64_t T = (h->L + o.N - 1) / o.N;
  int64_t G = h->num_sms / o.P;
  if (G < 1) G = 1;
  if (G > T) G = T;
  o.G = (int)G;
  o.kp = k <= 8 ? 16 : (k <= 16 ? 32 : 64);
  o.npow2 = 1;
  while (o.npow2 < o.G * o.kp) o.npow2 <<= 1;
  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t at = off; off += (bytes + 255) / 256 * 256; return at; };
  o.xa = take(fp8 ? (size_t)B * h->d : 0);
  o.xb = take(fp8 ? (size_t)B * h->d : 0);
  o.xinv = take(sizeof(float) * B);
  o.n1 = take(sizeof(float) * B);
  o.r1 = take(sizeof(float) * B);
  o.rflag = take(sizeof(int32_t) * B);
  o.wmax = take(sizeof(uint32_t));
  o.nfail = take(sizeof(int32_t));
  o.fail = take(sizeof(int32_t) * B);
  o.cs = take(sizeof(float) * (size_t)B * o.G * o.kp);
  o.ci = take(sizeof(int32_t) * (size_t)B * o.G * o.kp);
  o.thr = take(sizeof(float) * (size_t)B * o.G);
  o.tshare = take(sizeof(uint32_t) * (size_t)B);
  o.simt = take(topk_simt_workspace_bytes(h, B, k));
  o.total = off;
  return o;
}

constexpr size_t kScreenSmem = 1024 + kSStages * kSBox + sizeof(float) * kN * 128 + 2 * sizeof(float) * 64 * 128 +
                                sizeof(SmemS);
static_assert(kScreenSmem <= 232448, "screening kernel shared memory");

}  // namespace

bool topk_tc_supported(const elmo_head* h) {
  // the A operands (E4M3 hi and lo: 2 d bytes; bf16 X: 2 d bytes) must fit the
  // 384 TMEM columns (1536 bytes per lane) below the accumulators
  return h->d % 64 == 0 && h->d <= 768 && h->L <= (int64_t)INT32_MAX;
}

size_t topk_tc_workspace_bytes(const elmo_head* h, int32_t B, int32_t k) { return topk_layout(h, B, k).total; }

cudaError_t launch_topk_tc(elmo_head* h, const uint16_t* X, int32_t B, int32_t k, int32_t* idx, float* score,
                           cudaStream_t s) {
  const bool fp8 = h->dt == ELMO_FP8_E4M3;
  const TopkLayout o = topk_layout(h, B, k);
  uint8_t* ws = static_cast<uint8_t*>(h->cand);
  uint8_t* xa = ws + o.xa;
  uint8_t* xb = ws + o.xb;
  float* xinv = reinterpret_cast<float*>(ws + o.xinv);
  float* n1 = reinterpret_cast<float*>(ws + o.n1);
  float* r1 = reinterpret_cast<float*>(ws + o.r1);
  int32_t* rflag = reinterpret_cast<int32_t*>(ws + o.rflag);
  uint32_t* wmax = reinterpret_cast<uint32_t*>(ws + o.wmax);
  int32_t* nfail = reinterpret_cast<int32_t*>(ws + o.nfail);
  int32_t* fail = reinterpret_cast<int32_t*>(ws + o.fail);
  float* cs = reinterpret_cast<float*>(ws + o.cs);
  int32_t* ci = reinterpret_cast<int32_t*>(ws + o.ci);
  float* thr = reinterpret_cast<float*>(ws + o.thr);
  uint32_t* tshare = reinterpret_cast<uint32_t*>(ws + o.tshare);

  // stage 0
  cudaError_t e;
  {
    KernelScope sc(h, ELMO_K_PREP, s, 1);
    if (fp8) topk_xprep_kernel<1><<<B, kPrepT, 0, s>>>(X, h->d, xa, xb, xinv, n1, r1, rflag, wmax, nfail, tshare);
    else topk_xprep_kernel<0><<<B, kPrepT, 0, s>>>(X, h->d, xa, xb, xinv, n1, r1, rflag, wmax, nfail, tshare);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return e;

  // max|W| streams the head from HBM while the screening kernel (tensor-bound,
  // light on HBM) runs: a second stream, forked after the clears of stage 0
  // and joined before the selection
  if (!h->side) {
    if ((e = cudaStreamCreateWithFlags(&h->side, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&h->fork, cudaEventDisableTiming)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&h->join, cudaEventDisableTiming)) != cudaSuccess) return e;
  }
  if ((e = cudaEventRecord(h->fork, s)) != cudaSuccess) return e;
  if ((e = cudaStreamWaitEvent(h->side, h->fork, 0)) != cudaSuccess) return e;
  {
    KernelScope sc(h, ELMO_K_PREP, h->side, 1);
    const int64_t n16 = h->L * (int64_t)h->d * (fp8 ? 1 : 2) / 16;
    const int wgrid = h->num_sms * 4;
    if (fp8) topk_wmax_kernel<1><<<wgrid, 256, 0, h->side>>>(static_cast<const uint4*>(h->W), n16, wmax);
    else topk_wmax_kernel<0><<<wgrid, 256, 0, h->side>>>(static_cast<const uint4*>(h->W), n16, wmax);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = cudaEventRecord(h->join, h->side)) != cudaSuccess) return e;

  // stage 1
  CUtensorMap tmW;
  const int eb = fp8 ? 1 : 2;
  e = make_tma_map_2d(&tmW, h->W, eb, (uint64_t)h->d, (uint64_t)h->L, (uint64_t)h->d, (uint32_t)o.N);
  if (e != cudaSuccess) return e;
  const size_t smem = 1024 + kSStages * kSBox + sizeof(float) * kN * 128 + 2 * sizeof(float) * (size_t)o.kp * 128 +
                      sizeof(SmemS);
  auto ks = fp8 ? (h->w_e5m2 ? topk_screen_tc<1, 1> : topk_screen_tc<1>) : topk_screen_tc<0>;
  e = cudaFuncSetAttribute(ks, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kScreenSmem);
  if (e != cudaSuccess) return e;
  {
    KernelScope sc(h, ELMO_K_TOPK_SCORE, s, 1);
    ks<<<o.P * o.G, kSThreads, smem, s>>>(tmW, (int64_t)0, h->L, h->d, B, o.kp, o.G,
                                          fp8 ? xa : reinterpret_cast<const uint8_t*>(X), xb, xinv, cs, ci, thr, tshare,
                                          nullptr, h->status);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  // stage 2
  const int nkb = (h->d * eb + 127) / 128;
  const int nsteps = (fp8 ? 2 : 1) * nkb * 4;
  const float gamma = (float)((double)nsteps * 0x1p-20 + 1.01 * (double)h->d * 0x1p-24);
  const size_t ssmem = sizeof(float) * (2 * (size_t)o.npow2 + (size_t)h->d + 4 * (size_t)o.kp);
  e = cudaFuncSetAttribute(topk_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ssmem);
  if (e != cudaSuccess) return e;
  if ((e = cudaStreamWaitEvent(s, h->join, 0)) != cudaSuccess) return e;
  KernelScope sc(h, ELMO_K_TOPK_MERGE, s, 3);
  topk_select_kernel<<<B, kSelThreads, ssmem, s>>>(cs, ci, thr, o.G, o.kp, k, o.npow2, X, h->W, w_format(h), h->d,
                                                   gamma, n1, r1, rflag, wmax, idx, score, fail, nfail);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  // stage 3: the rows the certificate did not clear (a device-side list; usually empty)
  return launch_topk_simt_rows(h, X, B, k, fail, nfail, ws + o.simt, idx, score, s);
}

cudaError_t topk_uncertified_rows(elmo_head* h, int32_t B, int32_t k, int32_t* rows, cudaStream_t s) {
  const TopkLayout o = topk_layout(h, B, k);
  cudaError_t e = cudaMemcpyAsync(rows, static_cast<uint8_t*>(h->cand) + o.nfail, sizeof(int32_t),
                                  cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return e;
  return cudaStreamSynchronize(s);
}

cudaError_t launch_topk_screen_dump(elmo_head* h, const uint16_t* X, int32_t B, int64_t l0, int64_t l1, float* S,
                                    float* bound, cudaStream_t s) {
  const bool fp8 = h->dt == ELMO_FP8_E4M3;
  const TopkLayout o = topk_layout(h, B, 1);
  uint8_t* ws = static_cast<uint8_t*>(h->cand);
  uint8_t* xa = ws + o.xa;
  uint8_t* xb = ws + o.xb;
  float* xinv = reinterpret_cast<float*>(ws + o.xinv);
  float* n1 = reinterpret_cast<float*>(ws + o.n1);
  float* r1 = reinterpret_cast<float*>(ws + o.r1);
  int32_t* rflag = reinterpret_cast<int32_t*>(ws + o.rflag);
  uint32_t* wmax = reinterpret_cast<uint32_t*>(ws + o.wmax);
  int32_t* nfail = reinterpret_cast<int32_t*>(ws + o.nfail);
  uint32_t* tshare = reinterpret_cast<uint32_t*>(ws + o.tshare);
  h->launches += 4;
  if (fp8) topk_xprep_kernel<1><<<B, kPrepT, 0, s>>>(X, h->d, xa, xb, xinv, n1, r1, rflag, wmax, nfail, tshare);
  else topk_xprep_kernel<0><<<B, kPrepT, 0, s>>>(X, h->d, xa, xb, xinv, n1, r1, rflag, wmax, nfail, tshare);
  const int64_t n16 = h->L * (int64_t)h->d * (fp8 ? 1 : 2) / 16;
  if (fp8) topk_wmax_kernel<1><<<h->num_sms * 4, 256, 0, s>>>(static_cast<const uint4*>(h->W), n16, wmax);
  else topk_wmax_kernel<0><<<h->num_sms * 4, 256, 0, s>>>(static_cast<const uint4*>(h->W), n16, wmax);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap tmW;
  const int eb = fp8 ? 1 : 2;
  e = make_tma_map_2d(&tmW, h->W, eb, (uint64_t)h->d, (uint64_t)h->L, (uint64_t)h->d, (uint32_t)o.N);
  if (e != cudaSuccess) return e;
  auto ks = fp8 ? (h->w_e5m2 ? topk_screen_tc<1, 1> : topk_screen_tc<1>) : topk_screen_tc<0>;
  e = cudaFuncSetAttribute(ks, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kScreenSmem);
  if (e != cudaSuccess) return e;
  const int64_t nl = l1 - l0;
  int64_t G = h->num_sms / o.P;
  const int64_t T = (nl + kN - 1) / kN;
  if (G > T) G = T;
  if (G < 1) G = 1;
  const size_t smem = 1024 + kSStages * kSBox + sizeof(float) * kN * 128 + 2 * sizeof(float) * 16 * 128 +
                      sizeof(SmemS);
  ks<<<o.P * (int)G, kSThreads, smem, s>>>(tmW, l0, nl, h->d, B, 16, (int32_t)G,
                                           fp8 ? xa : reinterpret_cast<const uint8_t*>(X), xb, xinv, nullptr, nullptr,
                                           nullptr, tshare, S, h->status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int nkb = (h->d * eb + 127) / 128;
  const int nsteps = (fp8 ? 2 : 1) * nkb * 4;
  const float gamma = (float)((double)nsteps * 0x1p-20 + 1.01 * (double)h->d * 0x1p-24);
  topk_bound_kernel<<<(B + 127) / 128, 128, 0, s>>>(B, gamma, n1, r1, rflag, wmax, w_format(h), bound);
  return cudaGetLastError();
}

}  // namespace elmo
