// step_tc.cu -- the ELMO classifier-head step on sm_100a tensor cores.
//
// "ELMO: Efficiency via Low-precision and Peak Memory Optimization in Large
// Output Spaces", atlas summary "Approach": per label chunk the classifier
// gradient is fused with the momentum-free SGD update and applied with
// stochastic rounding, without FP32 master weights; chunking bounds the
// transient memory.  A label range (at most a few tens of MB of W and G, so
// that both stay in L2 between the two kernels) is processed by:
//
//   logits_grad_tc : Z^T[128 labels x B] = W_tile X^T on tcgen05 (TMEM
//                    accumulators, TMA-fed shared-memory operands), then
//                    G = sigmoid(Z) - Y formed in-tile by four epilogue warps
//                    and written as the next contraction's operand (bf16, or
//                    E4M3 of 2^8 G).
//   update_tc      : per (label tile, 128-column slice of d):
//                    dX^T[slice] += W_tile[:, slice]^T G_tile^T   (old W, TMEM-resident
//                                                                  across the CTA's tiles)
//                    dW = G_tile^T X[:, slice]                    (TMEM)
//                    W  = SR(W - lr dW)                           (epilogue, in place)
//                    one fp32 atomic flush of dX^T per run of tiles.
//
// Warp roles (192 threads): warp 0 issues TMA loads, warp 1 allocates TMEM and
// issues MMAs (one elected thread), warps 2-5 are the epilogue (warp w reads
// TMEM lanes 32*(w%4) .. +31).  Every wait is bounded; a wait that runs out
// records ELMO_ETIMEOUT in the status word and the CTA winds down.
#include <cuda.h>

#include "elmo_common.cuh"
#include "elmo_internal.h"
#include "tc_ptx.cuh"

namespace elmo {
namespace {

using namespace tc;

constexpr int kThreads = 192;
constexpr long long kWaitCycles = 4000000000LL;   // ~2 s at 2 GHz: only a broken pipeline waits this long
constexpr uint32_t kBox = 16384;                  // one 128-row x 128-byte TMA box

__device__ __forceinline__ void record_timeout(int32_t* status, volatile int* abort, int site) {
  *abort = 1;
  if (atomicCAS(status, 0, (int)ELMO_ETIMEOUT) == 0) status[1] = site;
}

// Positives of label `l` among the sorted keys (label << 8 | sample) in
// [k0, k1): a 256-bit sample mask.
__device__ __forceinline__ void label_mask(const uint32_t* __restrict__ keys, int k0, int k1, int64_t l,
                                           uint32_t (&m)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = 0;
  for (int i = k0; i < k1; ++i) {
    const uint32_t key = __ldg(keys + i);
    if ((int64_t)(key >> 8) == l) {
      const uint32_t b = key & 0xFFu;
#pragma unroll
      for (int w = 0; w < 8; ++w)
        if ((b >> 5) == (uint32_t)w) m[w] |= 1u << (b & 31);
    }
  }
}

// First key whose label is >= lab.
__device__ __forceinline__ int lower_bound_label(const uint32_t* keys, int n, int64_t lab) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if ((int64_t)(__ldg(keys + mid) >> 8) < lab) lo = mid + 1; else hi = mid;
  }
  return lo;
}

__device__ __forceinline__ float sigmoidf_fast(float z) { return __frcp_rn(1.0f + __expf(-z)); }

// ============================================================================
// Kernel A: logits and gradient operand of a label range.
// ============================================================================
constexpr int kStagesA = 4;
constexpr uint32_t kStageABytes = kBox + 32768;   // W k-block + X k-block (<= 256 rows)

struct SmemA {
  uint64_t full[kStagesA], empty[kStagesA], tfull[2], tempty[2];
  uint32_t tmem_base;
  int abort;
};

template <int kFp8>
__global__ void __launch_bounds__(kThreads, 1)
    logits_grad_tc(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX, int64_t L,
                   int32_t d, int32_t B, int32_t Bp, int64_t l0, int64_t l1, const uint32_t* __restrict__ keys,
                   const int32_t* __restrict__ nkeys, const float* __restrict__ xscale, void* __restrict__ gbuf,
                   float* __restrict__ Zout, float* __restrict__ Gout, int32_t* __restrict__ status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  SmemA* S = reinterpret_cast<SmemA*>(base + kStagesA * kStageABytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t span = l1 - l0;
  const int ntiles = (int)((span + 127) / 128);
  const int kb_elems = kFp8 ? 128 : 64;
  const int nkb = (d + kb_elems - 1) / kb_elems;
  const uint32_t x_bytes = (uint32_t)Bp * 128u;
  volatile int* abort = &S->abort;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesA; ++s) { mbar_init(&S->full[s], 1); mbar_init(&S->empty[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&S->tfull[b], 1); mbar_init(&S->tempty[b], 4); }
    S->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) { tmem_alloc(&S->tmem_base, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S->tmem_base;

  if (warp == 0) {
    if (elect_one()) {
      tma_prefetch_desc(&tmW);
      tma_prefetch_desc(&tmX);
      uint32_t it = 0;
      for (int t = blockIdx.x; t < ntiles && !*abort; t += gridDim.x) {
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % kStagesA;
          const uint32_t ph = (it / kStagesA) & 1;
          if (!mbar_wait(&S->empty[s], ph ^ 1, abort, kWaitCycles)) { record_timeout(status, abort, 1); break; }
          uint8_t* a = base + s * kStageABytes;
          mbar_arrive_expect_tx(&S->full[s], kBox + x_bytes);
          tma_load_2d(a, &tmW, &S->full[s], kb * kb_elems, (int32_t)(l0 + (int64_t)t * 128));
          tma_load_2d(a + kBox, &tmX, &S->full[s], kb * kb_elems, 0);
        }
      }
    }
  } else if (warp == 1) {
    if (elect_one()) {
      const uint32_t idesc = kFp8 ? make_idesc(0, 0, 0, 0, 128, (uint32_t)Bp) : make_idesc(1, 1, 0, 0, 128, (uint32_t)Bp);
      uint32_t it = 0, tc = 0;
      for (int t = blockIdx.x; t < ntiles && !*abort; t += gridDim.x, ++tc) {
        const uint32_t buf = tc & 1, use = tc >> 1;
        if (!mbar_wait(&S->tempty[buf], (use & 1) ^ 1, abort, kWaitCycles)) { record_timeout(status, abort, 2); break; }
        tc_fence_after();
        const uint32_t dcol = tmem + buf * 256;
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % kStagesA;
          const uint32_t ph = (it / kStagesA) & 1;
          if (!mbar_wait(&S->full[s], ph, abort, kWaitCycles)) { record_timeout(status, abort, 3); break; }
          tc_fence_after();
          const uint32_t a = smem_u32(base + s * kStageABytes);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t ad = sw128_desc(a + k * 32, 16, 1024);
            const uint64_t bd = sw128_desc(a + kBox + k * 32, 16, 1024);
            if (kFp8) mma_e4m3(dcol, ad, bd, idesc, (kb | k) != 0);
            else mma_bf16(dcol, ad, bd, idesc, (kb | k) != 0);
          }
          mma_commit(&S->empty[s]);
        }
        mma_commit(&S->tfull[buf]);
      }
    }
  } else {
    // epilogue: thread owns TMEM lane (label row) 32*(warp%4) + lane
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const float inv_sx = kFp8 ? xscale[1] : 1.0f;
    const int nk = *nkeys;
    uint32_t tc = 0;
    for (int t = blockIdx.x; t < ntiles && !*abort; t += gridDim.x, ++tc) {
      const uint32_t buf = tc & 1, use = tc >> 1;
      const int64_t lt0 = l0 + (int64_t)t * 128;
      const int64_t l = lt0 + row;
      const bool valid = (l - l0) < span;
      const int k0 = lower_bound_label(keys, nk, lt0);
      const int k1 = lower_bound_label(keys, nk, lt0 + 128);
      uint32_t mask[8];
      label_mask(keys, k0, k1, l, mask);
      if (!mbar_wait(&S->tfull[buf], use & 1, abort, kWaitCycles)) { record_timeout(status, abort, 4); break; }
      tc_fence_after();
      const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + buf * 256;
      for (int c = 0; c < Bp / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(taddr + c * 32, r);
        tmem_wait_ld();
        uint32_t mw = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) mw = (c == w) ? mask[w] : mw;
        float z[32], g[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          z[i] = __fmul_rn(__uint_as_float(r[i]), inv_sx);
          const float y = ((mw >> i) & 1u) ? 1.0f : 0.0f;
          g[i] = (c * 32 + i < B) ? sigmoidf_fast(z[i]) - y : 0.0f;
        }
        if (valid) {
          if (kFp8) {
            uint32_t packed[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              uint32_t v = 0;
#pragma unroll
              for (int e = 0; e < 4; ++e) v |= (uint32_t)f32_to_e4m3_rn(g[4 * i + e] * 256.0f) << (8 * e);
              packed[i] = v;
            }
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(gbuf) + (size_t)(l - l0) * Bp + c * 32);
            dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
            dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
            if (Gout) {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (c * 32 + i < B)
                  Gout[(size_t)(l - l0) * B + c * 32 + i] =
                      e4m3_to_f32((uint8_t)(packed[i >> 2] >> (8 * (i & 3)))) * 0.00390625f;
            }
          } else {
            uint32_t packed[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              packed[i] = (uint32_t)f32_to_bf16_rn(g[2 * i]) | ((uint32_t)f32_to_bf16_rn(g[2 * i + 1]) << 16);
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(gbuf) + (size_t)(l - l0) * Bp + c * 32);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
            if (Gout) {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (c * 32 + i < B)
                  Gout[(size_t)(l - l0) * B + c * 32 + i] = bf16_to_f32((uint16_t)(packed[i >> 1] >> (16 * (i & 1))));
            }
          }
          if (Zout) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (c * 32 + i < B) Zout[(size_t)(l - l0) * B + c * 32 + i] = z[i];
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S->tempty[buf]);
    }
  }
  __syncthreads();
  if (*abort) __nanosleep(20000);   // let copies in flight land before the shared memory goes away
  if (warp == 1) { tc_fence_after(); tmem_dealloc(tmem, 512); }
}

// ============================================================================
// Kernel B: input gradient, weight gradient and the SR update.
// ============================================================================
constexpr int kWSlots = 2;
constexpr int kGSlots = 3;
constexpr uint32_t kXBytes = 2 * 32768;     // X[:, slice]: up to two 64-column boxes of up to 256 rows
constexpr uint32_t kWSlotBytes = 2 * kBox;  // W[tile, slice]
constexpr uint32_t kGSlotBytes = 2 * kBox;  // one part of G^T[tile]: two boxes of 128 bytes of samples

struct SmemB {
  uint64_t xfull, xempty, dxfull, dxempty;
  uint64_t wfull[kWSlots], wempty[kWSlots];
  uint64_t gfull[kGSlots], gempty[kGSlots];
  uint64_t dwfull[2], dwempty[2];
  uint32_t tmem_base;
  int abort;
};

struct UnitRange {
  int u0, u1;  // [u0, u1) of units ordered (slice-major, tile-minor)
};

template <int kFp8>
__global__ void __launch_bounds__(kThreads, 1)
    update_tc(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
              const __grid_constant__ CUtensorMap tmG, void* __restrict__ Wglob, int64_t L, int32_t d, int32_t B,
              int32_t Bp, int64_t l0, int64_t l1, const float* __restrict__ xscale, float lr, uint64_t seed,
              uint64_t step, float* __restrict__ dX, int32_t* __restrict__ status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xs = base;
  uint8_t* ws = xs + kXBytes;
  uint8_t* gs = ws + kWSlots * kWSlotBytes;
  SmemB* S = reinterpret_cast<SmemB*>(gs + kGSlots * kGSlotBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t span = l1 - l0;
  const int T = (int)((span + 127) / 128);
  const int nD = (d + 127) / 128;
  const int U = T * nD;
  const int u0 = (int)((int64_t)U * blockIdx.x / gridDim.x);
  const int u1 = (int)((int64_t)U * (blockIdx.x + 1) / gridDim.x);
  constexpr int kElem = kFp8 ? 1 : 2;
  constexpr int kBoxCols = 128 / kElem;               // elements per 128-byte box row
  constexpr int kPart = kFp8 ? 256 : 128;             // samples per G part
  constexpr int kK = kFp8 ? 32 : 16;                  // MMA K
  const int nparts = (Bp + kPart - 1) / kPart;
  volatile int* abort = &S->abort;

  if (threadIdx.x == 0) {
    mbar_init(&S->xfull, 1); mbar_init(&S->xempty, 1);
    mbar_init(&S->dxfull, 1); mbar_init(&S->dxempty, 4);
    for (int s = 0; s < kWSlots; ++s) { mbar_init(&S->wfull[s], 1); mbar_init(&S->wempty[s], 4); }
    for (int s = 0; s < kGSlots; ++s) { mbar_init(&S->gfull[s], 1); mbar_init(&S->gempty[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&S->dwfull[b], 1); mbar_init(&S->dwempty[b], 4); }
    S->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) { tmem_alloc(&S->tmem_base, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S->tmem_base;

  if (warp == 0) {
    if (elect_one()) {
      tma_prefetch_desc(&tmW); tma_prefetch_desc(&tmX); tma_prefetch_desc(&tmG);
      int run = 0;
      uint32_t wit = 0, git = 0;
      for (int u = u0; u < u1 && !*abort;) {
        const int D = u / T;
        const int ue = min(u1, (D + 1) * T);
        const int D0 = D * 128;
        // X[:, slice] for this run, once the previous run's MMAs are done with it
        if (!mbar_wait(&S->xempty, (run & 1) ^ 1, abort, kWaitCycles)) { record_timeout(status, abort, 11); break; }
        {
          int nb = 0;
          for (int q = 0; q < 128 / kBoxCols; ++q) nb += (D0 + q * kBoxCols < d);
          mbar_arrive_expect_tx(&S->xfull, (uint32_t)nb * (uint32_t)Bp * 128u);
          for (int q = 0; q < 128 / kBoxCols; ++q)
            if (D0 + q * kBoxCols < d) tma_load_2d(xs + q * 32768, &tmX, &S->xfull, D0 + q * kBoxCols, 0);
        }
        for (; u < ue && !*abort; ++u) {
          const int t = u - D * T;
          const int32_t row0 = (int32_t)(l0 + (int64_t)t * 128);
          {
            const int s = wit % kWSlots;
            const uint32_t ph = (wit / kWSlots) & 1;
            ++wit;
            if (!mbar_wait(&S->wempty[s], ph ^ 1, abort, kWaitCycles)) { record_timeout(status, abort, 12); break; }
            int nb = 0;
            for (int q = 0; q < 128 / kBoxCols; ++q) nb += (D0 + q * kBoxCols < d);
            mbar_arrive_expect_tx(&S->wfull[s], (uint32_t)nb * kBox);
            for (int q = 0; q < 128 / kBoxCols; ++q)
              if (D0 + q * kBoxCols < d) tma_load_2d(ws + s * kWSlotBytes + q * kBox, &tmW, &S->wfull[s], D0 + q * kBoxCols, row0);
          }
          for (int p = 0; p < nparts; ++p) {
            const int s = git % kGSlots;
            const uint32_t ph = (git / kGSlots) & 1;
            ++git;
            if (!mbar_wait(&S->gempty[s], ph ^ 1, abort, kWaitCycles)) { record_timeout(status, abort, 13); break; }
            const int c0 = p * kPart;
            int nb = 0;
            for (int q = 0; q < 2; ++q) nb += (c0 + q * kBoxCols < Bp);
            mbar_arrive_expect_tx(&S->gfull[s], (uint32_t)nb * kBox);
            for (int q = 0; q < 2; ++q)
              if (c0 + q * kBoxCols < Bp)
                tma_load_2d(gs + s * kGSlotBytes + q * kBox, &tmG, &S->gfull[s], c0 + q * kBoxCols, t * 128);
          }
        }
        ++run;
      }
    }
  } else if (warp == 1) {
    if (elect_one()) {
      const uint32_t idesc_dw = kFp8 ? make_idesc(0, 0, 0, 1, 128, 128) : make_idesc(1, 1, 0, 1, 128, 128);
      int run = 0;
      uint32_t wit = 0, git = 0, dwit = 0;
      for (int u = u0; u < u1 && !*abort;) {
        const int D = u / T;
        const int ue = min(u1, (D + 1) * T);
        if (!mbar_wait(&S->xfull, run & 1, abort, kWaitCycles)) { record_timeout(status, abort, 21); break; }
        if (!mbar_wait(&S->dxempty, (run & 1) ^ 1, abort, kWaitCycles)) { record_timeout(status, abort, 22); break; }
        tc_fence_after();
        bool first = true;
        for (; u < ue && !*abort; ++u) {
          const int sw = wit % kWSlots;
          const uint32_t phw = (wit / kWSlots) & 1;
          ++wit;
          const uint32_t db = dwit & 1, duse = dwit >> 1;
          ++dwit;
          if (!mbar_wait(&S->wfull[sw], phw, abort, kWaitCycles)) { record_timeout(status, abort, 23); break; }
          if (!mbar_wait(&S->dwempty[db], (duse & 1) ^ 1, abort, kWaitCycles)) { record_timeout(status, abort, 24); break; }
          tc_fence_after();
          const uint32_t wa = smem_u32(ws + sw * kWSlotBytes);
          const uint32_t xa = smem_u32(xs);
          for (int p = 0; p < nparts; ++p) {
            const int sg = git % kGSlots;
            const uint32_t phg = (git / kGSlots) & 1;
            ++git;
            if (!mbar_wait(&S->gfull[sg], phg, abort, kWaitCycles)) { record_timeout(status, abort, 25); break; }
            tc_fence_after();
            const uint32_t ga = smem_u32(gs + sg * kGSlotBytes);
            const int np = min(kPart, Bp - p * kPart);   // samples in this part (multiple of 32)
            // dX^T[slice, part] += W^T G^T : M = 128 (columns of d), N = np, K = 128 labels
            const uint32_t idesc_dx = kFp8 ? make_idesc(0, 0, 1, 1, 128, (uint32_t)np)
                                           : make_idesc(1, 1, 1, 1, 128, (uint32_t)np);
            const uint32_t dxcol = tmem + (uint32_t)(p * kPart);
#pragma unroll 1
            for (int k = 0; k < 128 / kK; ++k) {
              const uint64_t ad = sw128_desc(wa + k * kK * 128, kBox, 1024);
              const uint64_t bd = sw128_desc(ga + k * kK * 128, kBox, 1024);
              if (kFp8) mma_e4m3(dxcol, ad, bd, idesc_dx, !(first && k == 0));
              else mma_bf16(dxcol, ad, bd, idesc_dx, !(first && k == 0));
            }
            // dW[tile, slice] += G^T[:, part] X[part, slice] : M = 128 labels, N = 128, K = np samples
            const uint32_t dwcol = tmem + 256 + db * 128;
#pragma unroll 1
            for (int k = 0; k < np / kK; ++k) {
              const int kb = (k * kK * kElem) / 128, kin = (k * kK * kElem) % 128;
              const uint64_t ad = sw128_desc(ga + kb * kBox + kin, 16, 1024);
              const uint64_t bd = sw128_desc(xa + (p * kPart + k * kK) * 128, 32768, 1024);
              if (kFp8) mma_e4m3(dwcol, ad, bd, idesc_dw, (p | k) != 0);
              else mma_bf16(dwcol, ad, bd, idesc_dw, (p | k) != 0);
            }
            mma_commit(&S->gempty[sg]);
          }
          mma_commit(&S->dwfull[db]);
          first = false;
        }
        mma_commit(&S->dxfull);
        mma_commit(&S->xempty);
        ++run;
      }
    }
  } else {
    const int q = warp & 3;
    const int row = q * 32 + lane;             // label row of dW; column of d for dX^T
    const float dw_scale = kFp8 ? 0.00390625f * xscale[1] : 1.0f;
    const float dx_scale = kFp8 ? 0.00390625f : 1.0f;
    int run = 0;
    uint32_t wit = 0, dwit = 0;
    for (int u = u0; u < u1 && !*abort;) {
      const int D = u / T;
      const int ue = min(u1, (D + 1) * T);
      const int D0 = D * 128;
      for (; u < ue && !*abort; ++u) {
        const int t = u - D * T;
        const int sw = wit % kWSlots;
        ++wit;
        const uint32_t db = dwit & 1, duse = dwit >> 1;
        ++dwit;
        if (!mbar_wait(&S->dwfull[db], duse & 1, abort, kWaitCycles)) { record_timeout(status, abort, 31); break; }
        tc_fence_after();
        const int64_t l = l0 + (int64_t)t * 128 + row;
        const bool valid = (l - l0) < span;
        const uint8_t* wrow = ws + sw * kWSlotBytes;
        const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + 256 + db * 128;
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(taddr + c * 32, r);
          tmem_wait_ld();
          const int j0 = D0 + c * 32;
          if (!valid || j0 >= d) continue;
          // old weights of (row, j0 .. j0+31) from the swizzled W tile
          uint32_t wold[kFp8 ? 8 : 16];
          if (kFp8) {
#pragma unroll
            for (int v = 0; v < 2; ++v) {
              const int chunk16 = c * 2 + v;
              const uint4 x = *reinterpret_cast<const uint4*>(wrow + row * 128 + ((chunk16 ^ (row & 7)) << 4));
              wold[4 * v] = x.x; wold[4 * v + 1] = x.y; wold[4 * v + 2] = x.z; wold[4 * v + 3] = x.w;
            }
          } else {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const int chunk16 = (c & 1) * 4 + v;
              const uint4 x = *reinterpret_cast<const uint4*>(wrow + (c >> 1) * kBox + row * 128 +
                                                              ((chunk16 ^ (row & 7)) << 4));
              wold[4 * v] = x.x; wold[4 * v + 1] = x.y; wold[4 * v + 2] = x.z; wold[4 * v + 3] = x.w;
            }
          }
          uint32_t wnew[kFp8 ? 8 : 16];
#pragma unroll
          for (int g8 = 0; g8 < 4; ++g8) {
            const uint64_t idx0 = (uint64_t)l * (uint64_t)d + (uint64_t)(j0 + 8 * g8);
            const u32x4 rb = sr_block(seed, step, idx0 >> 3);
            const uint32_t rw[4] = {rb.x, rb.y, rb.z, rb.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int i = 8 * g8 + e;
              const float dw = __fmul_rn(__uint_as_float(r[i]), dw_scale);
              float w;
              if (kFp8) w = e4m3_to_f32((uint8_t)(wold[i >> 2] >> (8 * (i & 3))));
              else w = bf16_to_f32((uint16_t)(wold[i >> 1] >> (16 * (i & 1))));
              const float v = __fsub_rn(w, __fmul_rn(lr, dw));
              const uint32_t k16 = (e & 1) ? (rw[e >> 1] >> 16) : (rw[e >> 1] & 0xFFFFu);
              if (kFp8) {
                const uint32_t cde = sr_e4m3(v, k16);
                if ((i & 3) == 0) wnew[i >> 2] = cde; else wnew[i >> 2] |= cde << (8 * (i & 3));
              } else {
                const uint32_t cde = sr_bf16(v, k16);
                if ((i & 1) == 0) wnew[i >> 1] = cde; else wnew[i >> 1] |= cde << 16;
              }
            }
          }
          uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(Wglob) + ((size_t)l * d + j0) * kElem);
#pragma unroll
          for (int v = 0; v < (kFp8 ? 2 : 4); ++v)
            dst[v] = make_uint4(wnew[4 * v], wnew[4 * v + 1], wnew[4 * v + 2], wnew[4 * v + 3]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) { mbar_arrive(&S->dwempty[db]); mbar_arrive(&S->wempty[sw]); }
      }
      if (*abort) break;
      // flush dX^T of this run: lane = column j of the slice, TMEM columns = samples
      if (!mbar_wait(&S->dxfull, run & 1, abort, kWaitCycles)) { record_timeout(status, abort, 32); break; }
      tc_fence_after();
      const int j = D0 + row;
      const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16);
      for (int c = 0; c < Bp / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(taddr + c * 32, r);
        tmem_wait_ld();
        if (j < d) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int b = c * 32 + i;
            if (b < B) atomicAdd(dX + (size_t)b * d + j, __uint_as_float(r[i]) * dx_scale);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S->dxempty);
      ++run;
    }
  }
  __syncthreads();
  if (*abort) __nanosleep(20000);
  if (warp == 1) { tc_fence_after(); tmem_dealloc(tmem, 512); }
}

// ---------------------------------------------------------------- host side
using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode_fn() {
  static EncodeFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  }
  return fn;
}

// 2-D row-major map [rows x cols] of 1- or 2-byte elements, box = 128 bytes x box_rows, 128B swizzle.
cudaError_t make_map(CUtensorMap* m, const void* ptr, int elem_bytes, uint64_t cols, uint64_t rows,
                     uint64_t row_stride_elems, uint32_t box_rows) {
  EncodeFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {row_stride_elems * (uint64_t)elem_bytes};
  const cuuint32_t box[2] = {(cuuint32_t)(128 / elem_bytes), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                        const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

constexpr size_t kSmemA = 1024 + kStagesA * kStageABytes + sizeof(SmemA);
constexpr size_t kSmemB = 1024 + kXBytes + kWSlots * kWSlotBytes + kGSlots * kGSlotBytes + sizeof(SmemB);
static_assert(kSmemA <= 232448, "kernel A shared memory");
static_assert(kSmemB <= 232448, "kernel B shared memory");

}  // namespace

// Samples are padded to whole 128-byte swizzle atoms of the operand type
// (64 bf16 or 128 E4M3 values): padded rows of X are zero-filled by TMA and
// the padded gradient entries are written as 0.
int32_t padded_batch(int32_t B, bool fp8) {
  const int32_t a = fp8 ? 128 : 64;
  return (B + a - 1) / a * a;
}

cudaError_t launch_logits_grad_tc(const elmo_head* h, const uint16_t* X, int32_t B, int64_t l0, int64_t l1,
                                  void* gbuf, float* Zout, float* Gout, cudaStream_t s) {
  if (l1 <= l0) return cudaSuccess;
  const bool fp8 = h->dt == ELMO_FP8_E4M3;
  const int eb = fp8 ? 1 : 2;
  const int32_t Bp = padded_batch(B, fp8);
  CUtensorMap tmW, tmX;
  cudaError_t e = make_map(&tmW, h->W, eb, (uint64_t)h->d, (uint64_t)h->L, (uint64_t)h->d, 128);
  if (e != cudaSuccess) return e;
  e = make_map(&tmX, fp8 ? static_cast<const void*>(h->xq) : static_cast<const void*>(X), eb, (uint64_t)h->d,
               (uint64_t)B, (uint64_t)h->d, (uint32_t)Bp);
  if (e != cudaSuccess) return e;
  const int ntiles = (int)((l1 - l0 + 127) / 128);
  const int grid = ntiles < h->num_sms ? ntiles : h->num_sms;
  auto kern = fp8 ? logits_grad_tc<1> : logits_grad_tc<0>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemA);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, kSmemA, s>>>(tmW, tmX, h->L, h->d, B, Bp, l0, l1, h->keys, h->nkeys, h->xscale, gbuf, Zout,
                                      Gout, h->status);
  return cudaGetLastError();
}

cudaError_t launch_update_tc(const elmo_head* h, const uint16_t* X, int32_t B, int64_t l0, int64_t l1,
                             const void* gbuf, float lr, uint64_t seed, uint64_t step, float* dX, cudaStream_t s) {
  if (l1 <= l0) return cudaSuccess;
  const bool fp8 = h->dt == ELMO_FP8_E4M3;
  const int eb = fp8 ? 1 : 2;
  const int32_t Bp = padded_batch(B, fp8);
  CUtensorMap tmW, tmX, tmG;
  cudaError_t e = make_map(&tmW, h->W, eb, (uint64_t)h->d, (uint64_t)h->L, (uint64_t)h->d, 128);
  if (e != cudaSuccess) return e;
  e = make_map(&tmX, fp8 ? static_cast<const void*>(h->xq) : static_cast<const void*>(X), eb, (uint64_t)h->d,
               (uint64_t)B, (uint64_t)h->d, (uint32_t)Bp);
  if (e != cudaSuccess) return e;
  e = make_map(&tmG, gbuf, eb, (uint64_t)Bp, (uint64_t)(l1 - l0), (uint64_t)Bp, 128);
  if (e != cudaSuccess) return e;
  const int T = (int)((l1 - l0 + 127) / 128);
  const int units = T * ((h->d + 127) / 128);
  const int grid = units < h->num_sms ? units : h->num_sms;
  auto kern = fp8 ? update_tc<1> : update_tc<0>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemB);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, kSmemB, s>>>(tmW, tmX, tmG, h->W, h->L, h->d, B, Bp, l0, l1, h->xscale, lr, seed, step, dX,
                                      h->status);
  return cudaGetLastError();
}

}  // namespace elmo
