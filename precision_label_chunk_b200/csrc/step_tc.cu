// step_tc.cu -- the ELMO classifier-head step on sm_100a tensor cores.
//
// "ELMO: Efficiency via Low-precision and Peak Memory Optimization in Large
// Output Spaces", atlas summary "Approach": per label chunk the classifier
// gradient is fused with the momentum-free SGD update and applied with
// stochastic rounding, without FP32 master weights; chunking bounds the
// transient memory.  A label range (the caller's chunk, split where its
// gradient operands would pass 128 MB) is processed by two kernels:
//
//   kernel A, Z = X W_tile^T and G = sigmoid(Z) - Y, written as the next
//   contraction's operand (bf16, or E4M3 / E5M2 of 2^8 G):
//     logits_grad_xt       : X resident in TMEM as the MMA's A operand, 64-label
//                            W k-blocks streamed by TMA through a 16-stage ring,
//                            G stored sample-major (E4M3 with B <= 256, bf16
//                            with B <= 128, d <= 768);
//     logits_grad_panel_tc : X panel resident in shared memory, Z^T = W X^T
//                            (bf16 with B > 128, or d > 768 when a panel fits);
//     logits_grad_tc       : X and W both streamed (the rest).
//   kernel B, update_tc, per (label tile, 128-column slice of d):
//     dX^T[slice] += W_tile[:, slice]^T G_tile^T   (old W, TMEM-resident across
//                                                   the CTA's tiles)
//     dW = G_tile^T X[:, slice]                    (TMEM)
//     W  = SR(W - lr dW)                           (epilogue, in place)
//     one fp32 atomic flush of dX^T per run of tiles.
//
// The gradient operands of a label range are stored tile by tile (128 labels
// x Bp samples) as 8-row x 16-byte core matrices, label-major (chunk j of
// samples and label group i at byte (j * 16 + i) * 128 of the tile) or
// sample-major (label chunk lc of sample b at ((b / 8) * nlc + lc) * 128 +
// (b % 8) * 16): kernel B fetches a tile part with one bulk copy and uses the
// same shared-memory block as both of its G operands (K-major for one
// contraction, MN-major for the other).
//
// Kernel B's warp roles (576 threads for E4M3, 320 for bf16): warp 0 issues
// TMA loads, warp 1 allocates TMEM and issues MMAs (one elected thread), the
// rest are the epilogue: warp w reads TMEM lanes 32*(w%4) .. +31 and an equal
// share of the 32-column chunks, so every SM sub-partition runs the same
// number of epilogue warps.  Every wait is bounded; a wait that runs out
// records ELMO_ETIMEOUT in the status word and the CTA winds down.
#include <cuda.h>
#include <stdlib.h>

#include <utility>

#include "step_common.cuh"

namespace elmo {
namespace {

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

template <int kFp8, int kG5 = 0, int kW5 = 0>
__global__ void __launch_bounds__(kThreads, 1)
    logits_grad_tc(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX, int64_t L,
                   int32_t d, int32_t B, int32_t Bp, int64_t l0, int64_t l1, const uint32_t* __restrict__ keys,
                   const int32_t* __restrict__ tile_ptr, const float* __restrict__ xscale, void* __restrict__ gbuf,
                   float* __restrict__ Zout, float* __restrict__ Gout, int32_t* __restrict__ status) {
  pdl_wait();      // G is written below: the previous range's kernel B must be done
  pdl_trigger();
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
    for (int b = 0; b < 2; ++b) { mbar_init(&S->tfull[b], 1); mbar_init(&S->tempty[b], kEpiWarps); }
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
      const uint32_t idesc = kFp8 ? make_idesc(kW5, 0, 0, 0, 128, (uint32_t)Bp) : make_idesc(1, 1, 0, 0, 128, (uint32_t)Bp);
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
    // epilogue: thread owns TMEM lane (label row) 32*(warp%4) + lane and the
    // 32-column chunks c with c % 4 == (warp - 2) / 4
    const int q = warp & 3;
    const int sub = (warp - 2) >> 2;
    const int row = q * 32 + lane;
    const float inv_sx = kFp8 ? xscale[1] : 1.0f;
    const float acc_lo = grad_acc_floor<kFp8 ? (kG5 ? 2 : 1) : 0>(inv_sx);
    uint32_t tc = 0;
    for (int t = blockIdx.x; t < ntiles && !*abort; t += gridDim.x, ++tc) {
      const uint32_t buf = tc & 1, use = tc >> 1;
      const int64_t lt0 = l0 + (int64_t)t * 128;
      const int64_t l = lt0 + row;
      const bool valid = (l - l0) < span;
      // positives of the 128-label tiles that overlap [lt0, lt0 + 128)
      const int k0 = __ldg(tile_ptr + (lt0 >> 7));
      const int k1 = __ldg(tile_ptr + min((lt0 + 127) >> 7, (L - 1) >> 7) + 1);
      uint32_t mask[8];
      label_mask(keys, k0, k1, l, mask);
      if (!mbar_wait(&S->tfull[buf], use & 1, abort, kWaitCycles)) { record_timeout(status, abort, 4); break; }
      tc_fence_after();
      const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + buf * 256;
      // this warp's 32-column chunks c = sub, sub + 4 (Bp <= 256): one load and wait each
      for (int c = sub; c < Bp / 32; c += 4) {
        uint32_t ra[32];
        tmem_ld32(taddr + c * 32, ra);
        tmem_wait_ld();
        const size_t rowoff = (size_t)(l - l0);
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int b0 = c * 32 + k * 16;
          grad16<kFp8, kG5>(ra + k * 16, inv_sx, acc_lo, mask16(mask, b0), b0, B,
                       static_cast<uint8_t*>(gbuf) + (size_t)t * 128 * Bp * (kFp8 ? 1 : 2), row, !valid,
                       Zout ? Zout + rowoff * B + b0 : nullptr, Gout ? Gout + rowoff * B + b0 : nullptr);
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
// Kernel A, resident-X variant: a panel of PN samples of X (all d columns) is
// loaded once per CTA and kept in shared memory; only W k-blocks stream from
// HBM, through a small ring.  Used whenever a panel of at least 64 samples
// fits (d * bytes <= 3 KB); several panels re-read W from L2.
// ============================================================================
constexpr uint32_t kPanelSmem = 229376;    // X panel + W ring (224 KB)
constexpr int kMaxStagesP = 8;

struct SmemP {
  uint64_t wfull[kMaxStagesP], wempty[kMaxStagesP], xfull, xempty, tfull[2], tempty[2];
  uint32_t tmem_base;
  int abort;
};

template <int kFp8, int kG5 = 0, int kW5 = 0>
__global__ void __launch_bounds__(kThreads, 1)
    logits_grad_panel_tc(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                         int64_t L, int32_t d, int32_t B, int32_t Bp, int32_t PN, int32_t nstages, int64_t l0,
                         int64_t l1,
                         const uint32_t* __restrict__ keys, const int32_t* __restrict__ tile_ptr,
                         const float* __restrict__ xscale, void* __restrict__ gbuf, float* __restrict__ Zout,
                         float* __restrict__ Gout, int32_t* __restrict__ status) {
  pdl_wait();      // G is written below: the previous range's kernel B must be done
  pdl_trigger();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int kb_elems = kFp8 ? 128 : 64;
  const int nkb = (d + kb_elems - 1) / kb_elems;
  uint8_t* xs = base;                                          // nkb k-blocks of [PN rows x 128 B]
  uint8_t* wst = base + (size_t)nkb * PN * 128;                // nstages W k-blocks
  SmemP* S = reinterpret_cast<SmemP*>(base + kPanelSmem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t span = l1 - l0;
  const int ntiles = (int)((span + 127) / 128);
  const int npanels = Bp / PN;
  const uint32_t xkb_bytes = (uint32_t)PN * 128u;
  volatile int* abort = &S->abort;

  if (threadIdx.x == 0) {
    for (int s = 0; s < nstages; ++s) { mbar_init(&S->wfull[s], 1); mbar_init(&S->wempty[s], 1); }
    mbar_init(&S->xfull, 1); mbar_init(&S->xempty, 1);
    for (int b = 0; b < 2; ++b) { mbar_init(&S->tfull[b], 1); mbar_init(&S->tempty[b], kEpiWarps); }
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
      for (int p = 0; p < npanels && !*abort; ++p) {
        if (!mbar_wait(&S->xempty, (p & 1) ^ 1, abort, kWaitCycles)) { record_timeout(status, abort, 41); break; }
        mbar_arrive_expect_tx(&S->xfull, (uint32_t)nkb * xkb_bytes);
        for (int kb = 0; kb < nkb; ++kb) tma_load_2d(xs + kb * xkb_bytes, &tmX, &S->xfull, kb * kb_elems, p * PN);
        for (int t = blockIdx.x; t < ntiles && !*abort; t += gridDim.x) {
          if (p == 0 && t == (int)blockIdx.x) {
            // warm L2 with this CTA's next tiles: HBM latency then hides behind the short ring
            for (int t2 = t; t2 < ntiles && t2 < t + 3 * (int)gridDim.x; t2 += gridDim.x)
              for (int kb = 0; kb < nkb; ++kb)
                tma_prefetch_l2(&tmW, kb * kb_elems, (int32_t)(l0 + (int64_t)t2 * 128));
          } else if (p == 0 && t + 2 * (int)gridDim.x < ntiles) {
            for (int kb = 0; kb < nkb; ++kb)
              tma_prefetch_l2(&tmW, kb * kb_elems, (int32_t)(l0 + (int64_t)(t + 2 * gridDim.x) * 128));
          }
          for (int kb = 0; kb < nkb; ++kb, ++it) {
            const int s = it % nstages;
            const uint32_t ph = (it / nstages) & 1;
            if (!mbar_wait(&S->wempty[s], ph ^ 1, abort, kWaitCycles)) { record_timeout(status, abort, 42); break; }
            mbar_arrive_expect_tx(&S->wfull[s], kBox);
            tma_load_2d(wst + s * kBox, &tmW, &S->wfull[s], kb * kb_elems, (int32_t)(l0 + (int64_t)t * 128));
          }
        }
      }
    }
  } else if (warp == 1) {
    if (elect_one()) {
      const uint32_t idesc = kFp8 ? make_idesc(kW5, 0, 0, 0, 128, (uint32_t)PN) : make_idesc(1, 1, 0, 0, 128, (uint32_t)PN);
      uint32_t it = 0, tc = 0;
      for (int p = 0; p < npanels && !*abort; ++p) {
        if (!mbar_wait(&S->xfull, p & 1, abort, kWaitCycles)) { record_timeout(status, abort, 43); break; }
        tc_fence_after();
        for (int t = blockIdx.x; t < ntiles && !*abort; t += gridDim.x, ++tc) {
          const uint32_t buf = tc & 1, use = tc >> 1;
          if (!mbar_wait(&S->tempty[buf], (use & 1) ^ 1, abort, kWaitCycles)) { record_timeout(status, abort, 44); break; }
          tc_fence_after();
          const uint32_t dcol = tmem + buf * 256;
          for (int kb = 0; kb < nkb; ++kb, ++it) {
            const int s = it % nstages;
            const uint32_t ph = (it / nstages) & 1;
            if (!mbar_wait(&S->wfull[s], ph, abort, kWaitCycles)) { record_timeout(status, abort, 45); break; }
            tc_fence_after();
            const uint32_t a = smem_u32(wst + s * kBox);
            const uint32_t xb = smem_u32(xs + kb * xkb_bytes);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint64_t ad = sw128_desc(a + k * 32, 16, 1024);
              const uint64_t bd = sw128_desc(xb + k * 32, 16, 1024);
              if (kFp8) mma_e4m3(dcol, ad, bd, idesc, (kb | k) != 0);
              else mma_bf16(dcol, ad, bd, idesc, (kb | k) != 0);
            }
            mma_commit(&S->wempty[s]);
          }
          mma_commit(&S->tfull[buf]);
        }
        mma_commit(&S->xempty);
      }
    }
  } else {
    const int q = warp & 3;
    const int sub = (warp - 2) >> 2;
    const int row = q * 32 + lane;
    const float inv_sx = kFp8 ? xscale[1] : 1.0f;
    const float acc_lo = grad_acc_floor<kFp8 ? (kG5 ? 2 : 1) : 0>(inv_sx);
    uint32_t tc = 0;
    for (int p = 0; p < npanels && !*abort; ++p) {
      for (int t = blockIdx.x; t < ntiles && !*abort; t += gridDim.x, ++tc) {
        const uint32_t buf = tc & 1, use = tc >> 1;
        const int64_t lt0 = l0 + (int64_t)t * 128;
        const int64_t l = lt0 + row;
        const bool valid = (l - l0) < span;
        const int k0 = __ldg(tile_ptr + (lt0 >> 7));
        const int k1 = __ldg(tile_ptr + min((lt0 + 127) >> 7, (L - 1) >> 7) + 1);
        uint32_t mask[8];
        label_mask(keys, k0, k1, l, mask);
        if (!mbar_wait(&S->tfull[buf], use & 1, abort, kWaitCycles)) { record_timeout(status, abort, 46); break; }
        tc_fence_after();
        const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + buf * 256;
        // this warp's 32-column chunks c = sub, sub + 4 of the panel: one load and wait each
        for (int c = sub; c < PN / 32; c += 4) {
          uint32_t ra[32];
          tmem_ld32(taddr + c * 32, ra);
          tmem_wait_ld();
          const size_t rowoff = (size_t)(l - l0);
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int cb = c * 32 + k * 16;             // panel column
            const int b0 = p * PN + cb;                 // sample
            grad16<kFp8, kG5>(ra + k * 16, inv_sx, acc_lo, mask16(mask, b0), b0, B,
                         static_cast<uint8_t*>(gbuf) + (size_t)t * 128 * Bp * (kFp8 ? 1 : 2), row, !valid,
                         Zout ? Zout + rowoff * B + b0 : nullptr, Gout ? Gout + rowoff * B + b0 : nullptr);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S->tempty[buf]);
      }
    }
  }
  __syncthreads();
  if (*abort) __nanosleep(20000);
  if (warp == 1) { tc_fence_after(); tmem_dealloc(tmem, 512); }
}

// ============================================================================
// Kernel A with X in tensor memory.  Z[samples x 64 labels] = X W_tile^T with
// X (up to 256 samples as 128-row M-blocks) as the MMA's A operand in TMEM,
// so shared memory holds a 16-stage ring of W k-blocks (64 labels x 128 B)
// instead of X.  The epilogue thread of sample b forms G = sigmoid(Z) - Y for
// its row of the tile and stores it sample-major: in each 128-label tile of
// the gradient buffer the 16-byte label chunk lc of sample b sits at byte
// ((b/8) * nlc + lc) * 128 + (b%8) * 16 (nlc = 8 chunks of 16 E4M3 or 16 of 8
// bf16 labels), i.e. core matrices of 8 samples x 16 bytes, which kernel B
// reads as the MN-major dW operand and the K-major dX^T operand.  Used when X fits the 384 TMEM columns below the
// accumulators: E4M3 with B <= 256 or bf16 with B <= 128, d <= 768.
// ============================================================================
constexpr int kXtThreads = 320;            // warp 0 TMA, warp 1 MMA + TMEM, warps 2-9 epilogue
constexpr int kXtEpi = 8;
constexpr int kXtN = 64;                   // labels per tile (the MMA's N)
constexpr uint32_t kXtBox = kXtN * 128;    // one W k-block: 64 labels x 128 bytes
constexpr int kXtStages = 16;
constexpr uint32_t kXtAcc = 384;           // first accumulator column

struct SmemXt {
  uint64_t wfull[kXtStages], wempty[kXtStages], tfull[2], tempty[2];
  uint64_t xready;              // X is in TMEM (one arrival per epilogue warp)
  uint64_t pmask[kXtEpi][32];   // per epilogue warp: its 32 samples' positives among the tile's labels
  uint32_t tmem_base;
  int abort;
};

template <int kFp8, int kG5 = 0, int kW5 = 0>
__global__ void __launch_bounds__(kXtThreads, 1)
    logits_grad_xt(const __grid_constant__ CUtensorMap tmW, int64_t L, int32_t d, int32_t B, int32_t Bp, int64_t l0,
                   int64_t l1, const uint8_t* __restrict__ xop, const uint32_t* __restrict__ keys,
                   const int32_t* __restrict__ tile_ptr, const float* __restrict__ xscale, void* __restrict__ gbuf,
                   float* __restrict__ Zout, float* __restrict__ Gout, int32_t* __restrict__ status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = base;
  SmemXt* S = reinterpret_cast<SmemXt*>(base + kXtStages * kXtBox);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t span = l1 - l0;
  const int T = 2 * (int)((span + 127) / 128);              // 64-label tiles of whole 128-label tiles
  const int t0 = (int)((int64_t)T * blockIdx.x / gridDim.x);
  const int t1 = (int)((int64_t)T * (blockIdx.x + 1) / gridDim.x);
  const int kbe = kFp8 ? 128 : 64;                          // elements of one 128-byte k-block
  const int nkb = (d + kbe - 1) / kbe;
  const uint32_t opcols = (uint32_t)nkb * 32;               // TMEM columns of one M-block of X
  const int nmb = (Bp + 127) / 128;                         // M-blocks of samples: 1 or 2
  // Two accumulator slots of 64 columns.  One M-block: the slots alternate
  // between tiles.  Two M-blocks: slot mb holds M-block mb of every tile, and
  // the MMAs run M-block by M-block, so the epilogue of one M-block overlaps
  // the MMAs of the other.  Either way the u-th use of the slots is slot u & 1.
  volatile int* abort = &S->abort;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kXtStages; ++s) { mbar_init(&S->wfull[s], 1); mbar_init(&S->wempty[s], 1); }
    for (int b2 = 0; b2 < 2; ++b2) { mbar_init(&S->tfull[b2], 1); mbar_init(&S->tempty[b2], nmb == 2 ? 4 : kXtEpi); }
    mbar_init(&S->xready, kXtEpi);
    S->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) { tmem_alloc(&S->tmem_base, 512); tmem_relinquish(); }
  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S->tmem_base;

  // X into TMEM: sample mb*128 + r of M-block mb in lane r, columns mb*opcols ...
  if (warp >= 2) {
    const int q = warp & 3, h = (warp - 2) >> 2;
    if (h < nmb) {
      const int b = h * 128 + q * 32 + lane;
      const size_t rowbytes = (size_t)d * (kFp8 ? 1 : 2);
      // E4M3: xop holds the codes by 16-byte column chunk (chunk c of row b at
      // (c * 256 + b) * 16), so a warp's load of one chunk covers 512
      // contiguous bytes; bf16: xop is X itself, row-major
      const uint8_t* src = kFp8 ? xop + (size_t)b * 16 : xop + (size_t)b * rowbytes;
      for (uint32_t c0 = 0; c0 < opcols; c0 += 64) {   // 64 columns (16 loads in flight) per round
        uint32_t v[2][32];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const size_t off = (size_t)(c0 + 4 * u) * 4;
          uint4 w4 = make_uint4(0u, 0u, 0u, 0u);
          if (b < B && off < rowbytes)
            w4 = *reinterpret_cast<const uint4*>(kFp8 ? src + (off >> 4) * (ELMO_MAX_BATCH * 16) : src + off);
          v[u >> 3][4 * (u & 7)] = w4.x; v[u >> 3][4 * (u & 7) + 1] = w4.y;
          v[u >> 3][4 * (u & 7) + 2] = w4.z; v[u >> 3][4 * (u & 7) + 3] = w4.w;
        }
        tmem_st32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)h * opcols + c0, v[0]);
        if (c0 + 32 < opcols) tmem_st32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)h * opcols + c0 + 32, v[1]);
      }
      tmem_wait_st();
    }
    // only the MMA warp needs X: the W stream starts while X is still filling
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&S->xready);
  }

  if (warp == 0) {
    if (elect_one()) {
      tma_prefetch_desc(&tmW);
      uint32_t it = 0;
      for (int t = t0; t < t1 && !*abort; ++t) {
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = (int)(it % kXtStages);
          const uint32_t ph = (it / kXtStages) & 1;
          if (!mbar_wait(&S->wempty[s], ph ^ 1, abort, kWaitCycles)) { record_timeout(status, abort, 71); break; }
          mbar_arrive_expect_tx(&S->wfull[s], kXtBox);
          tma_load_2d(ring + s * kXtBox, &tmW, &S->wfull[s], kb * kbe, (int32_t)(l0 + (int64_t)t * kXtN));
        }
      }
    }
  } else if (warp == 1) {
    if (elect_one()) {
      const uint32_t idesc = kFp8 ? make_idesc(0, kW5, 0, 0, 128, kXtN) : make_idesc(1, 1, 0, 0, 128, kXtN);
      uint32_t it = 0, u = 0;
      if (!mbar_wait(&S->xready, 0, abort, kWaitCycles)) record_timeout(status, abort, 75);
      tc_fence_after();
      for (int t = t0; t < t1 && !*abort; ++t) {
        for (int mb = 0; mb < nmb && !*abort; ++mb, ++u) {
          const uint32_t slot = u & 1, ph = (u >> 1) & 1;
          if (!mbar_wait(&S->tempty[slot], ph ^ 1, abort, kWaitCycles)) { record_timeout(status, abort, 72); break; }
          tc_fence_after();
          const uint32_t dcol = tmem + kXtAcc + slot * kXtN;
          for (int kb = 0; kb < nkb; ++kb) {
            const uint32_t its = it + (uint32_t)kb;             // the tile's kb-th W k-block
            const int s = (int)(its % kXtStages);
            if (mb == 0) {
              if (!mbar_wait(&S->wfull[s], (its / kXtStages) & 1, abort, kWaitCycles)) {
                record_timeout(status, abort, 73);
                break;
              }
              tc_fence_after();
            }
            const uint32_t bsm = smem_u32(ring + s * kXtBox);
#pragma unroll
            for (int k = 0; k < 4; ++k) {   // 32 bytes of K per MMA
              const uint32_t a = tmem + (uint32_t)mb * opcols + (uint32_t)kb * 32 + (uint32_t)k * 8;
              const uint64_t bd = sw128_desc(bsm + k * 32, 16, 1024);
              if (kFp8) mma_e4m3_ts(dcol, a, bd, idesc, (kb | k) != 0);
              else mma_bf16_ts(dcol, a, bd, idesc, (kb | k) != 0);
            }
            if (mb == nmb - 1) mma_commit(&S->wempty[s]);   // the k-block's last reader
          }
          mma_commit(&S->tfull[slot]);
        }
        it += (uint32_t)nkb;
      }
    }
  } else {
    // two warps per TMEM lane quadrant: with two M-blocks warp h takes M-block
    // h (all 64 labels), with one it takes label columns 32h .. 32h+31
    const int q = warp & 3, h = (warp - 2) >> 2;
    const int mb = nmb == 2 ? h : 0;
    const int c_lo = nmb == 2 ? 0 : 32 * h;
    const int ncol = nmb == 2 ? 64 : 32;
    const int b = mb * 128 + q * 32 + lane;                  // sample
    const bool bvalid = b < B;
    const bool bstore = b < Bp;
    const float inv_sx = kFp8 ? xscale[1] : 1.0f;
    const float acc_lo = grad_acc_floor<kFp8 ? (kG5 ? 2 : 1) : 0>(inv_sx);
    constexpr int kG = kFp8 ? (kG5 ? 2 : 1) : 0;                 // operand format of G
    constexpr int kEl = kFp8 ? 1 : 2;
    constexpr int kChunk = 16 / kEl;                          // labels per 16-byte chunk
    constexpr int kNlc = 128 / kChunk;                        // chunks per 128-label tile
    // the gradient buffer is free once the previous range's kernel B is done;
    // everything before the first store (X, W, the MMAs) overlaps its tail
    pdl_wait();
    uint32_t tc = 0;
    for (int t = t0; t < t1 && !*abort; ++t, ++tc) {
      const uint32_t u = nmb == 2 ? 2 * tc + (uint32_t)mb : tc;   // this thread's use of the slots
      const uint32_t buf = u & 1;
      if (!mbar_wait(&S->tfull[buf], (u >> 1) & 1, abort, kWaitCycles)) { record_timeout(status, abort, 74); break; }
      tc_fence_after();
      uint32_t v[64];
      const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + kXtAcc + buf * kXtN + (uint32_t)c_lo;
      tmem_ld32(taddr, *reinterpret_cast<uint32_t(*)[32]>(v));
      if (ncol == 64) tmem_ld32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S->tempty[buf]);
      // labels lc0 .. lc0 + ncol - 1 of this thread's row
      const int64_t lc0 = l0 + (int64_t)t * kXtN + c_lo;
      // positives of sample b among them, from the keys of the 128-label tiles
      // they touch.  The warp reads the keys together (32 per pass, coalesced)
      // and each key sets its bit in the mask of its sample, when that sample
      // is one of the warp's: a tile of a frequent label holds hundreds of keys,
      // which one thread per sample would each have to walk alone.
      uint64_t pm;
      {
        const int k0 = __ldg(tile_ptr + (lc0 >> 7));
        const int k1 = __ldg(tile_ptr + min((lc0 + ncol - 1) >> 7, (L - 1) >> 7) + 1);
        unsigned long long* wm = reinterpret_cast<unsigned long long*>(S->pmask[warp - 2]);
        wm[lane] = 0;
        __syncwarp();
        const int wb = b - lane;                              // the warp's first sample
        for (int i = k0 + lane; i < k1; i += 32) {
          const uint32_t key = __ldg(keys + i);
          const int sb = (int)(key & 0xFFu) - wb;
          const int64_t dl = (int64_t)(key >> 8) - lc0;
          if (sb >= 0 && sb < 32 && dl >= 0 && dl < ncol) atomicOr(wm + sb, 1ull << dl);
        }
        __syncwarp();
        pm = wm[lane];
      }
      uint8_t* gtile = static_cast<uint8_t*>(gbuf) + (size_t)(t >> 1) * 128 * Bp * kEl;
      const int lt = (t & 1) * kXtN + c_lo;                   // first label column within the 128-label tile
      for (int j = 0; j < ncol; j += 16) {
        // valid labels of this group: those below the range end, for a real sample
        const int64_t nv = l1 - (lc0 + j);
        const uint32_t vbits = !bvalid || nv <= 0 ? 0u : (nv >= 16 ? 0xFFFFu : (1u << nv) - 1u);
        uint32_t pk[8];
        grad_codes16<kG>(v + j, inv_sx, acc_lo, (uint32_t)(pm >> j) & 0xFFFFu, vbits, pk);
        if (kFp8) {
          if (bstore) {
            const int lc = (lt + j) / kChunk;
            *reinterpret_cast<uint4*>(gtile + ((size_t)(b >> 3) * kNlc + lc) * 128 + (b & 7) * 16) =
                make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        } else {
          if (bstore) {
            const int lc = (lt + j) / kChunk;
            *reinterpret_cast<uint4*>(gtile + ((size_t)(b >> 3) * kNlc + lc) * 128 + (b & 7) * 16) =
                make_uint4(pk[0], pk[1], pk[2], pk[3]);
            *reinterpret_cast<uint4*>(gtile + ((size_t)(b >> 3) * kNlc + lc + 1) * 128 + (b & 7) * 16) =
                make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        }
        if ((Zout || Gout) && bvalid) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int64_t l = lc0 + j + i;
            if (l >= l1) break;
            const size_t o = (size_t)(l - l0) * B + b;
            if (Zout) Zout[o] = __fmul_rn(__uint_as_float(v[j + i]), inv_sx);
            if (Gout)
              Gout[o] = grad_value<kG>(kFp8 ? (pk[i >> 2] >> (8 * (i & 3))) & 0xFFu
                                            : (pk[i >> 1] >> (16 * (i & 1))) & 0xFFFFu);
          }
        }
      }
    }
  }
  __syncthreads();
  if (*abort) __nanosleep(20000);
  if (warp == 1) { tc_fence_after(); tmem_dealloc(tmem, 512); }
}

// ============================================================================
// Kernel B: input gradient, weight gradient and the SR update.
// ============================================================================
constexpr int kWSlots = 4;                  // the most W slots (E4M3; bf16 has 2)
constexpr int kGSlots = 3;
constexpr uint32_t kXBytes = 2 * 32768;     // X[:, slice]: up to two 64-column boxes of up to 256 rows
constexpr uint32_t kWSlotBytes = 2 * kBox;  // W[tile, slice] (bf16: two boxes)
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

template <int kFp8, int kW5 = 0>
__global__ void __launch_bounds__(kFp8 ? kThreads : 320, 1)
    update_tc(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
              const uint8_t* __restrict__ gbuf, void* __restrict__ Wglob, int64_t L, int32_t d, int32_t B,
              int32_t Bp, int64_t l0, int64_t l1, const float* __restrict__ xscale, float lr, const PhiloxKeys rk,
              uint64_t step, uint64_t blk_base, float* __restrict__ dX, int gsm, uint32_t gfmt,
              int32_t* __restrict__ status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // E4M3 operands take half the bytes, which leaves room for 4 W slots: the
  // W load of a unit then starts two units ahead of its epilogue, so the
  // load -> MMA chain (about 2 us) stays off the epilogue's critical path
  constexpr int kWS = kFp8 ? 4 : 2;
  constexpr uint32_t kWSB = kFp8 ? kBox : 2 * kBox;           // bytes of one W slot
  constexpr uint32_t kXB = kFp8 ? 32768u : 2 * 32768u;        // bytes of X[:, slice]
  uint8_t* xs = base;
  uint8_t* ws = xs + kXB;
  uint8_t* gs = ws + kWS * kWSB;
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
  // epilogue warps: E4M3 16 (two 16-column groups each per unit), bf16 8 (two
  // pairs of groups each, a pair in flight together: measured faster for bf16,
  // whose cheaper SR leaves the Philox chains' latency exposed with 16 warps)
  constexpr int kEpiU = kFp8 ? 16 : 8;
  constexpr int kGrp = kFp8 ? 1 : 2;                  // 16-column groups per epilogue step
  const int nparts = (Bp + kPart - 1) / kPart;
  volatile int* abort = &S->abort;

  if (threadIdx.x == 0) {
    mbar_init(&S->xfull, 1); mbar_init(&S->xempty, 1);
    mbar_init(&S->dxfull, 1); mbar_init(&S->dxempty, kEpiU);
    for (int s = 0; s < kWS; ++s) { mbar_init(&S->wfull[s], 1); mbar_init(&S->wempty[s], kEpiU); }
    for (int s = 0; s < kGSlots; ++s) { mbar_init(&S->gfull[s], 1); mbar_init(&S->gempty[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&S->dwfull[b], 1); mbar_init(&S->dwempty[b], kEpiU); }
    S->abort = 0;
    fence_barrier_init();
  }
  pdl_trigger();
  if (warp == 1) { tmem_alloc(&S->tmem_base, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S->tmem_base;

  if (warp == 0) {
    if (elect_one()) {
      tma_prefetch_desc(&tmW); tma_prefetch_desc(&tmX);
      const size_t tile_bytes = (size_t)128 * Bp * kElem;
      bool g_ready = false;   // G comes from this range's kernel A: wait for it once, before the first read
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
            const int s = wit % kWS;
            const uint32_t ph = (wit / kWS) & 1;
            ++wit;
            if (!mbar_wait(&S->wempty[s], ph ^ 1, abort, kWaitCycles)) { record_timeout(status, abort, 12); break; }
            int nb = 0;
            for (int q = 0; q < 128 / kBoxCols; ++q) nb += (D0 + q * kBoxCols < d);
            mbar_arrive_expect_tx(&S->wfull[s], (uint32_t)nb * kBox);
            for (int q = 0; q < 128 / kBoxCols; ++q)
              if (D0 + q * kBoxCols < d) tma_load_2d(ws + s * kWSB + q * kBox, &tmW, &S->wfull[s], D0 + q * kBoxCols, row0);
          }
          for (int p = 0; p < nparts; ++p) {
            const int s = git % kGSlots;
            const uint32_t ph = (git / kGSlots) & 1;
            ++git;
            if (!mbar_wait(&S->gempty[s], ph ^ 1, abort, kWaitCycles)) { record_timeout(status, abort, 13); break; }
            // samples [p*kPart, p*kPart + np) of tile t: a contiguous run of 16-byte chunks
            const int np = min(kPart, Bp - p * kPart);
            const uint32_t bytes = (uint32_t)np * kElem * 128u;
            if (!g_ready) { pdl_wait(); g_ready = true; }
            mbar_arrive_expect_tx(&S->gfull[s], bytes);
            bulk_load(gs + s * kGSlotBytes, gbuf + (size_t)t * tile_bytes + (size_t)p * kPart * kElem * 128u, bytes,
                      &S->gfull[s]);
          }
        }
        ++run;
      }
    }
  } else if (warp == 1) {
    if (elect_one()) {
      // G stored label-major (kernel A with resident X) or sample-major (X in TMEM):
      // the same core matrices then serve as K- or MN-major operands
      const uint32_t gmn = gsm ? 1u : 0u;
      // E4M3 steps: G is E4M3 (gfmt 0) or E5M2 (gfmt 1); W and X are E4M3
      const uint32_t idesc_dw = kFp8 ? make_idesc(gfmt, 0, gmn, 1, 128, 128) : make_idesc(1, 1, gmn, 1, 128, 128);
      const uint32_t gstride = (uint32_t)(kFp8 ? 8 : 16) * 128u;   // sample-major: bytes between sample groups
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
          const int sw = wit % kWS;
          const uint32_t phw = (wit / kWS) & 1;
          ++wit;
          const uint32_t db = dwit & 1, duse = dwit >> 1;
          ++dwit;
          if (!mbar_wait(&S->wfull[sw], phw, abort, kWaitCycles)) { record_timeout(status, abort, 23); break; }
          if (!mbar_wait(&S->dwempty[db], (duse & 1) ^ 1, abort, kWaitCycles)) { record_timeout(status, abort, 24); break; }
          tc_fence_after();
          const uint32_t wa = smem_u32(ws + sw * kWSB);
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
            const uint32_t idesc_dx = kFp8 ? make_idesc(kW5, gfmt, 1, gmn ^ 1u, 128, (uint32_t)np)
                                           : make_idesc(1, 1, 1, gmn ^ 1u, 128, (uint32_t)np);
            const uint32_t dxcol = tmem + (uint32_t)(p * kPart);
#pragma unroll 1
            for (int k = 0; k < 128 / kK; ++k) {
              const uint64_t ad = sw128_desc(wa + k * kK * 128, kBox, 1024);
              // G part as B (N = samples, K = labels).  Label-major: MN-major, label
              // groups 128 B apart, 16-byte sample chunks 2048 B apart, kK / 8 groups per
              // MMA.  Sample-major: K-major, 16-byte label chunks 128 B apart, sample
              // groups gstride apart, 2 chunks per MMA.
              const uint64_t bd = gsm ? nosw_desc(ga + k * 2 * 128, 128, gstride)
                                      : nosw_desc(ga + k * (kK / 8) * 128, 128, 2048);
              if (kFp8) mma_e4m3(dxcol, ad, bd, idesc_dx, !(first && k == 0));
              else mma_bf16(dxcol, ad, bd, idesc_dx, !(first && k == 0));
            }
            // dW[tile, slice] += G^T[:, part] X[part, slice] : M = 128 labels, N = 128, K = np samples
            const uint32_t dwcol = tmem + 256 + db * 128;
#pragma unroll 1
            for (int k = 0; k < np / kK; ++k) {
              // G part as A (M = labels, K = samples).  Label-major: K-major, 16-byte
              // sample chunks 2048 B apart, label groups 128 B apart, 2 chunks per MMA.
              // Sample-major: MN-major, sample groups gstride apart, 16-byte label
              // chunks 128 B apart, kK / 8 groups per MMA.
              const uint64_t ad = gsm ? nosw_desc(ga + k * (kK / 8) * gstride, gstride, 128)
                                      : nosw_desc(ga + k * 2 * 2048, 2048, 128);
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
    const int sub = (warp - 2) >> 2;           // dW columns of width 128/(kEpiU/4); dX^T chunks c % (kEpiU/4) == sub
    const int row = q * 32 + lane;             // label row of dW; column of d for dX^T
    // lr * dW with dW = acc * 2^-8 / s_X (fp8) folds into one exact power-of-two scaled lr
    const float lrs = kFp8 ? lr * (0.00390625f * xscale[1]) : lr;
    const float dx_scale = kFp8 ? 0.00390625f : 1.0f;
    int run = 0;
    uint32_t wit = 0, dwit = 0;
    for (int u = u0; u < u1 && !*abort;) {
      const int D = u / T;
      const int ue = min(u1, (D + 1) * T);
      const int D0 = D * 128;
      for (; u < ue && !*abort; ++u) {
        const int t = u - D * T;
        const int sw = wit % kWS;
        ++wit;
        const uint32_t db = dwit & 1, duse = dwit >> 1;
        ++dwit;
        if (!mbar_wait(&S->dwfull[db], duse & 1, abort, kWaitCycles)) { record_timeout(status, abort, 31); break; }
        tc_fence_after();
        const int64_t l = l0 + (int64_t)t * 128 + row;
        const bool valid = (l - l0) < span;
        const uint8_t* wrow = ws + sw * kWSB;
        const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + 256 + db * 128;
#pragma unroll 1
        for (int hh = 0; hh < 2; ++hh) {
          const int jl = sub * 32 * kGrp + hh * 16 * kGrp;  // column within the 128-column slice
          uint32_t r[kGrp][16];
#pragma unroll
          for (int g = 0; g < kGrp; ++g) tmem_ld16(taddr + jl + 16 * g, r[g]);
          tmem_wait_ld();
          const int j0 = D0 + jl;
          if (!valid || j0 >= d) continue;
#pragma unroll
          for (int g = 0; g < kGrp; ++g) {
            uint32_t rw[8];
            sr_draws16(rk, step, blk_base, l, d, j0 + 16 * g, rw);
            update16<kFp8 ? (kW5 ? 2 : 1) : 0>(r[g], rw, wrow, row, jl + 16 * g, l, d, j0 + 16 * g, lrs, Wglob);
          }
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
      for (int c = sub; c < Bp / 32; c += kEpiU / 4) {
        uint32_t ra[32];
        tmem_ld32(taddr + c * 32, ra);
        tmem_wait_ld();
        if (j < d) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int b = c * 32 + i;
            if (b < B) atomicAdd(dX + (size_t)b * d + j, __uint_as_float(ra[i]) * dx_scale);
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
constexpr size_t kSmemA = 1024 + kStagesA * kStageABytes + sizeof(SmemA);
// the bf16 layout (X 64 KB, 2 W slots of 32 KB) is the larger of the two
// (E4M3: X 32 KB, 4 W slots of 16 KB)
constexpr size_t kSmemB = 1024 + kXBytes + 2 * kWSlotBytes + kGSlots * kGSlotBytes + sizeof(SmemB);
static_assert(32768 + kWSlots * kBox <= kXBytes + 2 * kWSlotBytes, "E4M3 kernel B layout");
constexpr size_t kSmemP = 1024 + kPanelSmem + sizeof(SmemP);
static_assert(kSmemA <= 232448, "kernel A shared memory");
static_assert(kSmemP <= 232448, "kernel A (resident X) shared memory");
static_assert(kSmemB <= 232448, "kernel B shared memory");

}  // namespace

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeFn encode_fn() {
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
cudaError_t make_tma_map_2d(CUtensorMap* m, const void* ptr, int elem_bytes, uint64_t cols, uint64_t rows,
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

// A row-major matrix seen as (128-byte k-block column, row, k-block): box
// {128 bytes, box_rows, box_kb} lands in shared memory as box_kb blocks of
// box_rows x 128 bytes, each in the 128B-swizzled K-major operand layout.
// One request per box (the W stream's rate follows the request count).
cudaError_t make_tma_map_kb3d(CUtensorMap* m, const void* ptr, int elem_bytes, uint64_t cols, uint64_t rows,
                              uint32_t box_rows, uint32_t box_kb) {
  EncodeFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  const uint64_t kbe = 128 / elem_bytes;                       // elements per k-block
  const cuuint64_t dims[3] = {kbe, rows, (cols + kbe - 1) / kbe};
  const cuuint64_t strides[2] = {cols * (uint64_t)elem_bytes, 128};
  const cuuint32_t box[3] = {(cuuint32_t)kbe, box_rows, box_kb};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 3,
                        const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Samples are padded to whole 128-byte swizzle atoms of the operand type
// (64 bf16 or 128 E4M3 values): padded rows of X are zero-filled by TMA and
// the padded gradient entries are written as 0.
int32_t padded_batch(int32_t B, bool fp8) {
  const int32_t a = fp8 ? 128 : 64;
  return (B + a - 1) / a * a;
}

// Launch with programmatic stream serialisation when `pdl` (the kernel's
// prologue then overlaps the tail of the previous kernel in the stream; each
// kernel orders its dependent accesses with griddepcontrol.wait).
template <typename... Params, typename... Args>
cudaError_t launch_k(void (*kern)(Params...), int grid, int block, size_t smem, cudaStream_t s, bool pdl,
                     Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3((unsigned)block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Kernel A keeps X in tensor memory (and stores G sample-major) when X fits
// the 384 TMEM columns below its accumulators; ELMO_STEP_XT=0 turns it off.
bool g_sample_major(const elmo_head* h, int32_t Bp) {
  const char* v = getenv("ELMO_STEP_XT");
  if (v && v[0] == '0') return false;
  const bool fp8 = h->dt == ELMO_FP8_E4M3;
  return h->d % 64 == 0 && h->d <= 768 && (fp8 ? Bp <= 256 : Bp <= 128);
}

constexpr size_t kSmemXt = 1024 + kXtStages * kXtBox + sizeof(SmemXt);
static_assert(kSmemXt <= 232448, "kernel A (X in TMEM) shared memory");

cudaError_t launch_logits_grad_tc(const elmo_head* h, const uint16_t* X, int32_t B, int64_t l0, int64_t l1,
                                  void* gbuf, float* Zout, float* Gout, cudaStream_t s, bool pdl) {
  if (l1 <= l0) return cudaSuccess;
  const bool fp8 = h->dt == ELMO_FP8_E4M3;
  const int eb = fp8 ? 1 : 2;
  const int32_t Bp = padded_batch(B, fp8);
  if (g_sample_major(h, Bp)) {
    CUtensorMap tmW64;
    cudaError_t e = make_tma_map_2d(&tmW64, h->W, eb, (uint64_t)h->d, (uint64_t)h->L, (uint64_t)h->d, kXtN);
    if (e != cudaSuccess) return e;
    const int T = 2 * (int)((l1 - l0 + 127) / 128);
    const int grid = T < h->num_sms ? T : h->num_sms;
    auto kx = fp8 ? (h->g_e5m2 ? logits_grad_xt<1, 1> : h->w_e5m2 ? logits_grad_xt<1, 0, 1> : logits_grad_xt<1>)
                  : logits_grad_xt<0>;
    e = cudaFuncSetAttribute(kx, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemXt);
    if (e != cudaSuccess) return e;
    const uint8_t* xop = fp8 ? h->xqt : reinterpret_cast<const uint8_t*>(X);
    return launch_k(kx, grid, kXtThreads, kSmemXt, s, pdl, tmW64, h->L, h->d, B, Bp, l0, l1, xop,
                    (const uint32_t*)h->keys, (const int32_t*)h->tile_ptr, (const float*)h->xscale, gbuf, Zout, Gout,
                    h->status);
  }
  CUtensorMap tmW, tmX;
  cudaError_t e = make_tma_map_2d(&tmW, h->W, eb, (uint64_t)h->d, (uint64_t)h->L, (uint64_t)h->d, 128);
  if (e != cudaSuccess) return e;
  e = make_tma_map_2d(&tmX, fp8 ? static_cast<const void*>(h->xq) : static_cast<const void*>(X), eb, (uint64_t)h->d,
               (uint64_t)B, (uint64_t)h->d, (uint32_t)Bp);
  if (e != cudaSuccess) return e;
  const int ntiles = (int)((l1 - l0 + 127) / 128);
  const int grid = ntiles < h->num_sms ? ntiles : h->num_sms;
  // resident-X panels: the largest multiple of 64 samples dividing Bp whose X
  // leaves room for a W ring of at least two 16 KB stages (measured: one large
  // panel with a short ring beats two panels with a deep ring, which re-read W)
  const int kb_elems = fp8 ? 128 : 64;
  const int64_t xrow = (int64_t)((h->d + kb_elems - 1) / kb_elems) * 128;   // bytes of one sample, k-block padded
  int32_t PN = 0, nst = 0;
  for (int32_t pn = (Bp < 256 ? Bp : 256); pn >= 64; pn -= 64) {
    if (Bp % pn) continue;
    const int64_t free_bytes = (int64_t)kPanelSmem - xrow * pn;
    const int st = (int)(free_bytes / kBox);
    if (st >= 2) { PN = pn; nst = st < kMaxStagesP ? st : kMaxStagesP; break; }
  }
  if (PN >= 64) {
    CUtensorMap tmXp;
    e = make_tma_map_2d(&tmXp, fp8 ? static_cast<const void*>(h->xq) : static_cast<const void*>(X), eb, (uint64_t)h->d,
                 (uint64_t)B, (uint64_t)h->d, (uint32_t)PN);
    if (e != cudaSuccess) return e;
    auto kp = fp8 ? (h->g_e5m2 ? logits_grad_panel_tc<1, 1>
                               : h->w_e5m2 ? logits_grad_panel_tc<1, 0, 1> : logits_grad_panel_tc<1>)
                  : logits_grad_panel_tc<0>;
    e = cudaFuncSetAttribute(kp, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemP);
    if (e != cudaSuccess) return e;
    return launch_k(kp, grid, kThreads, kSmemP, s, pdl, tmW, tmXp, h->L, h->d, B, Bp, PN, nst, l0, l1,
                    (const uint32_t*)h->keys, (const int32_t*)h->tile_ptr, (const float*)h->xscale, gbuf, Zout, Gout,
                    h->status);
  }
  auto kern = fp8 ? (h->g_e5m2 ? logits_grad_tc<1, 1> : h->w_e5m2 ? logits_grad_tc<1, 0, 1> : logits_grad_tc<1>)
                  : logits_grad_tc<0>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemA);
  if (e != cudaSuccess) return e;
  return launch_k(kern, grid, kThreads, kSmemA, s, pdl, tmW, tmX, h->L, h->d, B, Bp, l0, l1, (const uint32_t*)h->keys,
                  (const int32_t*)h->tile_ptr, (const float*)h->xscale, gbuf, Zout, Gout, h->status);
}

cudaError_t launch_update_tc(const elmo_head* h, const uint16_t* X, int32_t B, int64_t l0, int64_t l1,
                             const void* gbuf, float lr, uint64_t seed, uint64_t step, float* dX, cudaStream_t s,
                             bool pdl) {
  if (l1 <= l0) return cudaSuccess;
  const bool fp8 = h->dt == ELMO_FP8_E4M3;
  const int eb = fp8 ? 1 : 2;
  const int32_t Bp = padded_batch(B, fp8);
  CUtensorMap tmW, tmX;
  cudaError_t e = make_tma_map_2d(&tmW, h->W, eb, (uint64_t)h->d, (uint64_t)h->L, (uint64_t)h->d, 128);
  if (e != cudaSuccess) return e;
  e = make_tma_map_2d(&tmX, fp8 ? static_cast<const void*>(h->xq) : static_cast<const void*>(X), eb, (uint64_t)h->d,
               (uint64_t)B, (uint64_t)h->d, (uint32_t)Bp);
  if (e != cudaSuccess) return e;
  const int T = (int)((l1 - l0 + 127) / 128);
  const int units = T * ((h->d + 127) / 128);
  const int grid = units < h->num_sms ? units : h->num_sms;
  auto kern = fp8 ? (h->w_e5m2 ? update_tc<1, 1> : update_tc<1>) : update_tc<0>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemB);
  if (e != cudaSuccess) return e;
  return launch_k(kern, grid, fp8 ? kThreads : 320, kSmemB, s, pdl, tmW, tmX, static_cast<const uint8_t*>(gbuf), h->W,
                  h->L, h->d,
                  B, Bp, l0, l1, (const float*)h->xscale, lr, philox_keys(seed), step,
                  (uint64_t)h->label_base * (uint64_t)h->d / 8, dX, g_sample_major(h, Bp) ? 1 : 0,
                  h->g_e5m2 ? 1u : 0u, h->status);
}

}  // namespace elmo
