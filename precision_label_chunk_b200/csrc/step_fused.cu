// step_fused.cu -- the whole training step of a head in one persistent launch.
//
// "ELMO: Efficiency via Low-precision and Peak Memory Optimization in Large
// Output Spaces", atlas summary "Approach": per label chunk the classifier
// gradient is computed inside the momentum-free SGD update, applied with
// stochastic rounding, and the label axis is processed chunk by chunk so that
// the transient memory stays small.
//
// One CTA per SM, launched cooperatively so that every CTA is resident.  The
// CTAs split into two roles that run at the same time on different SMs:
//
//   role A (the first nA CTAs): Z = X W_tile^T and G = sigmoid(Z) - Y for
//     128-label tiles t = a, a + nA', ...: one M-block of X (128 samples) stays
//     in TMEM as the MMA's A operand, W k-blocks stream through a 128 KB TMA
//     ring, and the 16 epilogue warps write G (the next contractions'
//     operand, sample-major) into slot t % R of a ring of R tiles in global
//     memory, then count themselves in ready[slot].  With more than 128
//     samples two neighbouring CTAs form a tile, one M-block each.  E4M3: one
//     MMA chain of N = 128 labels per tile (X takes 192 TMEM columns, two
//     128-column accumulator slots follow); bf16: two of N = 64 (X takes 384);
////   role B (the other CTAs, nG groups x nD d-slices): the CTA of group g and
//     slice s runs the units (t, s) for t = g, g + nG, ...: it waits for
//     ready, copies G_t into shared memory (and counts itself in consumed[slot],
//     which role A waits on before it reuses the slot), and issues
//       dX^T[slice] += W_t[:, slice]^T G_t^T   (old W; TMEM-resident for the
//                                              whole launch, one flush at the end)
//       dW = G_t^T X[:, slice]                 (TMEM, never stored)
//     while its 16 epilogue warps apply W = SR(W - lr dW) in place.
//
// Role A's tensor work and W stream overlap role B's SR epilogue (issue-bound)
// across the GPU; W is read from HBM once, by role A, and role B finds its
// slice in L2 shortly after (the ring keeps role A at most R tiles ahead); G
// lives only in the R-tile ring.  The split nA : nB follows the two roles'
// work per tile.  Every wait is bounded; a wait that runs out records
// ELMO_ETIMEOUT in the status word, and the other CTAs stop at their next wait.
//
// Used for B <= 256, d <= 768, d a multiple of 64 (one M-block of X fits the
// TMEM columns below role A's accumulators); other shapes run the
// range-by-range kernels of step_tc.cu.
#include <stdlib.h>

#include <algorithm>
#include <utility>

#include "step_common.cuh"

namespace elmo {
namespace {

constexpr int kFThreads = 576;              // warp 0 TMA, warp 1 MMA + TMEM, warps 2-17 epilogue
constexpr int kFEpi = 16;
constexpr int kFStagesA = 24;               // role A: most W ring stages (4 of 48 KB are used)
constexpr uint32_t kFRingA = 192 * 1024;    // role A: bytes of the W ring
// role A: a 128-label tile is two halves of kN = 64 labels (the MMA's N),
// each accumulated in its own TMEM slot of 64 columns after one M-block of X
// (E4M3 192 columns at d = 768, bf16 384).  E4M3 has room for four slots:
// two epilogue groups, each with a slot per half; bf16 for two: one group.
template <int kFp8> struct RoleA {
  static constexpr int kN = 64;
  static constexpr int kHalves = 128 / kN;
  static constexpr int kGroups = kFp8 ? 2 : 1;
  static constexpr int kSlots = kGroups * kHalves;
  // a ring stage holds up to kKbs 128-byte k-blocks of a 64-label half
  // (48 KB): one TMA request per stage where the W rows divide into whole
  // k-blocks (a 3-D box), else one 2-D box per k-block.  The TMA engine's
  // rate follows its request count: 8 KB requests streamed about 25 bytes
  // per clock per SM on B200, 48 KB requests 75 (the HBM bound at 46 SMs).
  static constexpr int kKbs = 6;
  static constexpr uint32_t kKb = (uint32_t)kN * 128;       // one k-block of the half
  static constexpr uint32_t kStage = kKb * kKbs;
  static constexpr int kStages = (int)(kFRingA / kStage);
  static constexpr uint32_t kAcc = kFp8 ? 256 : 384;
};
constexpr int kFGSlots = 3;                 // role B: G tiles in shared memory
constexpr uint32_t kFGSlotBytes = 2 * kBox; // one G tile: 128 labels x up to 256 samples (E4M3) or 128 (bf16)
constexpr uint32_t kFXBytes = 2 * 32768;    // role B: X[:, slice]
constexpr uint32_t kFWBytes = 4 * kBox;     // role B: W slots (E4M3 4 x 16 KB, bf16 2 x 32 KB)

constexpr int kFQ = 8;                      // entries of a CTA's tile queue

struct SmemFA {
  uint64_t wfull[kFStagesA], wempty[kFStagesA], tfull[4], tempty[4];
  uint64_t xready;
  uint64_t qfull[kFQ], qempty[kFQ];           // the tile queue: tiles taken by the TMA warp, in order
  int tq[kFQ];
  uint64_t pmask[kFEpi][32];   // per epilogue warp: its 32 samples' positives among its labels
  int arrivals[4];             // epilogue warps done with a tile's G (by local tile index mod 4)
  uint32_t tmem_base;
  int abort;
};

struct SmemFB {
  uint64_t xfull, dxfull;
  uint64_t qfull[kFQ], qempty[kFQ];
  int tq[kFQ];
  int first_t;                                // the first tile taken (negative: none)
  uint64_t wfull[4], wempty[4];
  uint64_t gfull[kFGSlots], gempty[kFGSlots];
  uint64_t dwfull[2], dwempty[2];
  uint32_t tmem_base;
  int abort;
};

constexpr size_t kSmemF = 1024 + kFXBytes + kFWBytes + kFGSlots * kFGSlotBytes + 1024;
static_assert(kSmemF <= 232448, "fused step shared memory");
static_assert(kFRingA + sizeof(SmemFA) + 1024 <= kSmemF, "role A layout");
static_assert(sizeof(SmemFB) <= 1024, "role B barriers");

__device__ __forceinline__ int32_t ld_acquire(const int32_t* p) {
  int32_t v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ int32_t ld_relaxed(const int32_t* p) {
  int32_t v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(int32_t* p, int32_t v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void red_release_add(int32_t* p, int32_t v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// orders this thread's generic-proxy accesses of global memory with later
// async-proxy (TMA, bulk copy) accesses, and the other way round
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Bounded wait until *flag >= target (acquire).  Gives up when `abort` is set,
// when another CTA has recorded a timeout, or after `limit` clock cycles.
__device__ __forceinline__ bool wait_flag(const int32_t* flag, int32_t target, volatile int* abort,
                                          const int32_t* status, long long limit) {
  if (ld_acquire(flag) >= target) return true;
  const long long t0 = clock64();
  while (true) {
    __nanosleep(64);
    if (ld_acquire(flag) >= target) return true;
    if (*abort || *reinterpret_cast<const volatile int32_t*>(status) == (int32_t)ELMO_ETIMEOUT) return false;
    if (clock64() - t0 > limit) return false;
  }
}

template <int kFp8, int kG5, int kW5 = 0>
__global__ void __launch_bounds__(kFThreads, 1)
    step_fused(const __grid_constant__ CUtensorMap tmWa, const __grid_constant__ CUtensorMap tmWa3, int32_t wa3,
               const __grid_constant__ CUtensorMap tmWb,
               const __grid_constant__ CUtensorMap tmX, void* __restrict__ Wglob, int64_t L, int32_t d, int32_t B,
               int32_t Bp, const uint8_t* __restrict__ xop, const uint32_t* __restrict__ keys,
               const int32_t* __restrict__ tile_ptr, const float* __restrict__ xscale, uint8_t* __restrict__ gring,
               int32_t R, int32_t* __restrict__ ready, int32_t* __restrict__ consumed,
               int32_t* __restrict__ sched, int32_t nA, int32_t nG, float lr, const PhiloxKeys rk, uint64_t step, uint64_t blk_base, float* __restrict__ dX,
               int32_t* __restrict__ status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = (int)((L + 127) / 128);                       // 128-label tiles of the head
  const int nD = (d + 127) / 128;                             // 128-column d-slices
  constexpr int kEl = kFp8 ? 1 : 2;
  const size_t tile_bytes = (size_t)128 * Bp * kEl;           // one G tile in the ring

  if ((int)blockIdx.x < nA) {
    // ======================================================== role A
    using RA = RoleA<kFp8>;
    uint8_t* ring = base;
    SmemFA* S = reinterpret_cast<SmemFA*>(base + kFRingA);
    volatile int* abort = &S->abort;
    const int kbe = kFp8 ? 128 : 64;                          // elements of one 128-byte k-block
    const int nkb = (d + kbe - 1) / kbe;
    const int kbs = nkb < RA::kKbs ? nkb : RA::kKbs;          // k-blocks of one 3-D box
    const uint32_t opcols = (uint32_t)nkb * 32;               // TMEM columns of one M-block of X
    // Producers of a tile: one CTA holds the single M-block of X (up to 128
    // samples), or two neighbouring CTAs hold one M-block each and write
    // their halves of G.
    const int nprod = Bp > 128 ? 2 : 1;
    const int amb = nprod == 2 ? (int)(blockIdx.x & 1) : 0;   // the M-block held here
    // Tiles are handed out in order, one counter per M-block (sched[amb]): a
    // CTA's TMA warp takes the next tile and passes it to the MMA warp and the
    // epilogue through a queue in shared memory.
    constexpr int kGroups = RA::kGroups;                     // epilogue groups (alternate queue entries)
    constexpr int kWarpsG = kFEpi / kGroups;
    if (threadIdx.x == 0) {
      for (int i = 0; i < kFQ; ++i) { mbar_init(&S->qfull[i], 1); mbar_init(&S->qempty[i], 1 + kWarpsG); }
      for (int s = 0; s < RA::kStages; ++s) { mbar_init(&S->wfull[s], 1); mbar_init(&S->wempty[s], 1); }
      // each slot is drained by one group: both groups of eight (E4M3) or all sixteen warps (bf16)
      for (int b2 = 0; b2 < RA::kSlots; ++b2) { mbar_init(&S->tfull[b2], 1); mbar_init(&S->tempty[b2], kWarpsG); }
      mbar_init(&S->xready, kFEpi);
      for (int i = 0; i < 4; ++i) S->arrivals[i] = 0;
      S->abort = 0;
      fence_barrier_init();
    }
    if (warp == 1) { tmem_alloc(&S->tmem_base, 512); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S->tmem_base;

    if (warp >= 2) {
      // X into TMEM: sample amb*128 + r in lane r; warp (q, h) copies the
      // 64-column chunks c0 = 64 h, 64 h + 256, ... of its quadrant's lanes
      const int q = warp & 3, h = (warp - 2) >> 2;
      const int b = amb * 128 + q * 32 + lane;
      const size_t rowbytes = (size_t)d * kEl;
      // E4M3: xop holds the codes by 16-byte column chunk (chunk c of row b at
      // (c * 256 + b) * 16); bf16: xop is X itself, row-major
      const uint8_t* src = kFp8 ? xop + (size_t)b * 16 : xop + (size_t)b * rowbytes;
      for (uint32_t c0 = 64u * (uint32_t)h; c0 < opcols; c0 += 256) {
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
        tmem_st32(tmem + ((uint32_t)(q * 32) << 16) + c0, v[0]);
        if (c0 + 32 < opcols) tmem_st32(tmem + ((uint32_t)(q * 32) << 16) + c0 + 32, v[1]);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S->xready);
    }

    if (warp == 0) {
      if (elect_one()) {
        tma_prefetch_desc(&tmWa);
        uint32_t it = 0;
        // the next tile is taken one tile ahead, so that the counter's round
        // trip overlaps this tile's loads
        int t_next = atomicAdd(sched + amb, 1);
        for (uint32_t i = 0;; ++i) {
          const int qs = (int)(i % kFQ);
          if (!mbar_wait(&S->qempty[qs], ((i / kFQ) & 1) ^ 1, abort, kWaitCycles)) {
            record_timeout(status, abort, 80);
            break;
          }
          int t = t_next;
          if (t >= T || *abort) t = -1;
          else t_next = atomicAdd(sched + amb, 1);
          S->tq[qs] = t;
          mbar_arrive(&S->qfull[qs]);
          if (t < 0) {
            // a terminator for each epilogue group (they take alternate entries)
            for (int e = 1; e < kGroups; ++e) {
              const uint32_t i2 = i + (uint32_t)e;
              const int q2 = (int)(i2 % kFQ);
              if (!mbar_wait(&S->qempty[q2], ((i2 / kFQ) & 1) ^ 1, abort, kWaitCycles)) {
                record_timeout(status, abort, 80);
                break;
              }
              S->tq[q2] = -1;
              mbar_arrive(&S->qfull[q2]);
            }
            break;
          }
          // bring the W tile about two rounds of this M-block's CTAs ahead
          // into L2 (the first M-block's CTAs only: the second finds the same
          // tiles there), so that the ring's loads meet L2 rather than HBM latency
          if (amb == 0) {
            const int tp = t + 2 * (nA / nprod);
            if (tp < T)
              for (int hf = 0; hf < RA::kHalves; ++hf) {
                if (wa3)
                  for (int k0 = 0; k0 < nkb; k0 += RA::kKbs) tma_prefetch_l2_3d(&tmWa3, 0, tp * 128 + hf * RA::kN, k0);
                else
                  for (int kb = 0; kb < nkb; ++kb) tma_prefetch_l2(&tmWa, kb * kbe, tp * 128 + hf * RA::kN);
              }
          }
          bool stop = false;
          for (int hf = 0; hf < RA::kHalves && !stop; ++hf) {
            for (int k0 = 0; k0 < nkb; k0 += RA::kKbs, ++it) {
              const int s = (int)(it % RA::kStages);
              const uint32_t ph = (it / RA::kStages) & 1;
              if (!mbar_wait(&S->wempty[s], ph ^ 1, abort, kWaitCycles)) {
                record_timeout(status, abort, 81);
                stop = true;
                break;
              }
              const int nk = min(RA::kKbs, nkb - k0);        // k-blocks in this stage
              if (wa3) {
                // one box of kbs k-blocks (past the last k-block: zero fill, still counted)
                mbar_arrive_expect_tx(&S->wfull[s], (uint32_t)kbs * RA::kKb);
                tma_load_3d(ring + s * RA::kStage, &tmWa3, &S->wfull[s], 0, t * 128 + hf * RA::kN, k0);
              } else {
                mbar_arrive_expect_tx(&S->wfull[s], (uint32_t)nk * RA::kKb);
                for (int j = 0; j < nk; ++j)
                  tma_load_2d(ring + s * RA::kStage + j * RA::kKb, &tmWa, &S->wfull[s], (k0 + j) * kbe,
                              t * 128 + hf * RA::kN);
              }
            }
          }
          if (stop) break;
        }
      }
    } else if (warp == 1) {
      if (elect_one()) {
        const uint32_t idesc =
            kFp8 ? make_idesc(0, kW5, 0, 0, 128, RA::kN) : make_idesc(1, 1, 0, 0, 128, RA::kN);
        uint32_t it = 0;
        const uint64_t bdesc0 = sw128_desc(smem_u32(ring), 16, 1024);   // stage 0, k = 0
        if (!mbar_wait(&S->xready, 0, abort, kWaitCycles)) record_timeout(status, abort, 82);
        tc_fence_after();
        for (uint32_t i = 0; !*abort; ++i) {
          const int qs = (int)(i % kFQ);
          if (!mbar_wait(&S->qfull[qs], (i / kFQ) & 1, abort, kWaitCycles)) { record_timeout(status, abort, 87); break; }
          const int t = S->tq[qs];
          mbar_arrive(&S->qempty[qs]);
          if (t < 0) break;
          // tile i, half hf: slot (i % kGroups) kHalves + hf, its (i / kGroups)-th use
          for (int hf = 0; hf < RA::kHalves && !*abort; ++hf) {
            const uint32_t slot = (i % kGroups) * RA::kHalves + (uint32_t)hf, ph = (i / kGroups) & 1;
            if (!mbar_wait(&S->tempty[slot], ph ^ 1, abort, kWaitCycles)) { record_timeout(status, abort, 83); break; }
            tc_fence_after();
            const uint32_t dcol = tmem + RA::kAcc + slot * RA::kN;
            // descriptors advance by constants (the start address field counts
            // 16-byte units): few instructions per MMA for this thread, which
            // shares its scheduler with four busy epilogue warps
            for (int k0 = 0; k0 < nkb; k0 += RA::kKbs, ++it) {
              const int s = (int)(it % RA::kStages);
              if (!mbar_wait(&S->wfull[s], (it / RA::kStages) & 1, abort, kWaitCycles)) {
                record_timeout(status, abort, 84);
                break;
              }
              tc_fence_after();
              const int k1 = min(nkb, k0 + RA::kKbs);
              for (int kb = k0; kb < k1; ++kb) {
                // k-block kb - k0 of the stage: kKb bytes further in
                const uint64_t bd = bdesc0 + (uint64_t)((uint32_t)s * (RA::kStage >> 4) + (uint32_t)(kb - k0) * (RA::kKb >> 4));
                const uint32_t aa = tmem + (uint32_t)kb * 32;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  if (kFp8) mma_e4m3_ts(dcol, aa + (uint32_t)k * 8, bd + (uint64_t)(k * 2), idesc, (kb | k) != 0);
                  else mma_bf16_ts(dcol, aa + (uint32_t)k * 8, bd + (uint64_t)(k * 2), idesc, (kb | k) != 0);
                }
              }
              mma_commit(&S->wempty[s]);
            }
            mma_commit(&S->tfull[slot]);
          }
        }
      }
    } else {
      // Epilogue.  E4M3: two groups of eight warps take alternate tiles, group
      // g the slots 2 g and 2 g + 1 (one per 64-label half), so that one
      // group's waits (ring slot, positives, MMA) overlap the other's
      // arithmetic and the MMAs of one half overlap the epilogue of the other.
      // bf16: one group of sixteen with two slots.  Warp (q = warp % 4, hh) of
      // a group takes TMEM lanes 32 q .. 32 q + 31 (samples amb * 128 + 32 q +
      // lane) and label columns kColW hh .. kColW hh + kColW - 1 of each slot.
      constexpr int kColW = RA::kN / (kWarpsG / 4);           // 32 (E4M3) or 16 (bf16)
      const int gp = (warp - 2) / kWarpsG, wg = (warp - 2) % kWarpsG;
      const int q = warp & 3, hh = wg >> 2;
      const int c_lo = kColW * hh;
      const float inv_sx = kFp8 ? xscale[1] : 1.0f;
      const float acc_lo = grad_acc_floor<kFp8 ? (kG5 ? 2 : 1) : 0>(inv_sx);
      constexpr int kG = kFp8 ? (kG5 ? 2 : 1) : 0;
      constexpr int kChunk = 16 / kEl;                        // labels per 16-byte chunk
      constexpr int kNlc = 128 / kChunk;                      // chunks per 128-label tile
      unsigned long long* wm = reinterpret_cast<unsigned long long*>(S->pmask[warp - 2]);
      const int b = amb * 128 + q * 32 + lane;               // this thread's sample
      // queue entries gp, gp + kGroups, ...: this group's tiles, in the order taken
      for (uint32_t lt = (uint32_t)gp; !*abort; lt += kGroups) {
        const int qs = (int)(lt % kFQ);
        if (!mbar_wait(&S->qfull[qs], (lt / kFQ) & 1, abort, kWaitCycles)) { record_timeout(status, abort, 88); break; }
        const int t = S->tq[qs];
        __syncwarp();
        if (lane == 0) mbar_arrive(&S->qempty[qs]);
        if (t < 0) break;
        const int slot = t % R, round = t / R;
        uint8_t* gtile = gring + (size_t)slot * tile_bytes;
        // the ring slot's consumed count, read now and checked before the
        // stores (the slot is free once every d-slice's CTA has copied the
        // tile it held), and the tile's range of keys
        const int32_t cnow = round > 0 ? ld_relaxed(consumed + slot) : 0;
        const int k0 = __ldg(tile_ptr + t), k1 = __ldg(tile_ptr + t + 1);
        // positives among this thread's elements of the tile (bit kColW hf + c
        // for label column kN hf + c_lo + c), from the tile's keys: the warp
        // reads them together (a frequent label's tile holds hundreds) and
        // scatters each into the mask of its sample's lane
        uint64_t pm;
        {
          wm[lane] = 0;
          __syncwarp();
          const int64_t lbase = (int64_t)t * 128 + c_lo;
          for (int i = k0 + lane; i < k1; i += 32) {
            const uint32_t key = __ldg(keys + i);
            const int smp = (int)(key & 0xFFu);
            const int sl = smp - amb * 128 - 32 * q;                // the sample's lane here
            const int64_t dl = (int64_t)(key >> 8) - lbase;
            const int hk = dl >= RA::kN ? 1 : 0;                     // the half (bf16)
            const int64_t c = dl - hk * RA::kN;
            if (sl >= 0 && sl < 32 && dl >= 0 && c < kColW) atomicOr(wm + sl, 1ull << (kColW * hk + c));
          }
          __syncwarp();
          pm = wm[lane];
          __syncwarp();
        }
        bool stop = false;
        bool free_checked = round == 0;
        for (int hf = 0; hf < RA::kHalves && !stop; ++hf) {
          const uint32_t buf = (uint32_t)gp * RA::kHalves + (uint32_t)hf;
          const uint32_t ph = (lt / kGroups) & 1;
          if (!mbar_wait(&S->tfull[buf], ph, abort, kWaitCycles)) {
            record_timeout(status, abort, 86);
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + RA::kAcc + buf * RA::kN + (uint32_t)c_lo;
#pragma unroll
          for (int cc = 0; cc < kColW; cc += 32) {
            constexpr int kLd = kColW < 32 ? kColW : 32;
            uint32_t v[kLd];
            if (kLd == 32) tmem_ld32(tbase + cc, *reinterpret_cast<uint32_t(*)[32]>(v));
            else tmem_ld16(tbase + cc, *reinterpret_cast<uint32_t(*)[16]>(v));
            tmem_wait_ld();
            if (cc + 32 >= kColW) {                           // the last load from this slot
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&S->tempty[buf]);
            }
            if (!free_checked) {
              // the slot must be free before the first store into it
              bool ok = cnow >= nD * round;
              if (!ok) {
                if (lane == 0) ok = wait_flag(consumed + slot, nD * round, abort, status, kWaitCycles);
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
              }
              if (!ok) { if (lane == 0) record_timeout(status, abort, 85); stop = true; break; }
              free_checked = true;
            }
#pragma unroll
            for (int j = 0; j < kLd; j += 16) {
              const int col = hf * RA::kN + c_lo + cc + j;          // label column within the tile
              const int64_t nv = L - ((int64_t)t * 128 + col);
              const uint32_t vbits = b >= B || nv <= 0 ? 0u : (nv >= 16 ? 0xFFFFu : (1u << nv) - 1u);
              uint32_t pk[8];
              grad_codes16<kG>(v + j, inv_sx, acc_lo, (uint32_t)(pm >> (kColW * hf + cc + j)) & 0xFFFFu, vbits,
                               pk);
              if (b < Bp) {
                const int lc = col / kChunk;
                *reinterpret_cast<uint4*>(gtile + ((size_t)(b >> 3) * kNlc + lc) * 128 + (b & 7) * 16) =
                    make_uint4(pk[0], pk[1], pk[2], pk[3]);
                if (!kFp8)
                  *reinterpret_cast<uint4*>(gtile + ((size_t)(b >> 3) * kNlc + lc + 1) * 128 + (b & 7) * 16) =
                      make_uint4(pk[4], pk[5], pk[6], pk[7]);
              }
            }
          }
        }
        if (stop) break;
        // publish the tile once the group's warps have stored their parts:
        // each thread orders its stores with the async proxy (the bulk copies
        // that read them); the warp's stores are ordered before its arrival
        // at CTA scope (__syncwarp, then a CTA fence), and the last warp to
        // arrive makes every arrival's stores visible at GPU scope (its fence
        // is cumulative) and releases the flag.  No thread but that one waits
        // on a GPU-scope fence, and no barrier can be left waiting by a warp
        // that stopped early.
        fence_proxy_async_global();
        __syncwarp();
        if (lane == 0) {
          __threadfence_block();
          const int old = atomicAdd(&S->arrivals[lt & 3], 1);
          if (old == kWarpsG - 1) {
            S->arrivals[lt & 3] = 0;
            __threadfence();
            red_release_add(ready + slot, 1);      // nprod arrivals per round make the tile ready
          }
        }
      }
    }
    __syncthreads();
    if (*abort) __nanosleep(20000);   // let copies in flight land before the shared memory goes away
    if (warp == 1) { tc_fence_after(); tmem_dealloc(tmem, 512); }
    return;
  }

  // ========================================================== role B
  const int bid = (int)blockIdx.x - nA;
  const int g = bid / nD, sl = bid % nD;
  if (g >= nG) return;                                        // spare CTA
  constexpr int kWS = kFp8 ? 4 : 2;
  // bf16: the epilogue writes the new weights back into the W slot and the
  // TMA warp stores the slot (measured: 8.6M-label step 10.5 -> 8.9 ms, 500K
  // 0.86 -> 0.69 ms); E4M3: each thread stores its 16 codes (1 to 2 % faster
  // there, its slices being half as wide)
  constexpr bool kWB = !kFp8;
  constexpr uint32_t kWSB = kFp8 ? kBox : 2 * kBox;
  constexpr int kBoxCols = 128 / kEl;                         // elements per 128-byte box row
  constexpr int kK = kFp8 ? 32 : 16;                          // MMA K
  constexpr int kPart = kFp8 ? 256 : 128;                     // samples per G part (one 32 KB slot)
  const int nparts = (Bp + kPart - 1) / kPart;
  const int nprod = Bp > 128 ? 2 : 1;
  uint8_t* xs = base;
  uint8_t* ws = xs + kFXBytes;
  uint8_t* gs = ws + kFWBytes;
  SmemFB* S = reinterpret_cast<SmemFB*>(gs + kFGSlots * kFGSlotBytes);
  volatile int* abort = &S->abort;
  const int D0 = sl * 128;
  if (threadIdx.x == 0) {
    mbar_init(&S->xfull, 1);
    mbar_init(&S->dxfull, 1);
    // a W slot holds the unit's new weights once all sixteen epilogue warps
    // have written them back (the unit's MMAs, which read the old ones, have
    // completed before the epilogue starts); the TMA warp then stores it
    // (E4M3: free once the epilogue is done with it and the unit's dX^T MMAs
    // have completed: an mma_commit counts too)
    for (int s = 0; s < kWS; ++s) { mbar_init(&S->wfull[s], 1); mbar_init(&S->wempty[s], kWB ? kFEpi : kFEpi + 1); }
    for (int s = 0; s < kFGSlots; ++s) { mbar_init(&S->gfull[s], 1); mbar_init(&S->gempty[s], 1); }
    for (int b2 = 0; b2 < 2; ++b2) { mbar_init(&S->dwfull[b2], 1); mbar_init(&S->dwempty[b2], kFEpi); }
    // queue entries: read by the MMA warp and by every epilogue warp
    for (int i = 0; i < kFQ; ++i) { mbar_init(&S->qfull[i], 1); mbar_init(&S->qempty[i], 1 + kFEpi); }
    S->first_t = -1;
    S->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) { tmem_alloc(&S->tmem_base, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S->tmem_base;
  int nb = 0;                                                 // 128-byte boxes in this slice
  for (int qq = 0; qq < 128 / kBoxCols; ++qq) nb += (D0 + qq * kBoxCols < d);

  if (warp == 0) {
    if (elect_one()) {
      tma_prefetch_desc(&tmWb);
      tma_prefetch_desc(&tmX);
      mbar_arrive_expect_tx(&S->xfull, (uint32_t)nb * (uint32_t)Bp * 128u);
      for (int qq = 0; qq < 128 / kBoxCols; ++qq)
        if (D0 + qq * kBoxCols < d) tma_load_2d(xs + qq * 32768, &tmX, &S->xfull, D0 + qq * kBoxCols, 0);
      // units of this slice are handed out in tile order (sched[2 + slice]):
      // take the next, pass it to the MMA warp and the epilogue, then load
      // its W slice and copy its G tile once role A has published it
      uint32_t wit = 0, git = 0;
      int slot_t[kWS];                                        // the tile whose W slice a slot holds
      for (int s = 0; s < kWS; ++s) slot_t[s] = -1;
      // the new weights of the tile that slot s held go back to W with one
      // bulk tensor store per 128-byte column box (rows past L are clipped)
      auto store_slot = [&](int s) {
        for (int qq = 0; qq < 128 / kBoxCols; ++qq)
          if (D0 + qq * kBoxCols < d) tma_store_2d(&tmWb, ws + s * kWSB + qq * kBox, D0 + qq * kBoxCols, slot_t[s] * 128);
        bulk_commit_group();
      };
      int t_next = atomicAdd(sched + 2 + sl, 1);              // taken one unit ahead
      for (uint32_t i = 0;; ++i) {
        const int qs = (int)(i % kFQ);
        if (!mbar_wait(&S->qempty[qs], ((i / kFQ) & 1) ^ 1, abort, kWaitCycles)) {
          record_timeout(status, abort, 90);
          break;
        }
        int t = t_next;
        if (t >= T || *abort) t = -1;
        else t_next = atomicAdd(sched + 2 + sl, 1);
        if (i == 0) S->first_t = t;
        S->tq[qs] = t;
        mbar_arrive(&S->qfull[qs]);
        if (t < 0) break;
        {
          const int s = wit % kWS;
          const uint32_t ph = (wit / kWS) & 1;
          ++wit;
          if (!mbar_wait(&S->wempty[s], ph ^ 1, abort, kWaitCycles)) { record_timeout(status, abort, 91); break; }
          if (kWB && slot_t[s] >= 0) {
            store_slot(s);
            bulk_wait_read_all();                             // the store has read the slot
          }
          slot_t[s] = t;
          mbar_arrive_expect_tx(&S->wfull[s], (uint32_t)nb * kBox);
          for (int qq = 0; qq < 128 / kBoxCols; ++qq)
            if (D0 + qq * kBoxCols < d) tma_load_2d(ws + s * kWSB + qq * kBox, &tmWb, &S->wfull[s], D0 + qq * kBoxCols, t * 128);
        }
        const int slot = t % R, round = t / R;
        if (!wait_flag(ready + slot, nprod * (round + 1), abort, status, kWaitCycles)) {
          record_timeout(status, abort, 93);
          break;
        }
        fence_proxy_async_global();
        bool stop = false;
        for (int p = 0; p < nparts; ++p) {
          const int s = git % kFGSlots;
          const uint32_t ph = (git / kFGSlots) & 1;
          ++git;
          if (!mbar_wait(&S->gempty[s], ph ^ 1, abort, kWaitCycles)) { record_timeout(status, abort, 92); stop = true; break; }
          // samples [p kPart, p kPart + np): a contiguous run of 16-byte chunks
          const int np = min(kPart, Bp - p * kPart);
          const uint32_t bytes = (uint32_t)np * kEl * 128u;
          mbar_arrive_expect_tx(&S->gfull[s], bytes);
          bulk_load(gs + s * kFGSlotBytes, gring + (size_t)slot * tile_bytes + (size_t)p * kPart * kEl * 128u, bytes,
                    &S->gfull[s]);
        }
        if (stop) break;
      }
      // the last unit of each slot: its epilogue's completion is use
      // (n / kWS) of the slot's barrier, n the unit's index
      for (uint32_t n = wit > (uint32_t)kWS ? wit - kWS : 0u; kWB && n < wit && !*abort; ++n) {
        const int s = (int)(n % kWS);
        if (!mbar_wait(&S->wempty[s], (n / kWS) & 1, abort, kWaitCycles)) { record_timeout(status, abort, 91); break; }
        store_slot(s);
      }
      bulk_wait_all();
    }
  } else if (warp == 1) {
    if (elect_one()) {
      const uint32_t gfmt = kG5 ? 1u : 0u;
      // G is stored sample-major: K-major as dX^T's B operand, MN-major as dW's A operand
      const uint32_t idesc_dw = kFp8 ? make_idesc(gfmt, 0, 1, 1, 128, 128) : make_idesc(1, 1, 1, 1, 128, 128);
      const uint32_t gstride = (uint32_t)(kFp8 ? 8 : 16) * 128u;   // bytes between 8-sample groups
      uint32_t wit = 0, git = 0, dwit = 0;
      bool first = true;
      if (!mbar_wait(&S->xfull, 0, abort, kWaitCycles)) record_timeout(status, abort, 94);
      tc_fence_after();
      const uint32_t xa = smem_u32(xs);
      for (uint32_t i = 0; !*abort; ++i) {
        const int qs = (int)(i % kFQ);
        if (!mbar_wait(&S->qfull[qs], (i / kFQ) & 1, abort, kWaitCycles)) { record_timeout(status, abort, 89); break; }
        const int t = S->tq[qs];
        mbar_arrive(&S->qempty[qs]);
        if (t < 0) break;
        const int sw = wit % kWS;
        const uint32_t phw = (wit / kWS) & 1;
        ++wit;
        const uint32_t db = dwit & 1, duse = dwit >> 1;
        ++dwit;
        if (!mbar_wait(&S->wfull[sw], phw, abort, kWaitCycles)) { record_timeout(status, abort, 95); break; }
        if (!mbar_wait(&S->dwempty[db], (duse & 1) ^ 1, abort, kWaitCycles)) { record_timeout(status, abort, 96); break; }
        tc_fence_after();
        const uint32_t wa = smem_u32(ws + sw * kWSB);
        const uint32_t dwcol = tmem + 256 + db * 128;
        bool stop = false;
        // dW, then dX^T (which reads the old W in the slot).  bf16: the
        // epilogue waits for both, since it writes the new W into the same
        // slot; E4M3: for dW only.  The G parts (at most two) stay in their
        // slots until both are issued
        int sgs[2] = {0, 0};
        for (int p = 0; p < nparts; ++p) {
          const int sg = git % kFGSlots;
          const uint32_t phg = (git / kFGSlots) & 1;
          ++git;
          if (!mbar_wait(&S->gfull[sg], phg, abort, kWaitCycles)) { record_timeout(status, abort, 97); stop = true; break; }
          tc_fence_after();
          // G_t is in shared memory once its last part is: the ring slot may be
          // reused.  The copies that read it have completed, so the count
          // needs no release ordering (and the issuing thread no fence).
          if (p == nparts - 1) atomicAdd(consumed + t % R, 1);
          sgs[p] = sg;
          const uint32_t ga = smem_u32(gs + sg * kFGSlotBytes);
          const int np = min(kPart, Bp - p * kPart);
          // dW[tile, slice] += G_part^T X[part, slice] : M = 128 labels, N = 128, K = np samples
          {
            const uint64_t ad0 = nosw_desc(ga, gstride, 128);
            const uint64_t bd0 = sw128_desc(xa + p * kPart * 128, 32768, 1024);
#pragma unroll 4
            for (int k = 0; k < np / kK; ++k) {
              const uint64_t ad = ad0 + (uint64_t)(k * ((kK / 8) * gstride >> 4));
              const uint64_t bd = bd0 + (uint64_t)(k * (kK * 128 >> 4));
              if (kFp8) mma_e4m3(dwcol, ad, bd, idesc_dw, (p | k) != 0);
              else mma_bf16(dwcol, ad, bd, idesc_dw, (p | k) != 0);
            }
          }
        }
        if (stop) break;
        if (!kWB) mma_commit(&S->dwfull[db]);
        for (int p = 0; p < nparts; ++p) {
          const uint32_t ga = smem_u32(gs + sgs[p] * kFGSlotBytes);
          const int np = min(kPart, Bp - p * kPart);
          const uint32_t idesc_dx =
              kFp8 ? make_idesc(kW5, gfmt, 1, 0, 128, (uint32_t)np) : make_idesc(1, 1, 1, 0, 128, (uint32_t)np);
          // dX^T[slice, part] += W^T G_part^T : M = 128 (columns of d), N = np, K = 128 labels
          {
            const uint64_t ad0 = sw128_desc(wa, kBox, 1024);
            const uint64_t bd0 = nosw_desc(ga, 128, gstride);
#pragma unroll 4
            for (int k = 0; k < 128 / kK; ++k) {
              const uint64_t ad = ad0 + (uint64_t)(k * (kK * 128 >> 4));
              const uint64_t bd = bd0 + (uint64_t)(k * (2 * 128 >> 4));
              if (kFp8) mma_e4m3(tmem + (uint32_t)(p * kPart), ad, bd, idesc_dx, !(first && k == 0));
              else mma_bf16(tmem + (uint32_t)(p * kPart), ad, bd, idesc_dx, !(first && k == 0));
            }
          }
          mma_commit(&S->gempty[sgs[p]]);
        }
        mma_commit(kWB ? &S->dwfull[db] : &S->wempty[sw]);
        first = false;
      }
      mma_commit(&S->dxfull);
    }
  } else {
    // All sixteen warps take every unit: warp (q = warp % 4, sub) updates
    // label row 32 q + lane and columns 32 sub .. 32 sub + 31 of the slice.
    // The unit's dW slot (units alternate between two) is released as soon
    // as the warps have loaded it, so the MMA warp can form the next unit's
    // dW while this unit's update runs.
    const int q = warp & 3;
    const int sub = (warp - 2) >> 2;
    const int row = q * 32 + lane;                  // label row of dW; column of d for dX^T
    const float lrs = kFp8 ? lr * (0.00390625f * xscale[1]) : lr;
    const float dx_scale = kFp8 ? 0.00390625f : 1.0f;
    constexpr int kWf = kFp8 ? (kW5 ? 2 : 1) : 0;
    bool any = false;                               // the CTA took at least one unit
    for (uint32_t ui = 0; !*abort; ++ui) {
      const int qs = (int)(ui % kFQ);
      if (!mbar_wait(&S->qfull[qs], (ui / kFQ) & 1, abort, kWaitCycles)) { record_timeout(status, abort, 100); break; }
      const int t = S->tq[qs];
      if (ui == 0) any = S->first_t >= 0;
      __syncwarp();
      if (lane == 0) mbar_arrive(&S->qempty[qs]);
      if (t < 0) break;
      const int sw = (int)(ui % kWS);
      const uint32_t db = ui & 1, use = ui >> 1;
      const int64_t l = (int64_t)t * 128 + row;
      const int jl = sub * 32;                      // columns jl .. jl + 31 of the 128-column slice
      const int j0 = D0 + jl;
      const bool valid = l < L && j0 < d;           // d is a multiple of 64: all 32 columns or none
      // the draws do not depend on the gradient: form them while the MMAs run
      // (bf16: both chunks' four Philox blocks here, measured 4 % faster on the
      // 8.6M-label step; E4M3: the second chunk's after the first update,
      // 9 % faster on the 3M-label step)
      uint32_t rw[8], rw1[8];
      if (valid) {
        sr_draws16(rk, step, blk_base, l, d, j0, rw);
        if (!kFp8) sr_draws16(rk, step, blk_base, l, d, j0 + 16, rw1);
      }
      if (!mbar_wait(&S->dwfull[db], use & 1, abort, kWaitCycles)) { record_timeout(status, abort, 98); break; }
      tc_fence_after();
      const uint8_t* wrow = ws + sw * kWSB;
      const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + 256 + db * 128 + jl;
      uint32_t ra[16], rb[16];
      tmem_ld16(taddr, ra);
      tmem_ld16(taddr + 16, rb);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S->dwempty[db]);
      if (valid) {
        // bf16: the new codes go back into the slot, in place of the old ones
        update16<kWf, kWB>(ra, rw, wrow, row, jl, l, d, j0, lrs, Wglob);
        if (kFp8) sr_draws16(rk, step, blk_base, l, d, j0 + 16, rw1);
        update16<kWf, kWB>(rb, rw1, wrow, row, jl + 16, l, d, j0 + 16, lrs, Wglob);
        if (kWB) fence_proxy_async_smem();            // visible to the bulk store that reads the slot
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&S->wempty[sw]);
    }
    if (any && !*abort) {
      // flush dX^T of this CTA: lane = column j of the slice, TMEM columns = samples
      if (!mbar_wait(&S->dxfull, 0, abort, kWaitCycles)) {
        record_timeout(status, abort, 99);
      } else {
        tc_fence_after();
        const int j = D0 + row;
        const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16);
        for (int c = (warp - 2) >> 2; c < Bp / 32; c += 4) {
          uint32_t ra[32];
          tmem_ld32(taddr + c * 32, ra);
          tmem_wait_ld();
          if (j < d) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int bb = c * 32 + i;
              if (bb < B) atomicAdd(dX + (size_t)bb * d + j, __uint_as_float(ra[i]) * dx_scale);
            }
          }
        }
      }
    }
  }
  __syncthreads();
  if (*abort) __nanosleep(20000);
  if (warp == 1) { tc_fence_after(); tmem_dealloc(tmem, 512); }
}

}  // namespace

bool fused_step_supported(const elmo_head* h, int32_t B) {
  const char* v = getenv("ELMO_STEP_FUSED");
  if (v && v[0] == '0') return false;
  const bool fp8 = h->dt == ELMO_FP8_E4M3;
  const int32_t Bp = padded_batch(B, fp8);
  return h->d % 64 == 0 && h->d <= 768 && Bp <= 256;
}

// The split of the SMs between the roles follows their measured cost per
// 128-label tile on B200 at the workloads' shapes (d = 768): role A (Z and G
// of the tile; two CTAs per tile when B > 128) against role B (dX^T, dW and
// the SR update of the tile's weights for every d-slice).  Measured optima:
// E4M3 with two producers per tile 31 % of the SMs for role A (46 of 148; the
// 3M-label step at 2.48 ms against 2.55 at 44 and 2.63 at 48); bf16 with two
// producers 35 % (52; the 500K-label step at 0.70 ms against 0.72 at 48 and
// 0.75 at 56), with one 23 % (34; the 8.6M-label step at 8.8 ms, 9.1 at 32,
// 9.3 at 38).  E4M3 with one producer (no workload measured) 19 %, from the same
// per-tile costs.  ELMO_FUSED_A overrides nA.
void fused_split(int grid, int nD, int T, int nprod, bool fp8, int* nA, int* nG) {
  const int pct = fp8 ? (nprod == 2 ? 31 : 19) : (nprod == 2 ? 35 : 23);
  int a = (grid * pct + 50) / 100;
  const char* v = getenv("ELMO_FUSED_A");
  if (v && atoi(v) > 0) a = atoi(v);
  if (a > grid - nD) a = grid - nD;
  if (a > nprod * T) a = nprod * T;
  a = a / nprod * nprod;                            // whole groups of producers
  if (a < nprod) a = nprod;
  int gg = (grid - a) / nD;
  if (gg > T) gg = T;
  *nA = a;
  *nG = gg;
}

cudaError_t launch_step_fused(elmo_head* h, const uint16_t* X, int32_t B, float lr, uint64_t seed, uint64_t step,
                              float* dX, cudaStream_t s) {
  const bool fp8 = h->dt == ELMO_FP8_E4M3;
  const int eb = fp8 ? 1 : 2;
  const int32_t Bp = padded_batch(B, fp8);
  const int T = (int)((h->L + 127) / 128);
  const int nD = (h->d + 127) / 128;
  int nA = 0, nG = 0;
  fused_split(h->num_sms, nD, T, Bp > 128 ? 2 : 1, fp8, &nA, &nG);
  const int grid = nA + nG * nD;
  CUtensorMap tmWa, tmWa3, tmWb, tmX;
  cudaError_t e = make_tma_map_2d(&tmWa, h->W, eb, (uint64_t)h->d, (uint64_t)h->L, (uint64_t)h->d,
                                  fp8 ? RoleA<1>::kN : RoleA<0>::kN);
  if (e != cudaSuccess) return e;
  // role A's 3-D view needs rows of whole 128-byte k-blocks (else the view
  // would run into the next row): then one request per ring stage
  const int nkb = (int)((h->d * eb + 127) / 128);
  const int wa3 = (h->d * eb) % 128 == 0 ? 1 : 0;
  if (wa3) {
    e = make_tma_map_kb3d(&tmWa3, h->W, eb, (uint64_t)h->d, (uint64_t)h->L, RoleA<1>::kN,
                          (uint32_t)std::min(nkb, RoleA<1>::kKbs));
    if (e != cudaSuccess) return e;
  } else {
    tmWa3 = tmWa;                                   // not read
  }
  e = make_tma_map_2d(&tmWb, h->W, eb, (uint64_t)h->d, (uint64_t)h->L, (uint64_t)h->d, 128);
  if (e != cudaSuccess) return e;
  e = make_tma_map_2d(&tmX, fp8 ? static_cast<const void*>(h->xq) : static_cast<const void*>(X), eb, (uint64_t)h->d,
                      (uint64_t)B, (uint64_t)h->d, (uint32_t)Bp);
  if (e != cudaSuccess) return e;
  auto kern = fp8 ? (h->g_e5m2 ? step_fused<1, 1> : h->w_e5m2 ? step_fused<1, 0, 1> : step_fused<1, 0>)
                  : step_fused<0, 0>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemF);
  if (e != cudaSuccess) return e;
  // the ring's flags and the tile counters start at zero every step
  e = cudaMemsetAsync(h->ring_flags, 0, sizeof(int32_t) * (2 * (size_t)h->ring_tiles + kRingCounters), s);
  if (e != cudaSuccess) return e;
  const uint8_t* xop = fp8 ? h->xqt : reinterpret_cast<const uint8_t*>(X);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3((unsigned)kFThreads);
  cfg.dynamicSmemBytes = kSmemF;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeCooperative;   // every CTA resident: the roles wait on one another
  at[0].val.cooperative = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tmWa, tmWa3, wa3, tmWb, tmX, h->W, h->L, h->d, B, Bp, xop, (const uint32_t*)h->keys,
                            (const int32_t*)h->tile_ptr, (const float*)h->xscale, static_cast<uint8_t*>(h->ring),
                            h->ring_tiles, h->ring_flags, h->ring_flags + h->ring_tiles,
                            h->ring_flags + 2 * h->ring_tiles, nA, nG, lr, philox_keys(seed), step,
                            (uint64_t)h->label_base * (uint64_t)h->d / 8, dX, h->status);
}

}  // namespace elmo
