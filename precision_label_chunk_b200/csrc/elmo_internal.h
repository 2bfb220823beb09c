// elmo_internal.h -- host-side structures and kernel launchers of libelmo.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <vector>

#include "../../include/elmo.h"

struct CUtensorMap_st;   // cuda.h's TMA descriptor (CUtensorMap)

struct elmo_prof_rec {
  int cls;
  cudaEvent_t start, stop;
};

struct elmo_head {
  void* W = nullptr;           // borrowed [L x d] bf16 bits or E4M3 codes
  int64_t L = 0;
  int64_t label_base = 0;      // W holds the label rows [label_base, label_base + L) ...
  int64_t labels_total = 0;    // ... of a head of labels_total labels (0 and L when unsharded)
  int32_t d = 0;
  elmo_dtype dt = ELMO_BF16;    // format of W (and of X and G in the tensor cores): BF16 or E4M3
  bool g_e5m2 = false;         // E4M3 step whose gradient operand G is E5M2 (ELMO_FP8_E4M3_GE5M2)
  bool w_e5m2 = false;         // E5M2 weights (ELMO_FP8_E5M2 head): X and G stay E4M3
  int device = 0;
  int num_sms = 0;
  // workspace owned by the head
  int32_t* status = nullptr;   // [4]: status code, first bad index, spare
  uint32_t* keys = nullptr;    // [ELMO_MAX_NNZ] (label << 8 | sample) positives grouped by label tile
  int32_t* nkeys = nullptr;    // [1] number of valid keys
  int32_t* tile_ptr = nullptr; // [ceil(L/128) + 1] first key of every 128-label tile
  cudaStream_t side = nullptr; // second stream for work that overlaps a kernel of the caller's stream
  cudaEvent_t fork = nullptr, join = nullptr;
  float* xscale = nullptr;     // [2] s_X, 1/s_X (fp8 mode)
  uint8_t* xq = nullptr;       // [ELMO_MAX_BATCH x d] E4M3 codes of X * s_X (fp8 mode)
  uint8_t* xqt = nullptr;      // the same codes by 16-byte column chunk: [d/16][ELMO_MAX_BATCH][16]
  void* gbuf = nullptr;        // per-chunk gradient operands
  size_t gbuf_bytes = 0;
  void* ring = nullptr;        // the persistent step's ring of gradient-operand tiles
  int32_t* ring_flags = nullptr; // [2 * ring_tiles]: ready, then consumed; then kRingCounters tile counters (zeroed every step)
  int32_t ring_tiles = 0;
  size_t ring_bytes = 0;
  void* cand = nullptr;        // top-k candidates
  size_t cand_bytes = 0;
  size_t base_bytes = 0;       // bytes of the fixed part of the workspace
  // tracing
  bool prof = false;
  std::vector<elmo_prof_rec> prof_recs;
  std::vector<cudaEvent_t> prof_pool;
  int64_t launches = 0;
};

namespace elmo {
// Brackets the kernel launches of one class with events when tracing is on,
// and counts launches.  `n` is the number of kernels launched inside.
struct KernelScope {
  elmo_head* h;
  cudaStream_t s;
  elmo_prof_rec rec{};
  bool on;
  KernelScope(elmo_head* h_, int cls, cudaStream_t s_, int n = 1);
  ~KernelScope();
};
}  // namespace elmo

namespace elmo {

// The stored weights' grid: ELMO_BF16, ELMO_FP8_E4M3 or ELMO_FP8_E5M2.
inline int w_format(const elmo_head* h) { return h->w_e5m2 ? (int)ELMO_FP8_E5M2 : (int)h->dt; }

constexpr int kTileLabels = 128;        // labels per tensor-core tile

// Labels per pass of the tensor-core step: the caller's chunk, capped so that
// the gradient operands of one pass (the transient buffer chunking bounds)
// stay within 128 MB.  Longer passes amortise each kernel's fill and drain.
inline int64_t sub_chunk_labels(int32_t d, int32_t Bp, int elem_bytes) {
  (void)d;
  const int64_t per_label = (int64_t)Bp * elem_bytes;
  int64_t n = (int64_t(128) << 20) / per_label;
  n = n / 128 * 128;
  return n < 128 ? 128 : n;
}

// api.cu: the thread-local message elmo_last_error() returns
void set_last_error(const char* msg);

// prep.cu
cudaError_t launch_prep_labels(elmo_head* h, const int32_t* rowptr, const int32_t* cols, int32_t B,
                               int32_t nnz, cudaStream_t s);
cudaError_t launch_prep_x(elmo_head* h, const uint16_t* X, int32_t B, cudaStream_t s);
// the labels and (E4M3) X of a training step, in one launch
cudaError_t launch_prep_step(elmo_head* h, const int32_t* rowptr, const int32_t* cols, int32_t B, int32_t nnz,
                             const uint16_t* X, cudaStream_t s);

// step_tc.cu -- tensor-core step
// 2-D row-major TMA map [rows x cols] of 1- or 2-byte elements, box = 128 bytes
// x box_rows, 128-byte swizzle, zero fill outside the tensor.
cudaError_t make_tma_map_2d(CUtensorMap_st* m, const void* ptr, int elem_bytes, uint64_t cols, uint64_t rows,
                            uint64_t row_stride_elems, uint32_t box_rows);
cudaError_t make_tma_map_kb3d(CUtensorMap_st* m, const void* ptr, int elem_bytes, uint64_t cols, uint64_t rows,
                              uint32_t box_rows, uint32_t box_kb);
int32_t padded_batch(int32_t B, bool fp8);
cudaError_t launch_wait_check(long long limit_cycles, int32_t* status, cudaStream_t s);
// pdl: launch programmatically dependent on the previous kernel in the stream,
// which must be this step's kernel B (for A) or A (for B); the kernels wait
// for it before touching what it produces or consumes.
cudaError_t launch_logits_grad_tc(const elmo_head* h, const uint16_t* X, int32_t B, int64_t l0, int64_t l1,
                                  void* gbuf, float* Zout, float* Gout, cudaStream_t s, bool pdl = false);
cudaError_t launch_update_tc(const elmo_head* h, const uint16_t* X, int32_t B, int64_t l0, int64_t l1,
                             const void* gbuf, float lr, uint64_t seed, uint64_t step, float* dX, cudaStream_t s,
                             bool pdl = false);

// step_fused.cu -- the whole step in one persistent, cooperative launch (role A:
// logits and gradient operands into a ring of tiles; role B: dX, dW and the SR
// update), for the shapes whose X fits in TMEM
bool fused_step_supported(const elmo_head* h, int32_t B);
constexpr int32_t kRingTiles = 256;      // gradient-operand tiles in the ring
constexpr int32_t kRingCounters = 16;    // after the ring's flags: the persistent step's tile counters
cudaError_t launch_step_fused(elmo_head* h, const uint16_t* X, int32_t B, float lr, uint64_t seed, uint64_t step,
                              float* dX, cudaStream_t s);

// topk_simt.cu -- exact top-k on CUDA cores, for all rows (rows == null) or
// for the *nrows rows listed in rows (a list whose length lives on the device)
size_t topk_simt_workspace_bytes(const elmo_head* h, int32_t B, int32_t k);
cudaError_t launch_topk_simt_rows(const elmo_head* h, const uint16_t* X, int32_t B, int32_t k, const int32_t* rows,
                                  const int32_t* nrows, void* cand, int32_t* idx, float* score, cudaStream_t s);

// topk_tc.cu -- tensor-core screening, exact rescoring and certificate, with
// the CUDA-core path for the rows the certificate does not clear
bool topk_tc_supported(const elmo_head* h);
size_t topk_tc_workspace_bytes(const elmo_head* h, int32_t B, int32_t k);
cudaError_t launch_topk_tc(elmo_head* h, const uint16_t* X, int32_t B, int32_t k, int32_t* idx, float* score,
                           cudaStream_t s);
// rows of the last launch_topk_tc(B, k) that the certificate sent to the exact path (synchronises s)
cudaError_t topk_uncertified_rows(elmo_head* h, int32_t B, int32_t k, int32_t* rows, cudaStream_t s);
// inspection: screening scores S [B x (l1 - l0)] and each row's certificate bound [B]
cudaError_t launch_topk_screen_dump(elmo_head* h, const uint16_t* X, int32_t B, int64_t l0, int64_t l1, float* S,
                                    float* bound, cudaStream_t s);

// metrics.cu
cudaError_t launch_precision_at_k(const int32_t* idx, int32_t B, int32_t k, const int32_t* rowptr,
                                  const int32_t* cols, int32_t nnz, float* p, cudaStream_t s);

// sr.cu
cudaError_t launch_sr_round(const float* in, void* out, int64_t n, elmo_dtype dt, uint64_t seed,
                            uint64_t step, uint64_t base, cudaStream_t s);
cudaError_t launch_sr_draws(uint16_t* out, int64_t n, uint64_t seed, uint64_t step, uint64_t base,
                            cudaStream_t s);
cudaError_t launch_fill(void* W, int64_t n, elmo_dtype dt, float std, uint64_t seed, uint64_t index_base,
                        cudaStream_t s);
cudaError_t launch_sr_e5m2(const float* in, uint8_t* out, int64_t n, uint64_t seed, uint64_t step, uint64_t base,
                           cudaStream_t s);
cudaError_t launch_kahan_sgd(void* p, void* c, const void* g, int64_t n, float lr, cudaStream_t s);
cudaError_t launch_round_bf16(const float* in, void* out, int64_t n, cudaStream_t s);
// global label ids of a sharded head's top-k (idx += label_base)
cudaError_t launch_topk_offset(int32_t* idx, int64_t n, int64_t label_base, cudaStream_t s);
cudaError_t launch_topk_merge(const int32_t* idx, const float* score, int32_t P, int32_t B, int32_t k,
                              int32_t* idx_out, float* score_out, cudaStream_t s);

}  // namespace elmo
