/*
 * elmo.h -- C ABI of the B200 (sm_100a) ELMO classifier-head library.
 *
 * What it computes: the training step and the prediction of the extreme
 * multilabel classifier head of "ELMO: Efficiency via Low-precision and Peak
 * Memory Optimization in Large Output Spaces" (Zhang, Ullah, Schultheis,
 * Babbar, ICML 2025; arXiv 2510.11168).  The head W [L x d] is stored in pure
 * BF16 or unscaled FP8 E4M3 with no FP32 master copy (abstract; atlas summary,
 * "Approach" and "Surprising findings": E4M3 native range suffices) and is
 * trained by momentum-free SGD with stochastic rounding, the classifier
 * gradient fused with the update and the label axis processed in chunks
 * ("Approach": gradient fusion and chunking to cut transient memory).
 *
 * Conventions for every call:
 *   - Pointers named *_dev are device pointers owned by the caller; the
 *     library only borrows them for the duration of the work it enqueues.
 *   - All work is enqueued on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and is asynchronous: a call returns once the work is
 *     enqueued.  Argument errors are reported synchronously; data errors found
 *     by kernels (malformed label lists) and bounded-wait timeouts are written
 *     to a device status word and surface from elmo_sync_status() or from the
 *     next call on the same head.
 *   - Return values are elmo_status codes; elmo_last_error() gives a message
 *     (thread-local) for the most recent failure on the calling thread.
 *   - Matrices are row-major and densely packed; device pointers must be
 *     16-byte aligned unless the call says otherwise (the element-wise calls
 *     elmo_sr_round, elmo_kahan_sgd and elmo_round_bf16 take any alignment).
 *   - There is no CPU fallback: on a machine without an sm_100 GPU the calls
 *     return ELMO_ECUDA or ELMO_EUNSUPPORTED.
 */
#ifndef ELMO_H_
#define ELMO_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ELMO_BF16 = 0,           /* bfloat16 weights (8-bit exponent, 7-bit mantissa) */
  ELMO_FP8_E4M3 = 1,       /* OCP E4M3FN weights: max 448, no infinities, saturating */
  ELMO_FP8_E4M3_GE5M2 = 2, /* E4M3 weights (and X) as above; the training step's gradient
                              operand is OCP E5M2 of 2^8 G instead of E4M3 (heads only) */
  ELMO_FP8_E5M2 = 3        /* OCP E5M2 values (max 57344, with infinities): an SR output grid of
                              elmo_sr_round, and as a head E5M2 weights with X and the
                              gradient operand in E4M3 (the adjacent 8-bit format) */
} elmo_dtype;

typedef enum {
  ELMO_OK = 0,
  ELMO_EINVAL = 1,        /* bad argument: null pointer, shape, alignment, range */
  ELMO_ENOMEM = 2,        /* workspace allocation failed */
  ELMO_ECUDA = 3,         /* a CUDA runtime call failed (message has the CUDA error) */
  ELMO_ETIMEOUT = 4,      /* a kernel's bounded wait ran out; results are invalid */
  ELMO_EUNSUPPORTED = 5,  /* valid but beyond the library's limits (see each call) */
  ELMO_EDATA = 6          /* malformed labels: CSR out of order or column out of [0, L) */
} elmo_status;

/* Opaque handle: a borrowed weight matrix plus the head's workspace. */
typedef struct elmo_head elmo_head;

/* Limits of the library. */
#define ELMO_MAX_BATCH 256          /* B of a training step */
#define ELMO_MAX_NNZ 32768          /* positive labels per training step */
#define ELMO_MAX_LABELS (1LL << 24) /* L */
#define ELMO_MAX_TOPK 64            /* k of a prediction */
#define ELMO_MAX_PREDICT_BATCH 4096 /* B of a prediction */
#define ELMO_MAX_TOTAL_LABELS 2147483647LL /* labels of a head split over devices (int32 ids) */
#define ELMO_MAX_SHARDS 64          /* lists merged by elmo_topk_merge */

/*
 * elmo_init_head -- wrap a caller-owned weight matrix in a head.
 *
 * Passage: the classifier head W of L labels and width d, stored in BF16 or in
 * unscaled E4M3 (abstract; atlas summary "Approach", "Surprising findings").
 *
 *   out      : receives the new handle (host pointer).
 *   W_dev    : device pointer to W [L x d], bf16 bits (dt = ELMO_BF16), E4M3
 *              codes (ELMO_FP8_E4M3, ELMO_FP8_E4M3_GE5M2) or E5M2 codes
 *              (ELMO_FP8_E5M2: the weights are stored and stochastically rounded
 *              on the E5M2 grid, +-inf kept, finite values saturating at 57344;
 *              X and the gradient operand are E4M3 as for ELMO_FP8_E4M3);
 *              row-major, label-major.  Borrowed for the life of the head;
 *              updated in place by training steps.
 *   L        : number of labels, 1 <= L < ELMO_MAX_LABELS.
 *   d        : width, a multiple of 64 in [64, 4096].
 *   fill     : 0 = keep W as is; 1 = overwrite W with SR(init_std * N(0,1)),
 *              the normal draws and the rounding both from Philox4x32-10 keyed
 *              by `seed` (normal draws use step 2^64-2, the rounding step
 *              2^64-1; the normal transform is not bit-reproducible on a CPU).
 *   stream   : stream for the fill.
 * Allocates the head's workspace (device status word and label buckets);
 * returns ELMO_ENOMEM if that fails.  Larger per-step buffers are allocated on
 * first use (see elmo_train_step_chunked).
 */
elmo_status elmo_init_head(elmo_head** out, void* W_dev, int64_t L, int32_t d, elmo_dtype dt,
                           int fill, float init_std, uint64_t seed, void* stream);

/*
 * elmo_init_head_shard -- wrap the label rows [label_base, label_base + L) of
 * a head of labels_total labels that is split by labels over several devices.
 *
 * Passage: the head is the part of the model that grows with the label count
 * and dominates its compute and memory (abstract); split by label rows, each
 * device holds and trains its own rows.  The step of a label depends only on
 * its own weights, X and whether it is positive, so each device runs the same
 * step on its rows and the devices' dX add up to the whole head's dX (the
 * caller sums them, e.g. with one all-reduce).  Stochastic rounding and the
 * fill draw by the element's index in the whole head, (label_base + l) * d + j,
 * so the rows come out bit-identical to those of an unsplit head.
 *
 *   W_dev        : device pointer to this device's rows, [L x d], as in elmo_init_head.
 *   L            : rows held here, 1 <= L < ELMO_MAX_LABELS.
 *   label_base   : label id of row 0; 0 <= label_base <= labels_total - L.
 *   labels_total : labels of the whole head, <= ELMO_MAX_TOTAL_LABELS.
 * Training steps take the CSR of the whole head: positives with ids in
 * [0, labels_total) outside this device's rows are skipped, ids outside
 * [0, labels_total) set ELMO_EDATA.  elmo_topk_predict ranks this device's
 * rows and returns label ids of the whole head; elmo_topk_merge combines the
 * devices' lists.  elmo_forward_chunk's l0, l1 are row numbers of this device.
 * Other arguments and errors as in elmo_init_head, which is this call with
 * label_base = 0 and labels_total = L.
 */
elmo_status elmo_init_head_shard(elmo_head** out, void* W_dev, int64_t L, int32_t d, elmo_dtype dt,
                                 int64_t label_base, int64_t labels_total, int fill, float init_std,
                                 uint64_t seed, void* stream);

/* Releases the workspace (synchronising the device first); W is untouched. */
elmo_status elmo_head_destroy(elmo_head* h);

/*
 * elmo_train_step_chunked -- one fused SGD step of the head.
 *
 * Passage: atlas summary "Approach" (the classifier is trained in pure low
 * precision by stochastic rounding without master weights or momentum; its
 * gradient is computed inside the SGD update kernel, and the label dimension
 * is processed chunk by chunk so that transient memory stays small); the
 * abstract (gradient fusion and chunking).  For every label chunk W_c it computes
 *     Z   = X W_c^T                       (fp32 accumulation)
 *     G   = sigmoid(Z) - Y                (Y = 1 at the positive labels)
 *     dX += G W_c                         (OLD W_c, fp32)
 *     W_c = SR(W_c - lr * G^T X)          (in place, stochastic rounding)
 * without materialising Z, G or dW for all L labels.  In FP8 mode the tensor
 * core operands are E4M3: X is quantised with a per-step power-of-two scale
 * s_X = 2^floor(log2(448 / max|X|)) and G as E4M3(2^8 G); both scales are
 * undone exactly in fp32.  In BF16 mode G is rounded to bf16 (RNE).
 * SR of element (l, j) takes a 16-bit draw k from Philox4x32-10 with key
 * `seed`, counter (idx >> 3, step), idx = l * d + j (half idx & 1 of word
 * (idx >> 1) & 3), and rounds to the upper grid neighbour (in magnitude) iff
 * k < floor(2^16 f), f the fractional position between the neighbours: the
 * draw added to the first 16 bits of the discarded fraction carries.
 *
 *   X_dev      : bf16 [B x d] sample embeddings (device).
 *   B          : 1 <= B <= ELMO_MAX_BATCH.
 *   rowptr_dev : int32 [B + 1] CSR row pointers of the positive labels, rowptr[0] = 0.
 *   cols_dev   : int32 [nnz] label ids in [0, L); order within a row free;
 *                duplicates count once.
 *   nnz        : number of entries, 0 <= nnz <= ELMO_MAX_NNZ; must equal rowptr[B].
 *   lr         : learning rate (finite).
 *   chunk      : labels per chunk, >= 1.  A scheduling knob only: W is bit-for-
 *                bit independent of it; dX only up to fp32 summation order.
 *   seed, step : the stochastic-rounding stream; step 2^64-2 and 2^64-1 are
 *                reserved for the fill of elmo_init_head.
 *   dX_dev     : fp32 [B x d] (device), overwritten with the input gradient.
 * The transient gradient buffer of one label range (the chunk, capped so that
 * its operands stay within 128 MB; B padded to 64 (bf16) or 128 (E4M3) samples,
 * one operand byte (E4M3) or two (bf16) per label and sample) is allocated on
 * the first call that needs it (cudaMalloc: call once before
 * capturing the step in a CUDA graph).  A malformed CSR sets ELMO_EDATA in the
 * status word; the step then skips the malformed entries and W is undefined.
 */
elmo_status elmo_train_step_chunked(elmo_head* h, const void* X_dev, int32_t B,
                                    const int32_t* rowptr_dev, const int32_t* cols_dev, int32_t nnz,
                                    float lr, int64_t chunk, uint64_t seed, uint64_t step,
                                    float* dX_dev, void* stream);

/*
 * elmo_forward_chunk -- inspection: the logits and gradient operands of the
 * step for labels [l0, l1), exactly as elmo_train_step_chunked forms them
 * (same operand preparation and kernels), without touching W.
 *
 *   Z_dev : fp32 [(l1 - l0) x B] logits, label-major (may be NULL).
 *   G_dev : fp32 [(l1 - l0) x B] values of the rounded gradient operand (may be NULL).
 * Other arguments as in elmo_train_step_chunked.
 */
elmo_status elmo_forward_chunk(elmo_head* h, const void* X_dev, int32_t B,
                               const int32_t* rowptr_dev, const int32_t* cols_dev, int32_t nnz,
                               int64_t l0, int64_t l1, float* Z_dev, float* G_dev, void* stream);

/*
 * elmo_topk_predict -- chunked top-k labels per sample.
 *
 * Passage: the atlas summary's "Experimental setup" evaluates by precision at
 * 1, 3 and 5, which ranks labels by their logit; the label axis is processed in chunks as in
 * training ("Approach").  Score of (b, l) is the fp32 fused multiply-add chain
 * s = fma(x[b,j], w[l,j], s) over j = 0..d-1 from s = 0 with x the bf16 value
 * of X (unquantised) and w the stored weight; labels are ranked by score
 * descending, ties to the lower label index, NaN after every number.
 *
 *   X_dev     : bf16 [B x d] (device), 1 <= B <= ELMO_MAX_PREDICT_BATCH.
 *   k         : 1 <= k <= min(L, ELMO_MAX_TOPK).
 *   chunk     : labels per chunk (scheduling only; the result does not depend on it).
 *   idx_dev   : int32 [B x k] label ids (device), best first; label ids of the
 *               whole head for a head made by elmo_init_head_shard.
 *   score_dev : fp32 [B x k] their exact scores (device).
 */
elmo_status elmo_topk_predict(elmo_head* h, const void* X_dev, int32_t B, int32_t k, int64_t chunk,
                              int32_t* idx_dev, float* score_dev, void* stream);

/*
 * elmo_topk_uncertified_rows -- how many rows of the most recent
 * elmo_topk_predict(h, ..., B, k, ...) the screening could not certify, so
 * that their top-k came from the exact CUDA-core path over all labels.
 *
 * Passage: as elmo_topk_predict (a measurement of the chunked prediction).
 *   B, k  : the arguments of that call (they locate its counter).
 *   rows  : host int32, receives the count.
 * Synchronises `stream`.  ELMO_EINVAL if no tensor-core prediction ran.
 */
elmo_status elmo_topk_uncertified_rows(elmo_head* h, int32_t B, int32_t k, int32_t* rows, void* stream);

/*
 * elmo_topk_screen_scores -- inspection of the tensor-core screening of
 * elmo_topk_predict, for tests: the approximate scores it ranks labels
 * [l0, l1) by, and each row's bound on their distance to the exact score.
 *
 * Passage: as elmo_topk_predict.  The prediction keeps, per row, the labels
 * whose screening scores are highest, rescores them exactly, and accepts the
 * result when the k-th exact score exceeds every other label's screening
 * score by more than the row's bound (else the row is recomputed exactly);
 * this call exposes both quantities so that the bound can be checked.
 *
 *   X_dev     : bf16 [B x d] (device), 1 <= B <= ELMO_MAX_PREDICT_BATCH.
 *   l0, l1    : label rows, 0 <= l0 <= l1 <= L.
 *   S_dev     : fp32 [B x (l1 - l0)] (device): screening scores.
 *   bound_dev : fp32 [B] (device): the certificate's bound of each row (NaN
 *               where the row or the head holds non-finite values).
 * Uses (and grows) the head's top-k workspace; W is not modified.
 */
elmo_status elmo_topk_screen_scores(elmo_head* h, const void* X_dev, int32_t B, int64_t l0, int64_t l1,
                                    float* S_dev, float* bound_dev, void* stream);

/*
 * elmo_topk_merge -- the top-k of a head split over P devices from the
 * devices' own top-k lists (each device's elmo_topk_predict, gathered).
 *
 * Passage: as elmo_topk_predict.  The label sets of the lists are disjoint, so
 * the best k of their union, in the same order (score descending, NaN after
 * every number, ties to the lower label id), is the top-k of the whole head.
 *
 *   idx_dev, score_dev : int32 / fp32 [P x B x k] (device), list p of sample b
 *                        at ((p * B) + b) * k, each sorted best first.
 *   P                  : 1 <= P <= ELMO_MAX_SHARDS.
 *   B, k               : 1 <= B <= ELMO_MAX_PREDICT_BATCH, 1 <= k <= ELMO_MAX_TOPK.
 *   idx_out_dev, score_out_dev : int32 / fp32 [B x k] (device), best first;
 *                        must not overlap the inputs.
 */
elmo_status elmo_topk_merge(const int32_t* idx_dev, const float* score_dev, int32_t P, int32_t B, int32_t k,
                            int32_t* idx_out_dev, float* score_out_dev, void* stream);

/*
 * elmo_sr_round -- standalone stochastic rounding.
 *
 * Passage: stochastic rounding of the classifier weights replaces FP32 master
 * weights (abstract; atlas summary "Approach").  out[i] = SR(in[i]) with the
 * draw of element index_base + i of stream (seed, step), as in the step.
 * NaN -> canonical NaN (bf16 0x7FC0, E4M3 and E5M2 0x7F); E4M3: |v| >= 448 and
 * +-inf -> +-448; bf16 and E5M2 (dt = ELMO_FP8_E5M2, largest finite 57344):
 * finite |v| above the largest finite -> largest finite, +-inf kept.  Values
 * on the grid are returned unchanged; -0 stays -0.
 *
 *   in_dev  : fp32 [n] (device);  out_dev : bf16, E4M3 or E5M2 [n] (device).
 *   n       : >= 0 (0 is a no-op).
 */
elmo_status elmo_sr_round(const float* in_dev, void* out_dev, int64_t n, elmo_dtype dt,
                          uint64_t seed, uint64_t step, uint64_t index_base, void* stream);

/*
 * elmo_kahan_sgd -- one Kahan-compensated SGD step of a dense BF16 layer.
 *
 * Passage: the pages train the encoder in pure BF16 with Kahan summation in
 * place of FP32 master weights (atlas summary "Approach"; abstract).  For
 * every element, with one IEEE fp32 operation per step and the two stored
 * results rounded to nearest-even bf16 (NaN -> 0x7FC0):
 *     u = -(lr g),  y = u + c,  p' = bf16(p + y),  c' = bf16(y - (p' - p))
 * (Kahan's compensated summation of p and the increments: c carries what the
 * bf16 grid of p could not take).
 *
 *   p_dev : bf16 [n] parameters (device), updated in place.
 *   c_dev : bf16 [n] compensation (device), updated in place; zero it before
 *           the first step.
 *   g_dev : bf16 [n] gradient (device).
 *   n     : >= 0 (0 is a no-op);  lr : finite.
 * Buffers may have any alignment (16-byte aligned ones take the vector path).
 */
elmo_status elmo_kahan_sgd(void* p_dev, void* c_dev, const void* g_dev, int64_t n, float lr, void* stream);

/*
 * elmo_round_bf16 -- out[i] = bf16(in[i]), round to nearest-even, NaN -> 0x7FC0:
 * the head's fp32 dX handed to a BF16 encoder (atlas summary "Approach": the
 * whole model in pure BF16).
 *   in_dev : fp32 [n] (device);  out_dev : bf16 [n] (device);  n >= 0.
 */
elmo_status elmo_round_bf16(const float* in_dev, void* out_dev, int64_t n, void* stream);

/*
 * elmo_sr_draws -- the 16-bit uniform draws k that SR uses for
 * elements index_base .. index_base + n - 1 of stream (seed, step), as uint16
 * into out_dev [n] (device).  Philox4x32-10 of Salmon et al. (SC'11).
 */
elmo_status elmo_sr_draws(uint16_t* out_dev, int64_t n, uint64_t seed, uint64_t step,
                          uint64_t index_base, void* stream);

/*
 * elmo_sync_status -- synchronise `stream` and return the head's device status
 * word (ELMO_OK, ELMO_EDATA or ELMO_ETIMEOUT), clearing it.
 */
elmo_status elmo_sync_status(elmo_head* h, void* stream);

/* Bytes of device workspace the head currently holds (for peak-memory reports). */
elmo_status elmo_head_workspace_bytes(const elmo_head* h, size_t* bytes);

/*
 * Tracing.  When enabled, every kernel a head launches is bracketed by CUDA
 * events recorded on its launch stream and filed under one of these classes;
 * elmo_profile_read synchronises on the recorded events and returns the summed
 * device time and the number of launches of a class since the last reset.
 * elmo_launch_count counts every kernel launch of the head (tracing on or off).
 */
typedef enum {
  ELMO_K_PREP = 0,        /* label sort / validation, X quantisation */
  ELMO_K_LOGITS_GRAD = 1, /* Z = X W_c^T and G = sigmoid(Z) - Y for a label range */
  ELMO_K_INPUT_GRAD = 2,  /* dX contributions of a label range */
  ELMO_K_UPDATE = 3,      /* weight gradient fused with the SR update (and dX where fused) */
  ELMO_K_TOPK_SCORE = 4,  /* top-k scoring of label segments */
  ELMO_K_TOPK_MERGE = 5,  /* top-k merge / exact rescoring */
  ELMO_K_OTHER = 6,       /* fill, clears */
  ELMO_K_STEP = 7,        /* the whole step in one persistent launch: Z, G, dX, dW and the SR update */
  ELMO_K_COUNT = 8
} elmo_kernel_class;

elmo_status elmo_profile_enable(elmo_head* h, int enable);
elmo_status elmo_profile_reset(elmo_head* h);
elmo_status elmo_profile_read(elmo_head* h, int kernel_class, double* ms_total, int64_t* launches);
elmo_status elmo_launch_count(const elmo_head* h, int64_t* launches);

/*
 * elmo_train_step_noalloc -- the training step of elmo_train_step_chunked for
 * callers that cannot allocate device memory.  The paper has no counterpart:
 * this entry point exists for deployment, not for the method.
 *
 * Who needs it: code that issues the step while a stream is being captured
 * into a CUDA graph (allocation cannot be captured), runtimes that give the
 * library a fixed memory budget, and hosts whose device allocator belongs to
 * someone else.  Such callers cannot create an elmo_head (its workspace is
 * allocated) nor let the head grow its gradient buffer on first use.
 *
 * This call takes W directly and allocates nothing.  Its scratch (the
 * positives grouped by label tile, the tile index, quantised X and the
 * per-range gradient operands)
 * is one static device array of 11 MiB (ELMO_NOALLOC_SCRATCH_BYTES) that every
 * GPU loading the library holds until the process exits.  It supports the
 * same sizes as the head-based step -- 1 <= L < 2^24, d a multiple of 64 up to
 * 4096, 1 <= B <= 256, 0 <= nnz <= 32768 -- and rejects anything beyond them
 * with ELMO_EUNSUPPORTED; the label range per pass shrinks so that its gradient
 * operands fit the 8 MiB gradient part of the scratch (W stays bit-identical to
 * the head-based step; dX differs only by fp32 summation order).
 *
 * The first call on a device looks up the device address of the scratch array
 * (loading the library's device code on that device if needed); make that
 * first call before capturing any stream.  Every call on a device shares the
 * one array and each call rewrites it before reading it: calls whose work
 * overlaps on the GPU (different streams, or the same graph launched
 * concurrently) race on it and give wrong results -- serialise them.
 *
 *   W_dev, L, d, dt : the weights, as in elmo_init_head (updated in place).
 *   X_dev ... dX_dev: as in elmo_train_step_chunked.
 *   status_dev      : int32 [2] (device), zeroed by the call; a malformed label
 *                     list leaves ELMO_EDATA in [0] (and the first bad entry in
 *                     [1]) once the step has run.
 * Errors: ELMO_EINVAL / ELMO_EUNSUPPORTED synchronously (message in
 * elmo_last_error()), ELMO_ECUDA if a launch fails.
 */
#define ELMO_NOALLOC_SCRATCH_BYTES (11u << 20)
elmo_status elmo_train_step_noalloc(void* W_dev, int64_t L, int32_t d, elmo_dtype dt, const void* X_dev,
                                    int32_t B, const int32_t* rowptr_dev, const int32_t* cols_dev, int32_t nnz,
                                    float lr, int64_t chunk, uint64_t seed, uint64_t step, float* dX_dev,
                                    int32_t* status_dev, void* stream);

/*
 * elmo_precision_at_k -- P@1 .. P@k of top-k predictions ("ELMO: Efficiency
 * via Low-precision and Peak Memory Optimization in Large Output Spaces",
 * atlas summary, metrics P@1/3/5): p[j-1] = the mean over the B rows of
 * |{first j predicted labels} ∩ {positive labels}| / j.
 *
 *   idx_dev    : int32 [B x k] (device), each row's predictions in rank order
 *                (the idx output of elmo_topk_predict)
 *   B, k       : 1 <= B <= ELMO_MAX_PREDICT_BATCH, 1 <= k <= ELMO_MAX_TOPK
 *   rowptr_dev : int32 [B+1], cols_dev int32 [nnz] (device): each row's
 *                positive labels (CSR); entries outside [0, nnz) are clamped
 *   p_dev      : fp32 [k] (device), written: integer hit counts over j*B,
 *                divided in double and rounded once (independent of order)
 * Asynchronous on `stream`.  Errors: ELMO_EINVAL (null pointer, B or k out of
 * range), ELMO_ECUDA (launch).
 */
elmo_status elmo_precision_at_k(const int32_t* idx_dev, int32_t B, int32_t k, const int32_t* rowptr_dev,
                                const int32_t* cols_dev, int32_t nnz, float* p_dev, void* stream);

/*
 * elmo_check_bounded_wait -- runs, in one CTA, the bounded mbarrier wait that
 * every pipelined kernel of the library uses, on a barrier nothing ever
 * arrives on.  The paper has no counterpart: this checks the library's
 * failure detection without faulting anything.  The wait gives up after about
 * limit_cycles SM clock cycles, records ELMO_ETIMEOUT in status_dev[0] and
 * ELMO_WAIT_CHECK_SITE in status_dev[1] exactly as a kernel whose pipeline
 * stalled would, and the kernel returns normally, so the context stays usable.
 *
 *   limit_cycles : 1 .. 2^32 (about 2 s at the B200's clock)
 *   status_dev   : int32 [2] (device), cleared by the call
 * Asynchronous on `stream`: read status_dev after synchronising.  Errors:
 * ELMO_EINVAL (null status_dev, limit out of range), ELMO_ECUDA (launch).
 */
#define ELMO_WAIT_CHECK_SITE 99
elmo_status elmo_check_bounded_wait(int64_t limit_cycles, int32_t* status_dev, void* stream);

/* Message of the most recent failure on the calling thread ("" if none). */
const char* elmo_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* ELMO_H_ */
