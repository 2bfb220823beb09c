// api.cu -- the C ABI of libelmo (declared in include/elmo.h).
//
// Argument checking, workspace ownership and the chunk loop of the step;
// every arithmetic step runs in the kernels of this library.
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <new>
#include <string>

#include <nvtx3/nvToolsExt.h>

#include "../../include/elmo.h"
#include "elmo_internal.h"

namespace {

// An NVTX range named after the entry point around each call, so that a
// profiler's timeline groups the kernels of a call under the call's name.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};
#define ELMO_NVTX_RANGE() NvtxRange nvtx_range_(__func__)

thread_local std::string g_last_error;

elmo_status fail(elmo_status code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

elmo_status cuda_fail(cudaError_t e, const char* what) {
  return fail(ELMO_ECUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

#define ELMO_CUDA(call, what)                        \
  do {                                               \
    cudaError_t e_ = (call);                         \
    if (e_ != cudaSuccess) return cuda_fail(e_, what); \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

// ELMO_TOPK_SIMT=1 runs top-k prediction on CUDA cores only (every score by
// its exact chain), the comparison path of the tensor-core screening.
bool use_topk_simt() {
  const char* v = getenv("ELMO_TOPK_SIMT");
  return v && v[0] == '1';
}

// Fails with the status word's code if an earlier kernel recorded one.
// Reading it costs a synchronisation, so only elmo_sync_status does.
elmo_status check_device(elmo_head* h) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev != h->device) return fail(ELMO_EINVAL, "head lives on device %d, current device is %d", h->device, dev);
  return ELMO_OK;
}

elmo_status ensure_gbuf(elmo_head* h, size_t bytes) {
  if (h->gbuf_bytes >= bytes) return ELMO_OK;
  if (h->gbuf) cudaFree(h->gbuf);
  h->gbuf = nullptr;
  h->gbuf_bytes = 0;
  if (cudaMalloc(&h->gbuf, bytes) != cudaSuccess) {
    cudaGetLastError();
    return fail(ELMO_ENOMEM, "cannot allocate %zu bytes of gradient workspace", bytes);
  }
  h->gbuf_bytes = bytes;
  return ELMO_OK;
}

// The persistent step's ring: kRingTiles gradient-operand tiles of up to
// 128 labels x 256 samples (64 KB in bf16), its two flag arrays and the
// step's tile counters.
elmo_status ensure_ring(elmo_head* h) {
  const size_t tiles = elmo::kRingTiles;
  const size_t bytes = tiles * 65536 + sizeof(int32_t) * (2 * tiles + elmo::kRingCounters);
  if (h->ring_bytes >= bytes) return ELMO_OK;
  if (h->ring) cudaFree(h->ring);
  h->ring = nullptr;
  h->ring_bytes = 0;
  if (cudaMalloc(&h->ring, bytes) != cudaSuccess) {
    cudaGetLastError();
    return fail(ELMO_ENOMEM, "cannot allocate %zu bytes of gradient-operand ring", bytes);
  }
  h->ring_bytes = bytes;
  h->ring_tiles = (int32_t)tiles;
  h->ring_flags = reinterpret_cast<int32_t*>(static_cast<char*>(h->ring) + tiles * 65536);
  return ELMO_OK;
}

elmo_status ensure_cand(elmo_head* h, size_t bytes) {
  if (h->cand_bytes >= bytes) return ELMO_OK;
  if (h->cand) cudaFree(h->cand);
  h->cand = nullptr;
  h->cand_bytes = 0;
  if (cudaMalloc(&h->cand, bytes) != cudaSuccess) {
    cudaGetLastError();
    return fail(ELMO_ENOMEM, "cannot allocate %zu bytes of top-k workspace", bytes);
  }
  h->cand_bytes = bytes;
  return ELMO_OK;
}

elmo_status check_labels_args(const elmo_head* h, const void* X, int32_t B, const int32_t* rowptr,
                              const int32_t* cols, int32_t nnz) {
  if (!X || !rowptr) return fail(ELMO_EINVAL, "null X or rowptr");
  if (nnz > 0 && !cols) return fail(ELMO_EINVAL, "null cols with nnz > 0");
  if (B < 1 || B > ELMO_MAX_BATCH) return fail(ELMO_EINVAL, "B = %d outside [1, %d]", B, ELMO_MAX_BATCH);
  if (nnz < 0) return fail(ELMO_EINVAL, "nnz = %d < 0", nnz);
  if (nnz > ELMO_MAX_NNZ) return fail(ELMO_EUNSUPPORTED, "nnz = %d above %d", nnz, ELMO_MAX_NNZ);
  if (!aligned16(X)) return fail(ELMO_EINVAL, "X is not 16-byte aligned");
  (void)h;
  return ELMO_OK;
}

}  // namespace

namespace elmo {

void set_last_error(const char* msg) { g_last_error = msg ? msg : ""; }

KernelScope::KernelScope(elmo_head* h_, int cls, cudaStream_t s_, int n) : h(h_), s(s_), on(h_ && h_->prof) {
  if (h) h->launches += n;
  if (!on) return;
  auto take = [&]() {
    cudaEvent_t e = nullptr;
    if (!h->prof_pool.empty()) { e = h->prof_pool.back(); h->prof_pool.pop_back(); }
    else if (cudaEventCreate(&e) != cudaSuccess) { cudaGetLastError(); e = nullptr; }
    return e;
  };
  rec.cls = cls;
  rec.start = take();
  rec.stop = take();
  if (!rec.start || !rec.stop) { on = false; return; }
  cudaEventRecord(rec.start, s);
}

KernelScope::~KernelScope() {
  if (!on) return;
  cudaEventRecord(rec.stop, s);
  h->prof_recs.push_back(rec);
}

}  // namespace elmo

extern "C" {

elmo_status elmo_profile_enable(elmo_head* h, int enable) {
  if (!h) return fail(ELMO_EINVAL, "null head");
  h->prof = enable != 0;
  return ELMO_OK;
}

elmo_status elmo_profile_reset(elmo_head* h) {
  if (!h) return fail(ELMO_EINVAL, "null head");
  for (auto& r : h->prof_recs) {
    cudaEventSynchronize(r.stop);
    h->prof_pool.push_back(r.start);
    h->prof_pool.push_back(r.stop);
  }
  h->prof_recs.clear();
  return ELMO_OK;
}

elmo_status elmo_profile_read(elmo_head* h, int kernel_class, double* ms_total, int64_t* launches) {
  if (!h || !ms_total || !launches) return fail(ELMO_EINVAL, "null argument");
  double ms = 0.0;
  int64_t n = 0;
  for (auto& r : h->prof_recs) {
    if (r.cls != kernel_class) continue;
    ELMO_CUDA(cudaEventSynchronize(r.stop), "cudaEventSynchronize");
    float t = 0.0f;
    ELMO_CUDA(cudaEventElapsedTime(&t, r.start, r.stop), "cudaEventElapsedTime");
    ms += t;
    ++n;
  }
  *ms_total = ms;
  *launches = n;
  return ELMO_OK;
}

elmo_status elmo_launch_count(const elmo_head* h, int64_t* launches) {
  if (!h || !launches) return fail(ELMO_EINVAL, "null argument");
  *launches = h->launches;
  return ELMO_OK;
}


const char* elmo_last_error(void) { return g_last_error.c_str(); }

elmo_status elmo_init_head(elmo_head** out, void* W_dev, int64_t L, int32_t d, elmo_dtype dt, int fill,
                           float init_std, uint64_t seed, void* stream) {
  return elmo_init_head_shard(out, W_dev, L, d, dt, 0, L, fill, init_std, seed, stream);
}

elmo_status elmo_init_head_shard(elmo_head** out, void* W_dev, int64_t L, int32_t d, elmo_dtype dt,
                                 int64_t label_base, int64_t labels_total, int fill, float init_std, uint64_t seed,
                                 void* stream) {
  ELMO_NVTX_RANGE();
  g_last_error.clear();
  if (!out || !W_dev) return fail(ELMO_EINVAL, "null out or W");
  *out = nullptr;
  if (dt != ELMO_BF16 && dt != ELMO_FP8_E4M3 && dt != ELMO_FP8_E4M3_GE5M2 && dt != ELMO_FP8_E5M2)
    return fail(ELMO_EINVAL, "unknown dtype %d", (int)dt);
  const elmo_dtype fill_dt = dt == ELMO_FP8_E4M3_GE5M2 ? ELMO_FP8_E4M3 : dt;   // the weights' own grid
  const bool g_e5m2 = dt == ELMO_FP8_E4M3_GE5M2;
  const bool w_e5m2 = dt == ELMO_FP8_E5M2;
  if (g_e5m2 || w_e5m2) dt = ELMO_FP8_E4M3;          // the tensor-core operand path: X and G in E4M3 (or E5M2 G)
  if (L < 1 || L >= ELMO_MAX_LABELS) return fail(ELMO_EINVAL, "L = %lld outside [1, 2^24)", (long long)L);
  if (label_base < 0 || labels_total > ELMO_MAX_TOTAL_LABELS || label_base > labels_total - L)
    return fail(ELMO_EINVAL, "label rows [%lld, %lld) outside a head of %lld labels (at most %lld)",
                (long long)label_base, (long long)(label_base + L), (long long)labels_total,
                (long long)ELMO_MAX_TOTAL_LABELS);
  if (d < 64 || d > 4096 || d % 64 != 0) return fail(ELMO_EINVAL, "d = %d: need a multiple of 64 in [64, 4096]", d);
  if (!aligned16(W_dev)) return fail(ELMO_EINVAL, "W is not 16-byte aligned");
  if (fill && !(init_std >= 0.0f && init_std < 1e30f)) return fail(ELMO_EINVAL, "bad init_std");
  int dev = 0, nsm = 0, major = 0;
  ELMO_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  ELMO_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev), "cudaDeviceGetAttribute");
  if (major != 10) return fail(ELMO_EUNSUPPORTED, "device %d has compute capability %d.x; this library is built for sm_100a", dev, major);
  ELMO_CUDA(cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev), "cudaDeviceGetAttribute");
  elmo_head* h = new (std::nothrow) elmo_head();
  if (!h) return fail(ELMO_ENOMEM, "host allocation failed");
  h->W = W_dev;
  h->L = L;
  h->label_base = label_base;
  h->labels_total = labels_total;
  h->g_e5m2 = g_e5m2;
  h->w_e5m2 = w_e5m2;
  h->d = d;
  h->dt = dt;
  h->device = dev;
  h->num_sms = nsm;
  const size_t xq_bytes = (size_t)ELMO_MAX_BATCH * d;
  const size_t tp_bytes = (sizeof(int32_t) * (size_t)((L + 127) / 128 + 1) + 255) / 256 * 256;
  const size_t bytes = 64 + sizeof(uint32_t) * ELMO_MAX_NNZ + 64 + 2 * xq_bytes + tp_bytes;
  char* base = nullptr;
  if (cudaMalloc(&base, bytes) != cudaSuccess) {
    cudaGetLastError();
    delete h;
    return fail(ELMO_ENOMEM, "cannot allocate %zu bytes of head workspace", bytes);
  }
  h->status = reinterpret_cast<int32_t*>(base);
  h->nkeys = reinterpret_cast<int32_t*>(base + 16);
  h->xscale = reinterpret_cast<float*>(base + 32);
  h->keys = reinterpret_cast<uint32_t*>(base + 64);
  h->xq = reinterpret_cast<uint8_t*>(base + 64 + sizeof(uint32_t) * ELMO_MAX_NNZ + 64);
  h->tile_ptr = reinterpret_cast<int32_t*>(base + 64 + sizeof(uint32_t) * ELMO_MAX_NNZ + 64 + xq_bytes);
  h->xqt = reinterpret_cast<uint8_t*>(base + 64 + sizeof(uint32_t) * ELMO_MAX_NNZ + 64 + xq_bytes + tp_bytes);
  h->base_bytes = bytes;
  cudaStream_t s = as_stream(stream);
  cudaError_t e = cudaMemsetAsync(base, 0, 64, s);
  if (e == cudaSuccess && fill) {
    h->launches += 1;
    e = elmo::launch_fill(W_dev, L * (int64_t)d, fill_dt, init_std, seed, (uint64_t)label_base * (uint64_t)d, s);
  }
  if (e != cudaSuccess) {
    cudaFree(base);
    delete h;
    return cuda_fail(e, "elmo_init_head");
  }
  *out = h;
  return ELMO_OK;
}

elmo_status elmo_head_destroy(elmo_head* h) {
  ELMO_NVTX_RANGE();
  g_last_error.clear();
  if (!h) return ELMO_OK;
  cudaDeviceSynchronize();
  if (h->gbuf) cudaFree(h->gbuf);
  if (h->ring) cudaFree(h->ring);
  if (h->cand) cudaFree(h->cand);
  if (h->status) cudaFree(h->status);
  if (h->side) cudaStreamDestroy(h->side);
  if (h->fork) cudaEventDestroy(h->fork);
  if (h->join) cudaEventDestroy(h->join);
  for (auto& r : h->prof_recs) { cudaEventDestroy(r.start); cudaEventDestroy(r.stop); }
  for (auto e : h->prof_pool) cudaEventDestroy(e);
  delete h;
  return ELMO_OK;
}

elmo_status elmo_head_workspace_bytes(const elmo_head* h, size_t* bytes) {
  if (!h || !bytes) return fail(ELMO_EINVAL, "null argument");
  *bytes = h->base_bytes + h->gbuf_bytes + h->ring_bytes + h->cand_bytes;
  return ELMO_OK;
}

elmo_status elmo_sync_status(elmo_head* h, void* stream) {
  ELMO_NVTX_RANGE();
  g_last_error.clear();
  if (!h) return fail(ELMO_EINVAL, "null head");
  int32_t st[2] = {0, 0};
  cudaStream_t s = as_stream(stream);
  ELMO_CUDA(cudaMemcpyAsync(st, h->status, sizeof st, cudaMemcpyDeviceToHost, s), "status readback");
  ELMO_CUDA(cudaStreamSynchronize(s), "cudaStreamSynchronize");
  ELMO_CUDA(cudaMemsetAsync(h->status, 0, sizeof st, s), "status clear");
  ELMO_CUDA(cudaStreamSynchronize(s), "cudaStreamSynchronize");
  if (st[0] == ELMO_EDATA) return fail(ELMO_EDATA, "malformed labels (first bad entry %d; -1 = row pointers)", st[1]);
  if (st[0] == ELMO_ETIMEOUT) return fail(ELMO_ETIMEOUT, "a kernel's bounded wait ran out (site %d)", st[1]);
  if (st[0] != 0) return fail((elmo_status)st[0], "device status %d", st[0]);
  return ELMO_OK;
}

elmo_status elmo_sr_round(const float* in_dev, void* out_dev, int64_t n, elmo_dtype dt, uint64_t seed,
                          uint64_t step, uint64_t index_base, void* stream) {
  ELMO_NVTX_RANGE();
  g_last_error.clear();
  if (n < 0) return fail(ELMO_EINVAL, "n < 0");
  if (n == 0) return ELMO_OK;
  if (!in_dev || !out_dev) return fail(ELMO_EINVAL, "null pointer");
  if (dt != ELMO_BF16 && dt != ELMO_FP8_E4M3 && dt != ELMO_FP8_E5M2)
    return fail(ELMO_EINVAL, "dtype %d is not an SR output grid", (int)dt);
  if (index_base + (uint64_t)n < index_base) return fail(ELMO_EINVAL, "index range wraps around 2^64");
  if (dt == ELMO_FP8_E5M2)
    ELMO_CUDA(elmo::launch_sr_e5m2(in_dev, static_cast<uint8_t*>(out_dev), n, seed, step, index_base,
                                   as_stream(stream)), "sr_round");
  else
    ELMO_CUDA(elmo::launch_sr_round(in_dev, out_dev, n, dt, seed, step, index_base, as_stream(stream)), "sr_round");
  return ELMO_OK;
}

elmo_status elmo_sr_draws(uint16_t* out_dev, int64_t n, uint64_t seed, uint64_t step, uint64_t index_base,
                          void* stream) {
  ELMO_NVTX_RANGE();
  g_last_error.clear();
  if (n < 0) return fail(ELMO_EINVAL, "n < 0");
  if (n == 0) return ELMO_OK;
  if (!out_dev) return fail(ELMO_EINVAL, "null pointer");
  if (index_base + (uint64_t)n < index_base) return fail(ELMO_EINVAL, "index range wraps around 2^64");
  ELMO_CUDA(elmo::launch_sr_draws(out_dev, n, seed, step, index_base, as_stream(stream)), "sr_draws");
  return ELMO_OK;
}

elmo_status elmo_forward_chunk(elmo_head* h, const void* X_dev, int32_t B, const int32_t* rowptr_dev,
                               const int32_t* cols_dev, int32_t nnz, int64_t l0, int64_t l1, float* Z_dev,
                               float* G_dev, void* stream) {
  ELMO_NVTX_RANGE();
  g_last_error.clear();
  if (!h) return fail(ELMO_EINVAL, "null head");
  elmo_status st = check_labels_args(h, X_dev, B, rowptr_dev, cols_dev, nnz);
  if (st != ELMO_OK) return st;
  if (l0 < 0 || l1 > h->L || l0 > l1) return fail(ELMO_EINVAL, "label range [%lld, %lld) outside [0, %lld]",
                                                 (long long)l0, (long long)l1, (long long)h->L);
  if ((st = check_device(h)) != ELMO_OK) return st;
  if (l0 == l1) return ELMO_OK;
  cudaStream_t s = as_stream(stream);
  const uint16_t* X = static_cast<const uint16_t*>(X_dev);
  {
    elmo::KernelScope ks(h, ELMO_K_PREP, s, 1);
    ELMO_CUDA(elmo::launch_prep_step(h, rowptr_dev, cols_dev, B, nnz, X, s), "prep");
  }
  const bool fp8 = h->dt == ELMO_FP8_E4M3;
  const size_t esz = fp8 ? 1 : 2;
  const int32_t Bp = elmo::padded_batch(B, fp8);
  const int64_t sub = elmo::sub_chunk_labels(h->d, Bp, (int)esz);
  const int64_t span = l1 - l0 < sub ? l1 - l0 : sub;
  if ((st = ensure_gbuf(h, (size_t)((span + 127) / 128 * 128) * Bp * esz)) != ELMO_OK) return st;  // whole tiles
  for (int64_t a = l0; a < l1; a += span) {
    const int64_t e = a + span < l1 ? a + span : l1;
    elmo::KernelScope ks(h, ELMO_K_LOGITS_GRAD, s);
    float* Za = Z_dev ? Z_dev + (a - l0) * B : nullptr;
    float* Ga = G_dev ? G_dev + (a - l0) * B : nullptr;
    ELMO_CUDA(elmo::launch_logits_grad_tc(h, X, B, a, e, h->gbuf, Za, Ga, s), "logits_grad");
  }
  return ELMO_OK;
}

elmo_status elmo_train_step_chunked(elmo_head* h, const void* X_dev, int32_t B, const int32_t* rowptr_dev,
                                    const int32_t* cols_dev, int32_t nnz, float lr, int64_t chunk, uint64_t seed,
                                    uint64_t step, float* dX_dev, void* stream) {
  ELMO_NVTX_RANGE();
  g_last_error.clear();
  if (!h) return fail(ELMO_EINVAL, "null head");
  elmo_status st = check_labels_args(h, X_dev, B, rowptr_dev, cols_dev, nnz);
  if (st != ELMO_OK) return st;
  if (!dX_dev || !aligned16(dX_dev)) return fail(ELMO_EINVAL, "dX null or not 16-byte aligned");
  if (chunk < 1) return fail(ELMO_EINVAL, "chunk = %lld < 1", (long long)chunk);
  if (!(lr == lr) || lr > 3.0e38f || lr < -3.0e38f) return fail(ELMO_EINVAL, "lr is not finite");
  if ((st = check_device(h)) != ELMO_OK) return st;
  cudaStream_t s = as_stream(stream);
  const uint16_t* X = static_cast<const uint16_t*>(X_dev);
  {
    elmo::KernelScope ks(h, ELMO_K_PREP, s, 1);
    ELMO_CUDA(cudaMemsetAsync(dX_dev, 0, sizeof(float) * (size_t)B * h->d, s), "dX clear");
    ELMO_CUDA(elmo::launch_prep_step(h, rowptr_dev, cols_dev, B, nnz, X, s), "prep");
  }
  const bool fp8 = h->dt == ELMO_FP8_E4M3;
  const size_t esz = fp8 ? 1 : 2;
  const int32_t Bp = elmo::padded_batch(B, fp8);
  if (elmo::fused_step_supported(h, B)) {
    // one persistent launch; the chunk only bounds transient memory, which
    // the ring of gradient-operand tiles already does
    if ((st = ensure_ring(h)) != ELMO_OK) return st;
    elmo::KernelScope ks(h, ELMO_K_STEP, s);
    ELMO_CUDA(elmo::launch_step_fused(h, X, B, lr, seed, step, dX_dev, s), "step");
    return ELMO_OK;
  }
  const int64_t sub_max = elmo::sub_chunk_labels(h->d, Bp, (int)esz);
  const int64_t sub = chunk < sub_max ? chunk : sub_max;
  const int64_t span = h->L < sub ? h->L : sub;
  if ((st = ensure_gbuf(h, (size_t)((span + 127) / 128 * 128) * Bp * esz)) != ELMO_OK) return st;  // whole tiles
  for (int64_t c0 = 0; c0 < h->L; c0 += chunk) {
    const int64_t c1 = c0 + chunk < h->L ? c0 + chunk : h->L;
    for (int64_t a = c0; a < c1; a += span) {
      const int64_t e = a + span < c1 ? a + span : c1;
      // every kernel but the first follows one of the step's own kernels: programmatic launches
      {
        elmo::KernelScope ks(h, ELMO_K_LOGITS_GRAD, s);
        ELMO_CUDA(elmo::launch_logits_grad_tc(h, X, B, a, e, h->gbuf, nullptr, nullptr, s, a > 0), "logits_grad");
      }
      elmo::KernelScope ks(h, ELMO_K_UPDATE, s);
      ELMO_CUDA(elmo::launch_update_tc(h, X, B, a, e, h->gbuf, lr, seed, step, dX_dev, s, true), "update");
    }
  }
  return ELMO_OK;
}

elmo_status elmo_precision_at_k(const int32_t* idx_dev, int32_t B, int32_t k, const int32_t* rowptr_dev,
                                const int32_t* cols_dev, int32_t nnz, float* p_dev, void* stream) {
  ELMO_NVTX_RANGE();
  g_last_error.clear();
  if (!idx_dev || !rowptr_dev || !p_dev || (nnz > 0 && !cols_dev)) return fail(ELMO_EINVAL, "null pointer");
  if (B < 1 || B > ELMO_MAX_PREDICT_BATCH) return fail(ELMO_EINVAL, "B = %d outside [1, %d]", B, ELMO_MAX_PREDICT_BATCH);
  if (k < 1 || k > ELMO_MAX_TOPK) return fail(ELMO_EINVAL, "k = %d outside [1, %d]", k, ELMO_MAX_TOPK);
  if (nnz < 0) return fail(ELMO_EINVAL, "nnz = %d < 0", nnz);
  ELMO_CUDA(elmo::launch_precision_at_k(idx_dev, B, k, rowptr_dev, cols_dev, nnz, p_dev, as_stream(stream)),
            "precision_at_k");
  return ELMO_OK;
}

elmo_status elmo_check_bounded_wait(int64_t limit_cycles, int32_t* status_dev, void* stream) {
  g_last_error.clear();
  if (!status_dev) return fail(ELMO_EINVAL, "null status_dev");
  if (limit_cycles < 1 || limit_cycles > (int64_t(1) << 32))
    return fail(ELMO_EINVAL, "limit_cycles = %lld outside [1, 2^32]", (long long)limit_cycles);
  ELMO_CUDA(elmo::launch_wait_check((long long)limit_cycles, status_dev, as_stream(stream)), "wait check");
  return ELMO_OK;
}

elmo_status elmo_topk_predict(elmo_head* h, const void* X_dev, int32_t B, int32_t k, int64_t chunk,
                              int32_t* idx_dev, float* score_dev, void* stream) {
  ELMO_NVTX_RANGE();
  g_last_error.clear();
  if (!h) return fail(ELMO_EINVAL, "null head");
  if (!X_dev || !idx_dev || !score_dev) return fail(ELMO_EINVAL, "null pointer");
  if (B < 1 || B > ELMO_MAX_PREDICT_BATCH) return fail(ELMO_EINVAL, "B = %d outside [1, %d]", B, ELMO_MAX_PREDICT_BATCH);
  if (k < 1 || k > ELMO_MAX_TOPK || (int64_t)k > h->L) return fail(ELMO_EINVAL, "k = %d outside [1, min(L, %d)]", k, ELMO_MAX_TOPK);
  if (chunk < 1) return fail(ELMO_EINVAL, "chunk = %lld < 1", (long long)chunk);
  if (!aligned16(X_dev)) return fail(ELMO_EINVAL, "X is not 16-byte aligned");
  elmo_status st = check_device(h);
  if (st != ELMO_OK) return st;
  const uint16_t* X = static_cast<const uint16_t*>(X_dev);
  if (elmo::topk_tc_supported(h) && !use_topk_simt()) {
    if ((st = ensure_cand(h, elmo::topk_tc_workspace_bytes(h, B, k))) != ELMO_OK) return st;
    ELMO_CUDA(elmo::launch_topk_tc(h, X, B, k, idx_dev, score_dev, as_stream(stream)), "topk");
  } else {
    if ((st = ensure_cand(h, elmo::topk_simt_workspace_bytes(h, B, k))) != ELMO_OK) return st;
    elmo::KernelScope ks(h, ELMO_K_TOPK_SCORE, as_stream(stream), 2);
    ELMO_CUDA(elmo::launch_topk_simt_rows(h, X, B, k, nullptr, nullptr, h->cand, idx_dev, score_dev,
                                          as_stream(stream)),
              "topk");
  }
  if (h->label_base != 0) {     // label ids of the whole head
    h->launches += 1;
    ELMO_CUDA(elmo::launch_topk_offset(idx_dev, (int64_t)B * k, h->label_base, as_stream(stream)), "topk offset");
  }
  return ELMO_OK;
}

elmo_status elmo_topk_uncertified_rows(elmo_head* h, int32_t B, int32_t k, int32_t* rows, void* stream) {
  g_last_error.clear();
  if (!h || !rows) return fail(ELMO_EINVAL, "null argument");
  if (B < 1 || B > ELMO_MAX_PREDICT_BATCH) return fail(ELMO_EINVAL, "B = %d outside [1, %d]", B, ELMO_MAX_PREDICT_BATCH);
  if (k < 1 || k > ELMO_MAX_TOPK) return fail(ELMO_EINVAL, "k = %d outside [1, %d]", k, ELMO_MAX_TOPK);
  if (!elmo::topk_tc_supported(h) || !h->cand || h->cand_bytes < elmo::topk_tc_workspace_bytes(h, B, k))
    return fail(ELMO_EINVAL, "no tensor-core prediction of this shape has run on this head");
  ELMO_CUDA(elmo::topk_uncertified_rows(h, B, k, rows, as_stream(stream)), "uncertified rows");
  return ELMO_OK;
}

elmo_status elmo_topk_screen_scores(elmo_head* h, const void* X_dev, int32_t B, int64_t l0, int64_t l1,
                                    float* S_dev, float* bound_dev, void* stream) {
  ELMO_NVTX_RANGE();
  g_last_error.clear();
  if (!h) return fail(ELMO_EINVAL, "null head");
  if (!X_dev || !S_dev || !bound_dev) return fail(ELMO_EINVAL, "null pointer");
  if (B < 1 || B > ELMO_MAX_PREDICT_BATCH) return fail(ELMO_EINVAL, "B = %d outside [1, %d]", B, ELMO_MAX_PREDICT_BATCH);
  if (l0 < 0 || l1 > h->L || l0 > l1) return fail(ELMO_EINVAL, "label range [%lld, %lld) outside [0, %lld]",
                                                 (long long)l0, (long long)l1, (long long)h->L);
  if (!aligned16(X_dev)) return fail(ELMO_EINVAL, "X is not 16-byte aligned");
  if (!elmo::topk_tc_supported(h)) return fail(ELMO_EUNSUPPORTED, "this head has no tensor-core screening");
  elmo_status st = check_device(h);
  if (st != ELMO_OK) return st;
  if (l0 == l1) return ELMO_OK;
  if ((st = ensure_cand(h, elmo::topk_tc_workspace_bytes(h, B, 1))) != ELMO_OK) return st;
  ELMO_CUDA(elmo::launch_topk_screen_dump(h, static_cast<const uint16_t*>(X_dev), B, l0, l1, S_dev, bound_dev,
                                          as_stream(stream)), "screen scores");
  return ELMO_OK;
}

elmo_status elmo_kahan_sgd(void* p_dev, void* c_dev, const void* g_dev, int64_t n, float lr, void* stream) {
  ELMO_NVTX_RANGE();
  g_last_error.clear();
  if (n < 0) return fail(ELMO_EINVAL, "n = %lld < 0", (long long)n);
  if (n > 0 && (!p_dev || !c_dev || !g_dev)) return fail(ELMO_EINVAL, "null pointer");
  if (!(lr > -1e30f && lr < 1e30f)) return fail(ELMO_EINVAL, "lr is not finite");
  ELMO_CUDA(elmo::launch_kahan_sgd(p_dev, c_dev, g_dev, n, lr, as_stream(stream)), "kahan_sgd");
  return ELMO_OK;
}

elmo_status elmo_round_bf16(const float* in_dev, void* out_dev, int64_t n, void* stream) {
  ELMO_NVTX_RANGE();
  g_last_error.clear();
  if (n < 0) return fail(ELMO_EINVAL, "n = %lld < 0", (long long)n);
  if (n > 0 && (!in_dev || !out_dev)) return fail(ELMO_EINVAL, "null pointer");
  ELMO_CUDA(elmo::launch_round_bf16(in_dev, out_dev, n, as_stream(stream)), "round_bf16");
  return ELMO_OK;
}

elmo_status elmo_topk_merge(const int32_t* idx_dev, const float* score_dev, int32_t P, int32_t B, int32_t k,
                            int32_t* idx_out_dev, float* score_out_dev, void* stream) {
  ELMO_NVTX_RANGE();
  g_last_error.clear();
  if (!idx_dev || !score_dev || !idx_out_dev || !score_out_dev) return fail(ELMO_EINVAL, "null pointer");
  if (P < 1 || P > ELMO_MAX_SHARDS) return fail(ELMO_EINVAL, "P = %d outside [1, %d]", P, ELMO_MAX_SHARDS);
  if (B < 1 || B > ELMO_MAX_PREDICT_BATCH) return fail(ELMO_EINVAL, "B = %d outside [1, %d]", B, ELMO_MAX_PREDICT_BATCH);
  if (k < 1 || k > ELMO_MAX_TOPK) return fail(ELMO_EINVAL, "k = %d outside [1, %d]", k, ELMO_MAX_TOPK);
  ELMO_CUDA(elmo::launch_topk_merge(idx_dev, score_dev, P, B, k, idx_out_dev, score_out_dev, as_stream(stream)),
            "topk merge");
  return ELMO_OK;
}

}  // extern "C"
