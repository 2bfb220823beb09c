// noalloc.cu -- a training step that allocates no memory.
//
// Some callers cannot call cudaMalloc: code running while a stream is being
// captured into a CUDA graph (allocation is not a capturable operation),
// runtimes that hand the library a fixed memory budget and must not see it
// grow, and hosts whose allocator is owned by someone else.  They cannot
// create an elmo_head (its workspace is allocated) and cannot let the step
// grow its gradient buffer on first use.  elmo_train_step_noalloc serves them:
// it runs the same kernels as elmo_train_step_chunked, but all of its scratch
// lives in one statically sized device array defined in this file, which every
// GPU that loads the library holds until the process exits.
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <mutex>

#include "../../include/elmo.h"
#include "elmo_internal.h"

namespace {

// Layout of the scratch array (offsets are multiples of 256 bytes).
constexpr size_t kKeysBytes = sizeof(uint32_t) * ELMO_MAX_NNZ;                         // sorted positives
constexpr size_t kSmallBytes = 256;                                                    // key count, s_X, 1/s_X
constexpr size_t kXqBytes = (size_t)ELMO_MAX_BATCH * 4096;                             // E4M3 X
constexpr size_t kTilePtrBytes = (sizeof(int32_t) * ((ELMO_MAX_LABELS / 128) + 1) + 255) / 256 * 256;
constexpr size_t kGBytes = 8u << 20;                                                   // gradient operands
constexpr size_t kScratchBytes = kKeysBytes + kSmallBytes + 2 * kXqBytes + kTilePtrBytes + kGBytes;
static_assert(kScratchBytes <= ELMO_NOALLOC_SCRATCH_BYTES, "no-alloc scratch layout");

static __device__ __align__(256) unsigned char g_noalloc_scratch[ELMO_NOALLOC_SCRATCH_BYTES];

// Device address of the array, looked up once per device (host code must not
// use the symbol itself as a pointer: on the host it is only a stand-in).
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_dev[kMaxDevices] = {};

elmo_status fail(elmo_status code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  elmo::set_last_error(buf);          // read back through elmo_last_error()
  return code;
}

}  // namespace

extern "C" elmo_status elmo_train_step_noalloc(void* W_dev, int64_t L, int32_t d, elmo_dtype dt, const void* X_dev,
                                               int32_t B, const int32_t* rowptr_dev, const int32_t* cols_dev,
                                               int32_t nnz, float lr, int64_t chunk, uint64_t seed, uint64_t step,
                                               float* dX_dev, int32_t* status_dev, void* stream) {
  elmo::set_last_error("");
  // ---- arguments (the same limits as the head-based step; the scratch is sized for them)
  if (!W_dev || !X_dev || !rowptr_dev || !dX_dev || !status_dev) return fail(ELMO_EINVAL, "null pointer argument");
  if (nnz > 0 && !cols_dev) return fail(ELMO_EINVAL, "null cols with nnz > 0");
  if (dt != ELMO_BF16 && dt != ELMO_FP8_E4M3 && dt != ELMO_FP8_E4M3_GE5M2 && dt != ELMO_FP8_E5M2)
    return fail(ELMO_EINVAL, "unknown dtype %d", (int)dt);
  const bool g_e5m2 = dt == ELMO_FP8_E4M3_GE5M2;
  const bool w_e5m2 = dt == ELMO_FP8_E5M2;
  if (g_e5m2 || w_e5m2) dt = ELMO_FP8_E4M3;          // X and G in E4M3 (or E5M2 G)
  if (L < 1 || L >= ELMO_MAX_LABELS)
    return fail(ELMO_EUNSUPPORTED, "L = %lld: the no-allocation step supports 1 <= L < 2^24", (long long)L);
  if (d < 64 || d > 4096 || d % 64 != 0)
    return fail(ELMO_EUNSUPPORTED, "d = %d: the no-allocation step supports multiples of 64 up to 4096", d);
  if (B < 1 || B > ELMO_MAX_BATCH)
    return fail(ELMO_EUNSUPPORTED, "B = %d: the no-allocation step supports 1 <= B <= %d", B, ELMO_MAX_BATCH);
  if (nnz < 0 || nnz > ELMO_MAX_NNZ)
    return fail(ELMO_EUNSUPPORTED, "nnz = %d: the no-allocation step supports 0 <= nnz <= %d", nnz, ELMO_MAX_NNZ);
  if (chunk < 1) return fail(ELMO_EINVAL, "chunk = %lld < 1", (long long)chunk);
  if (!(lr == lr) || lr > 3.0e38f || lr < -3.0e38f) return fail(ELMO_EINVAL, "lr is not finite");
  const uintptr_t mis = reinterpret_cast<uintptr_t>(W_dev) | reinterpret_cast<uintptr_t>(X_dev) |
                        reinterpret_cast<uintptr_t>(dX_dev);
  if (mis & 15u) return fail(ELMO_EINVAL, "W, X and dX must be 16-byte aligned");

  // ---- the scratch array's device address, once per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(ELMO_ECUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(ELMO_EUNSUPPORTED, "device ordinal %d above %d", dev, kMaxDevices - 1);
  void* base = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_dev[dev]) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess || !p) return fail(ELMO_ECUDA, "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
      g_scratch_dev[dev] = p;
    }
    base = g_scratch_dev[dev];
  }
  int major = 0, nsm = 0;
  e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return fail(ELMO_ECUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
  if (major != 10) return fail(ELMO_EUNSUPPORTED, "device %d is not an sm_100 GPU", dev);

  // ---- a head on the host stack whose workspace pointers all point into the scratch array
  char* s = static_cast<char*>(base);
  elmo_head h;
  h.W = W_dev;
  h.L = L;
  h.labels_total = L;
  h.d = d;
  h.dt = dt;
  h.g_e5m2 = g_e5m2;
  h.w_e5m2 = w_e5m2;
  h.device = dev;
  h.num_sms = nsm;
  h.status = status_dev;
  h.keys = reinterpret_cast<uint32_t*>(s);
  h.nkeys = reinterpret_cast<int32_t*>(s + kKeysBytes);
  h.xscale = reinterpret_cast<float*>(s + kKeysBytes + 16);
  h.xq = reinterpret_cast<uint8_t*>(s + kKeysBytes + kSmallBytes);
  h.tile_ptr = reinterpret_cast<int32_t*>(s + kKeysBytes + kSmallBytes + kXqBytes);
  h.xqt = reinterpret_cast<uint8_t*>(s + kKeysBytes + kSmallBytes + kXqBytes + kTilePtrBytes);
  void* gbuf = s + kKeysBytes + kSmallBytes + 2 * kXqBytes + kTilePtrBytes;

  const bool fp8 = dt == ELMO_FP8_E4M3;
  const size_t esz = fp8 ? 1 : 2;
  const int32_t Bp = elmo::padded_batch(B, fp8);
  int64_t sub = elmo::sub_chunk_labels(d, Bp, (int)esz);
  const int64_t fit = (int64_t)(kGBytes / ((size_t)Bp * esz)) / 128 * 128;   // labels whose G fits the scratch
  if (sub > fit) sub = fit;
  if (sub > chunk) sub = chunk;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const uint16_t* X = static_cast<const uint16_t*>(X_dev);
  // the status word and dX must start at zero; everything else in the scratch is rewritten before it is read
  e = cudaMemsetAsync(status_dev, 0, 2 * sizeof(int32_t), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(dX_dev, 0, sizeof(float) * (size_t)B * d, st);
  if (e == cudaSuccess) e = elmo::launch_prep_step(&h, rowptr_dev, cols_dev, B, nnz, X, st);
  for (int64_t c0 = 0; e == cudaSuccess && c0 < L; c0 += chunk) {
    const int64_t c1 = c0 + chunk < L ? c0 + chunk : L;
    for (int64_t a = c0; e == cudaSuccess && a < c1; a += sub) {
      const int64_t b = a + sub < c1 ? a + sub : c1;
      e = elmo::launch_logits_grad_tc(&h, X, B, a, b, gbuf, nullptr, nullptr, st, a > 0);
      if (e == cudaSuccess) e = elmo::launch_update_tc(&h, X, B, a, b, gbuf, lr, seed, step, dX_dev, st, true);
    }
  }
  if (e != cudaSuccess) return fail(ELMO_ECUDA, "elmo_train_step_noalloc: %s", cudaGetErrorString(e));
  return ELMO_OK;
}
