// tsa_score_noalloc: token scoring for callers that cannot allocate device
// memory.
//
// tsa_score needs scratch for its per-split softmax partials and takes it from
// a caller-allocated workspace.  Some callers cannot make that allocation: a
// plugin running inside an engine that owns every byte of device memory, a
// latency-critical loop where a cudaMalloc (and the synchronisation it may
// imply) is not acceptable, or a deployment with a fixed memory budget that
// must not fail with out-of-memory part-way through a run.  This variant keeps
// the scratch in a fixed array that is part of the library itself, so the
// caller passes only the inputs and the output.  It runs the same kernels as
// tsa_score (tensor-core passes for bf16, SIMT passes for f32), so its scores
// are those of tsa_score.
//
// The array below is reserved on every GPU that loads this library and stays
// there until the process exits.  It is shared by all calls: two calls whose
// kernels overlap on the GPU (different streams, or different host threads)
// overwrite each other's partials and produce wrong scores.  The partials are
// written in full by the first pass before the second pass reads them, so no
// part of the array has to start at zero.  The device status word (a bounded
// wait that ran out) is cleared by each call and read back by
// tsa_check_status(NULL, 0, stream).
#include <math.h>

#include <mutex>

#include "internal.h"

namespace tsa {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t{1} << 20;  // 1 MiB of partials

// Host code sees these names only as stand-ins: their device addresses come
// from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) float g_score_scratch[kNoAllocScratchBytes / sizeof(float)];
static __device__ __align__(256) uint32_t g_score_status[64];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float* g_scratch_ptr[kMaxDevices] = {};
uint32_t* g_status_ptr[kMaxDevices] = {};

// Device addresses of the fixed scratch and status word on the current device
// (looked up on the first call made with that device current).
cudaError_t fixed_buffers_for_current_device(float** scratch, uint32_t** status) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_score_scratch);
    if (e != cudaSuccess) return e;
    void* s = nullptr;
    e = cudaGetSymbolAddress(&s, g_score_status);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = static_cast<float*>(p);
    g_status_ptr[dev] = static_cast<uint32_t*>(s);
  }
  *scratch = g_scratch_ptr[dev];
  *status = g_status_ptr[dev];
  return cudaSuccess;
}

}  // namespace

cudaError_t noalloc_status_word(uint32_t** word) {
  float* scratch = nullptr;
  return fixed_buffers_for_current_device(&scratch, word);
}

}  // namespace tsa

using namespace tsa;

extern "C" tsa_status tsa_score_noalloc(const tsa_desc* desc, const void* q, const void* k, int32_t window,
                                        float* scores, void* stream) {
  // Shape first, then the fixed scratch's size limit, then the pointers: a shape
  // the array cannot hold is refused before any pointer is looked at.
  Dims d;
  tsa_status s = check_desc(desc, &d);
  if (s != TSA_OK) return s;
  if ((s = check_window(d, window)) != TSA_OK) return s;
  if (score_partials_bytes(d, window) > kNoAllocScratchBytes) return TSA_ERR_WORKSPACE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(scores)) return TSA_ERR_INVALID_ARG;
  float* scratch = nullptr;
  uint32_t* status = nullptr;
  if (fixed_buffers_for_current_device(&scratch, &status) != cudaSuccess) return TSA_ERR_CUDA;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(status, 0, sizeof(uint32_t), st) != cudaSuccess) return TSA_ERR_CUDA;
  const cudaError_t e = d.dtype == TSA_BF16 ? launch_score_tc(d, q, k, window, scores, scratch, status, st)
                                            : launch_score_simt(d, q, k, window, scores, scratch, status, st);
  return e == cudaSuccess ? TSA_OK : TSA_ERR_CUDA;
}
