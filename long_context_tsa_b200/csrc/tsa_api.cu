// Host entry points of the C ABI declared in include/tsa.h: argument checks,
// workspace layout, launch planning and the device status word.
#include <math.h>

#include <atomic>

#include "device_common.cuh"
#include "internal.h"

namespace tsa {

static std::atomic<uint64_t> g_wait_limit{0};

uint64_t wait_limit() {
  const uint64_t v = g_wait_limit.load(std::memory_order_relaxed);
  return v ? v : (uint64_t{1} << 24);
}

static std::atomic<uint64_t> g_launches{0};

void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

static std::atomic<uint64_t> g_pair_launches{0};

void count_pair_launch() { g_pair_launches.fetch_add(1, std::memory_order_relaxed); }

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int window_rows_padded(const Dims& d, int window) {
  const int M = d.G * window;
  return (M + 63) / 64 * 64;
}

// Key-range splits per KV head of the SIMT score passes.  A function of L only:
// a KV head's scores do not depend on which other heads share the call, so a
// layer split by KV group across calls (or GPUs) gives bit-identical scores.
int score_splits(const Dims& d) {
  const int ntiles = (d.L + kScoreKeyTile - 1) / kScoreKeyTile;
  int s = ntiles < 74 ? ntiles : 74;
  s = s < kMaxScoreSplits ? s : kMaxScoreSplits;
  return s < 1 ? 1 : s;
}

WsLayout ws_layout(const Dims& d, int window) {
  WsLayout w;
  size_t off = 0;
  w.status = off;
  off += 256;
  const size_t n = (size_t)d.B * d.Hkv * d.L;
  w.scores = off;
  off += align256(n * sizeof(float));
  w.perm = off;
  off += align256(n * sizeof(int32_t));
  // Partials: the SIMT passes pad the window rows to 64, the tensor-core passes to 128 or 256.
  const int Mp_simt = window_rows_padded(d, window);
  const int Mp_tc = d.G * window > 128 ? 256 : 128;
  const int Mp = Mp_simt > Mp_tc ? Mp_simt : Mp_tc;
  w.part = off;
  off += align256((size_t)d.B * d.Hkv * kMaxScoreSplits * Mp * 2 * sizeof(float));
  w.lse = off;
  off += align256((size_t)d.B * d.Hkv * Mp * sizeof(float));
  w.budgets = off;
  off += align256((size_t)kMaxGroups * sizeof(int32_t));
  w.total = off;
  return w;
}

size_t score_partials_bytes(const Dims& d, int window) {
  const size_t groups = (size_t)d.B * d.Hkv;
  if (d.dtype == TSA_BF16) {  // tensor-core passes: window rows padded to 128 or 256
    const size_t Mp_tc = d.G * window > 128 ? 256 : 128;
    return groups * (size_t)score_tc_splits(d) * Mp_tc * 2 * sizeof(float);
  }
  return groups * (size_t)score_splits(d) * (size_t)window_rows_padded(d, window) * 2 * sizeof(float);
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

tsa_status check_desc(const tsa_desc* desc, Dims* d) {
  if (desc == nullptr) return TSA_ERR_INVALID_ARG;
  if (desc->B < 1 || desc->Hq < 1 || desc->Hkv < 1 || desc->L < 1 || desc->D < 1) return TSA_ERR_INVALID_ARG;
  if (desc->dtype != TSA_F32 && desc->dtype != TSA_BF16) return TSA_ERR_INVALID_ARG;
  if (desc->Hq % desc->Hkv != 0) return TSA_ERR_INVALID_ARG;
  if (!(desc->scale >= 0.f) && !(desc->scale < 0.f)) return TSA_ERR_INVALID_ARG;  // NaN
  if (desc->D != 64 && desc->D != 128) return TSA_ERR_UNSUPPORTED;
  const int G = desc->Hq / desc->Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16) return TSA_ERR_UNSUPPORTED;
  if ((long long)desc->B * desc->Hq * desc->L >= (1LL << 31)) return TSA_ERR_UNSUPPORTED;
  if ((long long)desc->B * desc->Hkv > kMaxGroups) return TSA_ERR_UNSUPPORTED;
  d->B = desc->B;
  d->Hq = desc->Hq;
  d->Hkv = desc->Hkv;
  d->L = desc->L;
  d->D = desc->D;
  d->G = G;
  d->dtype = desc->dtype;
  d->scale = desc->scale > 0.f ? desc->scale : 1.0f / sqrtf((float)desc->D);
  return TSA_OK;
}

tsa_status check_window(const Dims& d, int window) {
  if (window < 1 || window > d.L) return TSA_ERR_INVALID_ARG;
  if (d.G * window > kMaxWindowRows) return TSA_ERR_UNSUPPORTED;
  return TSA_OK;
}

namespace {

constexpr size_t kHeaderBytes = 256;

tsa_status load_budgets(const Dims& d, const int32_t* budget_host, Budgets* kb) {
  if (budget_host == nullptr) return TSA_ERR_INVALID_ARG;
  for (int i = 0; i < d.B * d.Hkv; ++i) {
    const int32_t x = budget_host[i];
    if (x < 1) return TSA_ERR_INVALID_ARG;
    kb->kept[i] = x < d.L ? x : d.L;
  }
  return TSA_OK;
}

uint32_t* status_word(void* ws) { return static_cast<uint32_t*>(ws); }

template <typename P>
P* ws_ptr(void* ws, size_t off) {
  return reinterpret_cast<P*>(static_cast<char*>(ws) + off);
}

tsa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? TSA_OK : TSA_ERR_CUDA; }

tsa_status run_score(const Dims& d, const void* q, const void* k, int window, float* scores, void* ws,
                     cudaStream_t st) {
  const WsLayout w = ws_layout(d, window);
  if (d.dtype == TSA_BF16)
    return cuda_status(launch_score_tc(d, q, k, window, scores, ws_ptr<float>(ws, w.part), status_word(ws), st));
  return cuda_status(launch_score_simt(d, q, k, window, scores, ws_ptr<float>(ws, w.part), status_word(ws), st));
}

tsa_status run_select(const Dims& d, const float* scores, const Budgets& kb, int32_t* perm, void* ws,
                      cudaStream_t st) {
  return cuda_status(launch_select(d, scores, kb, perm, status_word(ws), st));
}

tsa_status run_attend(const Dims& d, const void* q, const void* k, const void* v, const int32_t* perm,
                      const Budgets& kb, void* out, void* ws, cudaStream_t st, bool accumulate = false,
                      const uint8_t* block_mask = nullptr) {
  // The tensor-core kernel zero-fills the dropped rows itself (unless accumulating).
  if (d.dtype == TSA_BF16)
    return cuda_status(launch_attend_tc(d, q, k, v, perm, kb, out, status_word(ws), accumulate, block_mask, st));
  if (!accumulate) {
    const tsa_status s = cuda_status(launch_zero_fill(d, perm, kb, out, status_word(ws), st));
    if (s != TSA_OK) return s;
  }
  return cuda_status(launch_attend_simt(d, q, k, v, perm, kb, out, status_word(ws), accumulate, block_mask, st));
}

__global__ void debug_wait_kernel(uint32_t* status, const uint32_t* flag, uint64_t limit) {
  if (threadIdx.x == 0 && !bounded_wait_flag(flag, limit)) record_status(status, TSA_ERR_TIMEOUT);
}

}  // namespace

cudaError_t launch_debug_wait(uint32_t* status, uint32_t* flag, uint64_t limit, cudaStream_t st) {
  debug_wait_kernel<<<1, 32, 0, st>>>(status, flag, limit);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace tsa

using namespace tsa;

extern "C" {

size_t tsa_workspace_size(const tsa_desc* desc, int32_t window) {
  Dims d;
  if (check_desc(desc, &d) != TSA_OK || check_window(d, window) != TSA_OK) return 0;
  return ws_layout(d, window).total;
}

tsa_status tsa_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (!aligned16(ws) || ws_bytes < kHeaderBytes) return TSA_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(ws, 0, kHeaderBytes, static_cast<cudaStream_t>(stream)));
}

tsa_status tsa_score(const tsa_desc* desc, const void* q, const void* k, int32_t window, float* scores,
                     void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  tsa_status s = check_desc(desc, &d);
  if (s != TSA_OK) return s;
  if ((s = check_window(d, window)) != TSA_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(scores) || !aligned16(ws)) return TSA_ERR_INVALID_ARG;
  if (ws_bytes < ws_layout(d, window).total) return TSA_ERR_WORKSPACE;
  return run_score(d, q, k, window, scores, ws, static_cast<cudaStream_t>(stream));
}

tsa_status tsa_select(const tsa_desc* desc, const float* scores, const int32_t* budget_host, int32_t* perm,
                      void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  tsa_status s = check_desc(desc, &d);
  if (s != TSA_OK) return s;
  if (!aligned16(scores) || !aligned16(perm) || !aligned16(ws)) return TSA_ERR_INVALID_ARG;
  if (ws_bytes < kHeaderBytes) return TSA_ERR_WORKSPACE;
  Budgets kb;
  if ((s = load_budgets(d, budget_host, &kb)) != TSA_OK) return s;
  return run_select(d, scores, kb, perm, ws, static_cast<cudaStream_t>(stream));
}

tsa_status tsa_select_coverage(const tsa_desc* desc, const float* scores, double tau, int32_t* perm,
                               int32_t* budget_dev_out, void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  tsa_status s = check_desc(desc, &d);
  if (s != TSA_OK) return s;
  if (!(tau >= 0.0 && tau <= 1.0)) return TSA_ERR_INVALID_ARG;  // also rejects NaN
  if (!aligned16(scores) || !aligned16(perm) || !aligned16(ws) || budget_dev_out == nullptr ||
      (reinterpret_cast<uintptr_t>(budget_dev_out) & 3u) != 0)
    return TSA_ERR_INVALID_ARG;
  if (ws_bytes < kHeaderBytes) return TSA_ERR_WORKSPACE;
  return cuda_status(launch_select_coverage(d, scores, tau, perm, budget_dev_out, status_word(ws),
                                            static_cast<cudaStream_t>(stream)));
}

tsa_status tsa_attend(const tsa_desc* desc, const void* q, const void* k, const void* v, const int32_t* perm,
                      const int32_t* budget_host, void* out, void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  tsa_status s = check_desc(desc, &d);
  if (s != TSA_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(perm) || !aligned16(out) || !aligned16(ws))
    return TSA_ERR_INVALID_ARG;
  if (ws_bytes < kHeaderBytes) return TSA_ERR_WORKSPACE;
  Budgets kb;
  if ((s = load_budgets(d, budget_host, &kb)) != TSA_OK) return s;
  return run_attend(d, q, k, v, perm, kb, out, ws, static_cast<cudaStream_t>(stream));
}

size_t tsa_out_proj_workspace_size(const tsa_desc* desc) {
  Dims d;
  if (check_desc(desc, &d) != TSA_OK || d.Hkv > kOutProjMaxHkv) return 0;
  return out_proj_ws_layout(d).total;
}

tsa_status tsa_out_proj(const tsa_desc* desc, const void* attn_out, const int32_t* perm, const int32_t* budget_host,
                        const void* w_o, int32_t hidden, void* x, void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  tsa_status s = check_desc(desc, &d);
  if (s != TSA_OK) return s;
  if (d.Hkv > kOutProjMaxHkv) return TSA_ERR_UNSUPPORTED;
  if (hidden < 1) return TSA_ERR_INVALID_ARG;
  if (hidden % (d.dtype == TSA_BF16 ? 256 : 64) != 0) return TSA_ERR_UNSUPPORTED;
  if ((long long)d.B * d.L * hidden >= (1LL << 40)) return TSA_ERR_UNSUPPORTED;
  if (!aligned16(attn_out) || !aligned16(perm) || !aligned16(w_o) || !aligned16(x) || !aligned16(ws))
    return TSA_ERR_INVALID_ARG;
  if (ws_bytes < out_proj_ws_layout(d).total) return TSA_ERR_WORKSPACE;
  Budgets kb;
  if ((s = load_budgets(d, budget_host, &kb)) != TSA_OK) return s;
  return cuda_status(launch_out_proj(d, attn_out, perm, kb, w_o, hidden, x, ws, static_cast<cudaStream_t>(stream)));
}

tsa_status tsa_zero_dropped(const tsa_desc* desc, const int32_t* perm, const int32_t* budget_host, void* out,
                            void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  tsa_status s = check_desc(desc, &d);
  if (s != TSA_OK) return s;
  if (!aligned16(perm) || !aligned16(out) || !aligned16(ws)) return TSA_ERR_INVALID_ARG;
  if (ws_bytes < kHeaderBytes) return TSA_ERR_WORKSPACE;
  Budgets kb;
  if ((s = load_budgets(d, budget_host, &kb)) != TSA_OK) return s;
  return cuda_status(launch_zero_fill(d, perm, kb, out, status_word(ws), static_cast<cudaStream_t>(stream)));
}

tsa_status tsa_attend_accumulate(const tsa_desc* desc, const void* q, const void* k, const void* v,
                                 const int32_t* perm, const int32_t* budget_host, void* out, void* ws, size_t ws_bytes,
                                 void* stream) {
  Dims d;
  tsa_status s = check_desc(desc, &d);
  if (s != TSA_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(perm) || !aligned16(out) || !aligned16(ws))
    return TSA_ERR_INVALID_ARG;
  if (ws_bytes < kHeaderBytes) return TSA_ERR_WORKSPACE;
  Budgets kb;
  if ((s = load_budgets(d, budget_host, &kb)) != TSA_OK) return s;
  return run_attend(d, q, k, v, perm, kb, out, ws, static_cast<cudaStream_t>(stream), true);
}

tsa_status tsa_attend_block_sparse(const tsa_desc* desc, const void* q, const void* k, const void* v,
                                   const int32_t* perm, const int32_t* budget_host, const uint8_t* block_mask,
                                   void* out, void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  tsa_status s = check_desc(desc, &d);
  if (s != TSA_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(perm) || !aligned16(out) || !aligned16(ws) ||
      block_mask == nullptr)
    return TSA_ERR_INVALID_ARG;
  if (ws_bytes < kHeaderBytes) return TSA_ERR_WORKSPACE;
  Budgets kb;
  if ((s = load_budgets(d, budget_host, &kb)) != TSA_OK) return s;
  return run_attend(d, q, k, v, perm, kb, out, ws, static_cast<cudaStream_t>(stream), false, block_mask);
}

size_t tsa_drift_workspace_size(void) { return kDriftWsBytes; }

tsa_status tsa_drift(int64_t rows, int32_t hidden, int32_t dtype, const void* h_before, const void* h_after,
                     float* row_cos_or_null, double* drift, void* ws, size_t ws_bytes, void* stream) {
  if (dtype != TSA_F32 && dtype != TSA_BF16) return TSA_ERR_INVALID_ARG;
  const int64_t elem = dtype == TSA_BF16 ? 2 : 4;
  if (rows < 1 || hidden < 1 || (int64_t(hidden) * elem) % 16 != 0) return TSA_ERR_INVALID_ARG;
  if (rows > (int64_t(1) << 40) / hidden) return TSA_ERR_INVALID_ARG;  // bounds the row offsets
  if (!aligned16(h_before) || !aligned16(h_after) || !aligned16(ws) || drift == nullptr) return TSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(drift) & 7u) != 0) return TSA_ERR_INVALID_ARG;
  if (row_cos_or_null && (reinterpret_cast<uintptr_t>(row_cos_or_null) & 3u) != 0) return TSA_ERR_INVALID_ARG;
  if (ws_bytes < kDriftWsBytes) return TSA_ERR_WORKSPACE;
  return cuda_status(launch_drift(rows, hidden, dtype, h_before, h_after, row_cos_or_null, drift, ws,
                                  static_cast<cudaStream_t>(stream)));
}

tsa_status tsa_layer_stable(const double* history, int32_t n, int32_t window, double threshold, int32_t* stable) {
  if (stable == nullptr || window < 1 || n < 0 || (n > 0 && history == nullptr)) return TSA_ERR_INVALID_ARG;
  *stable = 0;
  if (n < window) return TSA_OK;
  double sum = 0.0;
  for (int32_t i = n - window; i < n; ++i) sum += history[i];
  *stable = sum / window < threshold ? 1 : 0;
  return TSA_OK;
}

tsa_status tsa_forward(const tsa_desc* desc, const void* q, const void* k, const void* v, int32_t window,
                       const int32_t* budget_host, float* scores_or_null, int32_t* perm_or_null, void* out,
                       void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  tsa_status s = check_desc(desc, &d);
  if (s != TSA_OK) return s;
  if ((s = check_window(d, window)) != TSA_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(ws))
    return TSA_ERR_INVALID_ARG;
  if ((scores_or_null && !aligned16(scores_or_null)) || (perm_or_null && !aligned16(perm_or_null)))
    return TSA_ERR_INVALID_ARG;
  const WsLayout w = ws_layout(d, window);
  if (ws_bytes < w.total) return TSA_ERR_WORKSPACE;
  Budgets kb;
  if ((s = load_budgets(d, budget_host, &kb)) != TSA_OK) return s;
  float* scores = scores_or_null ? scores_or_null : ws_ptr<float>(ws, w.scores);
  int32_t* perm = perm_or_null ? perm_or_null : ws_ptr<int32_t>(ws, w.perm);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = run_score(d, q, k, window, scores, ws, st)) != TSA_OK) return s;
  if ((s = run_select(d, scores, kb, perm, ws, st)) != TSA_OK) return s;
  return run_attend(d, q, k, v, perm, kb, out, ws, st);
}

tsa_status tsa_forward_coverage(const tsa_desc* desc, const void* q, const void* k, const void* v, int32_t window,
                                double tau, int32_t* budget_host_out, float* scores_or_null, int32_t* perm_or_null,
                                void* out, void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  tsa_status s = check_desc(desc, &d);
  if (s != TSA_OK) return s;
  if ((s = check_window(d, window)) != TSA_OK) return s;
  if (!(tau >= 0.0 && tau <= 1.0) || budget_host_out == nullptr) return TSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(ws))
    return TSA_ERR_INVALID_ARG;
  if ((scores_or_null && !aligned16(scores_or_null)) || (perm_or_null && !aligned16(perm_or_null)))
    return TSA_ERR_INVALID_ARG;
  const WsLayout w = ws_layout(d, window);
  if (ws_bytes < w.total) return TSA_ERR_WORKSPACE;
  float* scores = scores_or_null ? scores_or_null : ws_ptr<float>(ws, w.scores);
  int32_t* perm = perm_or_null ? perm_or_null : ws_ptr<int32_t>(ws, w.perm);
  int32_t* kdev = ws_ptr<int32_t>(ws, w.budgets);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = run_score(d, q, k, window, scores, ws, st)) != TSA_OK) return s;
  if ((s = cuda_status(launch_select_coverage(d, scores, tau, perm, kdev, status_word(ws), st))) != TSA_OK) return s;
  // The attention grid is sized from the budgets, so they come back to the host here.
  const size_t nb = (size_t)d.B * d.Hkv * sizeof(int32_t);
  if ((s = cuda_status(cudaMemcpyAsync(budget_host_out, kdev, nb, cudaMemcpyDeviceToHost, st))) != TSA_OK) return s;
  if ((s = cuda_status(cudaStreamSynchronize(st))) != TSA_OK) return s;
  Budgets kb;
  if ((s = load_budgets(d, budget_host_out, &kb)) != TSA_OK) return s;
  return run_attend(d, q, k, v, perm, kb, out, ws, st);
}

namespace {

// The device address of host memory that is mapped into this device's address
// space (pinned with the mapped flag, implied for cudaHostAlloc under unified
// addressing), or null for pageable memory.
const void* mapped_device_ptr(const void* host) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, host) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  return a.type == cudaMemoryTypeHost ? a.devicePointer : nullptr;
}

// Host-to-device bytes of tsa_forward_host; sparse: q and v are read in place.
size_t host_h2d_bytes(const Dims& d, int window, const Budgets& kb, bool sparse) {
  const size_t esz = d.dtype == TSA_F32 ? 4 : 2;
  const size_t row = (size_t)d.D * esz;
  const size_t kvbytes = (size_t)d.B * d.Hkv * d.L * row;
  if (!sparse) return (size_t)d.B * d.Hq * d.L * row + 2 * kvbytes;
  size_t kept = 0;
  for (int i = 0; i < d.B * d.Hkv; ++i) kept += (size_t)kb.kept[i];
  return kvbytes + (size_t)d.B * d.Hq * window * row + kept * (size_t)(d.G + 1) * row;
}

}  // namespace

tsa_status tsa_forward_host(const tsa_desc* desc, const void* q_host, const void* k_host, const void* v_host,
                            int32_t window, const int32_t* budget_host, void* out_host, void* q_dev, void* k_dev,
                            void* v_dev, void* out_dev, void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  tsa_status s = check_desc(desc, &d);
  if (s != TSA_OK) return s;
  if (!q_host || !k_host || !v_host || !out_host) return TSA_ERR_INVALID_ARG;
  const size_t esz = d.dtype == TSA_F32 ? 4 : 2;
  const size_t qbytes = (size_t)d.B * d.Hq * d.L * d.D * esz;
  const size_t kvbytes = (size_t)d.B * d.Hkv * d.L * d.D * esz;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!aligned16(q_dev) || !aligned16(k_dev) || !aligned16(v_dev) || !aligned16(out_dev)) return TSA_ERR_INVALID_ARG;
  if ((s = check_window(d, window)) != TSA_OK) return s;
  const WsLayout w = ws_layout(d, window);
  if (ws_bytes < w.total) return TSA_ERR_WORKSPACE;
  Budgets kb;
  if ((s = load_budgets(d, budget_host, &kb)) != TSA_OK) return s;
  const void* q_map = mapped_device_ptr(q_host);
  const void* v_map = mapped_device_ptr(v_host);
  if (q_map == nullptr || v_map == nullptr || !aligned16(q_map) || !aligned16(v_map)) {
    // Full copies of the three inputs, then the device forward.
    if (cudaMemcpyAsync(q_dev, q_host, qbytes, cudaMemcpyHostToDevice, st) != cudaSuccess) return TSA_ERR_CUDA;
    if (cudaMemcpyAsync(k_dev, k_host, kvbytes, cudaMemcpyHostToDevice, st) != cudaSuccess) return TSA_ERR_CUDA;
    if (cudaMemcpyAsync(v_dev, v_host, kvbytes, cudaMemcpyHostToDevice, st) != cudaSuccess) return TSA_ERR_CUDA;
    s = tsa_forward(desc, q_dev, k_dev, v_dev, window, budget_host, nullptr, nullptr, out_dev, ws, ws_bytes, stream);
    if (s != TSA_OK) return s;
  } else {
    // Mapped q and v: only what the step reads crosses the host link.  Every
    // key is scored, so K is copied in full; the score's queries are the last
    // `window` rows of each head (one strided copy); after the selection the
    // gather kernel reads the kept rows of Q and V in place.
    if (cudaMemcpyAsync(k_dev, k_host, kvbytes, cudaMemcpyHostToDevice, st) != cudaSuccess) return TSA_ERR_CUDA;
    const size_t pitch = (size_t)d.L * d.D * esz, wbytes = (size_t)window * d.D * esz;
    const size_t woff = (size_t)(d.L - window) * d.D * esz;
    if (cudaMemcpy2DAsync(static_cast<char*>(q_dev) + woff, pitch, static_cast<const char*>(q_host) + woff, pitch,
                          wbytes, (size_t)d.B * d.Hq, cudaMemcpyHostToDevice, st) != cudaSuccess)
      return TSA_ERR_CUDA;
    float* scores = ws_ptr<float>(ws, w.scores);
    int32_t* perm = ws_ptr<int32_t>(ws, w.perm);
    if ((s = run_score(d, q_dev, k_dev, window, scores, ws, st)) != TSA_OK) return s;
    if ((s = run_select(d, scores, kb, perm, ws, st)) != TSA_OK) return s;
    if ((s = cuda_status(launch_gather_kept_rows(d, q_map, v_map, perm, kb, q_dev, v_dev, status_word(ws), st))) !=
        TSA_OK)
      return s;
    if ((s = run_attend(d, q_dev, k_dev, v_dev, perm, kb, out_dev, ws, st)) != TSA_OK) return s;
  }
  if (cudaMemcpyAsync(out_host, out_dev, qbytes, cudaMemcpyDeviceToHost, st) != cudaSuccess) return TSA_ERR_CUDA;
  return TSA_OK;
}

size_t tsa_forward_host_h2d_bytes(const tsa_desc* desc, int32_t window, const int32_t* budget_host,
                                  const void* q_host, const void* v_host) {
  Dims d;
  if (check_desc(desc, &d) != TSA_OK || check_window(d, window) != TSA_OK) return 0;
  Budgets kb;
  if (load_budgets(d, budget_host, &kb) != TSA_OK) return 0;
  const void* q_map = q_host ? mapped_device_ptr(q_host) : nullptr;
  const void* v_map = v_host ? mapped_device_ptr(v_host) : nullptr;
  const bool sparse = q_map != nullptr && v_map != nullptr && aligned16(q_map) && aligned16(v_map);
  return host_h2d_bytes(d, window, kb, sparse);
}

tsa_status tsa_check_status(void* ws, size_t ws_bytes, void* stream) {
  uint32_t* word_dev = nullptr;
  if (ws == nullptr) {  // the status word of tsa_score_noalloc on the current device
    if (noalloc_status_word(&word_dev) != cudaSuccess) return TSA_ERR_CUDA;
  } else {
    if (!aligned16(ws) || ws_bytes < kHeaderBytes) return TSA_ERR_INVALID_ARG;
    word_dev = status_word(ws);
  }
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return TSA_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, word_dev, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return TSA_ERR_CUDA;
  if (cudaMemsetAsync(word_dev, 0, sizeof(word), st) != cudaSuccess) return TSA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return TSA_ERR_CUDA;
  switch (word) {
    case TSA_OK:
    case TSA_ERR_TIMEOUT:
    case TSA_ERR_DEVICE_BOUNDS:
      return static_cast<tsa_status>(word);
    default:
      return TSA_ERR_CUDA;
  }
}

const char* tsa_status_string(tsa_status s) {
  switch (s) {
    case TSA_OK: return "ok";
    case TSA_ERR_INVALID_ARG: return "invalid argument";
    case TSA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case TSA_ERR_WORKSPACE: return "workspace too small";
    case TSA_ERR_CUDA: return "CUDA runtime error";
    case TSA_ERR_TIMEOUT: return "device bounded wait timed out";
    case TSA_ERR_DEVICE_BOUNDS: return "device index out of bounds";
  }
  return "unknown status";
}

void tsa_debug_set_wait_limit(uint64_t polls) { g_wait_limit.store(polls, std::memory_order_relaxed); }

uint64_t tsa_debug_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

uint64_t tsa_debug_cta_pair_launch_count(void) { return g_pair_launches.load(std::memory_order_relaxed); }

tsa_status tsa_debug_exp2(const float* x, float* y, int32_t n, void* stream) {
  if (!aligned16(x) || !aligned16(y) || n < 2 || (n & 1)) return TSA_ERR_INVALID_ARG;
  return cuda_status(launch_debug_exp2(x, y, n, static_cast<cudaStream_t>(stream)));
}

tsa_status tsa_debug_wait_never_set(void* ws, size_t ws_bytes, void* stream) {
  if (!aligned16(ws) || ws_bytes < kHeaderBytes) return TSA_ERR_INVALID_ARG;
  uint32_t* base = status_word(ws);
  // base[1] is a header word nothing ever sets.
  return cuda_status(launch_debug_wait(base, base + 1, wait_limit(), static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
