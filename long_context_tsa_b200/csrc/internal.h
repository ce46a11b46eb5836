// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/tsa.h"

namespace tsa {

constexpr int kMaxGroups = 1024;      // B * Hkv limit (budgets travel as kernel parameters)
constexpr int kMaxWindowRows = 256;   // G * window limit
constexpr int kScoreKeyTile = 64;     // keys per SIMT score tile
constexpr int kMaxScoreSplits = 256;  // key-range splits per KV head in the score passes

struct Dims {
  int B, Hq, Hkv, L, D, G, dtype;
  float scale;  // resolved (> 0)
};

// Workspace regions, byte offsets from the workspace base (256-byte aligned).
struct WsLayout {
  size_t status;  // uint32 status word + counters (256 B header)
  size_t scores;  // [B,Hkv,L] f32 scratch for tsa_forward
  size_t perm;    // [B,Hkv,L] i32 scratch for tsa_forward
  size_t part;    // score partials [B*Hkv][splits][Mp] x {max, sum} f32
  size_t lse;     // combined per-row log-normaliser [B*Hkv][Mp] f32
  size_t budgets; // [B*Hkv] i32 budgets chosen on the device (coverage mode)
  size_t total;
};

WsLayout ws_layout(const Dims& d, int window);

// Argument checks shared by the entry points (same status codes everywhere).
bool aligned16(const void* p);
tsa_status check_desc(const tsa_desc* desc, Dims* d);  // fills d on TSA_OK
tsa_status check_window(const Dims& d, int window);
// Bytes of per-split score partials the score passes of d.dtype need.
size_t score_partials_bytes(const Dims& d, int window);
// Device address of tsa_score_noalloc's status word on the current device.
cudaError_t noalloc_status_word(uint32_t** word);
int score_splits(const Dims& d);
int window_rows_padded(const Dims& d, int window);  // Mp: G*window rounded up to 64

uint64_t wait_limit();  // polls for device bounded waits
void count_launches(int n);  // every launcher reports the kernels it enqueued
void count_pair_launch();    // the two-SM attention kernel reports each launch here too

// Kept counts clamped to L, one per (b, g); filled by the host entry points.
struct Budgets {
  int32_t kept[kMaxGroups];
};

// ---- launchers (return the CUDA error of the launch) ----
cudaError_t launch_score_simt(const Dims& d, const void* q, const void* k, int window, float* scores,
                              float* part, uint32_t* status, cudaStream_t st);
cudaError_t launch_score_tc(const Dims& d, const void* q, const void* k, int window, float* scores, float* part,
                            uint32_t* status, cudaStream_t st);
int score_tc_splits(const Dims& d);
cudaError_t launch_select(const Dims& d, const float* scores, const Budgets& kept, int32_t* perm,
                          uint32_t* status, cudaStream_t st);
cudaError_t launch_select_coverage(const Dims& d, const float* scores, double tau, int32_t* perm, int32_t* k_out,
                                   uint32_t* status, cudaStream_t st);
// block_mask: optional [B*Hkv][nb][nb] bytes (nb = ceil(L/128)) over 128-blocks of
// compacted (query, key) positions; null for plain causal attention.
cudaError_t launch_attend_simt(const Dims& d, const void* q, const void* k, const void* v,
                               const int32_t* perm, const Budgets& kept, void* out, uint32_t* status,
                               bool accumulate, const uint8_t* block_mask, cudaStream_t st);
cudaError_t launch_attend_tc(const Dims& d, const void* q, const void* k, const void* v, const int32_t* perm,
                             const Budgets& kept, void* out, uint32_t* status, bool accumulate,
                             const uint8_t* block_mask, cudaStream_t st);
// d = 128 on CTA pairs (cta_group::2): the same operation as launch_attend_tc.
cudaError_t launch_attend_tc_pair(const Dims& d, const void* q, const void* k, const void* v, const int32_t* perm,
                                  const Budgets& kept, void* out, uint32_t* status, bool accumulate,
                                  const uint8_t* block_mask, cudaStream_t st);
// Kept rows of Q (the G query heads of each group) and V, read from host
// memory mapped into the device address space, written to the same positions
// of the device buffers (host_gather.cu).
cudaError_t launch_gather_kept_rows(const Dims& d, const void* q_src, const void* v_src, const int32_t* perm,
                                    const Budgets& kept, void* q_dst, void* v_dst, uint32_t* status,
                                    cudaStream_t st);
cudaError_t launch_zero_fill(const Dims& d, const int32_t* perm, const Budgets& kept, void* out,
                             uint32_t* status, cudaStream_t st);
// Output projection (out_proj.cu): its own workspace, a 256-byte status header
// first, then the group masks of the positions and their counting sort.
constexpr int kOutProjMaxHkv = 16;  // the sort has one bucket per mask: 2^Hkv
struct OpWsLayout {
  size_t count, mask, hist, zero_end;  // [count, zero_end) is zeroed by each call
  size_t cursor, order, key, total;
};
OpWsLayout out_proj_ws_layout(const Dims& d);
cudaError_t launch_out_proj(const Dims& d, const void* attn, const int32_t* perm, const Budgets& kept,
                            const void* w_o, int N, void* x, void* ws, cudaStream_t st);
constexpr int kDriftMaxBlocks = 2048;  // drift partials held in its workspace
constexpr size_t kDriftWsBytes = 256 + sizeof(double) * kDriftMaxBlocks;
int drift_grid(int64_t rows);
cudaError_t launch_drift(int64_t rows, int hidden, int dtype, const void* a, const void* b, float* row_cos,
                         double* drift, void* ws, cudaStream_t st);
cudaError_t launch_debug_exp2(const float* x, float* y, int n, cudaStream_t st);
cudaError_t launch_debug_wait(uint32_t* status, uint32_t* flag, uint64_t limit, cudaStream_t st);

}  // namespace tsa
