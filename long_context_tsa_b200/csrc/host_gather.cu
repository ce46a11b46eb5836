// Kept-row gather from host memory for the host-buffer forward.
//
// "Token Sparse Attention Long Context" (skill page), Step 2 gather_tokens;
// "Token Sparse Attention: Efficient Long-Context Inference with Interleaved
// Token Selection", Figure 3, Stage 1 (each head's Q, K, V compressed to its
// token subset).  The attention reads, per KV group g, only the rows of Q (its
// G query heads) and V at the kept positions perm[b, g, 0:K].  When the
// caller's host buffers are mapped into the device's address space (pinned
// with the mapped flag, which unified addressing implies for cudaHostAlloc),
// this kernel reads exactly those rows over the host link and writes them to
// the same positions of the device copies of Q and V; the other device rows
// are left as they are, and the attention never reads them.
//
// Grid (row chunks of 128 kept positions, B*Hkv); 256 threads.  Item t of a
// chunk is one 16-byte piece of one row: consecutive threads take consecutive
// pieces of a row, so every row moves as whole contiguous segments.
#include <cuda_runtime.h>

#include "device_common.cuh"
#include "internal.h"

namespace tsa {
namespace {

constexpr int kGatherThreads = 256;
constexpr int kGatherRows = 128;  // kept positions per block

__global__ void __launch_bounds__(kGatherThreads) gather_kept_rows(const uint4* __restrict__ q_src,
                                                                   const uint4* __restrict__ v_src,
                                                                   const int32_t* __restrict__ perm, Budgets kept,
                                                                   uint4* __restrict__ q_dst, uint4* __restrict__ v_dst,
                                                                   int Hq, int Hkv, int L, int G, int row16,
                                                                   uint32_t* status) {
  const int grp = blockIdx.y;
  const int b = grp / Hkv, g = grp - b * Hkv;
  const int K = kept.kept[grp];
  const int i0 = blockIdx.x * kGatherRows;
  if (i0 >= K) return;
  const int n = min(kGatherRows, K - i0);
  const int per_pos = (G + 1) * row16;  // G query rows and one value row, in 16-byte pieces
  const int32_t* pm = perm + (size_t)grp * L;
  const int items = n * per_pos;
#pragma unroll 4
  for (int t = threadIdx.x; t < items; t += kGatherThreads) {
    const int ii = t / per_pos, rem = t - ii * per_pos;
    const int rr = rem / row16, c16 = rem - rr * row16;
    const int p = pm[i0 + ii];
    if ((unsigned)p >= (unsigned)L) {
      record_status(status, TSA_ERR_DEVICE_BOUNDS);
      continue;
    }
    if (rr < G) {
      const size_t off = ((size_t)(b * Hq + g * G + rr) * L + p) * row16 + c16;
      q_dst[off] = q_src[off];
    } else {
      const size_t off = ((size_t)(b * Hkv + g) * L + p) * row16 + c16;
      v_dst[off] = v_src[off];
    }
  }
}

}  // namespace

cudaError_t launch_gather_kept_rows(const Dims& d, const void* q_src, const void* v_src, const int32_t* perm,
                                    const Budgets& kept, void* q_dst, void* v_dst, uint32_t* status,
                                    cudaStream_t st) {
  int kmax = 0;
  for (int i = 0; i < d.B * d.Hkv; ++i) kmax = kept.kept[i] > kmax ? kept.kept[i] : kmax;
  if (kmax == 0) return cudaSuccess;
  const int esz = d.dtype == TSA_F32 ? 4 : 2;
  const int row16 = d.D * esz / 16;
  const dim3 grid((unsigned)((kmax + kGatherRows - 1) / kGatherRows), (unsigned)(d.B * d.Hkv));
  gather_kept_rows<<<grid, kGatherThreads, 0, st>>>(static_cast<const uint4*>(q_src), static_cast<const uint4*>(v_src),
                                                    perm, kept, static_cast<uint4*>(q_dst), static_cast<uint4*>(v_dst),
                                                    d.Hq, d.Hkv, d.L, d.G, row16, status);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace tsa
