// Representation drift between two hidden-state tensors, one streaming pass.
//
// "Token Sparse Attention Long Context" (skill page), Step 4,
// LayerStabilityAnalyzer.compute_representation_drift: each row of
// h_before and h_after ([rows, hidden]) is divided by max(its L2 norm, 1e-12)
// (torch.nn.functional.normalize), the two are dotted, and the drift is one
// minus the mean of those cosines over all rows.
//
// The pass reads every byte of both tensors exactly once, so it is bound by
// HBM bandwidth: algorithmic bytes = 2 * rows * hidden * sizeof(element)
// (+ 4 * rows when per-row cosines are written).  One warp owns one row at a
// time: its 32 lanes stream the row with 16-byte evict-first loads, several
// in flight per lane, and accumulate <a,b>, |a|^2 and |b|^2 in fp32.  The
// cosine of the row is formed once from those three sums:
//     <a,b> / (max(|a|, eps) * max(|b|, eps)),
// which is the normalise-then-dot of the definition up to rounding.  The
// mean over rows is summed in fp64: per warp, per block, then by the last
// block to finish over the blocks' partials in block order, so the result is
// the same on every run for a given grid.
#include <cuda_bf16.h>
#include <stdint.h>

#include "internal.h"

namespace tsa {
namespace {

constexpr int kDriftThreads = 256;  // 8 warps, one row each at a time
constexpr int kDriftUnroll = 4;     // 16-byte loads in flight per lane and tensor
constexpr float kNormEps = 1e-12f;  // torch.nn.functional.normalize default

struct DriftArgs {
  const uint4* a;   // [rows, vecs] 16-byte vectors of h_before
  const uint4* b;   // [rows, vecs] of h_after
  float* row_cos;   // [rows] or null
  double* partial;  // [gridDim.x]
  unsigned int* done;
  double* drift;    // [1]
  int64_t rows;
  int vecs;         // 16-byte vectors per row
};

__device__ __forceinline__ void accum(const uint4& x, const uint4& y, float& ab, float& aa, float& bb, __nv_bfloat16) {
  const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
  const uint32_t ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    // bf16 -> f32 is exact: the bf16 bits are the top half of the f32.
    const float x0 = __uint_as_float(xs[i] << 16), x1 = __uint_as_float(xs[i] & 0xffff0000u);
    const float y0 = __uint_as_float(ys[i] << 16), y1 = __uint_as_float(ys[i] & 0xffff0000u);
    ab = fmaf(x0, y0, ab);
    aa = fmaf(x0, x0, aa);
    bb = fmaf(y0, y0, bb);
    ab = fmaf(x1, y1, ab);
    aa = fmaf(x1, x1, aa);
    bb = fmaf(y1, y1, bb);
  }
}

__device__ __forceinline__ void accum(const uint4& x, const uint4& y, float& ab, float& aa, float& bb, float) {
  const float xs[4] = {__uint_as_float(x.x), __uint_as_float(x.y), __uint_as_float(x.z), __uint_as_float(x.w)};
  const float ys[4] = {__uint_as_float(y.x), __uint_as_float(y.y), __uint_as_float(y.z), __uint_as_float(y.w)};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    ab = fmaf(xs[i], ys[i], ab);
    aa = fmaf(xs[i], xs[i], aa);
    bb = fmaf(ys[i], ys[i], bb);
  }
}

template <typename T>
__global__ void __launch_bounds__(kDriftThreads) drift_kernel(DriftArgs p) {
  __shared__ double warp_sum[kDriftThreads / 32];
  __shared__ bool is_last;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t warps_total = int64_t(gridDim.x) * (kDriftThreads / 32);
  double my_sum = 0.0;  // lane 0: sum of this warp's row cosines

  for (int64_t r = int64_t(blockIdx.x) * (kDriftThreads / 32) + warp; r < p.rows; r += warps_total) {
    const uint4* ra = p.a + r * p.vecs;
    const uint4* rb = p.b + r * p.vecs;
    float ab = 0.f, aa = 0.f, bb = 0.f;
    int v = lane;
    for (; v + 32 * (kDriftUnroll - 1) < p.vecs; v += 32 * kDriftUnroll) {
      uint4 x[kDriftUnroll], y[kDriftUnroll];
#pragma unroll
      for (int u = 0; u < kDriftUnroll; ++u) {
        x[u] = __ldcs(ra + v + 32 * u);
        y[u] = __ldcs(rb + v + 32 * u);
      }
#pragma unroll
      for (int u = 0; u < kDriftUnroll; ++u) accum(x[u], y[u], ab, aa, bb, T());
    }
    for (; v < p.vecs; v += 32) accum(__ldcs(ra + v), __ldcs(rb + v), ab, aa, bb, T());
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      ab += __shfl_xor_sync(0xffffffffu, ab, o);
      aa += __shfl_xor_sync(0xffffffffu, aa, o);
      bb += __shfl_xor_sync(0xffffffffu, bb, o);
    }
    if (lane == 0) {
      const float c = ab / (fmaxf(sqrtf(aa), kNormEps) * fmaxf(sqrtf(bb), kNormEps));
      if (p.row_cos) p.row_cos[r] = c;
      my_sum += double(c);
    }
  }

  if (lane == 0) warp_sum[warp] = my_sum;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int w = 0; w < kDriftThreads / 32; ++w) s += warp_sum[w];
    p.partial[blockIdx.x] = s;
    __threadfence();
    is_last = atomicAdd(p.done, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!is_last || warp != 0) return;
  // Last block: fixed-order sum of every block's partial.
  __threadfence();
  double s = 0.0;
  for (int i = lane; i < int(gridDim.x); i += 32) s += __ldcg(p.partial + i);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) {
    *p.drift = 1.0 - s / double(p.rows);
    *p.done = 0;  // ready for the next call on this workspace
  }
}

}  // namespace

int drift_grid(int64_t rows) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int per_sm = 0;  // resident blocks per SM, so that the grid is one full wave
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, drift_kernel<__nv_bfloat16>, kDriftThreads, 0) !=
          cudaSuccess || per_sm < 1)
    per_sm = 1;
  const int64_t want = (rows + kDriftThreads / 32 - 1) / (kDriftThreads / 32);
  int64_t g = int64_t(sms) * per_sm;
  if (g > want) g = want;
  if (g > kDriftMaxBlocks) g = kDriftMaxBlocks;
  return int(g < 1 ? 1 : g);
}

cudaError_t launch_drift(int64_t rows, int hidden, int dtype, const void* a, const void* b, float* row_cos,
                         double* drift, void* ws, cudaStream_t st) {
  DriftArgs p;
  p.a = static_cast<const uint4*>(a);
  p.b = static_cast<const uint4*>(b);
  p.row_cos = row_cos;
  p.done = static_cast<unsigned int*>(ws);
  p.partial = reinterpret_cast<double*>(static_cast<char*>(ws) + 256);
  p.drift = drift;
  p.rows = rows;
  p.vecs = dtype == TSA_BF16 ? hidden / 8 : hidden / 4;
  cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(unsigned int), st);
  if (e != cudaSuccess) return e;
  const int grid = drift_grid(rows);
  if (dtype == TSA_BF16)
    drift_kernel<__nv_bfloat16><<<grid, kDriftThreads, 0, st>>>(p);
  else
    drift_kernel<float><<<grid, kDriftThreads, 0, st>>>(p);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace tsa
