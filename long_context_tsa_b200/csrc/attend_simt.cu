// Compressed causal attention on CUDA cores (exact fp32 arithmetic) and the
// zero fill of dropped rows.
//
// "Token Sparse Attention Long Context" (skill page), Step 2 gather_tokens /
// scatter_attention_output and Step 3 SparseAttentionHead.forward;
// "Token Sparse Attention: Efficient Long-Context Inference with Interleaved
// Token Selection", Figure 3.  For query head h of KV group g with K kept
// tokens at ascending positions perm[0:K]:
//   out[perm[i]] = sum_{r<=i} softmax_r(scale * q[perm[i]] . k[perm[r]]) v[perm[r]]
// The causal mask on compacted indices equals the mask on original
// positions because perm[0:K] is strictly ascending.  Rows perm[K:L] are 0.
#include <math.h>

#include "device_common.cuh"
#include "internal.h"

namespace tsa {
namespace {

constexpr int BR = 64;      // query rows per CTA
constexpr int BC = 64;      // keys per tile
constexpr int TS = BC + 4;  // stride of transposed tiles
constexpr int kZeroRows = 128;

struct AttendArgs {
  const void* q;
  const void* k;
  const void* v;
  const int32_t* perm;
  void* out;
  uint32_t* status;
  int Hq, Hkv, L, G;
  float scale;
  int accumulate;  // 1: out[kept rows] += attention
  const uint8_t* bmask;  // [B*Hkv][nb][nb] block mask over compacted (query, key) 128-blocks, or null
  int nb;
  Budgets kept;
};

__device__ __forceinline__ float max16(float x) {
#pragma unroll
  for (int o = 1; o < 16; o <<= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float sum16(float x) {
#pragma unroll
  for (int o = 1; o < 16; o <<= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Original position of compacted index c, with a bounds check.
__device__ __forceinline__ int checked_pos(const int32_t* pm, int c, int L, uint32_t* status) {
  const int p = pm[c];
  if ((unsigned)p >= (unsigned)L) {
    record_status(status, TSA_ERR_DEVICE_BOUNDS);
    return 0;
  }
  return p;
}

template <typename T, int D>
__global__ void __launch_bounds__(256) attend_simt(AttendArgs a) {
  constexpr int VS = D + 4;
  constexpr int DC = D / 16;
  extern __shared__ __align__(16) float sm[];
  float* Qs = sm;             // [D][TS]  query rows, transposed
  float* Ks = Qs + D * TS;    // [D][TS]  key rows, transposed
  float* Vs = Ks + D * TS;    // [BC][VS] value rows
  float* Ps = Vs + BC * VS;   // [BR][TS] probabilities

  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int g = h / a.G, grp = b * a.Hkv + g;
  const int K = a.kept.kept[grp];
  const int r0 = qb * BR;
  if (r0 >= K) return;
  const int L = a.L;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int32_t* pm = a.perm + (size_t)grp * L;
  const T* qh = static_cast<const T*>(a.q) + (size_t)(b * a.Hq + h) * L * D;
  const T* kg = static_cast<const T*>(a.k) + (size_t)grp * L * D;
  const T* vg = static_cast<const T*>(a.v) + (size_t)grp * L * D;

  for (int idx = tid; idx < BR * D; idx += blockDim.x) {
    const int n = idx / D, d = idx - n * D;
    const int r = r0 + n;
    float val = 0.f;
    if (r < K) val = to_f32(qh[(size_t)checked_pos(pm, r, L, a.status) * D + d]);
    Qs[d * TS + n] = val;
  }

  float m_i[4], l_i[4], o[4][DC];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m_i[i] = -INFINITY;
    l_i[i] = 0.f;
#pragma unroll
    for (int c = 0; c < DC; ++c) o[i][c] = 0.f;
  }

  const int nkeys = min(K, r0 + BR);
  const uint8_t* bm = a.bmask ? a.bmask + ((size_t)grp * a.nb + r0 / 128) * a.nb : nullptr;  // this CTA's block row
  for (int c0 = 0; c0 < nkeys; c0 += BC) {
    if (bm != nullptr && bm[c0 / 128] == 0) continue;  // block disabled (uniform over the CTA)
    __syncthreads();
    for (int idx = tid; idx < BC * D; idx += blockDim.x) {
      const int n = idx / D, d = idx - n * D;
      const int c = c0 + n;
      float kv = 0.f, vv = 0.f;
      if (c < K) {
        const size_t p = (size_t)checked_pos(pm, c, L, a.status);
        kv = to_f32(kg[p * D + d]);
        vv = to_f32(vg[p * D + d]);
      }
      Ks[d * TS + n] = kv;
      Vs[n * VS + d] = vv;
    }
    __syncthreads();

    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 8
    for (int d = 0; d < D; ++d) {
      const float4 qa = *reinterpret_cast<const float4*>(&Qs[d * TS + ty * 4]);
      const float4 kb = *reinterpret_cast<const float4*>(&Ks[d * TS + tx * 4]);
      const float qv[4] = {qa.x, qa.y, qa.z, qa.w};
      const float kv[4] = {kb.x, kb.y, kb.z, kb.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(qv[i], kv[j], acc[i][j]);
    }

#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = r0 + ty * 4 + i;
      float sv[4];
      float mt = -INFINITY;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = c0 + tx * 4 + j;
        const bool ok = (r < K) && (c < K) && (c <= r);
        sv[j] = ok ? acc[i][j] * a.scale : -INFINITY;
        mt = fmaxf(mt, sv[j]);
      }
      mt = max16(mt);
      const float mn = fmaxf(m_i[i], mt);
      float ps = 0.f;
      float alpha = 1.f;
      if (mn > -INFINITY) {
        alpha = (m_i[i] > -INFINITY) ? expf(m_i[i] - mn) : 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          sv[j] = (sv[j] > -INFINITY) ? expf(sv[j] - mn) : 0.f;
          ps += sv[j];
        }
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) sv[j] = 0.f;
      }
      ps = sum16(ps);
      l_i[i] = l_i[i] * alpha + ps;
      m_i[i] = mn;
#pragma unroll
      for (int c = 0; c < DC; ++c) o[i][c] *= alpha;
      *reinterpret_cast<float4*>(&Ps[(ty * 4 + i) * TS + tx * 4]) = make_float4(sv[0], sv[1], sv[2], sv[3]);
    }
    __syncthreads();
#pragma unroll 4
    for (int c = 0; c < BC; ++c) {
      float vv[DC];
#pragma unroll
      for (int dc = 0; dc < DC; ++dc) vv[dc] = Vs[c * VS + tx + 16 * dc];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float p = Ps[(ty * 4 + i) * TS + c];
#pragma unroll
        for (int dc = 0; dc < DC; ++dc) o[i][dc] = fmaf(p, vv[dc], o[i][dc]);
      }
    }
  }

  T* oh = static_cast<T*>(a.out) + (size_t)(b * a.Hq + h) * L * D;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = r0 + ty * 4 + i;
    if (r < K) {
      const size_t p = (size_t)checked_pos(pm, r, L, a.status);
      const float inv = l_i[i] > 0.f ? 1.f / l_i[i] : 0.f;  // no visible key (block mask): zeros
#pragma unroll
      for (int dc = 0; dc < DC; ++dc) {
        T* dst = oh + p * D + tx + 16 * dc;
        const float val = o[i][dc] * inv;
        *dst = from_f32<T>(a.accumulate ? to_f32(*dst) + val : val);
      }
    }
  }
}

// +0 into every dropped row perm[K:L] of every query head.
template <typename T, int D>
__global__ void __launch_bounds__(256) zero_fill(AttendArgs a) {
  constexpr int CPR = D * (int)sizeof(T) / 16;  // 16-byte chunks per row
  const int h = blockIdx.y, b = blockIdx.z;
  const int g = h / a.G, grp = b * a.Hkv + g;
  const int K = a.kept.kept[grp];
  const int L = a.L;
  const int u0 = K + blockIdx.x * kZeroRows;
  if (u0 >= L) return;
  const int nrow = min(kZeroRows, L - u0);
  const int32_t* pm = a.perm + (size_t)grp * L;
  uint4* ob = reinterpret_cast<uint4*>(static_cast<T*>(a.out) + (size_t)(b * a.Hq + h) * L * D);
  for (int idx = threadIdx.x; idx < nrow * CPR; idx += blockDim.x) {
    const int r = idx / CPR, c = idx - r * CPR;
    const int p = pm[u0 + r];
    if ((unsigned)p >= (unsigned)L) {
      record_status(a.status, TSA_ERR_DEVICE_BOUNDS);
      continue;
    }
    ob[(size_t)p * CPR + c] = make_uint4(0u, 0u, 0u, 0u);
  }
}

AttendArgs make_args(const Dims& d, const void* q, const void* k, const void* v, const int32_t* perm,
                     const Budgets& kept, void* out, uint32_t* status) {
  AttendArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.perm = perm;
  a.out = out;
  a.status = status;
  a.Hq = d.Hq;
  a.Hkv = d.Hkv;
  a.L = d.L;
  a.G = d.G;
  a.scale = d.scale;
  a.accumulate = 0;
  a.bmask = nullptr;
  a.nb = (d.L + 127) / 128;
  a.kept = kept;
  return a;
}

template <typename T, int D>
cudaError_t launch_attend_typed(const Dims& d, const AttendArgs& a, int maxK, cudaStream_t st) {
  const size_t sm = ((size_t)2 * D * TS + (size_t)BC * (D + 4) + (size_t)BR * TS) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(attend_simt<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  const dim3 grid((maxK + BR - 1) / BR, d.Hq, d.B);
  attend_simt<T, D><<<grid, 256, sm, st>>>(a);
  count_launches(1);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_zero_typed(const Dims& d, const AttendArgs& a, int minK, cudaStream_t st) {
  const int rows = d.L - minK;
  if (rows <= 0) return cudaSuccess;
  const dim3 grid((rows + kZeroRows - 1) / kZeroRows, d.Hq, d.B);
  zero_fill<T, D><<<grid, 256, 0, st>>>(a);
  count_launches(1);
  return cudaGetLastError();
}

void kept_range(const Dims& d, const Budgets& kept, int& mn, int& mx) {
  mn = d.L;
  mx = 0;
  for (int i = 0; i < d.B * d.Hkv; ++i) {
    mn = kept.kept[i] < mn ? kept.kept[i] : mn;
    mx = kept.kept[i] > mx ? kept.kept[i] : mx;
  }
}

}  // namespace

cudaError_t launch_attend_simt(const Dims& d, const void* q, const void* k, const void* v,
                               const int32_t* perm, const Budgets& kept, void* out, uint32_t* status,
                               bool accumulate, const uint8_t* block_mask, cudaStream_t st) {
  AttendArgs a = make_args(d, q, k, v, perm, kept, out, status);
  a.accumulate = accumulate ? 1 : 0;
  a.bmask = block_mask;
  int mn, mx;
  kept_range(d, kept, mn, mx);
  if (d.dtype == TSA_F32)
    return d.D == 64 ? launch_attend_typed<float, 64>(d, a, mx, st) : launch_attend_typed<float, 128>(d, a, mx, st);
  return d.D == 64 ? launch_attend_typed<__nv_bfloat16, 64>(d, a, mx, st)
                   : launch_attend_typed<__nv_bfloat16, 128>(d, a, mx, st);
}

cudaError_t launch_zero_fill(const Dims& d, const int32_t* perm, const Budgets& kept, void* out,
                             uint32_t* status, cudaStream_t st) {
  const AttendArgs a = make_args(d, nullptr, nullptr, nullptr, perm, kept, out, status);
  int mn, mx;
  kept_range(d, kept, mn, mx);
  if (d.dtype == TSA_F32)
    return d.D == 64 ? launch_zero_typed<float, 64>(d, a, mn, st) : launch_zero_typed<float, 128>(d, a, mn, st);
  return d.D == 64 ? launch_zero_typed<__nv_bfloat16, 64>(d, a, mn, st)
                   : launch_zero_typed<__nv_bfloat16, 128>(d, a, mn, st);
}

}  // namespace tsa
