// Token scoring on CUDA cores (exact fp32 arithmetic; any input dtype).
//
// Computes the per-KV-head importance of "Token Sparse Attention Long
// Context" (skill page), Step 1, method "entropy": softmax over keys of the
// scaled query-key logits, summed over queries -- restricted to an
// observation window of the last W queries, causal, and summed over the G
// query heads of a KV group.
//
// Two passes over the keys of each KV group, split into key ranges:
//   pass 1: per window row r, the running max m_r and normaliser
//           Z_r = sum_j exp(l_rj - m_r) over the split's keys  -> partials
//   pass 2: combine the partials into c_r = m_r + log Z_r, recompute the
//           logits and write score[j] = sum_r exp(l_rj - c_r).
// Window rows: r = hh*W + w is query head g*G+hh at position L-W+w.
#include <math.h>

#include "device_common.cuh"
#include "internal.h"

namespace tsa {
namespace {

constexpr int KT = kScoreKeyTile;  // keys per tile
constexpr int KS = KT + 4;         // row stride of the transposed key tile (floats)

struct ScoreArgs {
  const void* q;
  const void* k;
  float* scores;
  float* part;
  uint32_t* status;
  int Hq, Hkv, L, G, W, M, Mp, nsplit;
  float scale;
};

__device__ __forceinline__ void split_range(int s, int nsplit, int L, int& j0, int& j1) {
  const int ntiles = (L + KT - 1) / KT;
  const int t0 = (int)((long long)ntiles * s / nsplit);
  const int t1 = (int)((long long)ntiles * (s + 1) / nsplit);
  j0 = t0 * KT;
  j1 = min(L, t1 * KT);
}

// Window queries of group g, transposed: Qs[d * qstride + r].  Rows r >= M are 0.
template <typename T, int D>
__device__ void load_window(const ScoreArgs& a, int b, int g, float* Qs, int qstride) {
  const T* q = static_cast<const T*>(a.q);
  for (int idx = threadIdx.x; idx < a.Mp * D; idx += blockDim.x) {
    const int r = idx / D, d = idx - r * D;
    float val = 0.f;
    if (r < a.M) {
      const int hh = r / a.W, w = r - hh * a.W;
      const size_t row = (size_t)(b * a.Hq + g * a.G + hh) * a.L + (a.L - a.W + w);
      val = to_f32(q[row * D + d]);
    }
    Qs[d * qstride + r] = val;
  }
}

// Keys [jt, jt+KT) of one KV head, transposed: Ks[d * KS + n].  Keys >= j1 are 0.
template <typename T, int D>
__device__ void load_key_tile(const T* kp, int jt, int j1, float* Ks) {
  for (int idx = threadIdx.x; idx < KT * D; idx += blockDim.x) {
    const int n = idx / D, d = idx - n * D;
    const int j = jt + n;
    Ks[d * KS + n] = (j < j1) ? to_f32(kp[(size_t)j * D + d]) : 0.f;
  }
}

// 4x4 micro-tile of dot products: rows rb+ty*4+i, keys tx*4+j.
template <int D>
__device__ __forceinline__ void tile_dots(const float* Qs, int qstride, int rb, const float* Ks, int ty,
                                          int tx, float acc[4][4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 8
  for (int d = 0; d < D; ++d) {
    const float4 qa = *reinterpret_cast<const float4*>(&Qs[d * qstride + rb + ty * 4]);
    const float4 kb = *reinterpret_cast<const float4*>(&Ks[d * KS + tx * 4]);
    const float qv[4] = {qa.x, qa.y, qa.z, qa.w};
    const float kv[4] = {kb.x, kb.y, kb.z, kb.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(qv[i], kv[j], acc[i][j]);
  }
}

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

template <typename T, int D>
__global__ void __launch_bounds__(256) score_pass1(ScoreArgs a) {
  extern __shared__ __align__(16) float sm[];
  const int qstride = a.Mp + 4;
  float* Qs = sm;
  float* Ks = Qs + D * qstride;
  float* rm = Ks + D * KS;
  float* rz = rm + a.Mp;
  const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;

  load_window<T, D>(a, b, g, Qs, qstride);
  for (int r = tid; r < a.Mp; r += blockDim.x) {
    rm[r] = -INFINITY;
    rz[r] = 0.f;
  }
  int j0, j1;
  split_range(s, a.nsplit, a.L, j0, j1);
  const T* kp = static_cast<const T*>(a.k) + (size_t)(b * a.Hkv + g) * a.L * D;

  for (int jt = j0; jt < j1; jt += KT) {
    __syncthreads();
    load_key_tile<T, D>(kp, jt, j1, Ks);
    __syncthreads();
    for (int rb = 0; rb < a.Mp; rb += 64) {
      float acc[4][4];
      tile_dots<D>(Qs, qstride, rb, Ks, ty, tx, acc);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = rb + ty * 4 + i;
        const int pos = a.L - a.W + (r % a.W);
        float lv[4];
        float lmax = -INFINITY;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int jj = jt + tx * 4 + j;
          const bool ok = (r < a.M) && (jj < j1) && (jj <= pos);
          lv[j] = ok ? acc[i][j] * a.scale : -INFINITY;
          lmax = fmaxf(lmax, lv[j]);
        }
        lmax = max16(lmax);
        float ls = 0.f;
        if (lmax > -INFINITY) {
#pragma unroll
          for (int j = 0; j < 4; ++j) ls += expf(lv[j] - lmax);
        }
        ls = sum16(ls);
        if (tx == 0 && lmax > -INFINITY) {
          const float mo = rm[r], zo = rz[r];
          const float mn = fmaxf(mo, lmax);
          rz[r] = zo * expf(mo - mn) + ls * expf(lmax - mn);
          rm[r] = mn;
        }
      }
    }
  }
  __syncthreads();
  float* pp = a.part + ((size_t)(b * a.Hkv + g) * a.nsplit + s) * a.Mp * 2;
  for (int r = tid; r < a.Mp; r += blockDim.x) {
    pp[r] = rm[r];
    pp[a.Mp + r] = rz[r];
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(256) score_pass2(ScoreArgs a) {
  extern __shared__ __align__(16) float sm[];
  const int qstride = a.Mp + 4;
  float* Qs = sm;
  float* Ks = Qs + D * qstride;
  float* crow = Ks + D * KS;
  float* red = crow + a.Mp;  // [16][KT]
  const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;

  load_window<T, D>(a, b, g, Qs, qstride);
  const float* base = a.part + (size_t)(b * a.Hkv + g) * a.nsplit * a.Mp * 2;
  for (int r = tid; r < a.Mp; r += blockDim.x) {
    float mx = -INFINITY;
    for (int t = 0; t < a.nsplit; ++t) mx = fmaxf(mx, base[(size_t)t * a.Mp * 2 + r]);
    float z = 0.f;
    if (mx > -INFINITY) {
      for (int t = 0; t < a.nsplit; ++t) {
        const float mt = base[(size_t)t * a.Mp * 2 + r];
        if (mt > -INFINITY) z += base[(size_t)t * a.Mp * 2 + a.Mp + r] * expf(mt - mx);
      }
    }
    crow[r] = (r < a.M && mx > -INFINITY) ? mx + logf(z) : INFINITY;
  }
  int j0, j1;
  split_range(s, a.nsplit, a.L, j0, j1);
  const T* kp = static_cast<const T*>(a.k) + (size_t)(b * a.Hkv + g) * a.L * D;
  float* out = a.scores + (size_t)(b * a.Hkv + g) * a.L;

  for (int jt = j0; jt < j1; jt += KT) {
    __syncthreads();
    load_key_tile<T, D>(kp, jt, j1, Ks);
    __syncthreads();
    float col[4] = {0.f, 0.f, 0.f, 0.f};
    for (int rb = 0; rb < a.Mp; rb += 64) {
      float acc[4][4];
      tile_dots<D>(Qs, qstride, rb, Ks, ty, tx, acc);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = rb + ty * 4 + i;
        const int pos = a.L - a.W + (r % a.W);
        const float c = crow[r];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int jj = jt + tx * 4 + j;
          const bool ok = (r < a.M) && (jj < j1) && (jj <= pos);
          col[j] += ok ? expf(acc[i][j] * a.scale - c) : 0.f;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) red[ty * KT + tx * 4 + j] = col[j];
    __syncthreads();
    if (tid < KT) {
      float sum = 0.f;
#pragma unroll
      for (int t = 0; t < 16; ++t) sum += red[t * KT + tid];
      if (jt + tid < j1) out[jt + tid] = sum;
    }
  }
}

template <typename T, int D>
cudaError_t launch_typed(const Dims& d, const ScoreArgs& a, cudaStream_t st) {
  const size_t qs = (size_t)D * (a.Mp + 4) * sizeof(float);
  const size_t ks = (size_t)D * KS * sizeof(float);
  const size_t sm1 = qs + ks + 2 * (size_t)a.Mp * sizeof(float);
  const size_t sm2 = qs + ks + (size_t)a.Mp * sizeof(float) + 16 * KT * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(score_pass1<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(score_pass2<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2);
  if (e != cudaSuccess) return e;
  const dim3 grid(a.nsplit, d.Hkv, d.B);
  score_pass1<T, D><<<grid, 256, sm1, st>>>(a);
  count_launches(1);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  score_pass2<T, D><<<grid, 256, sm2, st>>>(a);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_score_simt(const Dims& d, const void* q, const void* k, int window, float* scores,
                              float* part, uint32_t* status, cudaStream_t st) {
  ScoreArgs a;
  a.q = q;
  a.k = k;
  a.scores = scores;
  a.part = part;
  a.status = status;
  a.Hq = d.Hq;
  a.Hkv = d.Hkv;
  a.L = d.L;
  a.G = d.G;
  a.W = window;
  a.M = d.G * window;
  a.Mp = window_rows_padded(d, window);
  a.nsplit = score_splits(d);
  a.scale = d.scale;
  if (d.dtype == TSA_F32) {
    return d.D == 64 ? launch_typed<float, 64>(d, a, st) : launch_typed<float, 128>(d, a, st);
  }
  return d.D == 64 ? launch_typed<__nv_bfloat16, 64>(d, a, st) : launch_typed<__nv_bfloat16, 128>(d, a, st);
}

}  // namespace tsa
