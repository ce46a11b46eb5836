// Top-K token selection per KV head: radix select + stable compaction.
//
// "Token Sparse Attention Long Context" (skill page), Step 1 select_top_k,
// with per-head budgets ("Token Sparse Attention: Efficient Long-Context
// Inference with Interleaved Token Selection", Figure 3: a token subset per
// head).  For each (b, g) with K kept tokens the kernel finds the exact
// 32-bit key T of the K-th largest score, keeps every score above T and the
// first (in index order) of those equal to T, and writes
//   perm[0:K]  = kept indices ascending,   perm[K:L] = dropped indices ascending.
//
// One thread-block cluster of kClusterCtas CTAs per (b, g); CTA `rank` owns a
// contiguous index slice.  Four 8-bit radix passes build per-CTA shared-memory
// histograms that every CTA sums over the cluster through distributed shared
// memory; each CTA then derives the same digit.  Compaction: the kept position
// of index i is  #(keys > T before i) + min(#(keys == T before i), ties_left),
// a block-wide scan per chunk plus the slice offsets exchanged over the cluster.
//
// Coverage mode (budgets from a token coverage tau, "Token Sparse Attention:
// Efficient Long-Context Inference with Interleaved Token Selection", dynamic
// token coverage, Figures 1 and 5): each score s carries the integer mass
// floor(clamp(s, 0, 256) * 2^S); the head's total M is summed over the
// cluster, the target is T = M - floor(double(M) * tau), and K is the fewest
// top-ranked tokens whose mass reaches T.  The four radix passes then build
// mass histograms (u64) beside the count histograms and descend to the digit
// where the mass from the top crosses the remaining target; at the end the
// key of the K-th token is known, with the count and mass of every key above
// it, and  K = above + ceil(remaining target / mass of that key).  Integer
// sums make K independent of the summation order.
#include <cooperative_groups.h>

#include "device_common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace tsa {
namespace {

constexpr int kClusterCtas = 8;
constexpr int kThreads = 1024;
constexpr int kPerThread = 8;
constexpr int kChunk = kThreads * kPerThread;
// A CTA's slice of sortable keys is staged in shared memory once when it holds
// at most this many (160 KB): every radix pass, the counts and the compaction
// then read shared memory instead of the scores in L2.
constexpr int kMaxStagedKeys = 40960;

struct SelectArgs {
  int staged;         // 1: the slice's keys are in dynamic shared memory
  const float* scores;
  int32_t* perm;
  uint32_t* status;
  int L, Hkv;
  int coverage;       // 1: K from tau (below), 0: K from kept
  double tau;
  float mass_scale;   // 2^S
  int32_t* k_out;     // [B * Hkv] chosen K (coverage mode), or null
  Budgets kept;
};

__device__ __forceinline__ uint64_t token_mass(float s, float mass_scale) {
  // fmaxf drops NaN; scaling by a power of two is exact, so v = s * 2^S is the
  // exact real value, and floor(v) is its significand shifted by its exponent
  // (integer bit operations; a float-to-64-bit conversion is much slower).
  const float v = fminf(fmaxf(s, 0.f), 256.f) * mass_scale;
  const uint32_t bits = __float_as_uint(v);
  const int k = (int)(bits >> 23) - 150;  // v = (1.f23 significand as integer) * 2^k for normal v
  if ((bits >> 23) == 0u || k <= -24) return 0u;  // zero, subnormal or below 1: floor is 0
  const uint64_t sig = (bits & 0x7FFFFFu) | 0x800000u;
  return k >= 0 ? sig << k : sig >> -k;
}

__device__ __forceinline__ void hist_add(uint32_t* h, bool match, uint32_t dg) {
  if (match) atomicAdd(&h[dg], 1u);
}

__device__ __forceinline__ float key_to_float(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// Inclusive scan over the 256 digit threads (tid < 256) of a u64 and a u32;
// named barrier 1 over those 256 threads.
__device__ __forceinline__ void digit_scan2(uint64_t m, uint32_t c, uint64_t* wm, uint32_t* wc, uint64_t& sm,
                                            uint32_t& sc) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  uint64_t xm = m;
  uint32_t xc = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint64_t ym = __shfl_up_sync(0xffffffffu, xm, o);
    const uint32_t yc = __shfl_up_sync(0xffffffffu, xc, o);
    if (lane >= o) {
      xm += ym;
      xc += yc;
    }
  }
  if (lane == 31) {
    wm[wid] = xm;
    wc[wid] = xc;
  }
  asm volatile("bar.sync 1, 256;" ::: "memory");
  uint64_t om = 0u;
  uint32_t oc = 0u;
  for (int w = 0; w < wid; ++w) {
    om += wm[w];
    oc += wc[w];
  }
  sm = om + xm;
  sc = oc + xc;
}

// Exclusive block scan of one u32 per thread (all kThreads threads call it).
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* warp_sums, uint32_t& total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[wid] = x;
  __syncthreads();
  if (wid == 0) {
    uint32_t w = warp_sums[lane];  // kThreads / 32 == 32 warps
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_sums[lane] = w;
  }
  __syncthreads();
  const uint32_t before = (wid > 0 ? warp_sums[wid - 1] : 0u) + x - v;
  total = warp_sums[31];
  __syncthreads();
  return before;
}

__global__ void __cluster_dims__(kClusterCtas, 1, 1) __launch_bounds__(kThreads, 1)
    select_radix(SelectArgs a) {
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int g = blockIdx.y, b = blockIdx.z;
  const int grp = b * a.Hkv + g;
  const int L = a.L;
  int K = a.kept.kept[grp];
  const float* sc = a.scores + (size_t)grp * L;
  int32_t* pm = a.perm + (size_t)grp * L;
  const int per = (L + kClusterCtas - 1) / kClusterCtas;
  const int lo = min(L, rank * per);
  const int hi = min(L, lo + per);
  const int tid = threadIdx.x;

  extern __shared__ uint32_t skeys[];  // [hi - lo] order keys when a.staged
  if (a.staged) {
    for (int i = lo + tid; i < hi; i += kThreads) skeys[i - lo] = order_key(sc[i]);
    __syncthreads();
  }
  auto key_at = [&](int i) -> uint32_t { return a.staged ? skeys[i - lo] : order_key(sc[i]); };
  __shared__ uint32_t hist[2][256];
  __shared__ uint32_t warp_sums[32];
  __shared__ uint32_t dig_warp[8];
  __shared__ uint32_t sh_digit, sh_above;
  __shared__ uint32_t cnt[2];  // this slice's (#key > T, #key == T)
  // Coverage mode: mass per digit as 32-bit halves (64-bit shared atomics are
  // much slower): lo wraps modulo 2^32 and every wrap adds one to hi.
  __shared__ uint32_t histml[2][256], histmh[2][256];
  __shared__ uint64_t dig_warp_m[8];
  __shared__ uint64_t sh_mass, sh_mabove;

  uint32_t prefix = 0u, mask = 0u, krem = 0u;
  bool have_T = false;  // coverage mode found the K-th key by mass
  if (a.coverage) {
    if (tid == 0) sh_mass = 0u;
    __syncthreads();
    uint64_t my = 0u;
    for (int i = lo + tid; i < hi; i += kThreads) my += token_mass(key_to_float(key_at(i)), a.mass_scale);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) my += __shfl_xor_sync(0xffffffffu, my, o);
    if ((tid & 31) == 0 && my) atomicAdd(reinterpret_cast<unsigned long long*>(&sh_mass), (unsigned long long)my);
    cluster.sync();
    uint64_t M = 0u;
    for (int r = 0; r < kClusterCtas; ++r) M += *cluster.map_shared_rank(&sh_mass, r);
    const uint64_t D = (uint64_t)floor(__ull2double_rn(M) * a.tau);
    uint64_t trem = D >= M ? 0u : M - D;
    if (trem == 0u) {
      K = 1;  // nothing has to be covered: keep the single top token
    } else {
      uint32_t above = 0u;
      for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        uint32_t* hc = hist[pass & 1];
        uint32_t* hml = histml[pass & 1];
        uint32_t* hmh = histmh[pass & 1];
        if (tid < 256) {
          hc[tid] = 0u;
          hml[tid] = 0u;
          hmh[tid] = 0u;
        }
        __syncthreads();
        for (int i = lo + tid; i < hi; i += kThreads) {
          const uint32_t key = key_at(i);
          const bool match = (key & mask) == prefix;
          const uint32_t dg = (key >> shift) & 255u;
          hist_add(hc, match, dg);
          if (match) {
            const uint64_t m = token_mass(key_to_float(key), a.mass_scale);
            const uint32_t mlo = (uint32_t)m;
            uint32_t mhi = (uint32_t)(m >> 32);
            if (mlo) {
              const uint32_t old = atomicAdd(&hml[dg], mlo);
              mhi += (old + mlo < old);  // the low word wrapped
            }
            if (mhi) atomicAdd(&hmh[dg], mhi);
          }
        }
        cluster.sync();
        if (tid < 256) {
          // Thread t stands for digit 255 - t: inclusive scans give the count
          // and mass of matching keys whose digit is >= 255 - t.
          uint32_t totc = 0u;
          uint64_t totm = 0u;
          for (int r = 0; r < kClusterCtas; ++r) {
            totc += cluster.map_shared_rank(hc, r)[255 - tid];
            totm += ((uint64_t)cluster.map_shared_rank(hmh, r)[255 - tid] << 32) +
                    cluster.map_shared_rank(hml, r)[255 - tid];
          }
          uint64_t Sm;
          uint32_t Sc;
          digit_scan2(totm, totc, dig_warp_m, dig_warp, Sm, Sc);
          if (Sm >= trem && Sm - totm < trem) {
            sh_digit = 255u - (uint32_t)tid;
            sh_mabove = Sm - totm;
            sh_above = Sc - totc;
          }
        }
        __syncthreads();
        prefix |= sh_digit << shift;
        mask |= 0xFFu << shift;
        trem -= sh_mabove;
        above += sh_above;
      }
      // Every key equal to the K-th carries the same mass, which is > 0
      // because that key's digit raised the running mass to the target.
      const uint64_t mk = token_mass(key_to_float(prefix), a.mass_scale);
      uint64_t need = 1u;
      if (mk == 0u) {
        record_status(a.status, TSA_ERR_DEVICE_BOUNDS);
      } else {
        need = (trem + mk - 1u) / mk;
      }
      K = (int)min((uint64_t)L, (uint64_t)above + need);
      krem = (uint32_t)K - above;
      have_T = true;
    }
    if (a.k_out && rank == 0 && tid == 0) a.k_out[grp] = K;
  }

  const bool partial = K < L;
  if (!have_T) krem = (uint32_t)K;
  if (partial && !have_T) {
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      uint32_t* h = hist[pass & 1];
      if (tid < 256) h[tid] = 0u;
      __syncthreads();
      for (int i = lo + tid; i < hi; i += kThreads) {
        const uint32_t key = key_at(i);
        hist_add(h, (key & mask) == prefix, (key >> shift) & 255u);
      }
      cluster.sync();
      if (tid < 256) {
        // Thread t stands for digit 255 - t, so an inclusive scan over t gives
        // the number of matching keys whose digit is >= 255 - t.
        uint32_t tot = 0u;
        for (int r = 0; r < kClusterCtas; ++r) tot += cluster.map_shared_rank(h, r)[255 - tid];
        const int lane = tid & 31, wid = tid >> 5;
        uint32_t x = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
          if (lane >= o) x += y;
        }
        if (lane == 31) dig_warp[wid] = x;
        asm volatile("bar.sync 1, 256;" ::: "memory");
        uint32_t off = 0u;
        for (int w = 0; w < wid; ++w) off += dig_warp[w];
        const uint32_t S = off + x;
        if (S >= krem && S - tot < krem) {
          sh_digit = 255u - (uint32_t)tid;
          sh_above = S - tot;
        }
      }
      __syncthreads();
      prefix |= sh_digit << shift;
      mask |= 0xFFu << shift;
      krem -= sh_above;
    }
  }
  const uint32_t T = prefix;

  // Per-slice counts, exchanged over the cluster.
  if (tid < 2) cnt[tid] = 0u;
  __syncthreads();
  if (partial) {
    uint32_t gt = 0u, eq = 0u;
    for (int i = lo + tid; i < hi; i += kThreads) {
      const uint32_t key = key_at(i);
      gt += key > T;
      eq += key == T;
    }
    if (gt) atomicAdd(&cnt[0], gt);
    if (eq) atomicAdd(&cnt[1], eq);
  }
  cluster.sync();
  uint32_t gt_before = 0u, eq_before = 0u;
  if (partial) {
    for (int r = 0; r < rank; ++r) {
      const uint32_t* rc = cluster.map_shared_rank(cnt, r);
      gt_before += rc[0];
      eq_before += rc[1];
    }
  } else {
    gt_before = (uint32_t)lo;  // everything is kept: index i lands at i
  }

  // A chunk's kept indices land in one contiguous range of perm[0:K] and its
  // dropped ones in one contiguous range of perm[K:L]: each index goes to its
  // place in a shared-memory copy of the chunk's two ranges (kept first), and
  // the ranges are then written out with consecutive threads on consecutive
  // addresses.
  __shared__ int32_t stage[kChunk];
  for (int base = lo; base < hi; base += kChunk) {
    const int n = min(kChunk, hi - base);
    const int i0 = base + tid * kPerThread;
    uint32_t isgt[kPerThread], iseq[kPerThread];
    uint32_t ngt = 0u, neq = 0u;
#pragma unroll
    for (int e = 0; e < kPerThread; ++e) {
      const int i = i0 + e;
      isgt[e] = 0u;
      iseq[e] = 0u;
      if (i < hi) {
        if (partial) {
          const uint32_t key = key_at(i);
          isgt[e] = key > T;
          iseq[e] = key == T;
        } else {
          isgt[e] = 1u;
        }
      }
      ngt += isgt[e];
      neq += iseq[e];
    }
    uint32_t total;
    const uint32_t ex = block_exclusive_scan((neq << 16) | ngt, warp_sums, total);
    const uint32_t tg = total & 0xFFFFu, te = total >> 16;
    const uint32_t kb0 = gt_before + min(eq_before, krem);            // kept indices before the chunk
    const uint32_t nk = gt_before + tg + min(eq_before + te, krem) - kb0;  // kept indices in the chunk
    uint32_t gb = gt_before + (ex & 0xFFFFu);
    uint32_t eb = eq_before + (ex >> 16);
#pragma unroll
    for (int e = 0; e < kPerThread; ++e) {
      const int i = i0 + e;
      if (i < hi) {
        const uint32_t S = gb + min(eb, krem);  // kept indices before i
        const bool keep = isgt[e] || (iseq[e] && eb < krem);
        // kept: S - kb0 in [0, nk); dropped: i - S dropped before i, minus those before the chunk
        const uint32_t local = keep ? S - kb0 : nk + ((uint32_t)i - S) - ((uint32_t)base - kb0);
        if (local < (uint32_t)n) {
          stage[local] = i;
        } else {
          record_status(a.status, TSA_ERR_DEVICE_BOUNDS);
        }
        gb += isgt[e];
        eb += iseq[e];
      }
    }
    __syncthreads();
    for (int x = tid; x < n; x += kThreads) {
      const uint32_t dst = (uint32_t)x < nk ? kb0 + (uint32_t)x : (uint32_t)K + ((uint32_t)base - kb0) + ((uint32_t)x - nk);
      if (dst < (uint32_t)L) {
        pm[dst] = stage[x];
      } else {
        record_status(a.status, TSA_ERR_DEVICE_BOUNDS);
      }
    }
    __syncthreads();  // the stage is rewritten by the next chunk
    gt_before += tg;
    eq_before += te;
  }
  cluster.sync();  // no CTA leaves while a peer may still read its shared memory
}

cudaError_t launch_radix(const Dims& d, SelectArgs& a, cudaStream_t st) {
  const int per = (d.L + kClusterCtas - 1) / kClusterCtas;
  a.staged = per <= kMaxStagedKeys ? 1 : 0;
  const int smem = a.staged ? per * (int)sizeof(uint32_t) : 0;
  cudaError_t e = cudaFuncSetAttribute(select_radix, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kMaxStagedKeys * (int)sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  const dim3 grid(kClusterCtas, d.Hkv, d.B);
  select_radix<<<grid, kThreads, smem, st>>>(a);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_select(const Dims& d, const float* scores, const Budgets& kept, int32_t* perm,
                          uint32_t* status, cudaStream_t st) {
  SelectArgs a;
  a.scores = scores;
  a.perm = perm;
  a.status = status;
  a.L = d.L;
  a.Hkv = d.Hkv;
  a.coverage = 0;
  a.tau = 0.0;
  a.mass_scale = 0.f;
  a.k_out = nullptr;
  a.kept = kept;
  return launch_radix(d, a, st);
}

cudaError_t launch_select_coverage(const Dims& d, const float* scores, double tau, int32_t* perm, int32_t* k_out,
                                   uint32_t* status, cudaStream_t st) {
  SelectArgs a;
  a.scores = scores;
  a.perm = perm;
  a.status = status;
  a.L = d.L;
  a.Hkv = d.Hkv;
  a.coverage = 1;
  a.tau = tau;
  int lg = 0;  // ceil(log2 L)
  while ((1ll << lg) < (long long)d.L) ++lg;
  a.mass_scale = ldexpf(1.f, 55 - lg);
  a.k_out = k_out;
  for (int i = 0; i < kMaxGroups; ++i) a.kept.kept[i] = 0;
  return launch_radix(d, a, st);
}

}  // namespace tsa
