// Token scoring on the tcgen05 tensor cores (bf16 in, fp32 accumulate).
//
// "Token Sparse Attention Long Context" (skill page), Step 1, method
// "entropy": per-key importance = softmax over keys of the scaled query-key
// logits, summed over queries -- here over an observation window of the last
// W queries of the G query heads of each KV group, causally masked.
//
// Window rows r = hh*W + w (query head g*G+hh, position L-W+w), padded to
// Mp = 128 or 256 rows.  Keys stream in tiles of 128 by plain tiled TMA; a
// CTA owns a contiguous range of key tiles ("split") of one (batch, KV group).
//   pass 1: S = Qw K^T (window rows on TMEM lanes); per row, over the split's
//           keys, m = max of x = l*log2(e) and Z = sum 2^(x - m)   -> partials
//   pass 2: S^T = K Qw^T (keys on TMEM lanes, window rows as columns); with
//           c_r = m_r + log2 Z_r combined over all splits,
//           score[j] = sum_r 2^(x_rj - c_r)  -- one thread per key, no
//           cross-thread reduction.
// Warp roles (576 threads): warps 0-15 read TMEM (four warpgroups), warp 16
// loads (TMA), warp 17 issues tcgen05.mma.  Two TMEM buffers alternate by step;
// in pass 1 each warpgroup pair reads every other step (whole rows), in pass 2
// each warpgroup pair reads every other key tile (one column half each), so on
// every SM sub-partition two reader warps load from TMEM while the other two
// compute.  TMEM loads run one 32-column chunk ahead.  Pass 1 merges the
// partial (m, Z) of the two step parities of each row; pass 2 adds the two
// halves of each key's sum into the scores, which pass 1 zeroed.  Bounded
// waits throughout.
#include <cuda.h>
#include <math.h>

#include "device_common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

#include "tma_maps.h"

namespace tsa {
namespace {

using namespace tc;

// ---- 2^t on the FMA pipe, for part of the column-sum exponentials ----
//
// The exponential unit (16 results per clock per SM) bounds both passes, so one
// pair in three of the exponentials is computed with FMA-pipe arithmetic
// instead (measured 6 % faster for pass 2).  Written from the math:
// t = j + f with j = floor(t) and f in [0, 1); 2^f by a degree-4 polynomial
// p(f) = 1 + f (c1 + f (c2 + f (c3 + f c4))) whose coefficients were fitted to
// 2^f on [0, 1) by iteratively reweighted least squares on the relative error
// (max relative error 3.0e-6 when evaluated in float32); 2^j by adding j to the
// exponent field.  floor(t) comes from one add of 1.5 * 2^23 rounded toward
// -infinity, whose low mantissa bits then hold j (the bits of 1.5 * 2^23 shift
// out of the exponent field).  t is clamped to >= -126 so the result stays a
// normal float: values below 2^-126 come out as 2^-126 instead of smaller, an
// absolute error below 1.2e-38 per term.  Valid for t < 128 (pass 2 has t <= 0;
// pass 1 clamps t to 127 first).
__device__ __forceinline__ uint64_t f2_add_rm(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rm.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ void ex2_fma_pair(float t0, float t1, float& p0, float& p1) {
  const uint64_t magic = 0x4B4000004B400000ull;  // (1.5 * 2^23, 1.5 * 2^23)
  const uint64_t tt = f2_pack(fmaxf(t0, -126.f), fmaxf(t1, -126.f));
  const uint64_t y = f2_add_rm(tt, magic);
  const uint64_t fr = f2_sub(tt, f2_sub(y, magic));
  uint64_t q = f2_fma(f2_pack(0.013426822610199451f, 0.013426822610199451f), fr,
                      f2_pack(0.052243269979953766f, 0.052243269979953766f));
  q = f2_fma(q, fr, f2_pack(0.2412789911031723f, 0.2412789911031723f));
  q = f2_fma(q, fr, f2_pack(0.6930451989173889f, 0.6930451989173889f));
  q = f2_fma(q, fr, f2_pack(1.f, 1.f));
  float q0, q1, y0, y1;
  f2_unpack(q, q0, q1);
  f2_unpack(y, y0, y1);
  p0 = __uint_as_float(__float_as_uint(q0) + (__float_as_uint(y0) << 23));
  p1 = __uint_as_float(__float_as_uint(q1) + (__float_as_uint(y1) << 23));
}

__global__ void debug_exp2_kernel(const float* x, float* y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) ex2_fma_pair(x[i], x[i + 1], y[i], y[i + 1]);
}

constexpr int kThreads = 576;
constexpr int kReaders = 512;  // warps 0-15: four warpgroups read TMEM
constexpr int kProducerWarp = 16;
constexpr int kMmaWarp = 17;
constexpr uint32_t kTeardownPolls = 1u << 26;

struct ScoreTcParams {
  float* scores;
  float* part;  // [groups][nsplit][Mp] x {m (log2 units), Z}
  uint32_t* status;
  int Hq, Hkv, L, G, W, M, nsplit;
  float scale_log2;
  uint64_t wait_limit;
};

template <int D, int RH>
struct SCfg {
  static constexpr int Mp = 128 * RH;
  static constexpr int NS = 4;
  static constexpr int HALVES = D / 64;
  static constexpr int QW_BYTES = Mp * D * 2;
  static constexpr int KT_BYTES = 128 * D * 2;
  static constexpr int OFF_QW = 0;
  static constexpr int OFF_K = QW_BYTES;
  static constexpr int OFF_CST = OFF_K + NS * KT_BYTES;  // pass 2: Mp floats
  static constexpr int OFF_RED = OFF_CST + 256 * 4;      // pass 1: partial (m, Z) of the other warpgroups
  static constexpr int OFF_BAR = OFF_RED + 4 * 256 * 4;
  // barriers: q, full[NS], empty[NS], sfull[2], sfree[2], teardown
  static constexpr int NBAR = 1 + 2 * NS + 4 + 1;
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;
};

__device__ __forceinline__ void split_tiles(int s, int nsplit, int ntiles, int& t0, int& t1) {
  t0 = (int)((long long)ntiles * s / nsplit);
  t1 = (int)((long long)ntiles * (s + 1) / nsplit);
}

template <int D, int RH, int PASS>
__global__ void __launch_bounds__(kThreads, 1)
    score_tc(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
             const ScoreTcParams p) {
  using C = SCfg<D, RH>;
  constexpr int Mp = C::Mp;
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int grp = b * p.Hkv + g;
  const int L = p.L;
  const int ntiles = (L + 127) / 128;
  int t0, t1;
  split_tiles(split, p.nsplit, ntiles, t0, t1);
  const int nt = t1 - t0;  // key tiles of this CTA
  const int j0 = t0 * 128, j1 = min(L, t1 * 128);
  // Steps: pass 1 with RH == 1 takes two key tiles per step (one per warpgroup);
  // otherwise one key tile per step.
  const int per_step = (PASS == 1 && RH == 1) ? 2 : 1;
  const int nstep = (nt + per_step - 1) / per_step;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sQ = base + C::OFF_QW, sK = base + C::OFF_K;
  float* cst = reinterpret_cast<float*>(gbase + C::OFF_CST);
  float* red = reinterpret_cast<float*>(gbase + C::OFF_RED);
  const uint32_t bar0 = base + C::OFF_BAR;
  const uint32_t bar_q = bar0;
  auto bar_full = [&](int s) { return bar0 + 8u * (1 + s); };
  auto bar_empty = [&](int s) { return bar0 + 8u * (1 + C::NS + s); };
  auto bar_sfull = [&](int i) { return bar0 + 8u * (1 + 2 * C::NS + i); };
  auto bar_sfree = [&](int i) { return bar0 + 8u * (3 + 2 * C::NS + i); };
  const uint32_t bar_td = bar0 + 8u * (5 + 2 * C::NS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + C::OFF_BAR + C::NBAR * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + C::OFF_BAR + C::NBAR * 8 + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_empty(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_sfull(i), 1);
      mbar_init(bar_sfree(i), kReaders / 2);  // one warpgroup pair reads each buffer
    }
    mbar_init(bar_td, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_map(&tmq);
    tma_prefetch_map(&tmk);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto fail = [&]() {
    record_status(p.status, TSA_ERR_TIMEOUT);
    *abort_flag = 1;
  };

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ loads
    // Window rows: lane l gathers rows 4l..4l+3 of each 128-row block; rows
    // past M repeat row M-1 (their results are never used).
    if (lane == 0) mbar_arrive_expect_tx(bar_q, C::QW_BYTES);
    __syncwarp();
#pragma unroll
    for (int rb = 0; rb < RH; ++rb) {
      int y[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = min(rb * 128 + 4 * lane + e, p.M - 1);
        const int hh = r / p.W, w = r - hh * p.W;
        y[e] = (b * p.Hq + g * p.G + hh) * L + (L - p.W + w);
      }
#pragma unroll
      for (int h = 0; h < C::HALVES; ++h)
        tma_gather4(sQ + h * (Mp * 128) + rb * 16384 + lane * 512, &tmq, bar_q, 64 * h, y[0], y[1], y[2], y[3]);
    }
    int issued = 0;
    if (lane == 0) {
      const int row0 = (b * p.Hkv + g) * L + j0;
      for (int u = 0; u < nt; ++u) {
        if (*abort_flag) break;
        const int s = u % C::NS;
        if (u >= C::NS && !mbar_wait(bar_empty(s), ((u / C::NS) - 1) & 1, p.wait_limit, abort_flag)) {
          fail();
          break;
        }
        mbar_arrive_expect_tx(bar_full(s), C::KT_BYTES);
#pragma unroll
        for (int h = 0; h < C::HALVES; ++h)
          tma_load_2d(sK + s * C::KT_BYTES + h * 16384, &tmk, bar_full(s), 64 * h, row0 + 128 * u);
        issued = u + 1;
      }
      if (*abort_flag) {
        mbar_wait(bar_q, 0, kTeardownPolls, nullptr);
        for (int u = (issued > C::NS ? issued - C::NS : 0); u < issued; ++u)
          mbar_wait(bar_full(u % C::NS), (u / C::NS) & 1, kTeardownPolls, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(bar_q, 0, p.wait_limit, abort_flag);
      if (PASS == 1) {
        constexpr uint32_t IDESC = idesc_bf16(128, 128, 0, 0);
        for (int i = 0; ok && i < nstep; ++i) {
          const int bf = i & 1;
          if (i >= 2 && !(ok = mbar_wait(bar_sfree(bf), ((i >> 1) - 1) & 1, p.wait_limit, abort_flag))) break;
          for (int w = 0; w < 2; ++w) {
            const int u = RH == 2 ? i : 2 * i + w;
            if (u >= nt) break;
            if ((RH == 1 || w == 0) && !(ok = mbar_wait(bar_full(u % C::NS), (u / C::NS) & 1, p.wait_limit,
                                                         abort_flag)))
              break;
            tc_fence_after();
            const uint32_t qb = sQ + (RH == 2 ? w * 16384 : 0);
            const uint32_t kb = sK + (u % C::NS) * C::KT_BYTES;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t qoff = (kk >> 2) * (Mp * 128) + (kk & 3) * 32;
              const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
              mma_bf16_ss(tmem + bf * 256 + w * 128, sdesc_sw128(qb + qoff, 16, 1024), sdesc_sw128(kb + koff, 16, 1024),
                          IDESC, kk > 0);
            }
            if (RH == 1 || w == 1) tc_commit(bar_empty(u % C::NS));
          }
          if (!ok) break;
          tc_commit(bar_sfull(bf));
        }
      } else {
        constexpr uint32_t IDESC = idesc_bf16(128, Mp, 0, 0);
        for (int u = 0; ok && u < nt; ++u) {
          const int bf = u & 1;
          if (u >= 2 && !(ok = mbar_wait(bar_sfree(bf), ((u >> 1) - 1) & 1, p.wait_limit, abort_flag))) break;
          if (!(ok = mbar_wait(bar_full(u % C::NS), (u / C::NS) & 1, p.wait_limit, abort_flag))) break;
          tc_fence_after();
          const uint32_t kb = sK + (u % C::NS) * C::KT_BYTES;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
            const uint32_t qoff = (kk >> 2) * (Mp * 128) + (kk & 3) * 32;
            mma_bf16_ss(tmem + bf * 256, sdesc_sw128(kb + koff, 16, 1024), sdesc_sw128(sQ + qoff, 16, 1024), IDESC,
                        kk > 0);
          }
          tc_commit(bar_empty(u % C::NS));
          tc_commit(bar_sfull(bf));
        }
      }
      if (!ok) fail();
      tc_commit(bar_td);
      mbar_wait(bar_td, 0, kTeardownPolls, nullptr);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ TMEM readers
    const int wg = warp >> 2;       // 0..3
    const int a = wg & 1;           // pass 1: row block (RH == 2) or tile of the step (RH == 1); pass 2: tile parity
    const int pr = wg >> 1;         // pass 1: step parity this pair reads; pass 2: column half
    const int ch = pr;
    const int rl = threadIdx.x & 127;  // TMEM lane of this thread
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    bool ok = true;
    if (PASS == 1) {
      // The two warpgroup pairs take alternate steps (buffer bf = step parity), so
      // one pair's TMEM loads overlap the other pair's exponentials; a thread reads
      // all 128 columns of its row in 32-column chunks, one chunk loaded ahead.
      const int r = RH == 2 ? a * 128 + rl : rl;  // window row
      const int pos = L - p.W + (r % p.W);
      const bool row_ok = r < p.M;
      // Pass 2 adds its two column halves into the scores: start them at zero.
      for (int j = j0 + threadIdx.x; j < j1; j += kReaders) p.scores[(size_t)grp * L + j] = 0.f;
      float m = -INFINITY, z = 0.f;
      // z is kept relative to a per-row reference m: any reference gives the
      // same m + log2 z.  The first chunk with a visible key sets m to its exact
      // max; later chunks sum 2^(x - m) directly and are redone against their own
      // max only if the sum leaves a safe range (a key far above m).
      auto chunk_sum = [&](const uint32_t (&v)[32], float ref) {
        const uint64_t negm2 = f2_pack(-ref, -ref), sc2 = f2_pack(p.scale_log2, p.scale_log2);
        uint64_t a2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int e2 = 0; e2 < 16; ++e2) {
          float t0, t1;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(v[2 * e2]), __uint_as_float(v[2 * e2 + 1])), sc2, negm2), t0, t1);
          float p0, p1;
          if (e2 % 3 == 2) {  // one pair in three on the FMA pipe; t <= 127 there (clamped: a
                              // larger t saturates at 2^127 and the sum check below redoes the chunk)
            ex2_fma_pair(fminf(t0, 127.f), fminf(t1, 127.f), p0, p1);
          } else {
            p0 = ex2_approx(t0);
            p1 = ex2_approx(t1);
          }
          a2[e2 & 3] = f2_add(a2[e2 & 3], f2_pack(p0, p1));
        }
        float s0, s1, s2, s3, s4, s5, s6, s7;
        f2_unpack(a2[0], s0, s1);
        f2_unpack(a2[1], s2, s3);
        f2_unpack(a2[2], s4, s5);
        f2_unpack(a2[3], s6, s7);
        return ((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7));
      };
      for (int i = pr; i < nstep; i += 2) {
        const int bf = i & 1;  // == pr
        ok = ok && __all_sync(0xffffffffu, mbar_wait(bar_sfull(bf), (i >> 1) & 1, p.wait_limit, abort_flag));
        if (!ok) break;
        tc_fence_after();
        const int u = RH == 2 ? i : 2 * i + a;  // key tile of this thread's row
        const bool have = u < nt;
        const uint32_t ta = tmem + lane_off + bf * 256 + a * 128;
        uint32_t va[32], vb[32];
        if (have) tmem_ld32(ta, va);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t(&v)[32] = (q & 1) ? vb : va;
          uint32_t(&vn)[32] = (q & 1) ? va : vb;
          if (have && q < 3) tmem_ld32_async(ta + (q + 1) * 32, vn);
          if (q == 3) {  // every column of this buffer is in registers: release it
            tc_fence_before();
            mbar_arrive(bar_sfree(bf));
          }
          if (have) {
            const int kbase = j0 + 128 * u + 32 * q;
            const int lim = row_ok ? min(j1 - 1, pos) - kbase + 1 : 0;  // visible keys in this chunk
            if (__any_sync(0xffffffffu, lim < 32)) {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (e >= lim) v[e] = 0xff800000u;  // -inf
            }
            float st = (m > -INFINITY) ? chunk_sum(v, m) : INFINITY;
            const bool exact = !(st <= 1.8446744e19f);  // > 2^64, NaN, or no reference yet
            if (__any_sync(0xffffffffu, exact)) {
              float mx8[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) mx8[e] = __uint_as_float(v[e]);
#pragma unroll
              for (int e = 8; e < 32; ++e) mx8[e & 7] = fmaxf(mx8[e & 7], __uint_as_float(v[e]));
              const float mt = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                     fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]))) * p.scale_log2;
              if (exact && mt > -INFINITY) {
                const float mn = fmaxf(m, mt);
                const float zs = (m > -INFINITY) ? z * ex2_approx(m - mn) : 0.f;
                m = mn;
                z = zs;
              }
              if (exact) st = (m > -INFINITY) ? chunk_sum(v, m) : 0.f;
            }
            z += st;
          }
          if (have && q < 3) tmem_wait_ld32(vn);
        }
      }
      // Merge the partial (m, Z) of the warpgroups that saw the same rows: both
      // step parities, and for RH == 1 also both tiles of a step.  The named
      // barrier is reached by all reader threads whatever happened above.
      const int slot = RH == 2 ? (pr * 2 + a) : wg;  // 4 slots of 128 (RH == 1) or 2 x 2 (RH == 2)
      red[slot * 128 + rl] = m;
      red[512 + slot * 128 + rl] = z;
      asm volatile("bar.sync 1, %0;" ::"n"(kReaders) : "memory");
      if (!ok) fail();
      const bool writer = RH == 2 ? (pr == 0) : (wg == 0);
      if (writer && !*abort_flag) {
        constexpr int NSRC = RH == 2 ? 2 : 4;  // partials per row
        float ms[NSRC], zs4[NSRC];
#pragma unroll
        for (int i = 0; i < NSRC; ++i) {
          const int sl = RH == 2 ? (i * 2 + a) : i;
          ms[i] = red[sl * 128 + rl];
          zs4[i] = red[512 + sl * 128 + rl];
        }
        float mn = -INFINITY;
#pragma unroll
        for (int i = 0; i < NSRC; ++i) mn = fmaxf(mn, ms[i]);
        float zz = 0.f;
        if (mn > -INFINITY) {
#pragma unroll
          for (int i = 0; i < NSRC; ++i)
            if (ms[i] > -INFINITY) zz += zs4[i] * ex2_approx(ms[i] - mn);
        }
        float* pp = p.part + ((size_t)grp * p.nsplit + split) * Mp * 2;
        pp[r] = mn;
        pp[Mp + r] = zz;
      }
    } else {
      // Combine the row partials of every split: c_r = m_r + log2 Z_r.
      const float* pbase = p.part + (size_t)grp * p.nsplit * Mp * 2;
      for (int r = threadIdx.x; r < Mp; r += kReaders) {
        float mx = -INFINITY;
        for (int s = 0; s < p.nsplit; ++s) mx = fmaxf(mx, pbase[(size_t)s * Mp * 2 + r]);
        float zs = 0.f;
        if (mx > -INFINITY) {
          for (int s = 0; s < p.nsplit; ++s) {
            const float ms = pbase[(size_t)s * Mp * 2 + r];
            if (ms > -INFINITY) zs += pbase[(size_t)s * Mp * 2 + Mp + r] * ex2_approx(ms - mx);
          }
        }
        cst[r] = (r < p.M && mx > -INFINITY) ? -(mx + log2f(zs)) : -INFINITY;  // -c_r
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kReaders) : "memory");
      float* out = p.scores + (size_t)grp * L;
      constexpr int HC = Mp / 2;  // columns (window rows) of this thread's half
      for (int u = a; u < nt; u += 2) {
        const int bf = u & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(bar_sfull(bf), (u >> 1) & 1, p.wait_limit, abort_flag));
        if (!ok) break;
        tc_fence_after();
        const int key = j0 + 128 * u + rl;
        // Only keys >= L-W are hidden from some window rows; decide per warp
        // (TMEM loads are warp-collective).
        const bool tail = __any_sync(0xffffffffu, key >= L - p.W);
        float acc4[4] = {0.f, 0.f, 0.f, 0.f};
        // 32-column chunks with the next chunk's TMEM load in flight; the buffer
        // is released once its last chunk is in registers.
        const uint32_t tb = tmem + lane_off + bf * 256 + ch * HC;
        uint32_t va[32], vb[32];
        tmem_ld32(tb, va);
#pragma unroll
        for (int q4 = 0; q4 < HC / 32; ++q4) {
          const int col0 = ch * HC + q4 * 32;  // first window row of this chunk
          uint32_t(&v)[32] = (q4 & 1) ? vb : va;
          uint32_t(&vn)[32] = (q4 & 1) ? va : vb;
          if (q4 + 1 < HC / 32) {
            tmem_ld32_async(tb + (q4 + 1) * 32, vn);
          } else {
            tc_fence_before();
            mbar_arrive(bar_sfree(bf));
          }
          const float* nc = cst + col0;
          if (!tail) {
            const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2);
            uint64_t a2[2] = {0ull, 0ull};
#pragma unroll
            for (int e2 = 0; e2 < 16; ++e2) {
              const uint64_t c2 = *reinterpret_cast<const uint64_t*>(nc + 2 * e2);  // (-c_r, -c_r+1)
              float t0, t1;
              f2_unpack(f2_fma(f2_pack(__uint_as_float(v[2 * e2]), __uint_as_float(v[2 * e2 + 1])), sc2, c2), t0, t1);
              float p0, p1;
              if (e2 % 3 == 2) {  // one pair in three on the FMA pipe
                ex2_fma_pair(t0, t1, p0, p1);
              } else {
                p0 = ex2_approx(t0);
                p1 = ex2_approx(t1);
              }
              a2[e2 & 1] = f2_add(a2[e2 & 1], f2_pack(p0, p1));
            }
            float s0, s1, s2, s3;
            f2_unpack(a2[0], s0, s1);
            f2_unpack(a2[1], s2, s3);
            acc4[0] += s0;
            acc4[1] += s1;
            acc4[2] += s2;
            acc4[3] += s3;
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int col = col0 + e;
              const float pe = ex2_approx(fmaf(__uint_as_float(v[e]), p.scale_log2, nc[e]));
              acc4[e & 3] += (key > L - p.W + (col % p.W)) ? 0.f : pe;
            }
          }
          if (q4 + 1 < HC / 32) tmem_wait_ld32(vn);
        }
        const float acc = (acc4[0] + acc4[1]) + (acc4[2] + acc4[3]);
        // Two column halves per key: 0 + h0 + h1 is the same in either order.
        if (key < j1) atomicAdd(out + key, acc);
      }
      if (!ok) fail();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D, int RH>
cudaError_t launch_passes(const Dims& d, const CUtensorMap& mq, const CUtensorMap& mk, const ScoreTcParams& prm,
                          cudaStream_t st) {
  const int smem = SCfg<D, RH>::SMEM;
  cudaError_t e = cudaFuncSetAttribute(score_tc<D, RH, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(score_tc<D, RH, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const dim3 grid(prm.nsplit, d.Hkv, d.B);
  score_tc<D, RH, 1><<<grid, kThreads, smem, st>>>(mq, mk, prm);
  count_launches(1);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  score_tc<D, RH, 2><<<grid, kThreads, smem, st>>>(mq, mk, prm);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

// Key-range splits per KV head: a function of L only (at most 18, so a layer of
// 8 KV heads is one wave of 144 CTAs, one per SM).  A KV head's scores therefore
// do not depend on which other heads share the call: a layer split by KV group
// across calls (or GPUs) gives bit-identical scores.
int score_tc_splits(const Dims& d) {
  const int ntiles = (d.L + 127) / 128;
  const int s = ntiles < 18 ? ntiles : 18;
  return s < kMaxScoreSplits ? s : kMaxScoreSplits;
}

cudaError_t launch_score_tc(const Dims& d, const void* q, const void* k, int window, float* scores, float* part,
                            uint32_t* status, cudaStream_t st) {
  CUtensorMap mq, mk;
  if (!make_row_map(&mq, q, (uint64_t)d.B * d.Hq * d.L, d.D) ||
      !make_tile_map(&mk, k, (uint64_t)d.B * d.Hkv * d.L, d.D, 128))
    return cudaErrorInvalidValue;
  ScoreTcParams prm;
  prm.scores = scores;
  prm.part = part;
  prm.status = status;
  prm.Hq = d.Hq;
  prm.Hkv = d.Hkv;
  prm.L = d.L;
  prm.G = d.G;
  prm.W = window;
  prm.M = d.G * window;
  prm.nsplit = score_tc_splits(d);
  prm.scale_log2 = d.scale * 1.4426950408889634f;
  prm.wait_limit = wait_limit();
  const bool two = prm.M > 128;
  if (d.D == 64) return two ? launch_passes<64, 2>(d, mq, mk, prm, st) : launch_passes<64, 1>(d, mq, mk, prm, st);
  return two ? launch_passes<128, 2>(d, mq, mk, prm, st) : launch_passes<128, 1>(d, mq, mk, prm, st);
}

cudaError_t launch_debug_exp2(const float* x, float* y, int n, cudaStream_t st) {
  debug_exp2_kernel<<<(n / 2 + 255) / 256, 256, 0, st>>>(x, y, n);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace tsa
