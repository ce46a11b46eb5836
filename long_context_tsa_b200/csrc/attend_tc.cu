// Compressed causal attention on the tcgen05 tensor cores (bf16 in, fp32
// accumulate), with the gather fused into the loads (16-byte cp.async copies of
// the selected rows straight into the swizzled shared-memory tiles) and the
// scatter fused into the epilogue.
//
// "Token Sparse Attention Long Context" (skill page), Steps 2-3;
// "Token Sparse Attention: Efficient Long-Context Inference with Interleaved
// Token Selection", Figure 3 (Stage 1: per-head compressed Q, K, V; Stage 2:
// attention on the compressed tensors, scattered back to the full layout).
//
// Work item = (batch, KV group g, chunk c).  A CTA owns two 128-row M tiles.
// With G = Hq/Hkv query heads per group and RP = 128/G, tile t row r is query
// head g*G + r/RP at compacted position c*2RP + t*RP + r%RP: the G heads of a
// group share every gathered K/V tile.  Keys come in tiles of 128 compacted
// positions; the causal mask on compacted indices equals the mask on original
// positions because perm[0:K] is ascending.
//
// Warp roles (512 threads, four warpgroups, 128 registers per thread):
//   warps 0-3, 4-7  softmax + epilogue of tile 0 / tile 1 (thread = TMEM lane = row)
//   warps 8-11      loads: each warp gathers 32 of the 128 rows of every Q/K/V
//                   tile with 16-byte cp.async (one warp per SM sub-partition:
//                   a single warp cannot pull gathered rows fast enough)
//   warp 12         MMA issuer (one thread): S_t = Q_t K^T, O_t += P_t V
//   warps 13-15     zero fill: this CTA's share of the group's dropped rows
//                   perm[K:L] gets +0 in every query head (HBM writes that
//                   overlap the tensor-bound work of the other warps)
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [256+D,256+2D);
// P_t (bf16) overwrites the first 64 columns of S_t once the softmax has read
// it, and PV reads it from there (A operand in TMEM).
// Shared memory: Q0 Q1 (128xD) and a ring of NS K/V tiles, K-major with the
// 128-byte swizzle (V is read MN-major).
//
// Online softmax in base 2 with a lazy rescale: the running max used for P
// moves only when a row max exceeds it by more than 8 (P <= 2^8), so O is
// rescaled in TMEM rarely.  Every mbarrier wait is bounded; on timeout the CTA
// records TSA_ERR_TIMEOUT, drains its own copies and MMAs, frees TMEM and exits.
#include <cuda.h>
#include <math.h>

#include <cstdlib>
#include <cstring>
#include <type_traits>

#include "device_common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

namespace tsa {
namespace {

using namespace tc;

constexpr int kThreads = 512;        // four warpgroups
constexpr int kProducerWarp0 = 8;    // warps 8-11: loads
constexpr int kProducerWarps = 4;
constexpr int kMmaWarp = 12;
constexpr int kZeroWarp0 = 13;       // warps 13-15: zero fill
constexpr int kZeroWarps = 3;

constexpr uint32_t kTeardownPolls = 1u << 26;
constexpr long long kFusedZeroMinCtas = 2 * 148;  // attention CTAs from which the zero fill is fused
constexpr float kRescaleThreshold = 8.0f;   // log2 units

struct TcAttendParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const int32_t* perm;
  void* out;
  uint32_t* status;
  int Hq, Hkv, L, G, RP, n_groups, cmax;
  float scale_log2;
  uint64_t wait_limit;
  int accumulate;  // 1: out[kept rows] += attention, dropped rows untouched
  int zero_fill;   // 1: warps 13-15 write the dropped rows (else a separate kernel did, or none are due)
  const uint8_t* block_mask;  // [B*Hkv][nb][nb] over 128-blocks of compacted (query, key), or null
  int nb;
  Budgets kept;
};

template <int D>
struct Cfg {
  static constexpr int NS = D == 128 ? 5 : 8;        // K/V ring stages
  static constexpr int Q_BYTES = 128 * D * 2;
  static constexpr int KV_BYTES = 128 * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = 2 * Q_BYTES;
  static constexpr int OFF_IDX = OFF_KV + NS * KV_BYTES;  // row tables: Q tiles (2 x 128), K/V tile (128)
  static constexpr int OFF_BAR = OFF_IDX + 3 * 128 * 4;
  // barriers: q (tile 0), full[NS], empty[NS], s[2], p[2], o[2], teardown, q (tile 1); then tmem slot, abort flag
  static constexpr int NBAR = 1 + 2 * NS + 6 + 1 + 1;  // + the second Q tile
  static constexpr int OFF_ZERO = (OFF_BAR + NBAR * 8 + 16 + 15) / 16 * 16;  // one row of zeros (bulk-copy source)
  static constexpr int SMEM = OFF_ZERO + D * 2 + 1024;  // + alignment slack
  static constexpr int CPR = D / 8;    // 16-byte chunks per row
  static constexpr int RPI = 32 / CPR;  // rows per warp-wide copy instruction
  static constexpr uint32_t O_COL0 = 256u;  // S_t lives at column 128 * t
};

__device__ __forceinline__ int load_pos(const int32_t* pm, int idx, int L, uint32_t* status) {
  const int p = pm[idx];
  if ((unsigned)p >= (unsigned)L) {
    record_status(status, TSA_ERR_DEVICE_BOUNDS);
    return 0;
  }
  return p;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attend_tc(const TcAttendParams p) {
  using C = Cfg<D>;
  const int bid = blockIdx.x;
  const int c = p.cmax - 1 - bid / p.n_groups;  // heaviest chunks first
  const int grp = bid % p.n_groups;
  const int K = p.kept.kept[grp];
  const int P2 = 2 * p.RP;  // positions per CTA
  if (c * P2 >= K) return;  // nothing to do for this group at this chunk
  const int b = grp / p.Hkv, g = grp - b * p.Hkv;
  const int L = p.L;
  const int last_pos = min(K, (c + 1) * P2) - 1;
  const int n_kt = last_pos / 128 + 1;  // key tiles 0..n_kt-1
  const int32_t* pm = p.perm + (size_t)grp * L;
  // Block-sparse composition: key tile kt is processed when the block mask
  // enables it for the 128-block of either M tile's positions (both tiles lie in
  // one block unless G = 1); every role walks the same list of active tiles, and
  // a tile disabled for only one M tile is fully masked in that tile's softmax.
  const uint8_t* bm = p.block_mask ? p.block_mask + (size_t)grp * p.nb * p.nb : nullptr;
  const int qb0 = (c * P2) / 128, qb1 = (c * P2 + p.RP) / 128;
  auto tile_on = [&](int t, int kt) -> bool { return bm == nullptr || bm[(t ? qb1 : qb0) * p.nb + kt] != 0; };
  auto active = [&](int kt) -> bool { return tile_on(0, kt) || tile_on(1, kt); };
  auto next_active = [&](int kt) -> int {
    int x = kt + 1;
    while (x < n_kt && !active(x)) ++x;
    return x;
  };

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sQ = base + C::OFF_Q, sKV = base + C::OFF_KV;
  const uint32_t bar0 = base + C::OFF_BAR;
  const uint32_t bar_q = bar0;
  auto bar_full = [&](int s) { return bar0 + 8u * (1 + s); };
  auto bar_empty = [&](int s) { return bar0 + 8u * (1 + C::NS + s); };
  auto bar_s = [&](int t) { return bar0 + 8u * (1 + 2 * C::NS + t); };
  auto bar_p = [&](int t) { return bar0 + 8u * (3 + 2 * C::NS + t); };
  auto bar_o = [&](int t) { return bar0 + 8u * (5 + 2 * C::NS + t); };
  const uint32_t bar_td = bar0 + 8u * (7 + 2 * C::NS);
  const uint32_t bar_q1 = bar0 + 8u * (8 + 2 * C::NS);  // Q tile 1 (bar_q: Q tile 0)
  int* qtab = reinterpret_cast<int*>(gbase + C::OFF_IDX);          // [2][128] global q rows
  int* kvtab = reinterpret_cast<int*>(gbase + C::OFF_IDX + 1024);  // [128] global k/v rows
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + C::OFF_BAR + C::NBAR * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + C::OFF_BAR + C::NBAR * 8 + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int n_act = n_kt;  // active key tiles
  if (bm != nullptr) {
    n_act = 0;
    for (int x0 = 0; x0 < n_kt; x0 += 32) n_act += __popc(__ballot_sync(0xffffffffu, x0 + lane < n_kt && active(x0 + lane)));
  }

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 32 * kProducerWarps);  // every producer lane arrives once its own copies land
    mbar_init(bar_q1, 32 * kProducerWarps);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(bar_full(s), 32 * kProducerWarps);
      mbar_init(bar_empty(s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar_s(t), 1);
      mbar_init(bar_p(t), 128);
      mbar_init(bar_o(t), 1);
    }
    mbar_init(bar_td, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto fail = [&]() {
    record_status(p.status, TSA_ERR_TIMEOUT);
    *abort_flag = 1;
  };

  if (warp >= 8) {
   if (warp < kProducerWarp0 + kProducerWarps) {
    // ------------------------------------------------------------ producer
    // Copies are 16-byte cp.async chunks written straight into the 128-byte
    // swizzled K-major layout the MMA reads; one warp instruction moves RPI
    // whole rows.  After issuing a tile every lane arrives on the tile's
    // barrier through cp.async.mbarrier.arrive, which fires once the lane's
    // copies have landed: no lane waits for its own copies, so loads of every
    // free ring stage are in flight at once.  Q tile 0 arrives on bar_q, Q tile 1
    // (issued right after K_0: the first QK waits only for Q tile 0 and K_0) on bar_q1, ring
    // load i (K_0, V_0, K_1, ...) on full[i % NS]; the MMA thread makes the
    // landed rows visible to the tensor core (proxy fence) after its wait.
    const int pw = warp - kProducerWarp0;  // this warp owns rows [32 pw, 32 pw + 32) of every tile
    const int my_c = lane % C::CPR, my_r = lane / C::CPR;
    const uint32_t chunk_off = (uint32_t)(my_c >> 3) * 16384u;
    auto issue_tile = [&](uint32_t dst, const __nv_bfloat16* src, const int* tab) {
#pragma unroll 4
      for (int n = 0; n < 32 / C::RPI; ++n) {
        const int row = 32 * pw + n * C::RPI + my_r;
        const __nv_bfloat16* g = src + (size_t)tab[row] * D + my_c * 8;
        cp_async16(dst + chunk_off + row * 128 + ((((uint32_t)my_c & 7u) ^ ((uint32_t)row & 7u)) << 4), g);
      }
    };
    // Row tables: lane l owns row 32 pw + l of each tile (the warp reads only its rows).
    const int my_row = 32 * pw + lane;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int hh = my_row / p.RP;
      const int pos = min(c * P2 + t * p.RP + (my_row - hh * p.RP), K - 1);
      qtab[t * 128 + my_row] = (b * p.Hq + g * p.G + hh) * L + load_pos(pm, pos, L, p.status);
    }
    __syncwarp();
    issue_tile(sQ, p.q, qtab);
    cp_async_mbar_arrive(bar_q);
    const int kv_row0 = (b * p.Hkv + g) * L;
    int kt_load = next_active(-1);  // the active tile whose rows y_next holds
    int y_next = kv_row0 + load_pos(pm, min(min(kt_load, n_kt - 1) * 128 + my_row, K - 1), L, p.status);
    for (int i = 0; i < 2 * n_act; ++i) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
      const int s = i % C::NS;
      if ((i & 1) == 0) {  // K of an active tile: its rows become current, fetch the next active tile's
        __syncwarp();
        kvtab[my_row] = y_next;
        __syncwarp();
        kt_load = next_active(kt_load);
        if (kt_load < n_kt) y_next = kv_row0 + load_pos(pm, min(kt_load * 128 + my_row, K - 1), L, p.status);
      }
      if (i >= C::NS) {  // wait until load i - NS (same stage) has been consumed
        const bool got = mbar_wait(bar_empty(s), ((i / C::NS) - 1) & 1, p.wait_limit, abort_flag);
        if (!__all_sync(0xffffffffu, got)) {
          if (lane == 0) fail();
          break;
        }
      }
      issue_tile(sKV + s * C::KV_BYTES, (i & 1) ? p.v : p.k, kvtab);
      cp_async_mbar_arrive(bar_full(s));
      if (i == 0) {  // Q tile 1 after K_0: the first QK needs only Q tile 0 and K_0
        issue_tile(sQ + C::Q_BYTES, p.q, qtab + 128);
        cp_async_mbar_arrive(bar_q1);
      }
    }
    cp_async_wait_all();  // no copy is still writing shared memory when the CTA exits
  } else if (warp >= kZeroWarp0) {
    // ------------------------------------------------------------ zero fill
    const int U = p.zero_fill ? L - K : 0;  // dropped rows of this group left to this kernel
    if (U > 0) {
      const int nc = (K + P2 - 1) / P2;  // CTAs of this group
      const int lo = (int)((long long)U * c / nc), hi = (int)((long long)U * (c + 1) / nc);
      // Each dropped row of each query head is one bulk (TMA) copy of a shared-memory
      // row of zeros: the copy engine moves the bytes, the warps only issue them
      // (plain 16-byte stores from these warps measured 2 % slower overall).
      constexpr int CPR = D * 2 / 16;  // 16-byte chunks per row
      const uint32_t szero = base + C::OFF_ZERO;
      const int zt = (warp - kZeroWarp0) * 32 + lane;  // 0 .. 32 * kZeroWarps - 1
      if (zt < CPR) st_shared_v4(szero + 16 * zt, 0u, 0u, 0u, 0u);
      fence_proxy_async_smem();  // the zeros are visible to the copy engine ...
      named_sync(3u, 32u * kZeroWarps);  // ... before any zero warp copies them
      __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(p.out) + (size_t)(b * p.Hq + g * p.G) * L * D;
      for (int u = lo + zt; u < hi; u += 32 * kZeroWarps) {
        const int pos = pm[K + u];
        if ((unsigned)pos >= (unsigned)L) {
          record_status(p.status, TSA_ERR_DEVICE_BOUNDS);
          continue;
        }
        for (int hh = 0; hh < p.G; ++hh) bulk_copy_s2g(ob + ((size_t)hh * L + pos) * D, szero, D * 2);
      }
      bulk_commit_wait_all();  // the source row stays valid and every copy is done before the CTA exits
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_QK = idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t IDESC_PV = idesc_bf16(128, D, 0, 1);
      bool ok = mbar_wait(bar_q, 0, p.wait_limit, abort_flag);
      fence_proxy_async_smem();  // rows landed by cp.async (generic proxy) are read by the tensor core
      auto wait_load = [&](int i) -> bool {
        const bool got = mbar_wait(bar_full(i % C::NS), (i / C::NS) & 1, p.wait_limit, abort_flag);
        fence_proxy_async_smem();
        return got;
      };
      auto qk = [&](int t, int i_k) {
        const uint32_t kbase = sKV + (i_k % C::NS) * C::KV_BYTES;
        const uint32_t qbase = sQ + t * C::Q_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16_ss(tmem + (uint32_t)t * 128u, sdesc_sw128(qbase + off, 16, 1024), sdesc_sw128(kbase + off, 16, 1024),
                      IDESC_QK, kk > 0);
        }
      };
      // P_t (bf16, two per column) sits in the first 64 columns of S_t.
      auto pv = [&](int t, int i_v, bool acc0) {
        const uint32_t vbase = sKV + (i_v % C::NS) * C::KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(tmem + C::O_COL0 + t * D, tmem + (uint32_t)t * 128u + kk * 8,
                      sdesc_sw128(vbase + kk * 2048, 16384, 1024), IDESC_PV, (acc0 || kk > 0) ? 1u : 0u);
      };
      if (ok && n_act > 0) ok = wait_load(0);
      if (ok && n_act > 0) {
        tc_fence_after();
        qk(0, 0);
        tc_commit(bar_s(0));
        ok = mbar_wait(bar_q1, 0, p.wait_limit, abort_flag);
        fence_proxy_async_smem();
        if (ok) {
          tc_fence_after();
          qk(1, 0);
          tc_commit(bar_s(1));
          tc_commit(bar_empty(0));  // K_0 consumed once both QKs complete
        }
      }
      for (int j = 0; ok && j < n_act; ++j) {  // j counts active tiles
        const int iv = 2 * j + 1, ik_next = 2 * j + 2;
        if (!(ok = wait_load(iv))) break;
        for (int t = 0; t < 2 && ok; ++t) {
          if (!(ok = mbar_wait(bar_p(t), j & 1, p.wait_limit, abort_flag))) break;
          tc_fence_after();
          pv(t, iv, j > 0);
          if (t == 1) tc_commit(bar_empty(iv % C::NS));  // V_j consumed
          if (j + 1 < n_act) {
            if (t == 0 && !(ok = wait_load(ik_next))) break;
            tc_fence_after();
            qk(t, ik_next);
            tc_commit(bar_s(t));
            if (t == 1) tc_commit(bar_empty(ik_next % C::NS));  // K_{j+1} consumed
          } else {
            tc_commit(bar_o(t));
          }
        }
      }
      if (!ok) fail();
      // Drain every MMA this thread issued before TMEM is released.
      tc_commit(bar_td);
      mbar_wait(bar_td, 0, kTeardownPolls, nullptr);
    }
    __syncwarp();
   }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int t = warp >> 2;
    const int r = threadIdx.x & 127;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + (uint32_t)t * 128u;
    const uint32_t tO = tmem + lane_off + C::O_COL0 + t * D;
    const int hh = r / p.RP;
    const int pos = c * P2 + t * p.RP + (r - hh * p.RP);
    float m_use = -INFINITY, l = 0.f;
    bool ok = true;
    // The two softmax warpgroups run independently: while one is in its
    // latency-bound max pass the other keeps the exponential unit busy.  (Taking
    // strict turns on the whole softmax phase measured 8 % slower.)
    int kt = next_active(-1);  // key tile of active step j
    for (int j = 0; j < n_act; ++j, kt = next_active(kt)) {
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_s(t), j & 1, p.wait_limit, abort_flag));
      if (!ok) continue;
      tc_fence_after();
      // Visible keys in this tile: causal, and none when the block mask disables it for this M tile.
      const int nvis = tile_on(t, kt) ? pos - kt * 128 + 1 : 0;
      // Only tiles on the diagonal hide keys from some rows (warp-uniform choice).
      const bool masked = __any_sync(0xffffffffu, nvis < 128);
      // Two passes over S_t, each in four 32-column chunks whose TMEM loads run one
      // chunk ahead (registers va / vb alternate).  Pass 1: the row max x_max.  The
      // reference m moves only when x_max * scale exceeds it by more than the
      // threshold (always on the first tile, where m = -inf); then alpha =
      // 2^(m_old - m_new) rescales l and O.  Pass 2: P = 2^(x * scale - m) for every
      // column against that final m (so P <= 2^threshold), summed into l and written
      // to TMEM as bf16 pairs over S columns [16 q, 16 q + 16), which pass 2 has
      // already read.  No decision inside the exponential loop.
      float alpha = 1.f;
      bool rescaled = false;  // warp-uniform: O must be rescaled by alpha
      uint64_t acc2 = 0ull;   // packed fp32 pair of the tile's row sum
      auto tile = [&](auto masked_c) {
        constexpr bool kMasked = decltype(masked_c)::value;
        auto xval = [&](const uint32_t* v, int q4, int e) -> float {
          const float x = __uint_as_float(v[e]);
          return (!kMasked || q4 * 32 + e < nvis) ? x : -INFINITY;
        };
        uint32_t va[32], vb[32];
        tmem_ld32(tS, va);
        float mxs[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};  // four independent chains
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t(&v)[32] = (q4 & 1) ? vb : va;
          uint32_t(&vn)[32] = (q4 & 1) ? va : vb;
          tmem_ld32_async(tS + ((q4 + 1) & 3) * 32, vn);  // after chunk 3: pass 2's chunk 0
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            mxs[0] = fmax3(mxs[0], xval(v, q4, e), xval(v, q4, e + 1));
            mxs[1] = fmax3(mxs[1], xval(v, q4, e + 2), xval(v, q4, e + 3));
            mxs[2] = fmax3(mxs[2], xval(v, q4, e + 4), xval(v, q4, e + 5));
            mxs[3] = fmax3(mxs[3], xval(v, q4, e + 6), xval(v, q4, e + 7));
          }
          tmem_wait_ld32(vn);
        }
        const float mx = fmaxf(fmaxf(mxs[0], mxs[1]), fmaxf(mxs[2], mxs[3]));
        const float mt = mx * p.scale_log2;
        const bool need = mt > m_use + kRescaleThreshold;  // always true on the first tile
        if (need) {
          alpha = ex2_approx(m_use - mt);  // 0 when m_use is -inf
          m_use = mt;
        }
        rescaled = j > 0 && __any_sync(0xffffffffu, need);
        const uint64_t scale2 = f2_pack(p.scale_log2, p.scale_log2);
        const float mref = m_use == -INFINITY ? 0.f : m_use;  // no visible key yet: P = 2^-inf = 0
        const uint64_t negm2 = f2_pack(-mref, -mref);
        uint64_t accq[2] = {0ull, 0ull};
        // Pairs of chunks per iteration of a rolled loop: the loop edge keeps the
        // scheduler from interleaving all four chunks (which ran out of registers).
#pragma unroll 1
        for (int qq = 0; qq < 4; qq += 2)
#pragma unroll
        for (int qi = 0; qi < 2; ++qi) {
          const int q4 = qq + qi;
          uint32_t(&v)[32] = qi ? vb : va;  // pass 2's chunk 0 sits in va
          uint32_t(&vn)[32] = qi ? va : vb;
          if (q4 < 3) tmem_ld32_async(tS + (q4 + 1) * 32, vn);
          uint32_t pk[16];
#pragma unroll
          for (int e2 = 0; e2 < 16; ++e2) {
            float t0, t1;
            f2_unpack(f2_fma(f2_pack(xval(v, q4, 2 * e2), xval(v, q4, 2 * e2 + 1)), scale2, negm2), t0, t1);
            const float p0 = ex2_approx(t0), p1 = ex2_approx(t1);
            accq[e2 & 1] = f2_add(accq[e2 & 1], f2_pack(p0, p1));
            pk[e2] = pack_bf16(p0, p1);
          }
          tmem_st16(tS + q4 * 16, pk);
          if (q4 < 3) tmem_wait_ld32(vn);
        }
        acc2 = f2_add(accq[0], accq[1]);
      };
      if (masked) {
        tile(std::true_type{});
      } else {
        tile(std::false_type{});
      }
      {
        float s0, s1;
        f2_unpack(acc2, s0, s1);
        l = l * alpha + (s0 + s1);
      }
      // O_t is idle here (the commit that released S_t(j) covers PV(t, j-1)).
      // TMEM access is warp-collective, so the whole warp rescales when any
      // lane needs it (alpha = 1 for the others).
      if (rescaled) {
#pragma unroll
        for (int q4 = 0; q4 < D / 32; ++q4) {
          uint32_t v[32];
          tmem_ld32(tO + q4 * 32, v);
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
          tmem_st32(tO + q4 * 32, v);
        }
      }
      tmem_st_wait();  // P (and a rescaled O) are in TMEM before the MMA warp is told
      tc_fence_before();
      mbar_arrive(bar_p(t));
    }
    if (ok && n_act > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar_o(t), 0, p.wait_limit, abort_flag));
    if (!ok) {
      fail();
    } else {
      tc_fence_after();
      const bool valid = pos < K;
      const int opos = valid ? load_pos(pm, pos, L, p.status) : 0;
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.out) + ((size_t)(b * p.Hq + g * p.G + hh) * L + opos) * D;
      const float inv = l > 0.f ? 1.f / l : 0.f;  // a row that saw no key (block mask) outputs zeros
#pragma unroll
      for (int q4 = 0; q4 < D / 32; ++q4) {
        uint32_t v[32];
        if (n_act > 0) {
          tmem_ld32(tO + q4 * 32, v);  // warp-collective: every lane loads, valid rows store
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = 0u;  // no active key tile: O was never written
        }
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + q4 * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float f[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) f[u] = __uint_as_float(v[8 * e + u]) * inv;
            if (p.accumulate) {  // scatter-add: the row's current value plus the attention output
              const uint4 old = dst[e];
              const uint32_t ow[4] = {old.x, old.y, old.z, old.w};
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&ow[u]);
                f[2 * u] += __bfloat162float(h.x);
                f[2 * u + 1] += __bfloat162float(h.y);
              }
            }
            uint4 o;
            o.x = pack_bf16(f[0], f[1]);
            o.y = pack_bf16(f[2], f[3]);
            o.z = pack_bf16(f[4], f[5]);
            o.w = pack_bf16(f[6], f[7]);
            dst[e] = o;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- host side

template <int D>
cudaError_t launch_tc(const Dims& d, const void* q, const void* k, const void* v, const int32_t* perm,
                      const Budgets& kept, void* out, uint32_t* status, bool accumulate, const uint8_t* block_mask,
                      cudaStream_t st) {
  TcAttendParams prm;
  prm.q = static_cast<const __nv_bfloat16*>(q);
  prm.k = static_cast<const __nv_bfloat16*>(k);
  prm.v = static_cast<const __nv_bfloat16*>(v);
  prm.perm = perm;
  prm.out = out;
  prm.status = status;
  prm.Hq = d.Hq;
  prm.Hkv = d.Hkv;
  prm.L = d.L;
  prm.G = d.G;
  prm.RP = 128 / d.G;
  prm.n_groups = d.B * d.Hkv;
  prm.scale_log2 = d.scale * 1.4426950408889634f;
  prm.wait_limit = wait_limit();
  prm.accumulate = accumulate ? 1 : 0;
  prm.kept = kept;
  int kmax = 0;
  for (int i = 0; i < prm.n_groups; ++i) kmax = kept.kept[i] > kmax ? kept.kept[i] : kmax;
  prm.cmax = (kmax + 2 * prm.RP - 1) / (2 * prm.RP);
  const long long nblk = (long long)prm.cmax * prm.n_groups;
  // The fused zero fill spreads the dropped rows over the attention CTAs; with
  // fewer of those than two per SM (small budgets) a separate full-grid zero
  // kernel writes them at HBM speed instead.
  prm.block_mask = block_mask;
  prm.nb = (d.L + 127) / 128;
  prm.zero_fill = 0;
  if (!accumulate) {
    if (nblk >= kFusedZeroMinCtas) {
      prm.zero_fill = 1;
    } else {
      const cudaError_t ez = launch_zero_fill(d, perm, kept, out, status, st);
      if (ez != cudaSuccess) return ez;
    }
  }
  const int smem = Cfg<D>::SMEM;
  cudaError_t e = cudaFuncSetAttribute(attend_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  attend_tc<D><<<(unsigned)nblk, kThreads, smem, st>>>(prm);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attend_tc(const Dims& d, const void* q, const void* k, const void* v, const int32_t* perm,
                             const Budgets& kept, void* out, uint32_t* status, bool accumulate,
                             const uint8_t* block_mask, cudaStream_t st) {
  if (d.D == 64) return launch_tc<64>(d, q, k, v, perm, kept, out, status, accumulate, block_mask, st);
  // The two-SM form (attend_tc2.cu) is opt-in: it measured slower than this
  // kernel at every bench size (the per-tile softmax chain, not the loads or
  // the MMA rate, bounds both).
  const char* pairs = getenv("TSA_ATTEND_CTA_PAIRS");
  if (pairs != nullptr && pairs[0] != '\0' && strcmp(pairs, "0") != 0)
    return launch_attend_tc_pair(d, q, k, v, perm, kept, out, status, accumulate, block_mask, st);
  return launch_tc<128>(d, q, k, v, perm, kept, out, status, accumulate, block_mask, st);
}

}  // namespace tsa
