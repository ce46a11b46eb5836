// Compressed causal attention on CTA pairs (tcgen05 cta_group::2), d = 128:
// the same operation, work split and softmax as attend_tc.cu, with two CTAs of
// a 2-CTA cluster sharing every tensor-core instruction.
//
// "Token Sparse Attention Long Context" (skill page), Steps 2-3;
// "Token Sparse Attention: Efficient Long-Context Inference with Interleaved
// Token Selection", Figure 3 (Stage 1: per-head compressed Q, K, V; Stage 2:
// attention on the compressed tensors, scattered back to the full layout).
//
// Work item = (batch, KV group g, chunk pair cp): CTA rank r of the cluster
// owns chunk c = 2 cp + r (two 128-row M tiles, as in attend_tc), and the pair
// walks the key tiles of chunk 2 cp + 1 (chunk 2 cp's rows see the extra
// tile, when there is one, fully masked).  Each M tile t of the pair is one
// M = 256 MMA: rows 0-127 from CTA 0's Q tile and TMEM, 128-255 from CTA 1's.
// The B operand is split along N: for S = Q K^T each CTA holds 64 of the 128
// keys of a tile (all 128 dims), for O += P V each CTA holds 64 of the 128
// value dims (all 128 keys) -- so each CTA gathers half of every K and V tile.
// CTA 0 (leader) issues the MMAs and commits every completion to both CTAs'
// barriers; CTA 1's MMA warp relays its producers' cp.async completions to the
// leader's barriers (async-proxy fence, then a cluster-scope release arrive);
// the softmax warps tell the leader that P is in TMEM with one arrive per warp
// on the leader's barrier (a local arrive in CTA 0, the CTA-scope remote arrive
// in CTA 1: the TMEM stores were already waited for and fenced, and a
// cluster-scope release there costs about a thousand cycles per step).  Warp
// roles, TMEM columns, the online softmax, the scatter epilogue and the fused
// zero fill are attend_tc's.  The library runs this kernel only on request
// (TSA_ATTEND_CTA_PAIRS): it measured slower than attend_tc, whose bound (the
// per-tile softmax-to-MMA chain) it shares.
// Every mbarrier wait is bounded; on timeout a CTA records TSA_ERR_TIMEOUT,
// drains its own copies and MMAs, meets its peer at the final cluster barrier,
// frees TMEM and exits.
#include <cuda.h>
#include <math.h>

#include <type_traits>

#include "device_common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

namespace tsa {
namespace {

using namespace tc;

constexpr int kThreads = 512;        // four warpgroups
constexpr int D = 128;
constexpr int kProducerWarp0 = 8;    // warps 8-11: loads
constexpr int kProducerWarps = 4;
constexpr int kMmaWarp = 12;
constexpr int kZeroWarp0 = 13;       // warps 13-15: zero fill
constexpr int kZeroWarps = 3;

constexpr uint32_t kTeardownPolls = 1u << 26;
constexpr long long kFusedZeroMinCtas = 2 * 148;  // attention CTAs from which the zero fill is fused
constexpr float kRescaleThreshold = 8.0f;   // log2 units

struct PairParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const int32_t* perm;
  void* out;
  uint32_t* status;
  int Hq, Hkv, L, G, RP, n_groups, cpmax;
  float scale_log2;
  uint64_t wait_limit;
  int accumulate;  // 1: out[kept rows] += attention, dropped rows untouched
  int zero_fill;   // 1: warps 13-15 write the dropped rows (else a separate kernel did, or none are due)
  const uint8_t* block_mask;  // [B*Hkv][nb][nb] over 128-blocks of compacted (query, key), or null
  int nb;
  Budgets kept;
};

struct C {
  static constexpr int NS = 8;                 // ring stages: a K half or a V half each
  static constexpr int Q_BYTES = 128 * D * 2;  // one M tile of this CTA
  static constexpr int HALF_BYTES = 128 * 128; // K half: 64 keys x 128 dims; V half: 128 keys x 64 dims
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = 2 * Q_BYTES;
  static constexpr int OFF_IDX = OFF_KV + NS * HALF_BYTES;  // row tables: Q tiles (2 x 128), K/V tile (128)
  static constexpr int OFF_BAR = OFF_IDX + 3 * 128 * 4;
  // barriers: q, full[NS], empty[NS], s[2], p[2], o[2], teardown; then tmem slot, abort flag
  static constexpr int NBAR = 1 + 2 * NS + 6 + 1;
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

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1) attend_tc2(const PairParams p) {
  const uint32_t rank = cluster_ctarank();  // 0: leader (issues the MMAs), 1: peer
  const int pid = blockIdx.x >> 1;
  const int cp = p.cpmax - 1 - pid / p.n_groups;  // heaviest chunk pairs first
  const int grp = pid % p.n_groups;
  const int K = p.kept.kept[grp];
  const int P2 = 2 * p.RP;  // positions per CTA
  if (2 * cp * P2 >= K) return;  // nothing to do for this group at this pair (both CTAs leave)
  const int c = 2 * cp + (int)rank;  // this CTA's chunk (past the last kept row: no rows, still a partner)
  const int b = grp / p.Hkv, g = grp - b * p.Hkv;
  const int L = p.L;
  const int last_pos = min(K, (2 * cp + 2) * P2) - 1;  // the pair's last row
  const int n_kt = last_pos / 128 + 1;  // key tiles 0..n_kt-1
  const int32_t* pm = p.perm + (size_t)grp * L;
  // Block-sparse composition: key tile kt is processed when the block mask
  // enables it for the 128-block of any of the pair's four M tiles; every role
  // of both CTAs walks the same list of active tiles, and a tile disabled for an
  // M tile is fully masked in that tile's softmax.
  const uint8_t* bm = p.block_mask ? p.block_mask + (size_t)grp * p.nb * p.nb : nullptr;
  auto qblock = [&](int cc, int t) { return (cc * P2 + t * p.RP) / 128; };
  auto tile_on = [&](int t, int kt) -> bool { return bm == nullptr || bm[qblock(c, t) * p.nb + kt] != 0; };
  auto active = [&](int kt) -> bool {
    if (bm == nullptr) return true;
    for (int cc = 2 * cp; cc < 2 * cp + 2; ++cc)
      for (int t = 0; t < 2; ++t)
        if (bm[qblock(cc, t) * p.nb + kt] != 0) return true;
    return false;
  };
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
    // Producer lanes arrive once their copies land; the leader's q / full
    // barriers also take one relayed arrival for the peer's copies.
    const uint32_t loads = 32 * kProducerWarps + (rank == 0 ? 1 : 0);
    mbar_init(bar_q, loads);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(bar_full(s), loads);
      mbar_init(bar_empty(s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar_s(t), 1);
      mbar_init(bar_p(t), 8);  // one arrive per softmax warp of both CTAs (used on the leader)
      mbar_init(bar_o(t), 1);
    }
    mbar_init(bar_td, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {  // warp 0 of both CTAs allocates the pair's TMEM (the same columns in each)
    tmem_alloc_pair(smem_u32(tmem_slot), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // barriers initialised and TMEM allocated in both CTAs
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
    // swizzled layouts the MMA reads.  Q tiles: this CTA's 2 x 128 rows, all
    // dims.  Ring load i (K_0, V_0, K_1, ...; stage i % NS): for K, keys
    // [64 r, 64 r + 64) of the tile with all 128 dims (two 8 KB halves of 64
    // dims); for V, all 128 keys with dims [64 r, 64 r + 64).  After issuing a
    // tile every lane arrives on the tile's barrier through
    // cp.async.mbarrier.arrive (no lane waits for its own copies).  The K/V row
    // table is shared by the four producer warps (named barrier 2).
    const int pw = warp - kProducerWarp0;  // this warp owns rows [32 pw, 32 pw + 32) of the tables
    const int ptid = pw * 32 + lane;       // 0..127
    const int my_c = lane % C::CPR, my_r = lane / C::CPR;
    const uint32_t chunk_off = (uint32_t)(my_c >> 3) * 16384u;
    auto issue_q = [&](uint32_t dst, const int* tab) {
#pragma unroll 4
      for (int n = 0; n < 32 / C::RPI; ++n) {
        const int row = 32 * pw + n * C::RPI + my_r;
        const __nv_bfloat16* gsrc = p.q + (size_t)tab[row] * D + my_c * 8;
        cp_async16(dst + chunk_off + row * 128 + ((((uint32_t)my_c & 7u) ^ ((uint32_t)row & 7u)) << 4), gsrc);
      }
    };
    auto issue_k_half = [&](uint32_t dst) {  // 64 keys x 16 chunks
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        const int ci = n * 128 + ptid;
        const int rr = ci >> 4, cc = ci & 15;
        const __nv_bfloat16* gsrc = p.k + (size_t)kvtab[64 * (int)rank + rr] * D + cc * 8;
        cp_async16(dst + (uint32_t)(cc >> 3) * 8192u + rr * 128 + ((((uint32_t)cc & 7u) ^ ((uint32_t)rr & 7u)) << 4),
                   gsrc);
      }
    };
    auto issue_v_half = [&](uint32_t dst) {  // 128 keys x 8 chunks of this CTA's 64 dims
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        const int ci = n * 128 + ptid;
        const int rr = ci >> 3, cc = ci & 7;
        const __nv_bfloat16* gsrc = p.v + (size_t)kvtab[rr] * D + 64 * (int)rank + cc * 8;
        cp_async16(dst + rr * 128 + ((((uint32_t)cc) ^ ((uint32_t)rr & 7u)) << 4), gsrc);
      }
    };
    // Row tables: lane l owns row 32 pw + l of each table.
    const int my_row = 32 * pw + lane;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int hh = my_row / p.RP;
      const int pos = min(c * P2 + t * p.RP + (my_row - hh * p.RP), K - 1);
      qtab[t * 128 + my_row] = (b * p.Hq + g * p.G + hh) * L + load_pos(pm, pos, L, p.status);
    }
    __syncwarp();
    issue_q(sQ, qtab);
    issue_q(sQ + C::Q_BYTES, qtab + 128);
    cp_async_mbar_arrive(bar_q);
    const int kv_row0 = (b * p.Hkv + g) * L;
    int kt_load = next_active(-1);  // the active tile whose rows y_next holds
    int y_next = kv_row0 + load_pos(pm, min(min(kt_load, n_kt - 1) * 128 + my_row, K - 1), L, p.status);
    // The producer warps leave the loop together, at a K load (the named
    // barriers there must see all four): a warp that hit a timeout or saw the
    // abort flag only stops issuing until then.
    bool stop = false;
    for (int i = 0; i < 2 * n_act; ++i) {
      stop = stop || __any_sync(0xffffffffu, *abort_flag != 0);
      const int s = i % C::NS;
      if ((i & 1) == 0) {  // K of an active tile: its rows become current, fetch the next active tile's
        stop = named_sync_or(2u, 32u * kProducerWarps, stop);  // every producer is done with the previous table
        if (stop) break;
        kvtab[my_row] = y_next;
        named_sync(2u, 32u * kProducerWarps);  // the new table is complete
        kt_load = next_active(kt_load);
        if (kt_load < n_kt) y_next = kv_row0 + load_pos(pm, min(kt_load * 128 + my_row, K - 1), L, p.status);
      }
      if (stop) continue;
      if (i >= C::NS) {  // wait until load i - NS (same stage) has been consumed
        const bool got = mbar_wait(bar_empty(s), ((i / C::NS) - 1) & 1, p.wait_limit, abort_flag);
        if (!__all_sync(0xffffffffu, got)) {
          if (lane == 0) fail();
          stop = true;
          continue;
        }
      }
      if (i & 1) {
        issue_v_half(sKV + s * C::HALF_BYTES);
      } else {
        issue_k_half(sKV + s * C::HALF_BYTES);
      }
      cp_async_mbar_arrive(bar_full(s));
    }
    cp_async_wait_all();  // no copy is still writing shared memory when the CTA exits
  } else if (warp >= kZeroWarp0) {
    // ------------------------------------------------------------ zero fill
    const int U = p.zero_fill ? L - K : 0;  // dropped rows of this group left to this kernel
    if (U > 0) {
      const int nc = 2 * ((K + 2 * P2 - 1) / (2 * P2));  // CTAs of this group (both of every pair)
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
    if (lane == 0 && rank == 0) {
      // ---------------------------------------------------------- MMA issuer (leader)
      constexpr uint32_t IDESC_QK = idesc_bf16(256, 128, 0, 0);
      constexpr uint32_t IDESC_PV = idesc_bf16(256, D, 0, 1);
      auto commit_both = [&](uint32_t bar) {  // the same barrier in both CTAs
        tc_commit_pair(bar);
        tc_commit_pair(mapa_shared(bar, 1));
      };
      bool ok = mbar_wait(bar_q, 0, p.wait_limit, abort_flag);
      fence_proxy_async_smem();  // rows landed by cp.async (generic proxy) are read by the tensor core
      auto wait_load = [&](int i) -> bool {
        const bool got = mbar_wait(bar_full(i % C::NS), (i / C::NS) & 1, p.wait_limit, abort_flag);
        fence_proxy_async_smem();
        return got;
      };
      auto qk = [&](int t, int i_k) {
        const uint32_t kbase = sKV + (i_k % C::NS) * C::HALF_BYTES;
        const uint32_t qbase = sQ + t * C::Q_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t qoff = (kk >> 2) * 16384 + (kk & 3) * 32;
          const uint32_t koff = (kk >> 2) * 8192 + (kk & 3) * 32;
          mma_pair_bf16_ss(tmem + (uint32_t)t * 128u, sdesc_sw128(qbase + qoff, 16, 1024),
                           sdesc_sw128(kbase + koff, 16, 1024), IDESC_QK, kk > 0);
        }
      };
      // P_t (bf16, two per column) sits in the first 64 columns of S_t of each CTA.
      auto pv = [&](int t, int i_v, bool acc0) {
        const uint32_t vbase = sKV + (i_v % C::NS) * C::HALF_BYTES;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_pair_bf16_ts(tmem + C::O_COL0 + t * D, tmem + (uint32_t)t * 128u + kk * 8,
                           sdesc_sw128(vbase + kk * 2048, 16384, 1024), IDESC_PV, (acc0 || kk > 0) ? 1u : 0u);
      };
      if (ok && n_act > 0) ok = wait_load(0);
      if (ok && n_act > 0) {
        tc_fence_after();
        qk(0, 0);
        commit_both(bar_s(0));
        qk(1, 0);
        commit_both(bar_s(1));
        commit_both(bar_empty(0));  // K_0 consumed once both QKs complete
      }
      for (int j = 0; ok && j < n_act; ++j) {  // j counts active tiles
        const int iv = 2 * j + 1, ik_next = 2 * j + 2;
        if (!(ok = wait_load(iv))) break;
        for (int t = 0; t < 2 && ok; ++t) {
          if (!(ok = mbar_wait(bar_p(t), j & 1, p.wait_limit, abort_flag))) break;
          tc_fence_after();
          pv(t, iv, j > 0);
          if (t == 1) commit_both(bar_empty(iv % C::NS));  // V_j consumed
          if (j + 1 < n_act) {
            if (t == 0 && !(ok = wait_load(ik_next))) break;
            tc_fence_after();
            qk(t, ik_next);
            commit_both(bar_s(t));
            if (t == 1) commit_both(bar_empty(ik_next % C::NS));  // K_{j+1} consumed
          } else {
            commit_both(bar_o(t));
          }
        }
      }
      if (!ok) fail();
      // Drain every MMA this thread issued before TMEM is released.
      tc_commit_pair(bar_td);
      mbar_wait(bar_td, 0, kTeardownPolls, nullptr);
    } else if (lane == 0) {
      // ---------------------------------------------------------- relay (peer)
      // The peer's copies arrive on its own barriers (cp.async arrivals are
      // CTA-local); this thread forwards each completed phase to the leader's
      // barrier, in the order the leader consumes them.
      auto relay = [&](uint32_t bar, uint32_t parity) -> bool {
        if (!mbar_wait(bar, parity, p.wait_limit, abort_flag)) return false;
        fence_proxy_async_smem();  // this CTA's landed rows are visible to the tensor core
        mbar_arrive_cluster(mapa_shared(bar, 0));
        return true;
      };
      bool ok = relay(bar_q, 0);
      for (int i = 0; ok && i < 2 * n_act; ++i) ok = relay(bar_full(i % C::NS), (i / C::NS) & 1);
      if (!ok) fail();
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
      tmem_st_wait();  // P (and a rescaled O) are in TMEM before the leader's MMA thread is told
      tc_fence_before();
      __syncwarp();
      // One arrive per warp on the leader's barrier: a local arrive there, the
      // plain remote form here (a cluster-scope release measured ~1000 cycles
      // per step on this critical path; the TMEM stores are already complete).
      if (lane == 0) {
        if (rank == 0) {
          mbar_arrive(bar_p(t));
        } else {
          mbar_arrive_remote(mapa_shared(bar_p(t), 0));
        }
      }
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
  cluster_sync_all();  // no MMA, commit or remote arrive still targets either CTA
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// ---------------------------------------------------------------- host side

}  // namespace

cudaError_t launch_attend_tc_pair(const Dims& d, const void* q, const void* k, const void* v, const int32_t* perm,
                                  const Budgets& kept, void* out, uint32_t* status, bool accumulate,
                                  const uint8_t* block_mask, cudaStream_t st) {
  PairParams prm;
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
  const int cmax = (kmax + 2 * prm.RP - 1) / (2 * prm.RP);
  prm.cpmax = (cmax + 1) / 2;
  const long long nblk = 2LL * prm.cpmax * prm.n_groups;
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
  cudaError_t e = cudaFuncSetAttribute(attend_tc2, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  attend_tc2<<<(unsigned)nblk, kThreads, C::SMEM, st>>>(prm);
  count_launches(1);
  count_pair_launch();
  return cudaGetLastError();
}

}  // namespace tsa
