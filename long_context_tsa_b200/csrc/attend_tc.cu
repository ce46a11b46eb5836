// Compressed causal attention on the tcgen05 tensor cores (bf16 in, fp32
// accumulate), with the gather fused into TMA tile::gather4 loads and the
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
// Warp roles (320 threads):
//   warps 0-3, 4-7  softmax + epilogue of tile 0 / tile 1 (thread = TMEM lane = row)
//   warp 8          producer: TMA gather4 of Q, K, V rows picked by perm
//   warp 9          MMA issuer (one thread): S_t = Q_t K^T, O_t += P_t V
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [256+D,256+2D).
// Shared memory: Q0 Q1 (128xD), P0 P1 (128x128 bf16), a ring of NS K/V tiles;
// every tile is K-major with the 128-byte swizzle (V is read MN-major).
//
// Online softmax in base 2 with a lazy rescale: the running max used for P
// moves only when a row max exceeds it by more than 8 (P <= 2^8), so O is
// rescaled in TMEM rarely.  Every mbarrier wait is bounded; on timeout the CTA
// records TSA_ERR_TIMEOUT, drains its own copies and MMAs, frees TMEM and exits.
#include <cuda.h>
#include <math.h>

#include "device_common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"
#include "tma_maps.h"

namespace tsa {
namespace {

using namespace tc;

constexpr int kThreads = 320;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr uint32_t kTeardownPolls = 1u << 26;
constexpr float kRescaleThreshold = 8.0f;

struct TcAttendParams {
  const int32_t* perm;
  void* out;
  uint32_t* status;
  int Hq, Hkv, L, G, RP, n_groups, cmax;
  float scale_log2;
  uint64_t wait_limit;
  Budgets kept;
};

template <int D>
struct Cfg {
  static constexpr int NS = D == 128 ? 3 : 4;        // K/V ring stages
  static constexpr int HALVES = D / 64;              // 64-column (128-byte) swizzle atoms per row
  static constexpr int Q_BYTES = 128 * D * 2;
  static constexpr int KV_BYTES = 128 * D * 2;
  static constexpr int P_BYTES = 128 * 128 * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_P = 2 * Q_BYTES;
  static constexpr int OFF_KV = OFF_P + 2 * P_BYTES;
  static constexpr int OFF_BAR = OFF_KV + NS * KV_BYTES;
  // barriers: q, full[NS], empty[NS], s[2], p[2], o[2], teardown; then tmem slot, abort flag
  static constexpr int NBAR = 1 + 2 * NS + 6 + 1;
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;  // + alignment slack
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
__global__ void __launch_bounds__(kThreads, 1)
    attend_tc(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
              const __grid_constant__ CUtensorMap tmv, const TcAttendParams p) {
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

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sQ = base + C::OFF_Q, sP = base + C::OFF_P, sKV = base + C::OFF_KV;
  const uint32_t bar0 = base + C::OFF_BAR;
  const uint32_t bar_q = bar0;
  auto bar_full = [&](int s) { return bar0 + 8u * (1 + s); };
  auto bar_empty = [&](int s) { return bar0 + 8u * (1 + C::NS + s); };
  auto bar_s = [&](int t) { return bar0 + 8u * (1 + 2 * C::NS + t); };
  auto bar_p = [&](int t) { return bar0 + 8u * (3 + 2 * C::NS + t); };
  auto bar_o = [&](int t) { return bar0 + 8u * (5 + 2 * C::NS + t); };
  const uint32_t bar_td = bar0 + 8u * (7 + 2 * C::NS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + C::OFF_BAR + C::NBAR * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + C::OFF_BAR + C::NBAR * 8 + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(bar_full(s), 1);
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
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_map(&tmq);
    tma_prefetch_map(&tmk);
    tma_prefetch_map(&tmv);
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
    // ------------------------------------------------------------ producer
    // Load i (K_0, V_0, K_1, V_1, ...) is fill number i / NS of stage i % NS.
    int issued = 0;
    // Q tiles: lane l gathers rows 4l..4l+3 of each tile.
    if (lane == 0) mbar_arrive_expect_tx(bar_q, 2 * C::Q_BYTES);
    __syncwarp();
    for (int t = 0; t < 2; ++t) {
      int y[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = 4 * lane + e;
        const int hh = r / p.RP;
        const int pos = min(c * P2 + t * p.RP + (r - hh * p.RP), K - 1);
        y[e] = (b * p.Hq + g * p.G + hh) * L + load_pos(pm, pos, L, p.status);
      }
#pragma unroll
      for (int h = 0; h < C::HALVES; ++h)
        tma_gather4(sQ + t * C::Q_BYTES + h * 16384 + lane * 512, &tmq, bar_q, 64 * h, y[0], y[1], y[2], y[3]);
    }
    const int kv_row0 = (b * p.Hkv + g) * L;
    for (int i = 0; i < 2 * n_kt; ++i) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
      const int j = i >> 1;
      const int s = i % C::NS;
      if (i >= C::NS) {  // wait until load i - NS (same stage) has been consumed
        const bool got = mbar_wait(bar_empty(s), ((i / C::NS) - 1) & 1, p.wait_limit, abort_flag);
        if (!__all_sync(0xffffffffu, got)) {
          if (lane == 0) fail();
          break;
        }
      }
      int y[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int kidx = min(j * 128 + 4 * lane + e, K - 1);
        y[e] = kv_row0 + load_pos(pm, kidx, L, p.status);
      }
      if (lane == 0) mbar_arrive_expect_tx(bar_full(s), C::KV_BYTES);
      __syncwarp();
      const CUtensorMap* map = (i & 1) ? &tmv : &tmk;
#pragma unroll
      for (int h = 0; h < C::HALVES; ++h)
        tma_gather4(sKV + s * C::KV_BYTES + h * 16384 + lane * 512, map, bar_full(s), 64 * h, y[0], y[1], y[2], y[3]);
      issued = i + 1;
    }
    // Drain after an abort: wait for the copies this warp issued (a fixed limit,
    // independent of the debug wait limit) before the CTA can exit.
    if (*abort_flag) {
      mbar_wait(bar_q, 0, kTeardownPolls, nullptr);
      for (int i = (issued > C::NS ? issued - C::NS : 0); i < issued; ++i)
        mbar_wait(bar_full(i % C::NS), (i / C::NS) & 1, kTeardownPolls, nullptr);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_QK = idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t IDESC_PV = idesc_bf16(128, D, 0, 1);
      bool ok = mbar_wait(bar_q, 0, p.wait_limit, abort_flag);
      auto wait_load = [&](int i) -> bool {
        return mbar_wait(bar_full(i % C::NS), (i / C::NS) & 1, p.wait_limit, abort_flag);
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
      auto pv = [&](int t, int i_v, bool acc0) {
        const uint32_t vbase = sKV + (i_v % C::NS) * C::KV_BYTES;
        const uint32_t pbase = sP + t * C::P_BYTES;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t aoff = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16_ss(tmem + C::O_COL0 + t * D, sdesc_sw128(pbase + aoff, 16, 1024),
                      sdesc_sw128(vbase + kk * 2048, 16384, 1024), IDESC_PV, (acc0 || kk > 0) ? 1u : 0u);
        }
      };
      if (ok) ok = wait_load(0);
      if (ok) {
        tc_fence_after();
        qk(0, 0);
        tc_commit(bar_s(0));
        qk(1, 0);
        tc_commit(bar_s(1));
        tc_commit(bar_empty(0));  // K_0 consumed once both QKs complete
      }
      for (int j = 0; ok && j < n_kt; ++j) {
        const int iv = 2 * j + 1, ik_next = 2 * j + 2;
        if (!(ok = wait_load(iv))) break;
        for (int t = 0; t < 2 && ok; ++t) {
          if (!(ok = mbar_wait(bar_p(t), j & 1, p.wait_limit, abort_flag))) break;
          tc_fence_after();
          pv(t, iv, j > 0);
          if (t == 1) tc_commit(bar_empty(iv % C::NS));  // V_j consumed
          if (j + 1 < n_kt) {
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
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int t = warp >> 2;
    const int r = threadIdx.x & 127;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + (uint32_t)t * 128u;
    const uint32_t tO = tmem + lane_off + C::O_COL0 + t * D;
    const int hh = r / p.RP;
    const int pos = c * P2 + t * p.RP + (r - hh * p.RP);
    const uint32_t prow = sP + t * C::P_BYTES + r * 128;
    const uint32_t sw = (uint32_t)(r & 7);
    float m_use = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kt; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar_s(t), j & 1, p.wait_limit, abort_flag));
      if (!ok) break;
      tc_fence_after();
      float x[128];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t v[32];
        tmem_ld32(tS + q4 * 32, v);
#pragma unroll
        for (int e = 0; e < 32; ++e) x[q4 * 32 + e] = __uint_as_float(v[e]) * p.scale_log2;
      }
      const int nvis = pos - j * 128 + 1;  // visible keys in this tile (causal)
      if (nvis < 128) {
#pragma unroll
        for (int e = 0; e < 128; ++e)
          if (e >= nvis) x[e] = -INFINITY;
      }
      float mt = -INFINITY;
#pragma unroll
      for (int e = 0; e < 128; ++e) mt = fmaxf(mt, x[e]);
      // Lazy rescale: move the reference max only when the tile max exceeds
      // it by more than the threshold (then alpha = 2^(old - new) rescales l
      // and O; P stays <= 2^threshold otherwise).
      const bool need = mt > m_use + kRescaleThreshold;
      const float alpha = need ? ex2_approx(m_use - mt) : 1.f;  // 0 when m_use is -inf
      if (need) {
        l *= alpha;
        m_use = mt;
      }
      float rs = 0.f;
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {
        uint32_t w4[4];
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) {
          const float p0 = ex2_approx(x[ch * 8 + 2 * e2] - m_use);
          const float p1 = ex2_approx(x[ch * 8 + 2 * e2 + 1] - m_use);
          rs += p0 + p1;
          w4[e2] = pack_bf16(p0, p1);
        }
        const uint32_t addr = prow + (ch >> 3) * 16384 + ((((uint32_t)ch & 7u) ^ sw) << 4);
        st_shared_v4(addr, w4[0], w4[1], w4[2], w4[3]);
      }
      l += rs;
      // O_t is idle here (the commit that released S_t(j) covers PV(t, j-1)).
      // TMEM access is warp-collective, so the whole warp rescales when any
      // lane needs it (alpha = 1 for the others).
      if (j > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll
        for (int q4 = 0; q4 < D / 32; ++q4) {
          uint32_t v[32];
          tmem_ld32(tO + q4 * 32, v);
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
          tmem_st32(tO + q4 * 32, v);
        }
        tmem_st_wait();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar_p(t));
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_o(t), 0, p.wait_limit, abort_flag));
    if (!ok) {
      fail();
    } else {
      tc_fence_after();
      const bool valid = pos < K;
      const int opos = valid ? load_pos(pm, pos, L, p.status) : 0;
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.out) + ((size_t)(b * p.Hq + g * p.G + hh) * L + opos) * D;
      const float inv = 1.f / l;
#pragma unroll
      for (int q4 = 0; q4 < D / 32; ++q4) {
        uint32_t v[32];
        tmem_ld32(tO + q4 * 32, v);  // warp-collective: every lane loads, valid rows store
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + q4 * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            uint4 o;
            o.x = pack_bf16(__uint_as_float(v[8 * e + 0]) * inv, __uint_as_float(v[8 * e + 1]) * inv);
            o.y = pack_bf16(__uint_as_float(v[8 * e + 2]) * inv, __uint_as_float(v[8 * e + 3]) * inv);
            o.z = pack_bf16(__uint_as_float(v[8 * e + 4]) * inv, __uint_as_float(v[8 * e + 5]) * inv);
            o.w = pack_bf16(__uint_as_float(v[8 * e + 6]) * inv, __uint_as_float(v[8 * e + 7]) * inv);
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
                      const Budgets& kept, void* out, uint32_t* status, cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  if (!make_row_map(&mq, q, (uint64_t)d.B * d.Hq * d.L, D) || !make_row_map(&mk, k, (uint64_t)d.B * d.Hkv * d.L, D) ||
      !make_row_map(&mv, v, (uint64_t)d.B * d.Hkv * d.L, D))
    return cudaErrorInvalidValue;
  TcAttendParams prm;
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
  prm.kept = kept;
  int kmax = 0;
  for (int i = 0; i < prm.n_groups; ++i) kmax = kept.kept[i] > kmax ? kept.kept[i] : kmax;
  prm.cmax = (kmax + 2 * prm.RP - 1) / (2 * prm.RP);
  const int smem = Cfg<D>::SMEM;
  cudaError_t e = cudaFuncSetAttribute(attend_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const long long nblk = (long long)prm.cmax * prm.n_groups;
  attend_tc<D><<<(unsigned)nblk, kThreads, smem, st>>>(mq, mk, mv, prm);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attend_tc(const Dims& d, const void* q, const void* k, const void* v, const int32_t* perm,
                             const Budgets& kept, void* out, uint32_t* status, cudaStream_t st) {
  return d.D == 64 ? launch_tc<64>(d, q, k, v, perm, kept, out, status, st)
                   : launch_tc<128>(d, q, k, v, perm, kept, out, status, st);
}

}  // namespace tsa
