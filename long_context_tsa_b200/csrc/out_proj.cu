// Output projection of the scattered attention output, added in place to the
// residual stream:
//   x[b, p, :] += sum over query heads h whose KV group kept p of
//                 attn[b, h, p, :] . W_o[:, h*D : (h+1)*D]^T
// "Token Sparse Attention Long Context" (skill page), Step 3: out_proj applied
// to the attention output of the selected tokens, then the scatter back to
// full length; "Token Sparse Attention: Efficient Long-Context Inference with
// Interleaved Token Selection", Figure 3: the residual is added after the
// scatter.  Rows of attn at positions a head's group dropped are not read
// (they are zero in what tsa_attend writes); rows no group kept are untouched.
//
// With one token subset per KV group, position p is kept by a set of groups
// m_p (a bitmask).  Only the G*D columns of W_o that belong to the groups in
// m_p meet a non-zero row, so the kept positions are counting-sorted by m_p:
// tiles of consecutive sorted positions then mostly share one mask, and a
// tile's K loop runs over the groups in the OR of its positions' masks only (a
// position's row of a group outside its own mask is loaded as zeros).  The
// tensor-core work stays close to the useful sum_g K_g * G*D * N
// multiply-adds instead of the dense L * Hq*D * N.  Every output row is
// written by exactly one CTA, with no atomics, and a row's value does not
// depend on which rows share its tile (groups outside its mask add exact
// zeros, and its own groups are always visited in ascending order).
//
// Kernels: op_mask (m_p by atomic OR over every group's kept list), op_hist,
// op_scan (one CTA), op_scatter (sorted order and keys); then op_tc (bf16,
// tcgen05: persistent CTAs over (tile of 128 sorted positions, 256 output
// columns) items; A rows gathered by cp.async, B = W_o tiles by TMA, fp32
// accumulators double-buffered in TMEM, epilogue adds the residual) or
// op_simt (f32).
#include <cuda.h>

#include "device_common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"
#include "tma_maps.h"

namespace tsa {
namespace {

using namespace tc;

// ------------------------------------------------------------ sort by group mask

struct OpSortArgs {
  const int32_t* perm;
  uint32_t* mask;    // [B*L]
  uint32_t* hist;    // [NB]
  uint32_t* cursor;  // [NB]
  int32_t* order;    // [B*L] sorted b*L + p
  uint32_t* key;     // [B*L] mask of each sorted entry
  uint32_t* count;   // [0]: number of kept positions (any group)
  uint32_t* status;
  int B, Hkv, L, NB;
  Budgets kept;
};

__global__ void __launch_bounds__(256) op_mask(const OpSortArgs a) {
  const int bg = blockIdx.y;
  const int b = bg / a.Hkv, g = bg - b * a.Hkv;
  const int K = a.kept.kept[bg];
  const int32_t* pm = a.perm + (size_t)bg * a.L;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < K; i += gridDim.x * blockDim.x) {
    const int p = pm[i];
    if ((unsigned)p >= (unsigned)a.L) {
      record_status(a.status, TSA_ERR_DEVICE_BOUNDS);
      continue;
    }
    atomicOr(a.mask + (size_t)b * a.L + p, 1u << g);
  }
}

__global__ void __launch_bounds__(256) op_hist(const OpSortArgs a) {
  const long long n = (long long)a.B * a.L;
  for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < n; t += (long long)gridDim.x * blockDim.x) {
    const uint32_t m = a.mask[t];
    if (m != 0u) atomicAdd(a.hist + m, 1u);
  }
}

// Exclusive scan of the bucket counts in the order (popcount descending, then
// by mask), one CTA of 1024 threads: positions kept by more groups come first,
// so the tiles' costs (one K pass per group in a tile's mask) fall along the
// sorted order.  Thread t owns the masks m = t (mod 1024); NB <= 65536.
__global__ void __launch_bounds__(1024) op_scan(const OpSortArgs a) {
  __shared__ uint32_t part[1024];
  __shared__ uint32_t level_base;
  if (threadIdx.x == 0) level_base = 0u;
  for (int pc = a.Hkv; pc >= 1; --pc) {
    uint32_t s = 0;
    for (int m = threadIdx.x; m < a.NB; m += 1024)
      if (__popc(m) == pc) s += a.hist[m];
    part[threadIdx.x] = s;
    __syncthreads();
    for (int off = 1; off < 1024; off <<= 1) {  // inclusive Hillis-Steele scan
      const uint32_t v = threadIdx.x >= off ? part[threadIdx.x - off] : 0u;
      __syncthreads();
      part[threadIdx.x] += v;
      __syncthreads();
    }
    uint32_t run = level_base + part[threadIdx.x] - s;
    for (int m = threadIdx.x; m < a.NB; m += 1024)
      if (__popc(m) == pc) {
        a.cursor[m] = run;
        run += a.hist[m];
      }
    __syncthreads();
    if (threadIdx.x == 1023) level_base += part[1023];
    __syncthreads();
  }
  if (threadIdx.x == 0) a.count[0] = level_base;
}

__global__ void __launch_bounds__(256) op_scatter(const OpSortArgs a) {
  const long long n = (long long)a.B * a.L;
  for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < n; t += (long long)gridDim.x * blockDim.x) {
    const uint32_t m = a.mask[t];
    if (m == 0u) continue;
    const uint32_t pos = atomicAdd(a.cursor + m, 1u);
    a.order[pos] = (int32_t)t;
    a.key[pos] = m;
  }
}

// ------------------------------------------------------------ tensor-core GEMM (bf16)

constexpr int kOpEpiWarps = 8;     // warps 0-7: epilogue (lane quarter w % 4, column half w / 4)
constexpr int kOpProdWarp0 = 8;    // warps 8-11 gather A rows; warp 8 lane 0 also loads B by TMA
constexpr int kOpMmaWarp = 12;
constexpr int kOpThreads = 13 * 32;
constexpr int kOpNS = 4;           // pipeline stages
constexpr int kOpBN = 256;         // output columns per item
constexpr int kOpA_BYTES = 128 * 128;    // 128 rows x 64 bf16, 128-byte swizzle
constexpr int kOpB_BYTES = kOpBN * 128;  // 256 W_o rows x 64 bf16
constexpr int kOpSTAGE = kOpA_BYTES + kOpB_BYTES;
constexpr int kOpOFF_EPI = kOpNS * kOpSTAGE;  // epilogue staging: per warp 32 rows x 64 bf16 (4 KB)
constexpr int kOpEPI_WARP_BYTES = 32 * 128;
constexpr int kOpOFF_BAR = kOpOFF_EPI + kOpEpiWarps * kOpEPI_WARP_BYTES;
// barriers: full[NS], empty[NS], accf[2], acce[2], teardown; then tmem slot, abort flag
constexpr int kOpNBAR = 2 * kOpNS + 5;
constexpr int kOpSMEM = kOpOFF_BAR + kOpNBAR * 8 + 16 + 1024;
constexpr uint32_t kOpTeardownPolls = 1u << 26;

struct OpTcParams {
  const __nv_bfloat16* attn;  // [B, Hq, L, D]
  __nv_bfloat16* x;           // [B, L, N]
  const int32_t* order;
  const uint32_t* key;
  const uint32_t* count;
  uint32_t* status;
  int Hq, G, L, D, N, cpg, ntn;  // cpg: 64-column chunks per group (G*D/64); ntn: N / 256
  uint64_t wait_limit;
};

__device__ __forceinline__ uint32_t tile_mask(const uint32_t* key, int e0, int U, int lane) {
  uint32_t m = 0u;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int e = e0 + lane + 32 * j;
    if (e < U) m |= key[e];
  }
  return __reduce_or_sync(0xffffffffu, m);
}

// Item j of this CTA: rounds of gridDim.x items, visited in a snake order (CTA c
// takes position c of even rounds and gridDim.x - 1 - c of odd rounds), so that
// with tiles sorted by falling cost every CTA gets a near-equal share.  Returns
// -1 past the last item.
__device__ __forceinline__ int op_item(int j, int n_items) {
  const int round = j, g = (int)gridDim.x, c = (int)blockIdx.x;
  const int item = round * g + ((round & 1) ? g - 1 - c : c);
  return item < n_items ? item : -1;
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__global__ void __launch_bounds__(kOpThreads, 1)
    op_tc(const __grid_constant__ CUtensorMap tmw, const OpTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t bar0 = base + kOpOFF_BAR;
  auto bar_full = [&](int s) { return bar0 + 8u * s; };
  auto bar_empty = [&](int s) { return bar0 + 8u * (kOpNS + s); };
  auto bar_accf = [&](int i) { return bar0 + 8u * (2 * kOpNS + i); };
  auto bar_acce = [&](int i) { return bar0 + 8u * (2 * kOpNS + 2 + i); };
  const uint32_t bar_td = bar0 + 8u * (2 * kOpNS + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kOpOFF_BAR + kOpNBAR * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + kOpOFF_BAR + kOpNBAR * 8 + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kOpNS; ++s) {
      mbar_init(bar_full(s), 32 * 4 + 1);  // every producer lane's copies land; +1 for the B load
      mbar_init(bar_empty(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_accf(i), 1);
      mbar_init(bar_acce(i), 32 * kOpEpiWarps);
    }
    mbar_init(bar_td, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (warp == kOpProdWarp0 && lane == 0) tma_prefetch_map(&tmw);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto fail = [&]() {
    record_status(p.status, TSA_ERR_TIMEOUT);
    *abort_flag = 1;
  };

  const int U = (int)p.count[0];
  const int n_items = ((U + 127) / 128) * p.ntn;

  if (warp >= kOpProdWarp0 && warp < kOpMmaWarp) {
    // ------------------------------------------------------------ producers
    // Each lane's copies arrive on the stage's full barrier when they land
    // (cp.async.mbarrier.arrive): no thread waits for its own copies, so up to
    // NS stages of loads are in flight.  The next item's row table is fetched
    // while the current item's copies are issued, and the one CTA that will
    // take column tile 0 of a tile in the next round prefetches that tile's
    // kept rows into L2, so the other column tiles' gathers hit L2.
    const int pw = warp - kOpProdWarp0;  // rows [32 pw, 32 pw + 32) of every A tile
    const int my_c = lane & 7, my_r = lane >> 3;  // 16-byte chunk, row within a 4-row copy
    const bool tma_lane = pw == 0 && lane == 0;
    const int hpc = p.D / 64;  // 64-column chunks per head
    int ci = 0;                // chunks issued by this CTA
    bool ok = true;
    auto row_table = [&](int item, uint32_t& tm, uint32_t& km, long long& rbase) {
      const int tile = item / p.ntn;
      const int e0 = tile * 128;
      tm = tile_mask(p.key, e0, U, lane);
      const int e = e0 + 32 * pw + lane;
      const int tok = e < U ? p.order[e] : -1;
      km = e < U ? p.key[e] : 0u;
      // Element offset of this lane's row in head 0, (b * Hq * L + p) * D; head h adds h * L * D.
      rbase = 0;
      if (tok >= 0) {
        const int bb = tok / p.L;
        rbase = ((long long)bb * p.Hq * p.L + (tok - bb * p.L)) * p.D;
      }
    };
    uint32_t tm = 0u, km = 0u;
    long long rbase = 0;
    int item = op_item(0, n_items);
    if (item >= 0) row_table(item, tm, km, rbase);
    for (int j = 0; ok && item >= 0; ++j) {
      const int nt = item % p.ntn;
      const int next = op_item(j + 1, n_items);
      uint32_t tm_n = 0u, km_n = 0u;
      long long rb_n = 0;
      if (next >= 0) {
        row_table(next, tm_n, km_n, rb_n);
        if (next % p.ntn == 0) {  // warm L2 with the next tile's kept rows (all its column tiles read them)
          for (uint32_t rem = km_n; rem != 0u; rem &= rem - 1u) {
            const int g = __ffs(rem) - 1;
            for (int hh = 0; hh < p.G; ++hh) {
              const __nv_bfloat16* row = p.attn + (size_t)(g * p.G + hh) * p.L * p.D + rb_n;
              for (int off = 0; off < p.D; off += 64) prefetch_l2(row + off);
            }
          }
        }
      }
      const uint32_t rb_lo = (uint32_t)rbase, rb_hi = (uint32_t)((unsigned long long)rbase >> 32);
      for (uint32_t rem = tm; ok && rem != 0u; rem &= rem - 1u) {
        const int g = __ffs(rem) - 1;
        for (int kc = 0; kc < p.cpg; ++kc, ++ci) {
          if (__any_sync(0xffffffffu, *abort_flag != 0)) {
            ok = false;
            break;
          }
          const int s = ci % kOpNS;
          if (ci >= kOpNS) {
            const bool got = mbar_wait(bar_empty(s), ((ci / kOpNS) - 1) & 1, p.wait_limit, abort_flag);
            if (!__all_sync(0xffffffffu, got)) {
              if (lane == 0) fail();
              ok = false;
              break;
            }
          }
          const uint32_t sA = base + s * kOpSTAGE, sB = sA + kOpA_BYTES;
          if (tma_lane) {
            mbar_arrive_expect_tx(bar_full(s), kOpB_BYTES);
            tma_load_2d(sB, &tmw, bar_full(s), g * p.G * p.D + kc * 64, nt * kOpBN);
          }
          const int h = g * p.G + kc / hpc;
          const __nv_bfloat16* hbase = p.attn + (size_t)h * p.L * p.D + (kc % hpc) * 64 + my_c * 8;
#pragma unroll
          for (int n = 0; n < 8; ++n) {
            const int rl = n * 4 + my_r;  // row within this warp's 32
            const uint32_t m = __shfl_sync(0xffffffffu, km, rl);
            const uint32_t lo = __shfl_sync(0xffffffffu, rb_lo, rl), hi = __shfl_sync(0xffffffffu, rb_hi, rl);
            const int row = 32 * pw + rl;
            const bool live = (m >> g) & 1u;  // rows past the last entry have m = 0
            const __nv_bfloat16* src = live ? hbase + (long long)(((unsigned long long)hi << 32) | lo) : p.attn;
            cp_async16_zfill(sA + row * 128 + ((((uint32_t)my_c) ^ ((uint32_t)row & 7u)) << 4), src, live ? 16u : 0u);
          }
          cp_async_mbar_arrive(bar_full(s));
        }
      }
      item = next;
      tm = tm_n;
      km = km_n;
      rbase = rb_n;
    }
    cp_async_wait_all();
    if (tma_lane) {  // every load has landed before the CTA can exit
      for (int c = (ci > kOpNS ? ci - kOpNS : 0); c < ci; ++c)
        mbar_wait(bar_full(c % kOpNS), (c / kOpNS) & 1, kOpTeardownPolls, nullptr);
    }
  } else if (warp == kOpMmaWarp) {
    // ------------------------------------------------------------ MMA issuer (lane 0; the warp reads the tile masks)
    constexpr uint32_t IDESC = idesc_bf16(128, kOpBN, 0, 0);
    bool ok = true;
    int ci = 0;
    int item = op_item(0, n_items);
    uint32_t tm_next = item >= 0 ? tile_mask(p.key, (item / p.ntn) * 128, U, lane) : 0u;
    for (int j = 0; ok && item >= 0; ++j) {
      const uint32_t tm = tm_next;
      const int buf = j & 1;
      if (lane == 0) {
        if (j >= 2) ok = mbar_wait(bar_acce(buf), ((j >> 1) - 1) & 1, p.wait_limit, abort_flag);
        const uint32_t d = tmem + (uint32_t)buf * kOpBN;
        int kc_item = 0;
        for (uint32_t rem = tm; ok && rem != 0u; rem &= rem - 1u) {
          for (int kc = 0; kc < p.cpg; ++kc, ++ci, ++kc_item) {
            const int s = ci % kOpNS;
            if (!(ok = mbar_wait(bar_full(s), (ci / kOpNS) & 1, p.wait_limit, abort_flag))) break;
            fence_proxy_async_smem();  // the cp.async rows (generic proxy) are read by the tensor core
            tc_fence_after();
            const uint32_t sA = base + s * kOpSTAGE, sB = sA + kOpA_BYTES;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16_ss(d, sdesc_sw128(sA + kk * 32, 16, 1024), sdesc_sw128(sB + kk * 32, 16, 1024), IDESC,
                          (kc_item > 0 || kk > 0) ? 1u : 0u);
            tc_commit(bar_empty(s));
          }
        }
        if (ok) tc_commit(bar_accf(buf));
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      item = op_item(j + 1, n_items);
      if (item >= 0) tm_next = tile_mask(p.key, (item / p.ntn) * 128, U, lane);
    }
    if (lane == 0) {
      if (!ok) fail();
      tc_commit(bar_td);
      mbar_wait(bar_td, 0, kOpTeardownPolls, nullptr);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    // Warp w owns rows 32 (w % 4) .. + 31 (its TMEM lane quarter) and columns
    // 128 (w / 4) .. + 127 of the item, in two passes of 64.  The residual is
    // read, and the result written, a whole 128-byte row segment per 8 lanes
    // (lane l: row 4 i + l / 8, 16-byte chunk l % 8) through a shared-memory
    // staging tile; thread r adds its TMEM row there.  Chunk c of staging row
    // r sits at chunk c ^ (r % 8), so both access patterns are conflict-free.
    const int qw = warp & 3, half = warp >> 2;
    const uint32_t lane_off = (uint32_t)(qw * 32) << 16;
    const uint32_t stg = base + kOpOFF_EPI + warp * kOpEPI_WARP_BYTES;
    const int lc = lane & 7, lr = lane >> 3;  // chunk, row within a 4-row access
    int item = op_item(0, n_items);
    for (int j = 0; item >= 0; ++j, item = op_item(j, n_items)) {
      const int tile = item / p.ntn, nt = item - tile * p.ntn;
      const int e = tile * 128 + qw * 32 + lane;  // this thread's TMEM row
      const int tok = e < U ? p.order[e] : -1;
      // Residual of one pass, lane-distributed: 8 accesses x 4 rows x 128 B.  Pass 0's
      // is loaded before the accumulator is ready, pass 1's while pass 0 computes.
      uint4 res[8];
      const size_t col0 = (size_t)nt * kOpBN + half * 128 + lc * 8;
      auto load_res = [&](int ps) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int t = __shfl_sync(0xffffffffu, tok, 4 * i + lr);
          res[i] = t >= 0 ? __ldcs(reinterpret_cast<const uint4*>(p.x + (size_t)t * p.N + col0 + ps * 64))
                          : make_uint4(0u, 0u, 0u, 0u);
        }
      };
      load_res(0);
      const int buf = j & 1;
      const bool got = __all_sync(0xffffffffu, mbar_wait(bar_accf(buf), (j >> 1) & 1, p.wait_limit, abort_flag));
      if (!got) {
        if (lane == 0) fail();
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int ps = 0; ps < 2; ++ps) {
        uint32_t va[32], vb[32];
        const uint32_t d = tmem + lane_off + (uint32_t)buf * kOpBN + half * 128 + ps * 64;
        tmem_ld32(d, va);
        tmem_ld32(d + 32, vb);
        if (ps == 1) {  // the accumulator is free once its last columns are in registers
          tc_fence_before();
          mbar_arrive(bar_acce(buf));
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {  // residual rows into the staging tile
          const int row = 4 * i + lr;
          st_shared_v4(stg + row * 128 + (((uint32_t)lc ^ (uint32_t)(row & 7)) << 4), res[i].x, res[i].y, res[i].z,
                       res[i].w);
        }
        if (ps == 0) load_res(1);
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 8; ++c) {  // this thread's row: residual + projection, rounded once
          const uint32_t a = stg + lane * 128 + (((uint32_t)c ^ (uint32_t)(lane & 7)) << 4);
          uint32_t w4[4];
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(w4[0]), "=r"(w4[1]), "=r"(w4[2]), "=r"(w4[3])
                       : "r"(a));
          const uint32_t* v = c < 4 ? va + 8 * c : vb + 8 * (c - 4);
          uint32_t nw[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const __nv_bfloat162 hv = *reinterpret_cast<const __nv_bfloat162*>(&w4[u]);
            const float f0 = __bfloat162float(hv.x) + __uint_as_float(v[2 * u]);
            const float f1 = __bfloat162float(hv.y) + __uint_as_float(v[2 * u + 1]);
            __nv_bfloat162 o = __floats2bfloat162_rn(f0, f1);
            nw[u] = *reinterpret_cast<uint32_t*>(&o);
          }
          st_shared_v4(a, nw[0], nw[1], nw[2], nw[3]);
        }
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 8; ++i) {  // whole row segments back to global memory
          const int row = 4 * i + lr;
          const int t = __shfl_sync(0xffffffffu, tok, row);
          uint32_t w4[4];
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(w4[0]), "=r"(w4[1]), "=r"(w4[2]), "=r"(w4[3])
                       : "r"(stg + row * 128 + (((uint32_t)lc ^ (uint32_t)(row & 7)) << 4)));
          if (t >= 0)
            __stcs(reinterpret_cast<uint4*>(p.x + (size_t)t * p.N + col0 + ps * 64), make_uint4(w4[0], w4[1], w4[2], w4[3]));
        }
        __syncwarp();
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

// ------------------------------------------------------------ SIMT (f32)

constexpr int kSimtRows = 64, kSimtCols = 64, kSimtK = 16;

struct OpSimtParams {
  const float* attn;
  float* x;
  const float* w;
  const int32_t* order;
  const uint32_t* key;
  const uint32_t* count;
  int Hq, G, L, D, N, ntn;
};

__global__ void __launch_bounds__(256) op_simt(const OpSimtParams p) {
  __shared__ float As[kSimtK][kSimtRows + 1];
  __shared__ float Bs[kSimtK][kSimtCols + 1];
  __shared__ int tok[kSimtRows];
  __shared__ uint32_t kms[kSimtRows];
  __shared__ uint32_t tmask;
  const int U = (int)p.count[0];
  const int n_items = ((U + kSimtRows - 1) / kSimtRows) * p.ntn;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int K = p.Hq * p.D;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int tile = item / p.ntn, nt = item - tile * p.ntn;
    __syncthreads();
    if (threadIdx.x == 0) tmask = 0u;
    __syncthreads();
    if (threadIdx.x < kSimtRows) {
      const int e = tile * kSimtRows + threadIdx.x;
      tok[threadIdx.x] = e < U ? p.order[e] : -1;
      kms[threadIdx.x] = e < U ? p.key[e] : 0u;
      atomicOr(&tmask, kms[threadIdx.x]);
    }
    __syncthreads();
    float acc[4][4] = {};
    for (uint32_t rem = tmask; rem != 0u; rem &= rem - 1u) {
      const int g = __ffs(rem) - 1;
      for (int k0 = 0; k0 < p.G * p.D; k0 += kSimtK) {
        const int h = g * p.G + k0 / p.D, d0 = k0 % p.D;
        for (int i = threadIdx.x; i < kSimtRows * kSimtK; i += 256) {
          const int rr = i / kSimtK, kk = i - rr * kSimtK;
          const int t = tok[rr];
          float v = 0.f;
          if (t >= 0 && ((kms[rr] >> g) & 1u)) {
            const int bb = t / p.L, pp = t - bb * p.L;
            v = p.attn[(((size_t)bb * p.Hq + h) * p.L + pp) * p.D + d0 + kk];
          }
          As[kk][rr] = v;
          const int cc = i / kSimtK;
          Bs[kk][cc] = p.w[(size_t)(nt * kSimtCols + cc) * K + g * p.G * p.D + k0 + kk];
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < kSimtK; ++kk) {
          float a4[4], b4[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            a4[u] = As[kk][ty * 4 + u];
            b4[u] = Bs[kk][tx * 4 + u];
          }
#pragma unroll
          for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(a4[u], b4[v], acc[u][v]);
        }
        __syncthreads();
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int t = tok[ty * 4 + u];
      if (t < 0) continue;
      float* xr = p.x + (size_t)t * p.N + nt * kSimtCols + tx * 4;
#pragma unroll
      for (int v = 0; v < 4; ++v) xr[v] += acc[u][v];
    }
  }
}

}  // namespace

// ------------------------------------------------------------ host side

OpWsLayout out_proj_ws_layout(const Dims& d) {
  OpWsLayout w;
  auto a256 = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t n = (size_t)d.B * d.L;
  const size_t nb = size_t{1} << d.Hkv;
  size_t off = 256;  // status header
  w.count = off;  // count, then mask and hist: one contiguous region zeroed per call
  off += 16;
  w.mask = off;
  off += n * 4;
  w.hist = off;
  off += nb * 4;
  w.zero_end = off;
  off = a256(off);
  w.cursor = off;
  off = a256(off + nb * 4);
  w.order = off;
  off = a256(off + n * 4);
  w.key = off;
  off = a256(off + n * 4);
  w.total = off;
  return w;
}

cudaError_t launch_out_proj(const Dims& d, const void* attn, const int32_t* perm, const Budgets& kept,
                            const void* w_o, int N, void* x, void* ws, cudaStream_t st) {
  const OpWsLayout wl = out_proj_ws_layout(d);
  char* wsb = static_cast<char*>(ws);
  uint32_t* status = reinterpret_cast<uint32_t*>(wsb);
  cudaError_t e = cudaMemsetAsync(wsb + wl.count, 0, wl.zero_end - wl.count, st);
  if (e != cudaSuccess) return e;
  OpSortArgs a;
  a.perm = perm;
  a.mask = reinterpret_cast<uint32_t*>(wsb + wl.mask);
  a.hist = reinterpret_cast<uint32_t*>(wsb + wl.hist);
  a.cursor = reinterpret_cast<uint32_t*>(wsb + wl.cursor);
  a.order = reinterpret_cast<int32_t*>(wsb + wl.order);
  a.key = reinterpret_cast<uint32_t*>(wsb + wl.key);
  a.count = reinterpret_cast<uint32_t*>(wsb + wl.count);
  a.status = status;
  a.B = d.B;
  a.Hkv = d.Hkv;
  a.L = d.L;
  a.NB = 1 << d.Hkv;
  a.kept = kept;
  int kmax = 1;
  for (int i = 0; i < d.B * d.Hkv; ++i) kmax = kept.kept[i] > kmax ? kept.kept[i] : kmax;
  const long long n = (long long)d.B * d.L;
  const int flat_grid = (int)((n + 255) / 256 < 4 * 148 ? (n + 255) / 256 : 4 * 148);
  op_mask<<<dim3((unsigned)((kmax + 255) / 256 < 64 ? (kmax + 255) / 256 : 64), (unsigned)(d.B * d.Hkv)), 256, 0,
            st>>>(a);
  op_hist<<<flat_grid, 256, 0, st>>>(a);
  op_scan<<<1, 1024, 0, st>>>(a);
  op_scatter<<<flat_grid, 256, 0, st>>>(a);
  count_launches(4);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // Work items are read from the device count; persistent grid of one CTA per SM.
  const int max_tiles = (int)((n + 127) / 128);
  if (d.dtype == TSA_BF16) {
    CUtensorMap mw;
    if (!make_tile_map(&mw, w_o, (uint64_t)N, d.Hq * d.D, kOpBN)) return cudaErrorInvalidValue;
    OpTcParams prm;
    prm.attn = static_cast<const __nv_bfloat16*>(attn);
    prm.x = static_cast<__nv_bfloat16*>(x);
    prm.order = a.order;
    prm.key = a.key;
    prm.count = a.count;
    prm.status = status;
    prm.Hq = d.Hq;
    prm.G = d.G;
    prm.L = d.L;
    prm.D = d.D;
    prm.N = N;
    prm.cpg = d.G * d.D / 64;
    prm.ntn = N / kOpBN;
    prm.wait_limit = wait_limit();
    if ((e = cudaFuncSetAttribute(op_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, kOpSMEM)) != cudaSuccess)
      return e;
    const long long items = (long long)max_tiles * prm.ntn;
    const int grid = (int)(items < 148 ? items : 148);
    op_tc<<<grid, kOpThreads, kOpSMEM, st>>>(mw, prm);
  } else {
    OpSimtParams prm;
    prm.attn = static_cast<const float*>(attn);
    prm.x = static_cast<float*>(x);
    prm.w = static_cast<const float*>(w_o);
    prm.order = a.order;
    prm.key = a.key;
    prm.count = a.count;
    prm.Hq = d.Hq;
    prm.G = d.G;
    prm.L = d.L;
    prm.D = d.D;
    prm.N = N;
    prm.ntn = N / kSimtCols;
    const long long items = (long long)((n + kSimtRows - 1) / kSimtRows) * prm.ntn;
    const int grid = (int)(items < 8 * 148 ? items : 8 * 148);
    op_simt<<<grid, 256, 0, st>>>(prm);
  }
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace tsa
