// Projection GEMM on the 5th-generation tensor cores: D = A B with bf16 operands, fp32 accumulation
// in TMEM and a bf16 (or fp32) result, for the projections either side of the decode path (GQLA
// explainer, section 2 "Methodology": W_UK folded into the query, W_UV after attention, the latent
// expanded into per-group keys and values; and the output projection after attention).
//
// Every projection is written with the large dimension as the MMA's M (rows of A, 128 per tile):
//   A rows   are K-major (the contraction is the row's unit-stride axis) and addressed through a
//            3-D tensor map {K, n1, n2}: a tile is a box of b1 x b2 rows (b1 * b2 = 128), which lets a
//            tile gather the rows of one head group across tokens (q[t, h, :] for h in a group).
//   B        is either K-major ([N, K] rows, W_UK[j]) or MN-major ([K, N] with unit stride along N,
//            W_UV[j], the expansion weights, W_O), 3-D {.., .., matrix index}.  The matrix a tile
//            uses comes from its rows (the head group) or from its columns (the expansion's groups
//            side by side).
// A tile is 128 rows x tn columns (tn a multiple of 64, <= 256); the K loop streams 64-wide blocks
// of A (16 KB) and B (tn x 128 bytes) through a ring of shared-memory stages.
//
// Warps: 0 TMA producer; 1 TMEM allocator and MMA issuer; 2-9 epilogue (warp w reads TMEM lane
// quadrant w % 4, column half (w - 2) / 4).  The kernel is persistent over tiles (grid = SM count at
// most) and double-buffers the accumulator in TMEM (2 x 256 columns), so a tile's epilogue overlaps
// the next tile's MMAs.  Every wait is bounded and records its site in the device error word.
#pragma once
#include <cstdint>
#include <cuda.h>
#include "lkv_ptx.cuh"
#include "../../include/lkv.h"

namespace lkv {

constexpr int kGemmThreads = 320;
constexpr int kGemmStages = 4;
constexpr int kGemmABytes = 16384;      // 128 rows x 64 K (bf16)
constexpr int kGemmBBytes = 32768;      // up to 256 N x 64 K (bf16)
constexpr int kGemmStageBytes = kGemmABytes + kGemmBBytes;
constexpr size_t kGemmSmemBytes = 1024 + static_cast<size_t>(kGemmStages) * kGemmStageBytes;
constexpr uint32_t kGemmTmemCols = 512;  // two accumulators of up to 256 columns
static_assert(kGemmSmemBytes <= 232448 - 1024, "shared memory budget");

// Wait sites of this kernel (added to LKV_SITE_WAIT_BASE in the error word; above the decode kernels').
enum GemmWaitSite { GW_EMPTY = LKV_SITE_WAIT_BASE + 120, GW_FULL, GW_TEMPTY, GW_TFULL, GW_DRAIN };

struct GemmParams {
  int k_blocks;       // ceil(K / 64)
  int tn;             // columns per tile (multiple of 64, <= 256)
  int n_tiles;        // tiles along the columns
  int n_valid;        // columns of the result (per group on the group axis)
  int b1, lg_b1, b2;  // rows of a tile along A's dims 1 and 2 (b1 a power of two, b1 * b2 = 128)
  int n1, n2;         // A's row extents
  int t1, t2;         // tiles along A's dims 1 and 2
  int rows_per_b;     // rows of dim 1 that share one B matrix (heads per group); 0: not row-selected
  int groups;         // B matrices applied to every row as separate column blocks (else 1)
  int nb;             // columns of one B matrix when the column axis spans several side by side
  int b_mn;           // B is MN-major
  int b_bytes;        // B bytes per stage
  int out_fp32;
  int vec_ok;         // every row start and column block is 16-byte aligned
  long long os1, os2; // result offset (elements) per unit of A's dims 1 and 2
  long long ocol;     // result column offset per group
  int total_tiles;
  void* out;
  int* err;
  unsigned long long wait_limit_ns;
  int m_tiles;        // weight-resident kernel: row tiles per column tile (t1 * t2)
  int res_groups;     // weight-resident kernel: CTAs per column tile (grid = res_groups * n_tiles)
};

struct __align__(8) GemmSmem {
  uint64_t full[kGemmStages];   // A and B of the stage landed
  uint64_t empty[kGemmStages];  // the MMAs reading the stage are done
  uint64_t tfull[2];            // accumulator b holds a finished tile
  uint64_t tempty[2];           // the 8 epilogue warps read accumulator b
  uint64_t drain;               // every MMA issued is complete
  uint32_t tmem_base;
  uint32_t abort;
  uint32_t zero;                // abort flag of the drain waits: never set
  int fills, consumed;
};

struct GemmTile {
  int nt, i1, i2, g;
};
__device__ __forceinline__ GemmTile gemm_tile(const GemmParams& p, int t) {
  GemmTile x;
  x.nt = t % p.n_tiles;
  t /= p.n_tiles;
  x.i1 = t % p.t1;
  t /= p.t1;
  x.i2 = t % p.t2;
  x.g = t / p.t2;
  return x;
}

// 32 consecutive fp32 results of one row (`n` of them in range) to global memory.
__device__ __forceinline__ void gemm_store32(const GemmParams& p, long long off, const uint32_t (&v)[32], int n) {
  if (n <= 0) return;
  if (p.out_fp32) {
    float* o = static_cast<float*>(p.out) + off;
    if (p.vec_ok && n >= 32) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        reinterpret_cast<uint4*>(o)[i] = make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (i < n) o[i] = __uint_as_float(v[i]);
    }
    return;
  }
  uint32_t h[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) h[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
  uint16_t* o = static_cast<uint16_t*>(p.out) + off;
  if (p.vec_ok && n >= 32) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      reinterpret_cast<uint4*>(o)[i] = make_uint4(h[4 * i], h[4 * i + 1], h[4 * i + 2], h[4 * i + 3]);
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i < n) o[i] = static_cast<uint16_t>(h[i >> 1] >> (16 * (i & 1)));
  }
}

// One epilogue warp's share of a finished tile: TMEM lane quadrant qd (row m of the tile), column
// half `half`, from the accumulator at TMEM address `acc` to the result rows.
__device__ __forceinline__ void gemm_store_tile(const GemmParams& p, const GemmTile& x, uint32_t acc, int qd, int half,
                                                int m) {
  const int hc = p.tn >> 1;
  const int u1 = x.i1 * p.b1 + (m & (p.b1 - 1));
  const int u2 = x.i2 * p.b2 + (m >> p.lg_b1);
  const bool row_ok = u1 < p.n1 && u2 < p.n2;
  const long long row_off = u1 * p.os1 + u2 * p.os2 + x.g * p.ocol;
  for (int c = half * hc; c < (half + 1) * hc; c += 32) {
    uint32_t v[32];
    tmem_ld32(acc + (static_cast<uint32_t>(32 * qd) << 16) + c, v);
    tmem_wait_ld();
    const int col = x.nt * p.tn + c;
    if (row_ok) gemm_store32(p, row_off + col, v, p.n_valid - col);
  }
}

__global__ void __launch_bounds__(kGemmThreads, 1)
    proj_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                     const GemmParams p) {
  extern __shared__ __align__(1024) uint8_t gemm_smem_raw[];
  __shared__ GemmSmem sm;
  uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gemm_smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  const uint32_t ring = smem_u32(dsm);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr int S = kGemmStages;
  auto bar = [](const uint64_t& b) { return smem_u32(&b); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(bar(sm.full[s]), 1);
      mbar_init(bar(sm.empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(sm.tfull[b]), 1);
      mbar_init(bar(sm.tempty[b]), 8);
    }
    mbar_init(bar(sm.drain), 1);
    sm.abort = 0;
    sm.zero = 0;
    sm.fills = 0;
    sm.consumed = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&sm.tmem_base), kGemmTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const WaitCtl wc{&sm.abort, p.err, p.wait_limit_ns};
  const WaitCtl wd{&sm.zero, p.err, p.wait_limit_ns};

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      tma_prefetch_desc(&map_a);
      tma_prefetch_desc(&map_b);
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < p.total_tiles; t += gridDim.x) {
        const GemmTile x = gemm_tile(p, t);
        const int row_b = p.rows_per_b ? (x.i1 * p.b1) / p.rows_per_b : 0;
        const int c_tile = x.nt * p.tn;
        for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
          const int s = it % S;
          if (!mbar_wait(bar(sm.empty[s]), ((it / S) & 1) ^ 1, wc, GW_EMPTY)) {
            ok = false;
            break;
          }
          const uint32_t a_dst = ring + s * kGemmStageBytes;
          const uint32_t b_dst = a_dst + kGemmABytes;
          const uint32_t fb = bar(sm.full[s]);
          mbar_arrive_expect_tx(fb, kGemmABytes + p.b_bytes);
          tma_load_3d(a_dst, &map_a, fb, kb * 64, x.i1 * p.b1, x.i2 * p.b2);
          if (p.b_mn) {
            for (int a = 0; a < (p.tn >> 6); ++a) {
              const int c0 = c_tile + 64 * a;
              tma_load_3d(b_dst + a * 8192, &map_b, fb, c0 % p.nb, kb * 64, x.g + row_b + c0 / p.nb);
            }
          } else {
            tma_load_3d(b_dst, &map_b, fb, kb * 64, c_tile, x.g + row_b);
          }
          sm.fills = it + 1;
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, p.tn, 0, p.b_mn);
      const uint32_t bstep = p.b_mn ? 2048u : 32u;  // one K step of 16: 16 rows of 128 B, or 32 B in a row
      const uint32_t blbo = p.b_mn ? 8192u : 16u;   // MN-major: 64-column blocks 8 KB apart
      int it = 0, lt = 0;
      bool issued = false, ok = true;
      for (int t = blockIdx.x; ok && t < p.total_tiles; t += gridDim.x, ++lt) {
        const int buf = lt & 1;
        if (!mbar_wait(bar(sm.tempty[buf]), ((lt >> 1) & 1) ^ 1, wc, GW_TEMPTY)) break;
        tc_fence_after();
        const uint32_t d = tmem + 256u * buf;
        for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
          const int s = it % S;
          if (!mbar_wait(bar(sm.full[s]), (it / S) & 1, wc, GW_FULL)) {
            ok = false;
            break;
          }
          sm.consumed = it + 1;
          tc_fence_after();
          const uint32_t a_addr = ring + s * kGemmStageBytes;
          const uint64_t ad = sdesc_sw128(a_addr, 16, 1024);
          const uint64_t bd = sdesc_sw128(a_addr + kGemmABytes, blbo, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_ss(d, desc_add(ad, kk * 32), desc_add(bd, kk * bstep), idesc, (kb | kk) ? 1u : 0u);
          issued = true;
          umma_commit(bar(sm.empty[s]));
        }
        if (ok) umma_commit(bar(sm.tfull[buf]));
      }
      if (issued) {
        umma_commit(bar(sm.drain));
        mbar_wait(bar(sm.drain), 0, wd, GW_DRAIN);
      }
    }
  } else {
    // ---------------- epilogue: TMEM -> registers -> global ----------------
    const int qd = warp & 3;
    const int half = (warp - 2) >> 2;
    const int m = 32 * qd + lane;
    int lt = 0;
    for (int t = blockIdx.x; t < p.total_tiles; t += gridDim.x, ++lt) {
      const GemmTile x = gemm_tile(p, t);
      const int buf = lt & 1;
      if (!mbar_wait(bar(sm.tfull[buf]), (lt >> 1) & 1, wc, GW_TFULL)) break;
      tc_fence_after();
      gemm_store_tile(p, x, tmem + 256u * buf, qd, half, m);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(sm.tempty[buf]));
    }
  }

  // Loads the MMA never waited for (after an abort) must land before the CTA's shared memory goes.
  __syncthreads();
  if (warp == 0 && lane == 0)
    for (int i = sm.consumed; i < sm.fills; ++i) mbar_wait(bar(sm.full[i % S]), (i / S) & 1, wd, GW_DRAIN);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kGemmTmemCols);
  }
}

// ------------------------------------------------------------------------------------------
// Weight-resident form, for an MN-major B shared by every row (the expansion, or an output
// projection with K <= 512): each CTA keeps one column tile's whole B (K x 128 columns) in shared
// memory for the whole launch and streams only A, so a tile's shared-memory fill is its 128 rows of
// A (the measured TMA fill of one SM, ~83 GB/s from L2, is what bounds the streaming form).  CTA i
// owns column tile i % n_tiles and row tiles i / n_tiles, + res_groups, ...: the n_tiles CTAs that
// need one row tile's A take it at about the same time, so it comes from HBM once and from L2 for
// the rest.  A streams in stages of two 64-wide K blocks (32 KB).  (Asking L2 for the next row
// tile's A ahead of time was measured slower.)
// ------------------------------------------------------------------------------------------
constexpr int kResTn = 128;                              // columns per tile
constexpr int kResMaxK = 512;                            // K of the resident B
constexpr int kResBBytes = kResMaxK * kResTn * 2;        // 128 KB
constexpr int kResStages = 3;
constexpr int kResStageBytes = 2 * kGemmABytes;          // two K blocks of A
constexpr size_t kResSmemBytes = 1024 + kResBBytes + static_cast<size_t>(kResStages) * kResStageBytes;
static_assert(kResSmemBytes <= 232448 - 1024, "shared memory budget");

struct __align__(8) GemmResSmem {
  uint64_t full[kResStages], empty[kResStages];
  uint64_t tfull[2], tempty[2];
  uint64_t bfull;     // the resident B landed
  uint64_t drain;
  uint32_t tmem_base, abort, zero;
  int fills, consumed, bloads;
};

__global__ void __launch_bounds__(kGemmThreads, 1)
    proj_gemm_resident_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                              const GemmParams p) {
  extern __shared__ __align__(1024) uint8_t gemm_res_raw[];
  __shared__ GemmResSmem sm;
  uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gemm_res_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  const uint32_t bres = smem_u32(dsm);
  const uint32_t ring = bres + kResBBytes;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr int S = kResStages;
  auto bar = [](const uint64_t& b) { return smem_u32(&b); };
  // this CTA's column tile and first row tile; its row tiles step by res_groups
  const int nt = blockIdx.x % p.n_tiles;
  const int mt0 = blockIdx.x / p.n_tiles;
  const int kpairs = (p.k_blocks + 1) >> 1;              // A stages per tile
  const uint32_t batom = static_cast<uint32_t>(p.k_blocks) * 8192u;  // bytes of one 64-column atom of B
  auto tile_of = [&](int mt) {
    GemmTile x;
    x.nt = nt;
    x.i1 = mt % p.t1;
    x.i2 = mt / p.t1;
    x.g = 0;
    return x;
  };

  if (threadIdx.x == 0) {
    for (int s2 = 0; s2 < S; ++s2) {
      mbar_init(bar(sm.full[s2]), 1);
      mbar_init(bar(sm.empty[s2]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(sm.tfull[b]), 1);
      mbar_init(bar(sm.tempty[b]), 8);
    }
    mbar_init(bar(sm.bfull), 1);
    mbar_init(bar(sm.drain), 1);
    sm.abort = 0;
    sm.zero = 0;
    sm.fills = 0;
    sm.consumed = 0;
    sm.bloads = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&sm.tmem_base), kGemmTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const WaitCtl wc{&sm.abort, p.err, p.wait_limit_ns};
  const WaitCtl wd{&sm.zero, p.err, p.wait_limit_ns};

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      tma_prefetch_desc(&map_a);
      tma_prefetch_desc(&map_b);
      int it = 0;
      bool ok = true;
      if (mt0 < p.m_tiles) {
        // this column tile's B, once
        mbar_arrive_expect_tx(bar(sm.bfull), static_cast<uint32_t>(2 * batom));
        for (int a = 0; a < 2; ++a) {
          const int c0 = nt * kResTn + 64 * a;
          for (int kb = 0; kb < p.k_blocks; ++kb)
            tma_load_3d(bres + a * batom + kb * 8192, &map_b, bar(sm.bfull), c0 % p.nb, kb * 64, c0 / p.nb);
        }
        sm.bloads = 1;
      }
      for (int mt = mt0; ok && mt < p.m_tiles; mt += p.res_groups) {
        const GemmTile x = tile_of(mt);
        for (int kp = 0; kp < kpairs; ++kp, ++it) {
          const int s2 = it % S;
          if (!mbar_wait(bar(sm.empty[s2]), ((it / S) & 1) ^ 1, wc, GW_EMPTY)) {
            ok = false;
            break;
          }
          const int nkb = (2 * kp + 1 < p.k_blocks) ? 2 : 1;
          const uint32_t fb = bar(sm.full[s2]);
          mbar_arrive_expect_tx(fb, static_cast<uint32_t>(nkb * kGemmABytes));
          for (int j = 0; j < nkb; ++j)
            tma_load_3d(ring + s2 * kResStageBytes + j * kGemmABytes, &map_a, fb, (2 * kp + j) * 64, x.i1 * p.b1,
                        x.i2 * p.b2);
          sm.fills = it + 1;
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, kResTn, 0, 1);
      const uint64_t bd0 = sdesc_sw128(bres, batom, 1024);  // MN-major: 64-column atoms batom apart
      int it = 0, lt = 0;
      bool issued = false;
      bool ok = mt0 >= p.m_tiles || mbar_wait(bar(sm.bfull), 0, wc, GW_FULL);
      for (int mt = mt0; ok && mt < p.m_tiles; mt += p.res_groups, ++lt) {
        const int buf = lt & 1;
        if (!mbar_wait(bar(sm.tempty[buf]), ((lt >> 1) & 1) ^ 1, wc, GW_TEMPTY)) break;
        tc_fence_after();
        const uint32_t d = tmem + 256u * buf;
        for (int kp = 0; kp < kpairs; ++kp, ++it) {
          const int s2 = it % S;
          if (!mbar_wait(bar(sm.full[s2]), (it / S) & 1, wc, GW_FULL)) {
            ok = false;
            break;
          }
          sm.consumed = it + 1;
          tc_fence_after();
          const int nkb = (2 * kp + 1 < p.k_blocks) ? 2 : 1;
          for (int j = 0; j < nkb; ++j) {
            const int kb = 2 * kp + j;
            const uint64_t ad = sdesc_sw128(ring + s2 * kResStageBytes + j * kGemmABytes, 16, 1024);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_ss(d, desc_add(ad, kk * 32), desc_add(bd0, kb * 8192 + kk * 2048), idesc, (kb | kk) ? 1u : 0u);
          }
          issued = true;
          umma_commit(bar(sm.empty[s2]));
        }
        if (!ok) break;
        umma_commit(bar(sm.tfull[buf]));
      }
      if (issued) {
        umma_commit(bar(sm.drain));
        mbar_wait(bar(sm.drain), 0, wd, GW_DRAIN);
      }
    }
  } else {
    // ---------------- epilogue ----------------
    const int qd = warp & 3;
    const int half = (warp - 2) >> 2;
    const int m = 32 * qd + lane;
    int lt = 0;
    for (int mt = mt0; mt < p.m_tiles; mt += p.res_groups, ++lt) {
      const GemmTile x = tile_of(mt);
      const int buf = lt & 1;
      if (!mbar_wait(bar(sm.tfull[buf]), (lt >> 1) & 1, wc, GW_TFULL)) break;
      tc_fence_after();
      gemm_store_tile(p, x, tmem + 256u * buf, qd, half, m);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(sm.tempty[buf]));
    }
  }

  // Copies the MMA never waited for (after an abort) must land before the CTA's shared memory goes.
  __syncthreads();
  if (warp == 0 && lane == 0) {
    for (int i = sm.consumed; i < sm.fills; ++i) mbar_wait(bar(sm.full[i % S]), (i / S) & 1, wd, GW_DRAIN);
    if (sm.bloads > 0) mbar_wait(bar(sm.bfull), (sm.bloads - 1) & 1, wd, GW_DRAIN);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kGemmTmemCols);
  }
}

// ------------------------------------------------------------------------------------------
// Split-K form, for few output tiles over a long K (a decode-size output projection: 64 tokens,
// K = 16384): the S CTAs of a cluster (S = 2, 4 or 8) take one tile and a contiguous S-th of its K
// blocks each.  Each CTA parks its fp32 partial tile in its own shared memory (the ring is free by
// then); after a cluster barrier CTA c sums rows [c * 128 / S, (c + 1) * 128 / S) of all S partials
// through distributed shared memory, in rank order (deterministic), and stores them.  Streaming
// producer and MMA as in proj_gemm_kernel, one tile per cluster.
// ------------------------------------------------------------------------------------------
constexpr int kSplitRowPitch = 256 * 4 + 16;  // bytes per partial row (padded against bank conflicts)
static_assert(128 * kSplitRowPitch <= kGemmStages * kGemmStageBytes, "partial tile fits the ring");

__global__ void __launch_bounds__(kGemmThreads, 1)
    proj_gemm_splitk_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                            const GemmParams p, int splits) {
  extern __shared__ __align__(1024) uint8_t gemm_sk_raw[];
  __shared__ GemmSmem sm;
  uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gemm_sk_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  const uint32_t ring = smem_u32(dsm);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr int S = kGemmStages;
  auto bar = [](const uint64_t& b) { return smem_u32(&b); };
  const int rank = static_cast<int>(cluster_ctarank());
  const int tile = blockIdx.x / splits;
  const int kb0 = static_cast<int>(static_cast<long long>(p.k_blocks) * rank / splits);
  const int kb1 = static_cast<int>(static_cast<long long>(p.k_blocks) * (rank + 1) / splits);
  const GemmTile x = gemm_tile(p, tile);

  if (threadIdx.x == 0) {
    for (int s2 = 0; s2 < S; ++s2) {
      mbar_init(bar(sm.full[s2]), 1);
      mbar_init(bar(sm.empty[s2]), 1);
    }
    mbar_init(bar(sm.tfull[0]), 1);
    mbar_init(bar(sm.drain), 1);
    sm.abort = 0;
    sm.zero = 0;
    sm.fills = 0;
    sm.consumed = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&sm.tmem_base), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const WaitCtl wc{&sm.abort, p.err, p.wait_limit_ns};
  const WaitCtl wd{&sm.zero, p.err, p.wait_limit_ns};
  bool have = false;  // epilogue: this CTA's partial is in TMEM

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&map_a);
      tma_prefetch_desc(&map_b);
      const int row_b = p.rows_per_b ? (x.i1 * p.b1) / p.rows_per_b : 0;
      const int c_tile = x.nt * p.tn;
      for (int kb = kb0, it = 0; kb < kb1; ++kb, ++it) {
        const int s2 = it % S;
        if (!mbar_wait(bar(sm.empty[s2]), ((it / S) & 1) ^ 1, wc, GW_EMPTY)) break;
        const uint32_t a_dst = ring + s2 * kGemmStageBytes;
        const uint32_t b_dst = a_dst + kGemmABytes;
        const uint32_t fb = bar(sm.full[s2]);
        mbar_arrive_expect_tx(fb, kGemmABytes + p.b_bytes);
        tma_load_3d(a_dst, &map_a, fb, kb * 64, x.i1 * p.b1, x.i2 * p.b2);
        if (p.b_mn) {
          for (int a = 0; a < (p.tn >> 6); ++a) {
            const int c0 = c_tile + 64 * a;
            tma_load_3d(b_dst + a * 8192, &map_b, fb, c0 % p.nb, kb * 64, x.g + row_b + c0 / p.nb);
          }
        } else {
          tma_load_3d(b_dst, &map_b, fb, kb * 64, c_tile, x.g + row_b);
        }
        sm.fills = it + 1;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, p.tn, 0, p.b_mn);
      const uint32_t bstep = p.b_mn ? 2048u : 32u;
      const uint32_t blbo = p.b_mn ? 8192u : 16u;
      bool issued = false, ok = true;
      for (int kb = kb0, it = 0; kb < kb1; ++kb, ++it) {
        const int s2 = it % S;
        if (!mbar_wait(bar(sm.full[s2]), (it / S) & 1, wc, GW_FULL)) {
          ok = false;
          break;
        }
        sm.consumed = it + 1;
        tc_fence_after();
        const uint32_t a_addr = ring + s2 * kGemmStageBytes;
        const uint64_t ad = sdesc_sw128(a_addr, 16, 1024);
        const uint64_t bd = sdesc_sw128(a_addr + kGemmABytes, blbo, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_ss(tmem, desc_add(ad, kk * 32), desc_add(bd, kk * bstep), idesc, (it | kk) ? 1u : 0u);
        issued = true;
        umma_commit(bar(sm.empty[s2]));
      }
      if (ok && issued) umma_commit(bar(sm.tfull[0]));
      if (issued) {
        umma_commit(bar(sm.drain));
        mbar_wait(bar(sm.drain), 0, wd, GW_DRAIN);
      }
    }
  } else {
    // park this CTA's partial: TMEM lane quadrant qd, column half `half`
    const int qd = warp & 3;
    const int half = (warp - 2) >> 2;
    const int m = 32 * qd + lane;
    have = kb1 > kb0 && mbar_wait(bar(sm.tfull[0]), 0, wc, GW_TFULL);
    have = __all_sync(0xffffffffu, have) != 0;
    if (have) {
      tc_fence_after();
      const int hc = p.tn >> 1;
      for (int c = half * hc; c < (half + 1) * hc; c += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(32 * qd) << 16) + c, v);
        tmem_wait_ld();
        float4* dst = reinterpret_cast<float4*>(dsm + m * kSplitRowPitch + c * 4);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]), __uint_as_float(v[4 * i + 2]),
                               __uint_as_float(v[4 * i + 3]));
      }
    }
  }
  // Loads the MMA never waited for (after an abort) must land before the ring is reused.
  __syncthreads();
  if (warp == 0 && lane == 0)
    for (int i = sm.consumed; i < sm.fills; ++i) mbar_wait(bar(sm.full[i % S]), (i / S) & 1, wd, GW_DRAIN);
  __syncthreads();
  // an empty K range (more splits than K blocks) parks zeros
  if (warp >= 2 && kb1 <= kb0) {
    const int m = 32 * (warp & 3) + lane;
    const int half = (warp - 2) >> 2;
    const int hc = p.tn >> 1;
    for (int c = half * hc; c < (half + 1) * hc; c += 4)
      *reinterpret_cast<float4*>(dsm + m * kSplitRowPitch + c * 4) = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  cluster_sync();  // every CTA's partial is parked
  if (warp >= 2) {
    // rows [r0, r0 + 128 / splits) of the tile, summed over the splits in rank order
    const int rows = 128 / splits;
    const int r0 = rank * rows;
    const int t = threadIdx.x - 64;             // 0 .. 255
    const int cpr = p.tn >> 2;                  // float4 columns per row
    const uint32_t base = smem_u32(dsm);
    for (int idx = t; idx < rows * cpr; idx += 256) {
      const int rr = r0 + idx / cpr, c4 = idx % cpr;
      const uint32_t off = base + static_cast<uint32_t>(rr * kSplitRowPitch + c4 * 16);
      float4 acc = ld_cluster_f32x4(map_to_peer(off, 0u));
      for (int k = 1; k < splits; ++k) {
        const float4 v = ld_cluster_f32x4(map_to_peer(off, static_cast<uint32_t>(k)));
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
      // the result row and column of this element group
      const int u1 = x.i1 * p.b1 + (rr & (p.b1 - 1));
      const int u2 = x.i2 * p.b2 + (rr >> p.lg_b1);
      const int col = x.nt * p.tn + 4 * c4;
      if (u1 >= p.n1 || u2 >= p.n2 || col >= p.n_valid) continue;
      const long long o = u1 * p.os1 + u2 * p.os2 + x.g * p.ocol + col;
      const int n = p.n_valid - col;
      const float a4[4] = {acc.x, acc.y, acc.z, acc.w};
      if (p.out_fp32) {
        float* y = static_cast<float*>(p.out) + o;
        if (p.vec_ok && n >= 4) {
          *reinterpret_cast<float4*>(y) = acc;
        } else {
          for (int i = 0; i < 4 && i < n; ++i) y[i] = a4[i];
        }
      } else {
        uint16_t* y = static_cast<uint16_t*>(p.out) + o;
        const uint32_t lo = pack_bf16x2(acc.x, acc.y), hi = pack_bf16x2(acc.z, acc.w);
        if (p.vec_ok && n >= 4) {
          *reinterpret_cast<uint2*>(y) = make_uint2(lo, hi);
        } else {
          const uint32_t w2[2] = {lo, hi};
          for (int i = 0; i < 4 && i < n; ++i) y[i] = static_cast<uint16_t>(w2[i >> 1] >> (16 * (i & 1)));
        }
      }
    }
  }
  tc_fence_before();
  cluster_sync();  // no CTA leaves while a peer still reads its partial
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ------------------------------------------------------------------------------------------
// CTA-pair form of the weight-resident GEMM (tcgen05 cta_group::2): a pair computes 256 rows x 256
// columns per tile, each CTA streaming its own 128 rows of A and holding its half (128 columns) of
// the column tile's B for the whole launch.  One pair MMA multiplies each CTA's A rows by both
// halves of B, so a CTA's A bytes carry twice the FLOPs of the one-CTA form (whose A stream, three
// 32 KB stages beside the 128 KB B, bounds it).  For A with one row dimension (n2 = 1).  Pairs own
// column tile pair % n_tiles and row tiles pair / n_tiles, + res_groups, ...; the A stages and B
// are counted on the even CTA's barriers (pair-form TMA) and released to both CTAs by the MMA's
// multicast commit, as in the MLA pair kernel.
// ------------------------------------------------------------------------------------------
constexpr int kPgTn = 256;
constexpr int kPgStages = 3;
constexpr int kPgStageBytes = 2 * kGemmABytes;
constexpr size_t kPgSmemBytes = 1024 + kResBBytes + static_cast<size_t>(kPgStages) * kPgStageBytes;
static_assert(kPgSmemBytes <= 232448 - 1024, "shared memory budget");
enum PairGemmWaitSite { PG_EMPTY = LKV_SITE_WAIT_BASE + 130, PG_FULL, PG_TEMPTY, PG_TFULL, PG_BFULL, PG_DRAIN };
constexpr uint16_t kPgBoth = 3, kPgEven = 1;  // multicast masks of a commit

struct __align__(8) GemmPairSmem {
  uint64_t full[kPgStages];   // even CTA: both CTAs' A of the stage landed
  uint64_t empty[kPgStages];  // each CTA: the MMAs reading the stage are done (multicast commit)
  uint64_t tfull[2];          // each CTA: accumulator b holds a finished tile (multicast commit)
  uint64_t tempty[2];         // even CTA: the 16 epilogue warps of both CTAs read accumulator b
  uint64_t bfull;             // even CTA: both CTAs' halves of B landed
  uint64_t drain;             // even CTA: every MMA issued is complete
  uint32_t tmem_base, abort;
  int fills, b_issued;                  // this CTA's producer counts
  int peer_fills, peer_b_issued;        // the odd CTA's, for the even CTA's drain
  int stage_bytes[kPgStages];           // bytes per CTA of the last phase armed on each stage
  int peer_stage_bytes[kPgStages];
};

__global__ void __launch_bounds__(kGemmThreads, 1)
    proj_gemm_pair_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                          const GemmParams p) {
  extern __shared__ __align__(1024) uint8_t gemm_pair_raw[];
  __shared__ GemmPairSmem sm;
  uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gemm_pair_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  const uint32_t bres = smem_u32(dsm);
  const uint32_t ring = bres + kResBBytes;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr int S = kPgStages;
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);
  const int pair = blockIdx.x >> 1;
  const int nt = pair % p.n_tiles;
  const int mt0 = pair / p.n_tiles;
  const int kpairs = (p.k_blocks + 1) >> 1;
  const uint32_t batom = static_cast<uint32_t>(p.k_blocks) * 8192u;
  auto bar = [](const uint64_t& b) { return smem_u32(&b); };
  auto lead = [&](const uint64_t& b) -> uint32_t { return map_to_peer(smem_u32(&b), 0u); };

  if (threadIdx.x == 0) {
    for (int s2 = 0; s2 < S; ++s2) {
      mbar_init(bar(sm.full[s2]), 1);
      mbar_init(bar(sm.empty[s2]), 1);
      sm.stage_bytes[s2] = 0;
      sm.peer_stage_bytes[s2] = 0;
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(sm.tfull[b]), 1);
      mbar_init(bar(sm.tempty[b]), 16);
    }
    mbar_init(bar(sm.bfull), 1);
    mbar_init(bar(sm.drain), 1);
    sm.abort = 0;
    sm.fills = 0;
    sm.b_issued = 0;
    sm.peer_fills = 0;
    sm.peer_b_issued = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(&sm.tmem_base), kGemmTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any remote arrive or pair load
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const WaitCtl wc{&sm.abort, p.err, p.wait_limit_ns};

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs) ----------------
    if (lane == 0) {
      tma_prefetch_desc(&map_a);
      tma_prefetch_desc(&map_b);
      int it = 0;
      bool ok = true;
      if (mt0 < p.m_tiles) {
        // this CTA's half of the column tile's B: columns 256 nt + 128 rank .. +127, once
        if (leader) mbar_arrive_expect_tx(bar(sm.bfull), 2u * 2u * batom);
        for (int a = 0; a < 2; ++a) {
          const int c0 = nt * kPgTn + 128 * static_cast<int>(rank) + 64 * a;
          for (int kb = 0; kb < p.k_blocks; ++kb)
            tma_load_3d_pair(bres + a * batom + kb * 8192, &map_b, lead(sm.bfull), c0 % p.nb, kb * 64, c0 / p.nb);
        }
        sm.b_issued = 1;
      }
      for (int mt = mt0; ok && mt < p.m_tiles; mt += p.res_groups) {
        const int row = (2 * mt + static_cast<int>(rank)) * 128;  // this CTA's 128 rows of the pair tile
        for (int kp = 0; kp < kpairs; ++kp, ++it) {
          const int s2 = it % S;
          if (!mbar_wait<true>(bar(sm.empty[s2]), ((it / S) & 1) ^ 1, wc, PG_EMPTY)) {
            ok = false;
            break;
          }
          const int nkb = (2 * kp + 1 < p.k_blocks) ? 2 : 1;
          const int bytes = nkb * kGemmABytes;
          if (leader) mbar_arrive_expect_tx(bar(sm.full[s2]), static_cast<uint32_t>(2 * bytes));
          sm.stage_bytes[s2] = bytes;
          for (int j = 0; j < nkb; ++j)
            tma_load_3d_pair(ring + s2 * kPgStageBytes + j * kGemmABytes, &map_a, lead(sm.full[s2]), (2 * kp + j) * 64,
                             row, 0);
          sm.fills = it + 1;
        }
      }
      if (!leader) {
        st_cluster_u32(map_to_peer(smem_u32(&sm.peer_fills), 0u), static_cast<uint32_t>(sm.fills));
        st_cluster_u32(map_to_peer(smem_u32(&sm.peer_b_issued), 0u), static_cast<uint32_t>(sm.b_issued));
        for (int s2 = 0; s2 < S; ++s2)
          st_cluster_u32(map_to_peer(smem_u32(&sm.peer_stage_bytes[s2]), 0u), static_cast<uint32_t>(sm.stage_bytes[s2]));
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (even CTA) ----------------
    if (leader && lane == 0) {
      const uint32_t idesc = idesc_bf16(256, kPgTn, 0, 1);   // 128 rows per CTA, B MN-major
      const uint64_t bd0 = sdesc_sw128(bres, batom, 1024);
      int it = 0, lt = 0;
      bool issued = false;
      bool ok = mt0 >= p.m_tiles || mbar_wait<true>(bar(sm.bfull), 0, wc, PG_BFULL);
      for (int mt = mt0; ok && mt < p.m_tiles; mt += p.res_groups, ++lt) {
        const int buf = lt & 1;
        if (!mbar_wait<true>(bar(sm.tempty[buf]), ((lt >> 1) & 1) ^ 1, wc, PG_TEMPTY)) break;
        tc_fence_after();
        const uint32_t d = tmem + 256u * buf;
        for (int kp = 0; kp < kpairs; ++kp, ++it) {
          const int s2 = it % S;
          if (!mbar_wait<true>(bar(sm.full[s2]), (it / S) & 1, wc, PG_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int nkb = (2 * kp + 1 < p.k_blocks) ? 2 : 1;
          for (int j = 0; j < nkb; ++j) {
            const int kb = 2 * kp + j;
            const uint64_t ad = sdesc_sw128(ring + s2 * kPgStageBytes + j * kGemmABytes, 16, 1024);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_pair_ss(d, desc_add(ad, kk * 32), desc_add(bd0, kb * 8192 + kk * 2048), idesc, (kb | kk) ? 1u : 0u);
          }
          issued = true;
          umma_pair_commit(bar(sm.empty[s2]), kPgBoth);
        }
        if (!ok) break;
        umma_pair_commit(bar(sm.tfull[buf]), kPgBoth);
      }
      if (issued) {
        umma_pair_commit(bar(sm.drain), kPgEven);
        uint32_t zero = 0;
        const WaitCtl dc{&zero, p.err, p.wait_limit_ns};
        mbar_wait(bar(sm.drain), 0, dc, PG_DRAIN);
      }
    }
  } else {
    // ---------------- epilogue (both CTAs): this CTA's 128 rows x all 256 columns ----------------
    const int qd = warp & 3;
    const int half = (warp - 2) >> 2;
    const int m = 32 * qd + lane;
    int lt = 0;
    for (int mt = mt0; mt < p.m_tiles; mt += p.res_groups, ++lt) {
      const int buf = lt & 1;
      const bool okw = __all_sync(0xffffffffu, mbar_wait<true>(bar(sm.tfull[buf]), (lt >> 1) & 1, wc, PG_TFULL)) != 0;
      if (!okw) break;
      tc_fence_after();
      GemmTile x;
      x.nt = nt;
      x.i1 = 2 * mt + static_cast<int>(rank);
      x.i2 = 0;
      x.g = 0;
      gemm_store_tile(p, x, tmem + 256u * buf, qd, half, m);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_pair(lead(sm.tempty[buf]));
    }
  }

  // ---------------- teardown ----------------
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the odd CTA's producer counts are visible; every remote arrive has been made
  if (leader && warp == 0 && lane == 0) {
    // Drain: no copy may still be landing in either CTA when they exit.  A phase one producer
    // issued and the other did not (after a wait gave up) is completed for the missing side here.
    uint32_t zero = 0;
    const WaitCtl dc{&zero, p.err, p.wait_limit_ns};
    const int nl = sm.fills, np = sm.peer_fills;
    const int nmax = nl > np ? nl : np;
    for (int i = (nmax > S ? nmax - S : 0); i < nmax; ++i) {
      const uint32_t fb = bar(sm.full[i % S]);
      if (i < nl && i >= np) mbar_complete_tx(fb, static_cast<uint32_t>(sm.stage_bytes[i % S]));
      if (i >= nl && i < np) mbar_arrive_expect_tx(fb, static_cast<uint32_t>(sm.peer_stage_bytes[i % S]));
      mbar_wait(fb, static_cast<uint32_t>((i / S) & 1), dc, PG_DRAIN);
    }
    if (sm.b_issued || sm.peer_b_issued) {
      const uint32_t bb = bar(sm.bfull);
      if (sm.b_issued && !sm.peer_b_issued) mbar_complete_tx(bb, 2u * batom);
      if (!sm.b_issued && sm.peer_b_issued) mbar_arrive_expect_tx(bb, 2u * batom);
      mbar_wait(bb, 0, dc, PG_DRAIN);
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kGemmTmemCols);
  }
}

}  // namespace lkv
