// GLA decode with the keys in the MMA's M dimension, for units of at most 64 query rows (a latent
// group of d_h = 256 that serves as key and value, and the shared RoPE key).
//
// Per latent group j the GLA article (section "GLA") attends the group's heads to c_j (key and
// value in the absorbed form) plus the RoPE key.  A unit holds hpg x s_q <= 64 rows, so with the
// rows in M the MMAs run half empty and the O accumulator (64 rows x 256 columns) crowds S out of
// TMEM.  Transposed, as lkv_decode_swap.cuh does for d_h = 128:
//   S^T[key, row] = c[key, :] . Q[row, :]        M = 128 keys, N = 64 rows, K = 256 + 64 columns
//   O^T[d, row]  += c^T[d, key] . P^T[key, row]   two MMAs of M = 128 (value columns 0..127 and
//                                                 128..255), N = 64, K = 128 keys
//
// Warps: 0 TMA producer; 1 TMEM allocator and QK issuer; 2 PV issuer; 3 idle; 4-11 softmax /
// epilogue.  Softmax warp w owns lane quadrant w % 4 (keys 32 (w % 4) .. +31 of the tile, value
// columns d and 128 + d of O^T likewise) and the 32 rows 32 h .. 32 h + 31, h = (w - 4) / 4.  A
// row's tile max is a reduce-scatter over the warp's lanes (31 shuffles, lane l ends with row l),
// then the 4 quadrant warps' values through shared memory; the row sums stay per thread and are
// reduced once per unit.
//
// TMEM (256 columns): S^T buffers at 0 and 64 (128 keys x 64 rows), O^T at 128 (value columns
// 0..127) and 192 (128..255).  Shared memory: a ring of two 80 KB stages (four 64-column boxes of
// the group's latent and the RoPE key box), the unit's Q as the K-major B operand of QK (64 rows x
// 320 columns, five 128-byte-swizzled boxes) and one P^T buffer, the MN-major B operand of PV
// (128 keys x 64 rows of bf16, 128-byte swizzle).
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "lkv_ptx.cuh"
#include "lkv_sched.cuh"
#include "lkv_decode_tc.cuh"
#include "lkv_decode_swap.cuh"

namespace lkv {

constexpr int kWideMaxRows = 64;  // N of every MMA: the unit's rows, zero-padded

struct WideCfg {
  static constexpr int kTile = 128;                   // keys per tile = M of QK
  static constexpr int kN = kWideMaxRows;
  static constexpr int kDH = 256;                     // latent (key and value) columns of a group
  static constexpr int kBoxBytes = kTile * 128;       // 128 keys x 64 bf16, 128-byte swizzle
  static constexpr int kStageBytes = 5 * kBoxBytes;   // latent (4 boxes) + RoPE key (1 box)
  static constexpr int kStages = 2;
  static constexpr int kQBoxBytes = kN * 128;         // 64 rows x 64 bf16
  static constexpr int kQBytes = 5 * kQBoxBytes;
  static constexpr int kPBytes = kTile * kN * 2;      // 128 keys x 64 bf16
  static constexpr size_t kRingBytes = static_cast<size_t>(kStages) * kStageBytes;
  static constexpr size_t kSmemBytes = 1024 + kRingBytes + kQBytes + kPBytes;
  static constexpr uint32_t S0 = 0, O0 = 128;
  static constexpr int kTmemCols = 256;
  static constexpr int kSiteBase = LKV_SITE_WAIT_BASE + 280;  // wait sites of this kernel
};
static_assert(WideCfg::kSmemBytes <= 232448 - 8192, "shared memory budget");

struct __align__(16) WideSmem {
  uint64_t full[WideCfg::kStages], empty[WideCfg::kStages];
  uint64_t s_full[2], s_free[2], p_full, o_done;
  uint64_t q_ready, o_free, drain;
  uint64_t xb4[2];                  // the 8 softmax warps posted one value per row (double-buffered)
  alignas(16) float red[2][8][32];  // [buffer][softmax warp][row of its half]
  alignas(16) float msub[8][32];    // per warp: the tile's row max (log2 units), subtracted in the exponent
  alignas(16) float fac[8][32];     // per warp: 2^(tile max - running max) per row
  alignas(16) float arow[8][32];    // per warp: O rescale factor per row, then 1 / l at the end
  uint32_t tmem_base;
  uint32_t abort;
  long long t_begin, t_end, unit_t0;
  int b0, k0;
};

// Reduce-scatter over the warp, 32 values (rows) per lane: lane l ends with row l reduced over the
// 32 lanes (31 shuffles; at each level a lane keeps the half of its rows that matches its lane bit).
template <bool kMax>
__device__ __forceinline__ float warp_rows_reduce32(float (&v)[32], int lane) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const bool up = (lane & s) != 0;
#pragma unroll
    for (int j = 0; j < s; ++j) {
      const float send = up ? v[j] : v[j + s];
      const float keep = up ? v[j + s] : v[j];
      v[j] = rop<kMax>(keep, __shfl_xor_sync(0xffffffffu, send, s));
    }
  }
  return v[0];
}

__global__ void __launch_bounds__(kSwapThreads, 1)
    decode_swap_wide_kernel(const __grid_constant__ CUtensorMap map_c,  // latent [rows, g*256], box 64 x 128
                            const __grid_constant__ CUtensorMap map_r,  // RoPE key [rows, 64], box 64 x 128
                            const TcParams p) {
  using Cfg = WideCfg;
  constexpr int TN = Cfg::kTile;
  constexpr int KS = Cfg::kStages;
  constexpr int kBoxBytes = Cfg::kBoxBytes;
  constexpr int kStageBytes = Cfg::kStageBytes;
  constexpr uint32_t S0 = Cfg::S0, O0 = Cfg::O0;
  constexpr int SB = Cfg::kSiteBase;

  extern __shared__ __align__(1024) uint8_t wide_smem_raw[];
  __shared__ WideSmem sm;
  uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(wide_smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  const uint32_t stage_base = smem_u32(dsm);
  uint8_t* qsm = dsm + Cfg::kRingBytes;
  const uint32_t q_base = smem_u32(qsm);
  uint8_t* psm = qsm + Cfg::kQBytes;
  const uint32_t p_base = smem_u32(psm);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int range = blockIdx.x;

  SchedArgs sa0;
  sa0.cu = p.cu;
  sa0.B = p.B;
  sa0.s_q = p.s_q;
  sa0.tile = TN;
  sa0.units_per_req = p.G;
  sa0.per_query_units = 0;
  sa0.P = p.P;
  const bool lockstep = lockstep_groups(sa0);
  const SchedArgs sa = request_space(sa0);
  const int sched_range = lockstep ? range / p.G : range;
  const int kfix = lockstep ? range % p.G : 0;
  auto next_seg = [&](SegCursor& c, Segment& sg) -> bool {
    const bool r = c.next(sa, sg);
    if (r && lockstep) {
      sg.k = kfix;
      sg.unit_id = sg.b * p.G + kfix;
    }
    return r;
  };

  if (tid == 0) {
    for (int s = 0; s < KS; ++s) {
      mbar_init(smem_u32(&sm.full[s]), 1);
      mbar_init(smem_u32(&sm.empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&sm.s_full[b]), 1);
      mbar_init(smem_u32(&sm.s_free[b]), 8);  // the 8 softmax warps
      mbar_init(smem_u32(&sm.xb4[b]), 8);
    }
    mbar_init(smem_u32(&sm.p_full), 8);
    mbar_init(smem_u32(&sm.o_done), 1);
    mbar_init(smem_u32(&sm.q_ready), 8);
    mbar_init(smem_u32(&sm.o_free), 8);
    mbar_init(smem_u32(&sm.drain), 2);  // one commit from each issuer
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    bool malformed = false;
    SegCursor c = locate_range(sa, sched_range, &malformed);
    if (lane == 0) {
      if (malformed && range == 0) record_error(p.err, LKV_SITE_BAD_LENGTH);
      sm.t_begin = c.t_begin;
      sm.t_end = c.t_end;
      sm.unit_t0 = c.unit_t0;
      sm.b0 = c.b;
      sm.k0 = c.k;
      p.seg_info[2 * range] = -1;
      p.seg_info[2 * range + 1] = -1;
      tma_prefetch_desc(&map_c);
      tma_prefetch_desc(&map_r);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&sm.tmem_base), Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (tid == 0) griddep_launch_dependents();  // the split combine may start launching
  const uint32_t tbase = sm.tmem_base;
  const WaitCtl wc{&sm.abort, p.err, p.wait_limit_ns};

  SegCursor cur0;
  cur0.t_begin = sm.t_begin;
  cur0.t_end = sm.t_end;
  cur0.unit_t0 = sm.unit_t0;
  cur0.b = sm.b0;
  cur0.k = sm.k0;
  cur0.produced = 0;

  if (warp == 0) {
    // ============================================================ TMA producer
    if (lane == 0) {
      SegCursor cur = cur0;
      Segment sg;
      int n = 0;
      bool ok = true;
      while (ok && next_seg(cur, sg)) {
        for (int t = sg.tile_lo; t < sg.tile_hi; ++t) {
          const int st = n % KS;
          if (!mbar_wait(smem_u32(&sm.empty[st]), static_cast<uint32_t>(((n / KS) & 1) ^ 1), wc, SB + W_EMPTY)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&sm.full[st]);
          mbar_arrive_expect_tx(fb, kStageBytes);
          const uint32_t dst = stage_base + st * kStageBytes;
          const int row = sg.cu_b + t * TN;
          const int c0 = Cfg::kDH * sg.k;
#pragma unroll
          for (int bx = 0; bx < 4; ++bx) tma_load_2d(dst + bx * kBoxBytes, &map_c, fb, c0 + 64 * bx, row);
          tma_load_2d(dst + 4 * kBoxBytes, &map_r, fb, 0, row);
          ++n;
        }
      }
      // no copy may still be landing when the CTA exits: wait for the last ones issued
      uint32_t zero = 0;
      const WaitCtl dc{&zero, p.err, p.wait_limit_ns};
      for (int m = (n > KS ? n - KS : 0); m < n; ++m)
        mbar_wait(smem_u32(&sm.full[m % KS]), static_cast<uint32_t>((m / KS) & 1), dc, SB + W_DRAIN);
    }
  }
  else if (warp == 1 || warp == 2) {
    // ============================================================ MMA issuers
    if (lane == 0) {
      SegCursor cur = cur0;
      Segment sg;
      int n = 0, seg = 0;
      bool ok = true;
      if (warp == 1) {
        // S^T[key, row] = c[key, :] . Q[row, :]: A = the stage (K-major: latent boxes 0-3, then the
        // RoPE box 4); B = Q, K-major (each row's 320 columns); M = 128 keys, N = 64 rows
        const uint32_t id_qk = idesc_bf16(128, Cfg::kN, 0, 0);
        const uint64_t qdesc = sdesc_sw128(q_base, 16, 1024);
        while (ok && next_seg(cur, sg)) {
          for (int t = sg.tile_lo; t < sg.tile_hi; ++t, ++n) {
            const int st = n % KS;
            const int sb = n & 1;
            if (!mbar_wait(smem_u32(&sm.full[st]), static_cast<uint32_t>((n / KS) & 1), wc, SB + W_FULL) ||
                (n >= 2 && !mbar_wait(smem_u32(&sm.s_free[sb]), static_cast<uint32_t>(((n - 2) >> 1) & 1), wc,
                                      SB + W_SFREE)) ||
                (t == sg.tile_lo &&
                 !mbar_wait(smem_u32(&sm.q_ready), static_cast<uint32_t>(seg & 1), wc, SB + W_QREADY))) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t kdesc = sdesc_sw128(stage_base + st * kStageBytes, 16, 1024);
#pragma unroll
            for (int ks = 0; ks < 20; ++ks) {
              const int bx = ks >> 2, kk = ks & 3;
              umma_ss(tbase + S0 + Cfg::kN * sb, desc_add(kdesc, bx * kBoxBytes + kk * 32),
                      desc_add(qdesc, bx * Cfg::kQBoxBytes + kk * 32), id_qk, ks ? 1u : 0u);
            }
            umma_commit(smem_u32(&sm.s_full[sb]));
          }
          ++seg;
        }
      } else {
        // O^T[d, row] += c^T[d, key] P^T[key, row] for d in 128 h .. 128 h + 127: A = latent boxes
        // 2h and 2h + 1 read MN-major (LBO between them), B = P^T, MN-major in the 128-byte swizzle
        // (one atom of 64 rows wide, 8-key atoms of 1 KB); M = 128, N = 64, 16 keys per MMA
        const uint32_t id_pv = idesc_bf16(128, Cfg::kN, 1, 1);
        const uint64_t pdesc = sdesc_sw128(p_base, 16, 1024);
        while (ok && next_seg(cur, sg)) {
          for (int t = sg.tile_lo; t < sg.tile_hi; ++t, ++n) {
            const bool first = (t == sg.tile_lo);
            if (!mbar_wait(smem_u32(&sm.p_full), static_cast<uint32_t>(n & 1), wc, SB + W_PFULL) ||
                (first && seg > 0 &&
                 !mbar_wait(smem_u32(&sm.o_free), static_cast<uint32_t>((seg - 1) & 1), wc, SB + W_OFREE))) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t stage = stage_base + static_cast<uint32_t>(n % KS) * kStageBytes;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint64_t adesc = sdesc_sw128(stage + 2 * h * kBoxBytes, kBoxBytes, 1024);
#pragma unroll
              for (int kk = 0; kk < TN / 16; ++kk)
                umma_ss(tbase + O0 + Cfg::kN * h, desc_add(adesc, kk * 2048), desc_add(pdesc, kk * 2048), id_pv,
                        (first && kk == 0) ? 0u : 1u);
            }
            umma_commit(smem_u32(&sm.o_done));
            umma_commit(smem_u32(&sm.empty[n % KS]));  // the stage served as key and value
          }
          ++seg;
        }
      }
      // every MMA of this thread complete before TMEM is released (both issuers arrive)
      umma_commit(smem_u32(&sm.drain));
      uint32_t zero = 0;
      const WaitCtl dc{&zero, p.err, p.wait_limit_ns};
      mbar_wait(smem_u32(&sm.drain), 0, dc, SB + W_DRAIN);
    }
  }
  else if (warp >= 4) {
    // ============================================================ softmax / epilogue
    const int sw = warp - 4;                 // softmax warp 0..7
    const int q4 = warp & 3;                 // TMEM lane quadrant
    const int hh = sw >> 2;                  // rows 32 hh .. 32 hh + 31
    const int rb = 32 * hh;
    const int k = q4 * 32 + lane;            // key of the tile = S^T lane; value columns k, 128 + k of O^T
    const uint32_t lb = static_cast<uint32_t>(q4 * 32);
    auto wait_all = [&](uint32_t bar, uint32_t par, int site) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, par, wc, site)) != 0;
    };
    auto warp_arrive = [&](uint32_t bar) {
      __syncwarp();
      if (lane == 0) mbar_arrive(bar);
    };
    // every warp posts one value per row (row rb + lane) and reads back the posts of the 4 warps of
    // its row half (the 4 lane quadrants, i.e. all 128 keys)
    int xc = 0;
    auto xchg4 = [&](float v, float (&all)[4]) -> bool {
      const int b = xc & 1;
      sm.red[b][sw][lane] = v;
      warp_arrive(smem_u32(&sm.xb4[b]));
      const bool okx = wait_all(smem_u32(&sm.xb4[b]), static_cast<uint32_t>((xc >> 1) & 1), SB + W_XCHG);
#pragma unroll
      for (int w = 0; w < 4; ++w) all[w] = sm.red[b][4 * hh + w][lane];
      ++xc;
      return okx;
    };
    // the unit's Q (rows padded with zeros to 64) as the K-major B operand: 40 chunks of 16 bytes a row
    auto load_q = [&](const Segment& sg) {
      for (int idx = sw * 32 + lane; idx < Cfg::kN * 40; idx += 256) {
        const int r = idx / 40, c = idx % 40;
        const int bx = c >> 3, cc = c & 7;
        uint4 x = make_uint4(0u, 0u, 0u, 0u);
        if (r < p.R) {
          const int i = r / p.hpg;
          const int h = sg.k * p.hpg + (r - i * p.hpg);
          const size_t qrow = (static_cast<size_t>(sg.b) * p.s_q + i) * p.h_q + h;
          x = bx < 4 ? __ldg(reinterpret_cast<const uint4*>(p.q_nope + qrow * p.dq + 64 * bx) + cc)
                     : __ldg(reinterpret_cast<const uint4*>(p.q_rope + qrow * 64) + cc);
        }
        *reinterpret_cast<uint4*>(qsm + bx * Cfg::kQBoxBytes + r * 128 + ((cc ^ (r & 7)) << 4)) = x;
      }
      fence_proxy_async_smem();
      warp_arrive(smem_u32(&sm.q_ready));
    };

    const int qi0 = rb / p.hpg, rr0 = rb - qi0 * p.hpg;  // query and head offset of row rb
    SegCursor cur = cur0;
    Segment sg, nx;
    bool ok = true;
    int n = 0;
    // running max of row rb + lane (log2 units); per row j of this warp, this thread's (key lane k)
    // running sum of the fp32 weights (the lse and the normaliser)
    float m_run = -INFINITY;
    float lt[32];
    bool have = next_seg(cur, sg);
    if (have) load_q(sg);
    while (ok && have) {
      bool have_nx = false;
      const int lim0 = sg.L - p.s_q;  // query i sees keys 0 .. lim0 + i of the request
      for (int t = sg.tile_lo; t < sg.tile_hi; ++t, ++n) {
        const int sb = n & 1;
        if (!wait_all(smem_u32(&sm.s_full[sb]), static_cast<uint32_t>((n >> 1) & 1), SB + W_SFULL)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t a[32];
        tmem_ld32(tm_addr(tbase, lb, S0 + Cfg::kN * sb + rb), a);
        tmem_wait_ld();
        tc_fence_before();
        warp_arrive(smem_u32(&sm.s_free[sb]));
        if (t == sg.tile_hi - 1 && (have_nx = next_seg(cur, nx))) load_q(nx);  // this unit's QKs are done
        if (t == sg.tile_lo) {
          m_run = -INFINITY;
#pragma unroll
          for (int j = 0; j < 32; ++j) lt[j] = 0.f;
        }
        // row rb + j is query (rb + j) / hpg; rows >= R are padding.  A tile whose last key every
        // query sees, with no padding row, needs no mask.
        const int kg = t * TN + k;  // key index in the request
        float sv[32];
        if ((t + 1) * TN - 1 <= lim0 && p.R == kWideMaxRows) {
#pragma unroll
          for (int j = 0; j < 32; ++j) sv[j] = __uint_as_float(a[j]);
        } else {
          int qi = qi0, rr = rr0;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const bool vis = (rb + j < p.R) && (kg <= lim0 + qi);
            sv[j] = vis ? __uint_as_float(a[j]) : -INFINITY;
            if (++rr == p.hpg) {
              rr = 0;
              ++qi;
            }
          }
        }
        // the tile's max per row over the 128 keys (raw scores: the scale is positive)
        float mx[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) mx[j] = sv[j];
        const float mw = warp_rows_reduce32<true>(mx, lane);
        float all4[4];
        if (!xchg4(mw, all4)) {
          ok = false;
          break;
        }
        const float mt = fmaxf(fmaxf(all4[0], all4[1]), fmaxf(all4[2], all4[3])) * p.sl2;
        bool rescale = false;
        float m_new = m_run;
        if (mt > m_run + 8.f) {  // lazy rescale: keep the running max unless it grows by 2^8
          m_new = mt;
          rescale = (m_run != -INFINITY);
        }
        // exponents centred on the tile max (<= 0, so the fp16 argument of the best keys is exact
        // or nearly so), times f = 2^(mt - m_new) <= 2^8 in fp32
        sm.msub[sw][lane] = (mt == -INFINITY) ? 0.f : mt;
        sm.fac[sw][lane] = (mt == -INFINITY) ? 0.f : ex2_approx(mt - m_new);
        sm.arow[sw][lane] = rescale ? ex2_approx(m_run - m_new) : 1.f;
        m_run = m_new;
        __syncwarp();
        const bool any_rescale = __any_sync(0xffffffffu, rescale) != 0;
        if (any_rescale) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float4 a4 = reinterpret_cast<const float4*>(sm.arow[sw])[j];
            lt[4 * j] *= a4.x, lt[4 * j + 1] *= a4.y, lt[4 * j + 2] *= a4.z, lt[4 * j + 3] *= a4.w;
          }
        }
        // this key's weight for the warp's 32 rows: half of row k of P^T
        uint32_t pw[16];
#pragma unroll
        for (int j4 = 0; j4 < 8; ++j4) {
          const float4 m4 = reinterpret_cast<const float4*>(sm.msub[sw])[j4];
          const float4 f4 = reinterpret_cast<const float4*>(sm.fac[sw])[j4];
          const uint32_t h0 = ex2_f16x2(fmaf(sv[4 * j4], p.sl2, -m4.x), fmaf(sv[4 * j4 + 1], p.sl2, -m4.y));
          const uint32_t h1 = ex2_f16x2(fmaf(sv[4 * j4 + 2], p.sl2, -m4.z), fmaf(sv[4 * j4 + 3], p.sl2, -m4.w));
          const float e0 = f16_lo(h0) * f4.x, e1 = f16_hi(h0) * f4.y;
          const float e2 = f16_lo(h1) * f4.z, e3 = f16_hi(h1) * f4.w;
          pw[2 * j4] = pack_bf16x2(e0, e1);
          pw[2 * j4 + 1] = pack_bf16x2(e2, e3);
          lt[4 * j4] += e0;
          lt[4 * j4 + 1] += e1;
          lt[4 * j4 + 2] += e2;
          lt[4 * j4 + 3] += e3;
        }
        // the P buffer and O^T were last used by PV(n - 1)
        if (n >= 1 && !wait_all(smem_u32(&sm.o_done), static_cast<uint32_t>((n - 1) & 1), SB + W_ODONE)) {
          ok = false;
          break;
        }
        {
          // row k of P^T is 128 bytes in the 128-byte swizzle (16-byte chunk c at c ^ (k & 7));
          // this warp's rows are chunks 4 hh .. 4 hh + 3
          uint8_t* prow = psm + k * 128;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            *reinterpret_cast<uint4*>(prow + (((4 * hh + c) ^ (k & 7)) << 4)) =
                make_uint4(pw[4 * c], pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3]);
        }
        // keys past the request belong to another request or to unwritten cache: their P is 0, but
        // 0 * NaN would still poison O, so each such latent row is cleared (boxes 2 hh, 2 hh + 1 by
        // row half hh)
        const int in_unit = sg.keys - t * TN;
        if (in_unit < TN && k >= in_unit) {
          uint8_t* vb = dsm + (n % KS) * kStageBytes;
#pragma unroll
          for (int bx = 0; bx < 2; ++bx)
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4*>(vb + (2 * hh + bx) * kBoxBytes + k * 128 + c * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
        if (any_rescale && t != sg.tile_lo) {
          // O^T holds this unit's tiles up to n-1 (PV(n-1) is done): scale column r by alpha_r
          tc_fence_after();
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t o[32];
            tmem_ld32(tm_addr(tbase, lb, O0 + Cfg::kN * h + rb), o);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * sm.arow[sw][j]);
            tmem_st32(tm_addr(tbase, lb, O0 + Cfg::kN * h + rb), o);
          }
          tmem_wait_st();
        }
        tc_fence_before();
        warp_arrive(smem_u32(&sm.p_full));
        if (t != sg.tile_hi - 1) continue;
        // ---------------------------------------------------------- unit epilogue
        const float lw = warp_rows_reduce32<false>(lt, lane);
        float lt4[4];
        if (!xchg4(lw, lt4)) {
          ok = false;
          break;
        }
        const float l_tot = (lt4[0] + lt4[1]) + (lt4[2] + lt4[3]);  // row rb + lane
        const float inv_l = l_tot > 0.f ? 1.f / l_tot : 0.f;
        const float lse_v = l_tot > 0.f ? (m_run + __log2f(l_tot)) * 0.69314718055994531f : -INFINITY;
        sm.arow[sw][lane] = inv_l;
        __syncwarp();
        if (!wait_all(smem_u32(&sm.o_done), static_cast<uint32_t>(n & 1), SB + W_ODONE)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const size_t slot_row = static_cast<size_t>(2 * range + (sg.complete ? 0 : sg.slot)) * p.rmax;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t o[32];
          tmem_ld32(tm_addr(tbase, lb, O0 + Cfg::kN * h + rb), o);
          tmem_wait_ld();
          const int d = Cfg::kDH / 2 * h + k;
          int qi = qi0, rr = rr0;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            if (rb + j < p.R) {
              const size_t orow = (static_cast<size_t>(sg.b) * p.s_q + qi) * p.h_q + sg.k * p.hpg + rr;
              const float val = __uint_as_float(o[j]) * sm.arow[sw][j];
              if (sg.complete)
                p.out[orow * p.dv_total + d] = __float2bfloat16_rn(val);
              else
                p.part_o[(slot_row + rb + j) * p.dv_total + d] = val;
            }
            if (++rr == p.hpg) {
              rr = 0;
              ++qi;
            }
          }
        }
        if (q4 == 0 && rb + lane < p.R) {
          const int r = rb + lane;
          const int i = r / p.hpg;
          const size_t orow = (static_cast<size_t>(sg.b) * p.s_q + i) * p.h_q + sg.k * p.hpg + (r - i * p.hpg);
          if (sg.complete)
            p.lse[orow] = lse_v;
          else
            p.part_lse[slot_row + r] = lse_v;
        }
        if (!sg.complete && sw == 0 && lane == 0) p.seg_info[2 * range + sg.slot] = sg.unit_id;
        tc_fence_before();
        warp_arrive(smem_u32(&sm.o_free));
      }
      if (!ok) break;
      have = have_nx;
      if (have) sg = nx;
    }
  }
  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, Cfg::kTmemCols);
  }
}

}  // namespace lkv
