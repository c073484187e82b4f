// Tensor-core (tcgen05 / TMEM) split-KV decode attention for sm_100a.
//
// One persistent CTA (MLA: one CTA pair, a thread-block cluster of 2) per work range
// (lkv_sched.cuh).  Per CTA, 8 warps:
//   warp 0      TMA producer: streams 64-token key/value tiles of the cache into a ring of
//               shared-memory stages (2-D tiles of 64 rows x 64 bf16, 128-byte swizzle).
//   warp 1      TMEM owner and UMMA issuer (one thread): S = Q K^T into TMEM, then
//               O += P V into TMEM.  The non-RoPE part of Q and P are A operands read from
//               TMEM; the RoPE part of Q is an A operand in shared memory; K and V are B
//               operands in the stage (V is read MN-major from the very same swizzled tile
//               that served as K where K = V).
//   warps 4..7  softmax / epilogue: thread r owns row r (TMEM lane r): stages the unit's
//               query, reads S, masks, runs the online softmax in the exp2 domain, writes P
//               (bf16) into TMEM, rescales O when the running max moves, and at the end of a
//               segment writes out / lse (or fp32 partials).
//
// TMEM columns: O [0, DV) | S [DV, DV+64) | P0, P1 [DV+64, DV+128) | Q [DV+128, ...).
// P is double buffered so the softmax of tile n+1 never waits for the PV of tile n.
//
// MLA absorbed path (h_q = 128 heads share the latent, GQLA explainer section 2): the
// 128 x 512 fp32 output accumulator alone fills a whole TMEM, so a CTA pair splits it:
// rank 0 owns value columns 0..255 and computes the partial scores over latent columns
// 0..255 plus the 64 RoPE columns; rank 1 owns value columns 256..511 and the partial
// scores over latent columns 256..511.  The two partial score tiles are exchanged through
// distributed shared memory and summed (in the same order on both CTAs, so both derive the
// same P), and each CTA accumulates its own half of O.  Each CTA streams only the cache
// columns it needs, so the pair reads every cache byte once.  The softmax runs one tile
// behind the score stream: tile n's partial scores are sent before tile n-1 is finished,
// which hides the exchange latency.
//
// GQLA (g groups of expanded K_j, V_j) and GLA (latent groups, K_j = V_j) run one unit per
// CTA: rows = heads of the group x new tokens (<= 128), padded to the M = 128 UMMA shape.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "lkv_ptx.cuh"
#include "lkv_sched.cuh"
#include "../../include/lkv.h"

// Error-word code of a bounded wait that gave up: base + 20 * mode + site.
#define LKV_WAIT(x) (LKV_SITE_WAIT_BASE + 20 * kMode + (x))

namespace lkv {

constexpr int kBoxBytes = 64 * 64 * 2;  // one TMA box: 64 rows x 64 bf16
constexpr int kMaxBoxes = 5;
constexpr int kStageBytes = kMaxBoxes * kBoxBytes;  // 40 KB
constexpr int kQropeBytes = 128 * 128;             // 128 rows x 64 bf16, swizzled
constexpr int kTcThreads = 256;
constexpr int kXRow = 68;                          // floats per exchange row (64 + padding)
constexpr int kXBufBytes = 128 * kXRow * 4;
constexpr int kTmemCols = 512;

enum DecodeMode { MODE_MLA = 0, MODE_GQLA = 1, MODE_GLA = 2 };

// Wait sites (added to LKV_SITE_WAIT_BASE in the error word).
enum WaitSite {
  W_EMPTY = 1, W_FULL, W_SFREE, W_QREADY, W_PFULL, W_OFREE, W_SFULL, W_ODONE, W_XFREE, W_XFULL,
  W_DRAIN
};

struct TcParams {
  const __nv_bfloat16* q_nope;  // [B, s_q, h_q, dq]
  const __nv_bfloat16* q_rope;  // [B, s_q, h_q, 64]
  int dq;                       // row length of q_nope
  const int* cu;
  int B, s_q, h_q, G, hpg, R;   // R = valid rows per unit
  float sl2;                    // scale * log2(e)
  __nv_bfloat16* out;           // [B, s_q, h_q, dv_total]
  float* lse;                   // [B, s_q, h_q]
  int dv_total;
  int* seg_info;                // [2P]
  float* part_lse;              // [2P][rmax]
  float* part_o;                // [2P][rmax][dv_total]
  int rmax;
  int P;
  int* err;
  unsigned long long wait_limit_ns;
};

template <int kMode>
struct ModeCfg {
  static constexpr bool kPair = (kMode == MODE_MLA);
  static constexpr int kDV = (kMode == MODE_GQLA) ? 128 : 256;  // value columns per CTA
  static constexpr int kStages = kPair ? 3 : 5;
  static constexpr int kNope = (kMode == MODE_GQLA) ? 2 : 4;    // non-RoPE Q boxes (in TMEM)
  static constexpr int kRopeBox = (kMode == MODE_GQLA) ? 2 : 4; // stage box holding k_rope
  static constexpr int kVBox0 = (kMode == MODE_GQLA) ? 3 : 0;   // first stage box holding V
  static constexpr int kNV = kDV / 64;
  static constexpr uint32_t S0 = kDV, P0 = kDV + 64, Q0 = kDV + 128;
  static constexpr size_t kSmemBytes =
      1024 + static_cast<size_t>(kStages) * kStageBytes + kQropeBytes + (kPair ? 2 * kXBufBytes : 0);
  __device__ static bool has_rope(uint32_t rank) { return !kPair || rank == 0; }
  __device__ static int n_stage_boxes(uint32_t rank) { return kPair ? (rank == 0 ? 5 : 4) : 5; }
};
static_assert(ModeCfg<MODE_MLA>::Q0 + 32 * ModeCfg<MODE_MLA>::kNope <= kTmemCols, "TMEM budget");
static_assert(ModeCfg<MODE_GLA>::Q0 + 32 * ModeCfg<MODE_GLA>::kNope <= kTmemCols, "TMEM budget");
static_assert(ModeCfg<MODE_MLA>::kSmemBytes <= 232448, "shared memory budget");
static_assert(ModeCfg<MODE_GLA>::kSmemBytes <= 232448, "shared memory budget");

template <int kStagesT>
struct __align__(16) TcSmem {
  uint64_t full[kStagesT];
  uint64_t empty[kStagesT];
  uint64_t s_full, s_free, o_free, q_ready, drain;
  uint64_t p_full[2], o_done[2], x_full[2], x_free[2];
  uint32_t tmem_base;
  uint32_t abort;
  long long t_begin, t_end, unit_t0;
  int b0, k0;
};

__device__ __forceinline__ uint32_t tm_addr(uint32_t base, uint32_t lane_base, uint32_t col) {
  return base + (lane_base << 16) + col;
}

template <int kMode>
__global__ void __launch_bounds__(kTcThreads, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap map_a,  // MLA ckv | GQLA k | GLA clat
                     const __grid_constant__ CUtensorMap map_r,  // k_rope
                     const __grid_constant__ CUtensorMap map_v,  // GQLA v (unused otherwise)
                     const TcParams p) {
  using Cfg = ModeCfg<kMode>;
  constexpr int DV = Cfg::kDV;
  constexpr int KS = Cfg::kStages;
  constexpr bool kPair = Cfg::kPair;
  constexpr uint32_t S0 = Cfg::S0, P0 = Cfg::P0, Q0 = Cfg::Q0;

  extern __shared__ __align__(1024) uint8_t dsmem_raw[];
  __shared__ TcSmem<KS> sm;
  uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  const uint32_t stage_base = smem_u32(dsm);
  uint8_t* qrope_smem = dsm + KS * kStageBytes;
  const uint32_t qrope_base = smem_u32(qrope_smem);
  float* xbuf = reinterpret_cast<float*>(qrope_smem + kQropeBytes);  // MLA only: [2][128][kXRow]

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const uint32_t rank = kPair ? cluster_ctarank() : 0u;
  const int range = kPair ? (blockIdx.x >> 1) : blockIdx.x;
  const int n_sm_warps = (p.R + 31) >> 5;  // softmax warps holding valid rows
  const int n_sm_threads = n_sm_warps * 32;

  SchedArgs sa;
  sa.cu = p.cu;
  sa.B = p.B;
  sa.s_q = p.s_q;
  sa.units_per_req = kPair ? p.s_q : p.G;
  sa.per_query_units = kPair ? 1 : 0;
  sa.P = p.P;

  // ---------------------------------------------------------------- set-up
  if (tid == 0) {
    for (int s = 0; s < KS; ++s) {
      mbar_init(smem_u32(&sm.full[s]), 1);
      mbar_init(smem_u32(&sm.empty[s]), 1);
    }
    mbar_init(smem_u32(&sm.s_full), 1);
    mbar_init(smem_u32(&sm.s_free), n_sm_threads);
    mbar_init(smem_u32(&sm.o_free), n_sm_threads);
    mbar_init(smem_u32(&sm.q_ready), n_sm_threads);
    mbar_init(smem_u32(&sm.drain), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&sm.p_full[b]), n_sm_threads);
      mbar_init(smem_u32(&sm.o_done[b]), 1);
      mbar_init(smem_u32(&sm.x_full[b]), 128);
      mbar_init(smem_u32(&sm.x_free[b]), 128);
    }
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    bool malformed = false;
    SegCursor c = locate_range(sa, range, &malformed);
    if (lane == 0) {
      // a request shorter than s_q gets no tiles (its outputs are left unwritten): report it
      if (malformed && range == 0 && rank == 0) record_error(p.err, LKV_SITE_BAD_LENGTH);
      sm.t_begin = c.t_begin;
      sm.t_end = c.t_end;
      sm.unit_t0 = c.unit_t0;
      sm.b0 = c.b;
      sm.k0 = c.k;
      if (rank == 0) {
        p.seg_info[2 * range] = -1;
        p.seg_info[2 * range + 1] = -1;
      }
      tma_prefetch_desc(&map_a);
      tma_prefetch_desc(&map_r);
      if (kMode == MODE_GQLA) tma_prefetch_desc(&map_v);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&sm.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  if (kPair) cluster_sync();  // the peer's barriers exist before any remote arrive
  tc_fence_after();
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
      const int nbox = Cfg::n_stage_boxes(rank);
      const uint32_t bytes = nbox * kBoxBytes;
      SegCursor cur = cur0;
      Segment sg;
      long long n = 0;
      bool ok = true;
      while (ok && cur.next(sa, sg)) {
        for (int t = sg.tile_lo; t < sg.tile_hi; ++t, ++n) {
          const int st = static_cast<int>(n % KS);
          const uint32_t par = static_cast<uint32_t>(((n / KS) & 1) ^ 1);
          if (!mbar_wait(smem_u32(&sm.empty[st]), par, wc, LKV_WAIT(W_EMPTY))) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&sm.full[st]);
          mbar_arrive_expect_tx(fb, bytes);
          const uint32_t dst = stage_base + st * kStageBytes;
          const int row = sg.cu_b + t * kTileN;
          if (kMode == MODE_MLA) {
            const int c0 = 256 * static_cast<int>(rank);
            for (int bx = 0; bx < 4; ++bx) tma_load_2d(dst + bx * kBoxBytes, &map_a, fb, c0 + 64 * bx, row);
            if (rank == 0) tma_load_2d(dst + 4 * kBoxBytes, &map_r, fb, 0, row);
          } else if (kMode == MODE_GQLA) {
            const int c0 = 128 * sg.k;
            tma_load_2d(dst, &map_a, fb, c0, row);
            tma_load_2d(dst + kBoxBytes, &map_a, fb, c0 + 64, row);
            tma_load_2d(dst + 2 * kBoxBytes, &map_r, fb, 0, row);
            tma_load_2d(dst + 3 * kBoxBytes, &map_v, fb, c0, row);
            tma_load_2d(dst + 4 * kBoxBytes, &map_v, fb, c0 + 64, row);
          } else {
            const int c0 = 256 * sg.k;
            for (int bx = 0; bx < 4; ++bx) tma_load_2d(dst + bx * kBoxBytes, &map_a, fb, c0 + 64 * bx, row);
            tma_load_2d(dst + 4 * kBoxBytes, &map_r, fb, 0, row);
          }
        }
      }
      // never leave copies in flight into a CTA that is about to exit
      const long long inflight = n < KS ? n : KS;
      uint32_t zero = 0;
      const WaitCtl dc{&zero, p.err, p.wait_limit_ns};  // ignores the abort flag, keeps the limit
      for (long long m = n - inflight; m < n; ++m)
        mbar_wait(smem_u32(&sm.full[m % KS]), static_cast<uint32_t>((m / KS) & 1), dc, LKV_WAIT(W_DRAIN));
    }
  } else if (warp == 1) {
    // ============================================================ UMMA issuer
    if (lane == 0) {
      const bool rope = Cfg::has_rope(rank);
      const uint32_t id_qk = idesc_bf16(128, kTileN, 0, 0);
      const uint32_t id_pv = idesc_bf16(128, DV, 0, 1);
      SegCursor cur = cur0;
      Segment sg;
      long long n = 0;   // global tile counter
      int seg = 0;       // segments started
      bool ok = true;
      bool pend = false, pend_first = false;   // PV of tile pend_n not yet issued
      int pend_seg = 0;
      long long pend_n = 0;
      auto issue_pv = [&]() -> bool {
        const int pb = static_cast<int>(pend_n & 1);
        if (!mbar_wait(smem_u32(&sm.p_full[pb]), static_cast<uint32_t>((pend_n >> 1) & 1), wc,
                       LKV_WAIT(W_PFULL)))
          return false;
        if (pend_first && pend_seg > 0 &&
            !mbar_wait(smem_u32(&sm.o_free), static_cast<uint32_t>((pend_seg - 1) & 1), wc, LKV_WAIT(W_OFREE)))
          return false;
        tc_fence_after();
        const uint32_t vbase = stage_base + static_cast<uint32_t>(pend_n % KS) * kStageBytes + Cfg::kVBox0 * kBoxBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t bd = sdesc_sw128(vbase + kk * 2048, kBoxBytes, 1024);
          umma_ts(tbase, tbase + P0 + 32 * pb + kk * 8, bd, id_pv, (pend_first && kk == 0) ? 0u : 1u);
        }
        umma_commit(smem_u32(&sm.o_done[pb]));
        umma_commit(smem_u32(&sm.empty[pend_n % KS]));
        pend = false;
        return true;
      };
      while (ok && cur.next(sa, sg)) {
        for (int t = sg.tile_lo; t < sg.tile_hi; ++t, ++n) {
          const int st = static_cast<int>(n % KS);
          if (!mbar_wait(smem_u32(&sm.full[st]), static_cast<uint32_t>((n / KS) & 1), wc, LKV_WAIT(W_FULL)) ||
              (n > 0 && !mbar_wait(smem_u32(&sm.s_free), static_cast<uint32_t>((n - 1) & 1), wc, LKV_WAIT(W_SFREE))) ||
              (t == sg.tile_lo &&
               !mbar_wait(smem_u32(&sm.q_ready), static_cast<uint32_t>(seg & 1), wc, LKV_WAIT(W_QREADY)))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t kb = stage_base + st * kStageBytes;
#pragma unroll
          for (int bx = 0; bx < Cfg::kNope; ++bx) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t bd = sdesc_sw128(kb + bx * kBoxBytes + kk * 32, 16, 1024);
              umma_ts(tbase + S0, tbase + Q0 + bx * 32 + kk * 8, bd, id_qk, (bx | kk) ? 1u : 0u);
            }
          }
          if (rope) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = sdesc_sw128(qrope_base + kk * 32, 16, 1024);
              const uint64_t bd = sdesc_sw128(kb + Cfg::kRopeBox * kBoxBytes + kk * 32, 16, 1024);
              umma_ss(tbase + S0, ad, bd, id_qk, 1u);
            }
          }
          umma_commit(smem_u32(&sm.s_full));
          if (pend && !issue_pv()) {
            ok = false;
            break;
          }
          pend = true;
          pend_first = (t == sg.tile_lo);
          pend_seg = seg;
          pend_n = n;
        }
        ++seg;
      }
      if (ok && pend) issue_pv();
      // all tcgen05 work of this thread done before TMEM is released
      umma_commit(smem_u32(&sm.drain));
      uint32_t zero = 0;
      const WaitCtl dc{&zero, p.err, p.wait_limit_ns};
      mbar_wait(smem_u32(&sm.drain), 0, dc, LKV_WAIT(W_DRAIN));
    }
  } else if (warp >= 4 && (warp - 4) < n_sm_warps) {
    // ============================================================ softmax / epilogue
    const int r = tid - 128;                 // row == TMEM lane
    const uint32_t lb = static_cast<uint32_t>((warp & 3) * 32);
    const bool row_ok = r < p.R;
    const uint32_t peer = rank ^ 1u;
    uint32_t x_remote[2] = {0u, 0u}, xfull_remote[2] = {0u, 0u}, xfree_remote[2] = {0u, 0u};
    if (kPair) {
      for (int b = 0; b < 2; ++b) {
        x_remote[b] = map_to_peer(smem_u32(xbuf + (b * 128 + r) * kXRow), peer);
        xfull_remote[b] = map_to_peer(smem_u32(&sm.x_full[b]), peer);
        xfree_remote[b] = map_to_peer(smem_u32(&sm.x_free[b]), peer);
      }
    }
    const int col_base = kPair ? 256 * static_cast<int>(rank) : 0;

    // every lane of a softmax warp takes the same branch after a wait (tcgen05.ld/st are
    // warp-collective), so a wait that gives up in one lane ends the loop in all of them
    auto wait_all = [&](uint32_t bar, uint32_t par, int site) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, par, wc, site)) != 0;
    };
    auto wait_all_cl = [&](uint32_t bar, uint32_t par, int site) -> bool {
      return __all_sync(0xffffffffu, mbar_wait<true>(bar, par, wc, site)) != 0;
    };
    // (query token, head) of this row in a unit
    auto row_map = [&](const Segment& sg, int& i, int& h) {
      if (kPair) {
        i = sg.k;
        h = r;
      } else {
        i = r / p.hpg;
        h = sg.k * p.hpg + (r % p.hpg);
      }
    };
    // Stage the unit's query: non-RoPE part into TMEM (A operand), RoPE part into the
    // swizzled shared-memory A operand.
    auto load_q = [&](const Segment& sg) {
      int i, h;
      row_map(sg, i, h);
      const size_t qrow = (static_cast<size_t>(sg.b) * p.s_q + i) * p.h_q + h;
#pragma unroll 1
      for (int bx = 0; bx < Cfg::kNope; ++bx) {
        uint32_t w[32];
        if (row_ok) {
          const uint4* src = reinterpret_cast<const uint4*>(p.q_nope + qrow * p.dq + col_base + 64 * bx);
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const uint4 x = __ldg(src + v);
            w[4 * v] = x.x;
            w[4 * v + 1] = x.y;
            w[4 * v + 2] = x.z;
            w[4 * v + 3] = x.w;
          }
        } else {
#pragma unroll
          for (int v = 0; v < 32; ++v) w[v] = 0u;
        }
        tmem_st32(tm_addr(tbase, lb, Q0 + bx * 32), w);
      }
      if (Cfg::has_rope(rank)) {
        const uint4* src = reinterpret_cast<const uint4*>(p.q_rope + qrow * 64);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 x = row_ok ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
          *reinterpret_cast<uint4*>(qrope_smem + r * 128 + ((c ^ (r & 7)) << 4)) = x;
        }
        fence_proxy_async_smem();
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&sm.q_ready));
    };

    float m_run = -INFINITY, l_run = 0.f;
    // Softmax of one tile whose full scores are in s[]; writes P(n); runs the segment
    // epilogue after the unit's last tile of this range.
    auto process = [&](float (&s)[64], const Segment& sg, int t, long long n) -> bool {
      int qi, qh;
      row_map(sg, qi, qh);
      if (t == sg.tile_lo) {
        m_run = -INFINITY;
        l_run = 0.f;
      }
      const int lim = kPair ? sg.keys : (sg.L - p.s_q + qi + 1);  // keys visible to this row
      const int key0 = t * kTileN;
      float mx = -INFINITY;
      if (key0 + kTileN <= lim) {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          s[c] *= p.sl2;
          mx = fmaxf(mx, s[c]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          s[c] = (key0 + c < lim) ? s[c] * p.sl2 : -INFINITY;
          mx = fmaxf(mx, s[c]);
        }
      }
      // lazy rescale: keep the running max unless the tile max exceeds it by 2^8
      bool rescale = false;
      float m_new = m_run;
      if (mx > m_run + 8.f) {
        m_new = mx;
        rescale = (m_run != -INFINITY);
      }
      const float alpha = rescale ? ex2_approx(m_run - m_new) : 1.f;
      const float msub = (m_new == -INFINITY) ? 0.f : m_new;
      uint32_t pw[32];
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float e0 = ex2_approx(s[2 * c] - msub);
        const float e1 = ex2_approx(s[2 * c + 1] - msub);
        sum += e0 + e1;
        pw[c] = pack_bf16x2(e0, e1);
      }
      l_run = l_run * alpha + sum;
      m_run = m_new;
      const int pb = static_cast<int>(n & 1);
      // P buffer pb was last read by PV(n-2)
      if (n >= 2 && !wait_all(smem_u32(&sm.o_done[pb]), static_cast<uint32_t>(((n - 2) >> 1) & 1), LKV_WAIT(W_ODONE)))
        return false;
      if (__any_sync(0xffffffffu, rescale) && t != sg.tile_lo) {
        // O holds this segment's tiles up to n-1: wait for PV(n-1), then scale in place
        if (!wait_all(smem_u32(&sm.o_done[pb ^ 1]), static_cast<uint32_t>(((n - 1) >> 1) & 1), LKV_WAIT(W_ODONE)))
          return false;
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < DV; c += 32) {
          uint32_t o[32];
          tmem_ld32(tm_addr(tbase, lb, c), o);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
          tmem_st32(tm_addr(tbase, lb, c), o);
        }
      }
      tc_fence_after();
      tmem_st32(tm_addr(tbase, lb, P0 + 32 * pb), pw);
      if (key0 + kTileN > sg.keys) {
        // Rows past the unit's last key belong to another request or to unwritten cache:
        // their P is 0, but 0 * NaN would still poison O, so clear those V rows first.
        const int first = sg.keys - key0;
        const int per_box = (kTileN - first) * 8;  // 16-byte chunks per V box
        uint8_t* vb = dsm + (n % KS) * kStageBytes + Cfg::kVBox0 * kBoxBytes;
        for (int idx = r; idx < per_box * Cfg::kNV; idx += n_sm_threads) {
          const int bx = idx / per_box, rem = idx % per_box;
          *reinterpret_cast<uint4*>(vb + bx * kBoxBytes + (first + rem / 8) * 128 + (rem % 8) * 16) =
              make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&sm.p_full[pb]));
      if (t != sg.tile_hi - 1) return true;
      // ---------------------------------------------------------- segment epilogue
      if (!wait_all(smem_u32(&sm.o_done[pb]), static_cast<uint32_t>((n >> 1) & 1), LKV_WAIT(W_ODONE)))
        return false;
      tc_fence_after();
      const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
      const float lse_v = l_run > 0.f ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
      const size_t orow = (static_cast<size_t>(sg.b) * p.s_q + qi) * p.h_q + qh;
      if (sg.complete) {
        __nv_bfloat16* dst = p.out + orow * p.dv_total + col_base;
#pragma unroll 1
        for (int c = 0; c < DV; c += 32) {
          uint32_t o[32];
          tmem_ld32(tm_addr(tbase, lb, c), o);
          tmem_wait_ld();
          if (row_ok) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(o[8 * v + 0]) * inv_l, __uint_as_float(o[8 * v + 1]) * inv_l);
              w.y = pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv_l, __uint_as_float(o[8 * v + 3]) * inv_l);
              w.z = pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv_l, __uint_as_float(o[8 * v + 5]) * inv_l);
              w.w = pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv_l, __uint_as_float(o[8 * v + 7]) * inv_l);
              d4[v] = w;
            }
          }
        }
        if (row_ok && rank == 0) p.lse[orow] = lse_v;
      } else {
        const size_t prow = static_cast<size_t>(2 * range + sg.slot) * p.rmax + r;
        float* dst = p.part_o + prow * p.dv_total + col_base;
#pragma unroll 1
        for (int c = 0; c < DV; c += 32) {
          uint32_t o[32];
          tmem_ld32(tm_addr(tbase, lb, c), o);
          tmem_wait_ld();
          if (row_ok) {
            float4* d4 = reinterpret_cast<float4*>(dst + c);
#pragma unroll
            for (int v = 0; v < 8; ++v)
              d4[v] = make_float4(__uint_as_float(o[4 * v]) * inv_l, __uint_as_float(o[4 * v + 1]) * inv_l,
                                  __uint_as_float(o[4 * v + 2]) * inv_l, __uint_as_float(o[4 * v + 3]) * inv_l);
          }
        }
        if (row_ok && rank == 0) p.part_lse[prow] = lse_v;
        if (r == 0 && rank == 0) p.seg_info[2 * range + sg.slot] = sg.unit_id;
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&sm.o_free));
      return true;
    };

    SegCursor cur = cur0;
    Segment sgA, nx;
    bool haveA = cur.next(sa, sgA);
    int tA = haveA ? sgA.tile_lo : 0;
    long long nA = 0;
    // tile waiting for the peer's partial scores (MLA only)
    float prev[64];
    Segment sgB;
    int tB = 0;
    long long nB = 0;
    bool haveB = false;
    bool ok = true;
    if (haveA) load_q(sgA);
    while (ok && (haveA || haveB)) {
      float cs[64];
      bool gotA = false;
      Segment sgAc;
      int tAc = 0;
      long long nAc = 0;
      if (haveA) {
        if (!wait_all(smem_u32(&sm.s_full), static_cast<uint32_t>(nA & 1), LKV_WAIT(W_SFULL))) {
          ok = false;
          break;
        }
        tc_fence_after();
        {
          uint32_t a[32], b2[32];
          tmem_ld32(tm_addr(tbase, lb, S0), a);
          tmem_ld32(tm_addr(tbase, lb, S0 + 32), b2);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            cs[c] = __uint_as_float(a[c]);
            cs[32 + c] = __uint_as_float(b2[c]);
          }
        }
        tc_fence_before();
        mbar_arrive(smem_u32(&sm.s_free));
        const bool last = (tA == sgA.tile_hi - 1);
        bool have_nx = false;
        if (last) {
          // QK of this tile is done, so the query operands are free: stage the next unit's
          have_nx = cur.next(sa, nx);
          if (have_nx) load_q(nx);
        }
        if (kPair) {
          const int xb = static_cast<int>(nA & 1);
          if (nA >= 2 && !wait_all_cl(smem_u32(&sm.x_free[xb]), static_cast<uint32_t>(((nA - 2) >> 1) & 1),
                                      LKV_WAIT(W_XFREE))) {
            ok = false;
            break;
          }
#pragma unroll
          for (int c = 0; c < 64; c += 4) st_cluster_v4(x_remote[xb] + c * 4, cs[c], cs[c + 1], cs[c + 2], cs[c + 3]);
          mbar_arrive_remote(xfull_remote[xb]);
        }
        gotA = true;
        sgAc = sgA;
        tAc = tA;
        nAc = nA;
        ++nA;
        ++tA;
        if (last) {
          haveA = have_nx;
          if (haveA) {
            sgA = nx;
            tA = sgA.tile_lo;
          }
        }
      }
      if (kPair) {
        if (haveB) {
          const int xb = static_cast<int>(nB & 1);
          if (!wait_all_cl(smem_u32(&sm.x_full[xb]), static_cast<uint32_t>((nB >> 1) & 1), LKV_WAIT(W_XFULL))) {
            ok = false;
            break;
          }
          const float4* xr = reinterpret_cast<const float4*>(xbuf + (xb * 128 + r) * kXRow);
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const float4 x = xr[c];
            prev[4 * c] += x.x;
            prev[4 * c + 1] += x.y;
            prev[4 * c + 2] += x.z;
            prev[4 * c + 3] += x.w;
          }
          mbar_arrive_remote(xfree_remote[xb]);
          if (!process(prev, sgB, tB, nB)) {
            ok = false;
            break;
          }
        }
        haveB = gotA;
        if (gotA) {
#pragma unroll
          for (int c = 0; c < 64; ++c) prev[c] = cs[c];
          sgB = sgAc;
          tB = tAc;
          nB = nAc;
        }
      } else if (gotA) {
        if (!process(cs, sgAc, tAc, nAc)) {
          ok = false;
          break;
        }
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
  if (kPair) cluster_sync();
}

}  // namespace lkv
