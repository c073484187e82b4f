// Tensor-core (tcgen05 / TMEM) split-KV decode attention for sm_100a: the grouped forms.
//
// GQLA (g groups of expanded K_j, V_j), GLA (latent groups, K_j = V_j) and GTA (tied groups,
// K_j = V_j) run one persistent CTA per work range (lkv_sched.cuh) with one unit per segment:
// rows = heads of the group x new tokens (<= 128), padded to the M = 128 UMMA shape.  The MLA
// absorbed path runs on CTA pairs in lkv_mla_pair.cuh.  12 warps:
//   warp 0      TMA producer: streams key/value tiles of the cache (64 keys for GLA, 128 for
//               GQLA and GTA) into rings of shared-memory stages (2-D boxes of tile rows x 64
//               bf16, 128-byte swizzle).
//   warp 1      TMEM owner and QK issuer (one thread): S = Q K^T into TMEM.  The non-RoPE part
//               of Q is an A operand in TMEM, the RoPE part one in shared memory; K is the B
//               operand in the stage.
//   warp 2      PV issuer (one thread): O += P V into TMEM, P an A operand in TMEM, V read
//               MN-major from the very same swizzled tile that served as K where K = V.
//   warps 4-11  softmax / epilogue: warp 4 + q + 4h owns TMEM lane quadrant q and key-column
//               half h of each tile; the two halves of a row agree on the running max through a
//               bounded shared-memory exchange.
//
// TMEM columns: O [0, DV) | S [DV, DV+T) | P0, P1 [DV+T, DV+2T) | Q [DV+2T, ...) for T keys/tile.
// P is double buffered so the softmax of tile n+1 never waits for the PV of tile n.
//
// GTA over FP8 cache rows (MODE_GTA8): the producer loads the group's e4m3 codes, the tokens'
// power-of-two scales and the RoPE key; warps 6, 7, 10 and 11 (idle in the other modes when a unit
// has at most 64 rows) convert the codes into the bf16 tied state of the stage, exactly (a 4-bit
// significand times a power of two), after which the tile is used as in MODE_GTA.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include "lkv_ptx.cuh"
#include "lkv_sched.cuh"
#include "../../include/lkv.h"

// Error-word code of a bounded wait that gave up: base + 20 * mode + site.
#define LKV_WAIT(x) (LKV_SITE_WAIT_BASE + 20 * kMode + (x))

namespace lkv {

constexpr int kTcThreads = 384;
constexpr int kTmemCols = 512;

// Sum of the two bf16 values packed in w.
__device__ __forceinline__ float bf16x2_sum(uint32_t w) {
  return __uint_as_float(w << 16) + __uint_as_float(w & 0xffff0000u);
}

// MODE_GTA: grouped-tied attention, the GQLA shapes with K_j = V_j (one tied state per group).
// (Mode 0, the MLA absorbed path, runs in lkv_mla_pair.cuh; the numbering keeps wait-site codes stable.)
// MODE_GTA8: MODE_GTA over FP8 (e4m3) cache rows.
enum DecodeMode { MODE_GQLA = 1, MODE_GLA = 2, MODE_GTA = 3, MODE_GTA8 = 5 };

// Wait sites (added to LKV_SITE_WAIT_BASE in the error word).
enum WaitSite {
  W_EMPTY = 1, W_FULL, W_SFREE, W_QREADY, W_PFULL, W_OFREE, W_SFULL, W_ODONE, W_DRAIN = 11, W_XCHG = 13, W_CONV
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
  int fp8_scale_col;            // MODE_GTA8: column (4-byte units) of a row's scale
  int fp8_rope_col;             // MODE_GTA8: column (bf16 units) of a row's RoPE key
};

template <int kMode>
struct ModeCfg {
  static constexpr bool kFp8 = (kMode == MODE_GTA8);
  static constexpr bool kTied128 = (kMode == MODE_GTA || kMode == MODE_GTA8);  // one tied 128-wide state
  static constexpr bool kHead128 = (kMode == MODE_GQLA || kTied128);  // d_h = 128 groups
  // Keys per tile.  GQLA runs 128-key tiles so that every QK UMMA is N = 128 (one issuing
  // thread then keeps the tensor pipe at full rate); GLA keeps 64-key tiles because a
  // 128-column S tile would not fit next to its 256-column O accumulator and resident Q.
  static constexpr int kTile = kHead128 ? 128 : 64;
  static constexpr int kBoxBytes = kTile * 128;                 // one TMA box: kTile rows x 64 bf16
  // GQLA keeps K (+ k_rope) and V in separate rings: a K slot is refilled as soon as its QK
  // is done, while V waits for its PV.  Where K = V (GLA, GTA) one ring holds the tile.
  static constexpr bool kSplitKV = (kMode == MODE_GQLA);
  static constexpr int kKBoxes = kHead128 ? 2 : 4;  // 64-column boxes of the non-RoPE key per stage
  static constexpr int kRopeBoxBytes = kBoxBytes;  // the whole 64-column RoPE key
  // FP8 stages also hold the codes (kTile rows x 128 bytes) and scales (kTile rows x 16 bytes) that
  // the bf16 state is converted from
  static constexpr int kCodesOff = kKBoxes * kBoxBytes + kRopeBoxBytes;
  static constexpr int kScalesOff = kCodesOff + kTile * 128;
  static constexpr int kStageBytes = kKBoxes * kBoxBytes + kRopeBoxBytes + (kFp8 ? kTile * (128 + 16) : 0);
  // bytes the producer's copies bring into a stage
  static constexpr int kTmaBytes = kFp8 ? kTile * (128 + 16) + kRopeBoxBytes : kStageBytes;
  static constexpr int kVStageBytes = 2 * kBoxBytes;                  // V ring (GQLA)
  static constexpr int kDV = kHead128 ? 128 : 256;  // value columns per CTA
  // GTA holds a stage from its load to its PV (K = V), so it gets the ring depth that GQLA
  // splits between its K ring (2) and V ring (3)
  static constexpr int kStages = (kMode == MODE_GQLA) ? 2 : (kMode == MODE_GTA ? 4 : (kFp8 ? 3 : 5));
  static constexpr int kVStages = kSplitKV ? 3 : 1;
  static constexpr int kNope = kHead128 ? 2 : 4;    // non-RoPE Q boxes (in TMEM)
  static constexpr int kRopeBox = kKBoxes;          // stage box holding k_rope
  static constexpr int kVBox0 = 0;                              // first V box (V ring or stage)
  static constexpr int kNV = kDV / 64;
  static constexpr int kPCols = kTile / 2;                      // bf16 P per buffer
  static constexpr uint32_t S0 = kDV, P0 = kDV + kTile, Q0 = kDV + 2 * kTile;
  static constexpr size_t kRingBytes =
      static_cast<size_t>(kStages) * kStageBytes + (kSplitKV ? static_cast<size_t>(kVStages) * kVStageBytes : 0);
  // The RoPE part of the query sits in shared memory as an A operand: 128 rows of 64 columns
  // (128-byte swizzle).
  static constexpr int kQropeBytes = 128 * 128;
  static constexpr int kRopeSteps = 4;  // QK K-steps over the RoPE columns
  static constexpr size_t kSmemBytes = 1024 + kRingBytes + kQropeBytes;
};
static_assert(ModeCfg<MODE_GLA>::Q0 + 32 * ModeCfg<MODE_GLA>::kNope <= kTmemCols, "TMEM budget");
static_assert(ModeCfg<MODE_GQLA>::Q0 + 32 * ModeCfg<MODE_GQLA>::kNope <= kTmemCols, "TMEM budget");
static_assert(ModeCfg<MODE_GTA>::Q0 + 32 * ModeCfg<MODE_GTA>::kNope <= kTmemCols, "TMEM budget");
static_assert(ModeCfg<MODE_GLA>::kSmemBytes <= 232448, "shared memory budget");
static_assert(ModeCfg<MODE_GQLA>::kSmemBytes <= 232448, "shared memory budget");
static_assert(ModeCfg<MODE_GTA>::kSmemBytes <= 232448, "shared memory budget");
static_assert(ModeCfg<MODE_GTA>::kStageBytes == 3 * ModeCfg<MODE_GTA>::kBoxBytes, "GTA stage: tied state + RoPE key");
static_assert(ModeCfg<MODE_GTA8>::Q0 + 32 * ModeCfg<MODE_GTA8>::kNope <= kTmemCols, "TMEM budget");
static_assert(ModeCfg<MODE_GTA8>::kSmemBytes <= 232448, "shared memory budget");
static_assert(ModeCfg<MODE_GTA8>::kScalesOff % 1024 == 0 && ModeCfg<MODE_GTA8>::kStageBytes % 1024 == 0,
              "FP8 stage fields on 1024-byte boundaries");

// Two e4m3 codes (the low byte first) times a power-of-two scale, packed as bf16x2: exact, since
// every e4m3 value is an f16 normal (or zero) with a 4-bit significand.
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t two_codes, float s) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two_codes & 0xffffu), __NV_E4M3);
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
  return pack_bf16x2(f.x * s, f.y * s);
}

// Advance a shared-memory descriptor by a byte offset (start-address field, 16-byte units).
template <int kStagesT, int kVStagesT>
struct __align__(16) TcSmem {
  uint64_t full[kStagesT];
  uint64_t empty[kStagesT];
  uint64_t conv[kStagesT];          // MODE_GTA8: the stage's codes are converted to bf16
  uint64_t vfull[kVStagesT];
  uint64_t vempty[kVStagesT];
  uint64_t s_full, s_free;         // the S buffer
  uint64_t o_free, q_ready, drain;
  uint64_t p_full[2], o_done[2];
  uint64_t xbar[4][2];              // per lane quadrant: both column halves posted a value
  float xch[2][2][128];             // [buffer][column half][row] values swapped between the halves
  uint32_t tmem_base;
  uint32_t abort;
  long long t_begin, t_end, unit_t0;
  int b0, k0;
};

__device__ __forceinline__ uint32_t tm_addr(uint32_t base, uint32_t lane_base, uint32_t col) {
  return base + (lane_base << 16) + col;
}

// Rarely executed per-row blocks of the softmax warps, kept out of line so that the per-tile loops
// stay short in the instruction cache.  `trow` is the TMEM address of this thread's row at column
// c0; every lane of the warp calls them together (tcgen05.ld / st are warp-collective).
// O[row, c0 .. c0+ncols) *= alpha.
__device__ __noinline__ void tmem_scale_row(uint32_t trow, int ncols, float alpha) {
#pragma unroll 1
  for (int c = 0; c < ncols; c += 32) {
    uint32_t o[32];
    tmem_ld32(trow + c, o);
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
    tmem_st32(trow + c, o);
  }
  tmem_wait_st();
}
// dst[0 .. ncols) = bf16(O[row, c0 ..] * inv_l) (stores skipped for a padding row).
__device__ __noinline__ void tmem_row_to_bf16(uint32_t trow, int ncols, float inv_l, __nv_bfloat16* dst, bool store) {
#pragma unroll 1
  for (int c = 0; c < ncols; c += 32) {
    uint32_t o[32];
    tmem_ld32(trow + c, o);
    tmem_wait_ld();
    if (store) {
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
}
// dst[0 .. ncols) = O[row, c0 ..] * inv_l in fp32 (a split partial).
__device__ __noinline__ void tmem_row_to_f32(uint32_t trow, int ncols, float inv_l, float* dst, bool store) {
#pragma unroll 1
  for (int c = 0; c < ncols; c += 32) {
    uint32_t o[32];
    tmem_ld32(trow + c, o);
    tmem_wait_ld();
    if (store) {
      float4* d4 = reinterpret_cast<float4*>(dst + c);
#pragma unroll
      for (int v = 0; v < 8; ++v)
        d4[v] = make_float4(__uint_as_float(o[4 * v]) * inv_l, __uint_as_float(o[4 * v + 1]) * inv_l,
                            __uint_as_float(o[4 * v + 2]) * inv_l, __uint_as_float(o[4 * v + 3]) * inv_l);
    }
  }
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
  constexpr int TN = Cfg::kTile;
  constexpr int kBoxBytes = Cfg::kBoxBytes;
  constexpr int kStageBytes = Cfg::kStageBytes;
  constexpr uint32_t S0 = Cfg::S0, P0 = Cfg::P0, Q0 = Cfg::Q0;

  extern __shared__ __align__(1024) uint8_t dsmem_raw[];
  constexpr int VS = Cfg::kVStages;
  constexpr bool kSplit = Cfg::kSplitKV;
  __shared__ TcSmem<KS, VS> sm;
  uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  const uint32_t stage_base = smem_u32(dsm);
  uint8_t* vring = dsm + KS * kStageBytes;                 // GQLA V ring
  const uint32_t vring_base = smem_u32(vring);
  uint8_t* qrope_smem = dsm + Cfg::kRingBytes;
  const uint32_t qrope_base = smem_u32(qrope_smem);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int range = blockIdx.x;
  const int n_row_warps = (p.R + 31) >> 5;  // lane quadrants holding valid rows
  const int n_sm_warps = 2 * n_row_warps;     // softmax warps: two column halves per quadrant
  const int n_sm_threads = n_sm_warps * 32;

  SchedArgs sa0;
  sa0.cu = p.cu;
  sa0.B = p.B;
  sa0.s_q = p.s_q;
  sa0.tile = TN;
  sa0.units_per_req = p.G;
  sa0.per_query_units = 0;
  sa0.P = p.P;
  // grouped units in lockstep (lkv_sched.cuh): the cursor walks request space, and this range
  // serves group kfix of block range / G
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

  // ---------------------------------------------------------------- set-up
  if (tid == 0) {
    for (int s = 0; s < KS; ++s) {
      mbar_init(smem_u32(&sm.full[s]), 1);
      mbar_init(smem_u32(&sm.empty[s]), 1);
      mbar_init(smem_u32(&sm.conv[s]), 4);  // one arrival per converter warp
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(smem_u32(&sm.vfull[s]), 1);
      mbar_init(smem_u32(&sm.vempty[s]), 1);
    }
    mbar_init(smem_u32(&sm.s_full), 1);
    // softmax-side barriers take one arrival per softmax warp (lane 0, after a __syncwarp)
    mbar_init(smem_u32(&sm.s_free), n_sm_warps);
    mbar_init(smem_u32(&sm.o_free), n_sm_warps);
    mbar_init(smem_u32(&sm.q_ready), n_sm_warps);
    mbar_init(smem_u32(&sm.drain), 2);  // one commit from each UMMA issuer
    for (int q = 0; q < 4; ++q)
      for (int b = 0; b < 2; ++b) mbar_init(smem_u32(&sm.xbar[q][b]), 2);
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&sm.p_full[b]), n_sm_warps);
      mbar_init(smem_u32(&sm.o_done[b]), 1);
    }
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    bool malformed = false;
    SegCursor c = locate_range(sa, sched_range, &malformed);
    if (lane == 0) {
      // a request shorter than s_q gets no tiles (its outputs are left unwritten): report it
      if (malformed && range == 0) record_error(p.err, LKV_SITE_BAD_LENGTH);
      sm.t_begin = c.t_begin;
      sm.t_end = c.t_end;
      sm.unit_t0 = c.unit_t0;
      sm.b0 = c.b;
      sm.k0 = c.k;
      p.seg_info[2 * range] = -1;
      p.seg_info[2 * range + 1] = -1;
      tma_prefetch_desc(&map_a);
      tma_prefetch_desc(&map_r);
      if (kMode == MODE_GQLA || kMode == MODE_GTA8) tma_prefetch_desc(&map_v);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&sm.tmem_base), kTmemCols);
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
      const uint32_t bytes = Cfg::kTmaBytes;
      SegCursor cur = cur0;
      Segment sg;
      int n = 0, nv = 0;   // K (or whole) tiles and V tiles issued (a CTA's tile count fits an int)
      bool ok = true;
      while (ok && next_seg(cur, sg)) {
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
          const int row = sg.cu_b + t * TN;
          if constexpr (kMode == MODE_GQLA) {
            const int c0 = 128 * sg.k;
            tma_load_2d(dst, &map_a, fb, c0, row);
            tma_load_2d(dst + kBoxBytes, &map_a, fb, c0 + 64, row);
            tma_load_2d(dst + 2 * kBoxBytes, &map_r, fb, 0, row);
            // V goes to its own ring slot, freed only by the PV of this tile
            const int vs = static_cast<int>(n % VS);
            if (!mbar_wait(smem_u32(&sm.vempty[vs]), static_cast<uint32_t>(((n / VS) & 1) ^ 1), wc,
                           LKV_WAIT(W_EMPTY))) {
              ok = false;
              ++n;  // this tile's K copies are in flight: the drain below must wait for them
              break;
            }
            const uint32_t vb = smem_u32(&sm.vfull[vs]);
            mbar_arrive_expect_tx(vb, Cfg::kVStageBytes);
            const uint32_t vdst = vring_base + vs * Cfg::kVStageBytes;
            tma_load_2d(vdst, &map_v, vb, c0, row);
            tma_load_2d(vdst + kBoxBytes, &map_v, vb, c0 + 64, row);
            ++nv;
          } else if constexpr (kMode == MODE_GTA) {
            // the group's tied state (key without RoPE, and value) and the shared RoPE key
            const int c0 = 128 * sg.k;
            tma_load_2d(dst, &map_a, fb, c0, row);
            tma_load_2d(dst + kBoxBytes, &map_a, fb, c0 + 64, row);
            tma_load_2d(dst + 2 * kBoxBytes, &map_r, fb, 0, row);
          } else if constexpr (kMode == MODE_GTA8) {
            // the group's 128 codes per row, the rows' scales (with their 12 zero bytes) and the
            // shared RoPE key; the converter warps fill the bf16 state at the stage's start
            tma_load_2d(dst + Cfg::kCodesOff, &map_a, fb, 128 * sg.k, row);
            tma_load_2d(dst + Cfg::kScalesOff, &map_v, fb, p.fp8_scale_col, row);
            tma_load_2d(dst + 2 * kBoxBytes, &map_r, fb, p.fp8_rope_col, row);
          } else {
            const int c0 = 256 * sg.k;
            for (int bx = 0; bx < 4; ++bx) tma_load_2d(dst + bx * kBoxBytes, &map_a, fb, c0 + 64 * bx, row);
            tma_load_2d(dst + 4 * kBoxBytes, &map_r, fb, 0, row);
          }
        }
      }
      // never leave copies in flight into a CTA that is about to exit
      const int inflight = n < KS ? n : KS;
      uint32_t zero = 0;
      const WaitCtl dc{&zero, p.err, p.wait_limit_ns};  // ignores the abort flag, keeps the limit
      for (int m = n - inflight; m < n; ++m)
        mbar_wait(smem_u32(&sm.full[m % KS]), static_cast<uint32_t>((m / KS) & 1), dc, LKV_WAIT(W_DRAIN));
      if (kSplit) {
        // V copies: issued for every tile whose K was issued, except possibly the last one when
        // its vempty wait gave up; wait only for those actually issued (counted by nv)
        const int vin = nv < VS ? nv : VS;
        for (int m = nv - vin; m < nv; ++m)
          mbar_wait(smem_u32(&sm.vfull[m % VS]), static_cast<uint32_t>((m / VS) & 1), dc, LKV_WAIT(W_DRAIN));
      }
    }
  } else if (warp == 1 || warp == 2) {
    // ============================================================ UMMA issuers
    // Warp 1 issues the QK products and warp 2 the PV products.  Two issuing threads keep
    // more MMAs in flight than one, and neither chain stalls behind the other's operands: a
    // QK waits only for its key tile and a free S, a PV only for its P (and a free O).
    if (lane == 0) {
      SegCursor cur = cur0;
      Segment sg;
      int n = 0;         // tile counter of this CTA
      int seg = 0;       // segments started
      bool ok = true;
      if (warp == 1) {
        const uint32_t id_qk = idesc_bf16(128, TN, 0, 0);
        const uint64_t qrope_desc = sdesc_sw128(qrope_base, 16, 1024);
        while (ok && next_seg(cur, sg)) {
          for (int t = sg.tile_lo; t < sg.tile_hi; ++t, ++n) {
            const int st = static_cast<int>(n % KS);
            // one S buffer: tile n's QK waits until the softmax has read tile n-1's scores
            const uint32_t kbar = Cfg::kFp8 ? smem_u32(&sm.conv[st]) : smem_u32(&sm.full[st]);
            if (!mbar_wait(kbar, static_cast<uint32_t>((n / KS) & 1), wc, LKV_WAIT(Cfg::kFp8 ? W_CONV : W_FULL)) ||
                (n >= 1 && !mbar_wait(smem_u32(&sm.s_free), static_cast<uint32_t>((n - 1) & 1), wc, LKV_WAIT(W_SFREE))) ||
                (t == sg.tile_lo &&
                 !mbar_wait(smem_u32(&sm.q_ready), static_cast<uint32_t>(seg & 1), wc, LKV_WAIT(W_QREADY)))) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t kdesc = sdesc_sw128(stage_base + st * kStageBytes, 16, 1024);
#pragma unroll
            for (int ks = 0; ks < 4 * Cfg::kNope; ++ks) {
              const int bx = ks >> 2, kk = ks & 3;
              umma_ts(tbase + S0, tbase + Q0 + bx * 32 + kk * 8, desc_add(kdesc, bx * kBoxBytes + kk * 32), id_qk,
                      ks ? 1u : 0u);
            }
            const uint32_t rope_addr = stage_base + st * kStageBytes + Cfg::kRopeBox * kBoxBytes;
            const uint64_t rdesc = sdesc_sw128(rope_addr, 16, 1024);
#pragma unroll
            for (int kk = 0; kk < Cfg::kRopeSteps; ++kk)
              umma_ss(tbase + S0, desc_add(qrope_desc, kk * 32), desc_add(rdesc, kk * 32), id_qk, 1u);
            umma_commit(smem_u32(&sm.s_full));
            if (kSplit) umma_commit(smem_u32(&sm.empty[st]));  // the K slot is free once QK is done
          }
          ++seg;
        }
      } else {
        const uint32_t id_pv = idesc_bf16(128, DV, 0, 1);
        while (ok && next_seg(cur, sg)) {
          for (int t = sg.tile_lo; t < sg.tile_hi; ++t, ++n) {
            const int pb = static_cast<int>(n & 1);
            const bool first = (t == sg.tile_lo);
            if (!mbar_wait(smem_u32(&sm.p_full[pb]), static_cast<uint32_t>((n >> 1) & 1), wc, LKV_WAIT(W_PFULL)) ||
                (first && seg > 0 &&
                 !mbar_wait(smem_u32(&sm.o_free), static_cast<uint32_t>((seg - 1) & 1), wc, LKV_WAIT(W_OFREE))) ||
                (kSplit && !mbar_wait(smem_u32(&sm.vfull[n % VS]), static_cast<uint32_t>((n / VS) & 1), wc,
                                      LKV_WAIT(W_FULL)))) {
              ok = false;
              break;
            }
            tc_fence_after();
            // P(n) exists only after S(n) was read, so QK(n) is complete and the whole stage
            // (K and V, where they share it) is free once this PV completes
            const uint32_t vaddr = kSplit ? vring_base + static_cast<uint32_t>(n % VS) * Cfg::kVStageBytes
                                          : stage_base + static_cast<uint32_t>(n % KS) * kStageBytes;
            const uint64_t vdesc = sdesc_sw128(vaddr + Cfg::kVBox0 * kBoxBytes, kBoxBytes, 1024);
            const uint32_t pa = tbase + P0 + Cfg::kPCols * pb;
#pragma unroll
            for (int kk = 0; kk < TN / 16; ++kk)
              umma_ts(tbase, pa + kk * 8, desc_add(vdesc, kk * 2048), id_pv, (first && kk == 0) ? 0u : 1u);
            umma_commit(smem_u32(&sm.o_done[pb]));
            umma_commit(kSplit ? smem_u32(&sm.vempty[n % VS]) : smem_u32(&sm.empty[n % KS]));
          }
          ++seg;
        }
      }
      // all tcgen05 work of both issuers done before TMEM is released
      umma_commit(smem_u32(&sm.drain));
      uint32_t zero = 0;
      const WaitCtl dc{&zero, p.err, p.wait_limit_ns};
      mbar_wait(smem_u32(&sm.drain), 0, dc, LKV_WAIT(W_DRAIN));
    }
  } else if (Cfg::kFp8 && warp >= 4 && warp < 12 && ((warp - 4) & 3) >= 2) {
    // ============================================================ FP8 converters (MODE_GTA8)
    // Thread `row` turns key row `row` of each tile from 128 e4m3 codes (128-byte swizzled box)
    // into 128 bf16 values in the stage's two 64-column state boxes (the layout a TMA copy with
    // 128-byte swizzle writes).  Rows past the unit's keys become zeros.
    const int row = 64 * ((warp - 4) >> 2) + 32 * (((warp - 4) & 3) - 2) + lane;
    SegCursor cur = cur0;
    Segment sg;
    int n = 0;
    bool ok = true;
    while (ok && next_seg(cur, sg)) {
      for (int t = sg.tile_lo; t < sg.tile_hi; ++t, ++n) {
        const int st = static_cast<int>(n % KS);
        if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.full[st]), static_cast<uint32_t>((n / KS) & 1), wc,
                                               LKV_WAIT(W_FULL)))) {
          ok = false;
          break;
        }
        uint8_t* sb = dsm + st * kStageBytes;
        const bool valid = t * TN + row < sg.keys;
        const float sc = valid ? *reinterpret_cast<const float*>(sb + Cfg::kScalesOff + row * 16) : 0.f;
        const int sw = row & 7;
        const uint8_t* crow = sb + Cfg::kCodesOff + row * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j) {  // codes 16 j .. 16 j + 15 -> bf16 chunks 2 (j % 4), +1 of box j / 4
          const uint4 c = valid ? *reinterpret_cast<const uint4*>(crow + ((j ^ sw) << 4)) : make_uint4(0u, 0u, 0u, 0u);
          const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
          uint32_t o[8];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            o[2 * k] = e4m3x2_to_bf16x2(cw[k], sc);
            o[2 * k + 1] = e4m3x2_to_bf16x2(cw[k] >> 16, sc);
          }
          uint8_t* box = sb + (j >> 2) * kBoxBytes + row * 128;
          const int cc = 2 * (j & 3);
          *reinterpret_cast<uint4*>(box + ((cc ^ sw) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
          *reinterpret_cast<uint4*>(box + (((cc + 1) ^ sw) << 4)) = make_uint4(o[4], o[5], o[6], o[7]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.conv[st]));
      }
    }
  } else if (warp >= 4 && warp < 12 && ((warp - 4) & 3) < n_row_warps) {
    // ============================================================ softmax / epilogue
    const int q4 = (warp - 4) & 3;             // TMEM lane quadrant
    const int hf = (warp - 4) >> 2;            // key-column half of the tile
    const int r = q4 * 32 + lane;              // row == TMEM lane
    const uint32_t lb = static_cast<uint32_t>(q4 * 32);
    const bool row_ok = r < p.R;
    const int sidx = hf * n_row_warps * 32 + r;  // 0 .. n_sm_threads-1
    constexpr int HC = TN / 2;                 // key columns of this thread per tile
    constexpr int HW = HC / 2;                 // packed fp16 / bf16 pairs
    const int c0 = hf * HC;

    // every lane of a softmax warp takes the same branch after a wait (tcgen05.ld/st are
    // warp-collective), so a wait that gives up in one lane ends the loop in all of them
    auto wait_all = [&](uint32_t bar, uint32_t par, int site) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, par, wc, site)) != 0;
    };
    auto warp_arrive = [&](uint32_t bar) {
      __syncwarp();
      if (lane == 0) mbar_arrive(bar);
    };
    auto wait_all_cl = [&](uint32_t bar, uint32_t par, int site) -> bool {
      return __all_sync(0xffffffffu, mbar_wait<true>(bar, par, wc, site)) != 0;
    };
    // Swap one value per row with the other column half of this quadrant (double-buffered,
    // bounded wait: a partner that gave up ends this warp's loop too).
    int xc = 0;
    auto pair_xchg = [&](float v, float& other) -> bool {
      const int b = xc & 1;
      sm.xch[b][hf][r] = v;
      warp_arrive(smem_u32(&sm.xbar[q4][b]));
      const bool okx = wait_all(smem_u32(&sm.xbar[q4][b]), static_cast<uint32_t>((xc >> 1) & 1), LKV_WAIT(W_XCHG));
      other = sm.xch[b][hf ^ 1][r];
      ++xc;
      return okx;
    };
    // (query token, head) of this row in a unit
    auto row_map = [&](const Segment& sg, int& i, int& h) {
      i = r / p.hpg;
      h = sg.k * p.hpg + (r % p.hpg);
    };
    // Stage the unit's query: non-RoPE part into TMEM (A operand; each half writes every
    // other 64-column box), RoPE part (half 0) into the swizzled shared-memory A operand.
    auto load_q = [&](const Segment& sg) {
      int i, h;
      row_map(sg, i, h);
      const size_t qrow = (static_cast<size_t>(sg.b) * p.s_q + i) * p.h_q + h;
#pragma unroll 1
      for (int bx = hf; bx < Cfg::kNope; bx += 2) {
        uint32_t w[32];
        if (row_ok) {
          const uint4* src = reinterpret_cast<const uint4*>(p.q_nope + qrow * p.dq + 64 * bx);
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
      if (hf == 0) {
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
      warp_arrive(smem_u32(&sm.q_ready));
    };

    // Running max (shared by both halves of a row) and this half's running sums.
    float m_run = -INFINITY, l_run = 0.f, lb_run = 0.f;
    // Lazy rescale: keep the running max unless the tile max exceeds it by 2^8.
    auto new_max = [&](float mx, bool& rescale, float& alpha) -> float {
      rescale = false;
      float m_new = m_run;
      if (mx > m_run + 8.f) {
        m_new = mx;
        rescale = (m_run != -INFINITY);
      }
      alpha = rescale ? ex2_approx(m_run - m_new) : 1.f;
      return m_new;
    };
    // Grouped modes: softmax of this half of one tile whose scores are in s[] -> P bits in
    // pw[], the running max / sum updated; `alpha` rescales O when the running max moved.
    auto softmax_tile = [&](float (&s)[HC], const Segment& sg, int t, int qi, uint32_t (&pw)[HW], bool& rescale,
                            float& alpha) -> bool {
      if (t == sg.tile_lo) {
        m_run = -INFINITY;
        l_run = 0.f;
        lb_run = 0.f;
      }
      // keys of this half of the tile visible to this row
      const int rem = (sg.L - p.s_q + qi + 1) - (t * TN + c0);
      // max of the raw scores (the scale is positive), then one FMA per score for the
      // exponent in log2 units
      if (rem < HC) {
#pragma unroll
        for (int c = 0; c < HC; ++c) s[c] = (c < rem) ? s[c] : -INFINITY;
      }
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c = 0; c < HC; ++c) m4[c & 3] = fmaxf(m4[c & 3], s[c]);
      const float mh = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * p.sl2;
      float mo;
      if (!pair_xchg(mh, mo)) return false;
      const float mx = fmaxf(mh, mo);  // this tile's row max
      const float m_new = new_max(mx, rescale, alpha);
      // exponents centred on the tile max (<= 0, so the fp16 argument of the best keys is exact
      // or nearly so), times f = 2^(mx - m_new) <= 2^8 in fp32
      const float msub = (mx == -INFINITY) ? 0.f : mx;
      const float f = (mx == -INFINITY) ? 0.f : ex2_approx(mx - m_new);
      float s4[4] = {0.f, 0.f, 0.f, 0.f}, b4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < HW; ++c) {
        const uint32_t h = ex2_f16x2(fmaf(s[2 * c], p.sl2, -msub), fmaf(s[2 * c + 1], p.sl2, -msub));
        const float e0 = f16_lo(h) * f, e1 = f16_hi(h) * f;
        s4[c & 3] += e0 + e1;
        pw[c] = pack_bf16x2(e0, e1);
        b4[c & 3] += bf16x2_sum(pw[c]);
      }
      // l_run (fp32 weights) gives the lse; lb_run sums the bf16 weights PV actually used
      l_run = l_run * alpha + ((s4[0] + s4[1]) + (s4[2] + s4[3]));
      lb_run = lb_run * alpha + ((b4[0] + b4[1]) + (b4[2] + b4[3]));
      m_run = m_new;
      return true;
    };
    // Common tail of a tile: publish this half of P(n) (after the PV that last read its
    // buffer), rescale this half of O's columns if the running max moved, and run the segment
    // epilogue after the unit's last tile here.
    auto finish_tile = [&](uint32_t (&pw)[HW], bool rescale, float alpha, const Segment& sg, int t,
                           int n) -> bool {
      int qi, qh;
      row_map(sg, qi, qh);
      const int key0 = t * TN;
      const int pb = static_cast<int>(n & 1);
      // P buffer pb was last read by PV(n-2)
      if (n >= 2 && !wait_all(smem_u32(&sm.o_done[pb]), static_cast<uint32_t>(((n - 2) >> 1) & 1), LKV_WAIT(W_ODONE)))
        return false;
      if (__any_sync(0xffffffffu, rescale ? 1 : 0) && t != sg.tile_lo) {
        // O holds this segment's tiles up to n-1: wait for PV(n-1), then scale in place
        if (!wait_all(smem_u32(&sm.o_done[pb ^ 1]), static_cast<uint32_t>(((n - 1) >> 1) & 1), LKV_WAIT(W_ODONE)))
          return false;
        tc_fence_after();
        tmem_scale_row(tm_addr(tbase, lb, hf * (DV / 2)), DV / 2, alpha);
      }
      tc_fence_after();
      {
        const uint32_t pcol = P0 + Cfg::kPCols * pb + hf * HW;
        if constexpr (HW == 16) {
          tmem_st16(tm_addr(tbase, lb, pcol), pw);
        } else {
#pragma unroll
          for (int c = 0; c < HW; c += 32) {
            uint32_t w[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) w[j] = pw[c + j];
            tmem_st32(tm_addr(tbase, lb, pcol + c), w);
          }
        }
      }
      if (!Cfg::kFp8 && key0 + TN > sg.keys) {
        // (The FP8 converters write zeros there themselves.)
        // Rows past the unit's last key belong to another request or to unwritten cache:
        // their P is 0, but 0 * NaN would still poison O, so clear those V rows first.
        const int first = sg.keys - key0;
        const int per_box = (TN - first) * 8;  // 16-byte chunks per V box
        if (kSplit && !wait_all(smem_u32(&sm.vfull[n % VS]), static_cast<uint32_t>((n / VS) & 1), LKV_WAIT(W_FULL)))
          return false;  // the copy must land before it is overwritten
        uint8_t* vb = (kSplit ? vring + (n % VS) * Cfg::kVStageBytes : dsm + (n % KS) * kStageBytes) +
                      Cfg::kVBox0 * kBoxBytes;
        for (int idx = sidx; idx < per_box * Cfg::kNV; idx += n_sm_threads) {
          const int bx = idx / per_box, rem = idx % per_box;
          *reinterpret_cast<uint4*>(vb + bx * kBoxBytes + (first + rem / 8) * 128 + (rem % 8) * 16) =
              make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
      }
      tmem_wait_st();
      tc_fence_before();
      warp_arrive(smem_u32(&sm.p_full[pb]));
      if (t != sg.tile_hi - 1) return true;
      // ---------------------------------------------------------- segment epilogue
      float l_other, lb_other;
      if (!pair_xchg(l_run, l_other) || !pair_xchg(lb_run, lb_other)) return false;
      const float l_tot = l_run + l_other, lb_tot = lb_run + lb_other;
      if (!wait_all(smem_u32(&sm.o_done[pb]), static_cast<uint32_t>((n >> 1) & 1), LKV_WAIT(W_ODONE)))
        return false;
      tc_fence_after();
      const float inv_l = lb_tot > 0.f ? 1.f / lb_tot : 0.f;
      const float lse_v = l_tot > 0.f ? (m_run + __log2f(l_tot)) * 0.69314718055994531f : -INFINITY;
      const size_t orow = (static_cast<size_t>(sg.b) * p.s_q + qi) * p.h_q + qh;
      if (sg.complete) {
        tmem_row_to_bf16(tm_addr(tbase, lb, hf * (DV / 2)), DV / 2, inv_l, p.out + orow * p.dv_total + hf * (DV / 2),
                         row_ok);
        if (row_ok && hf == 0) p.lse[orow] = lse_v;
      } else {
        const size_t prow = static_cast<size_t>(2 * range + sg.slot) * p.rmax + r;
        tmem_row_to_f32(tm_addr(tbase, lb, hf * (DV / 2)), DV / 2, inv_l, p.part_o + prow * p.dv_total + hf * (DV / 2),
                        row_ok);
        if (row_ok && hf == 0) p.part_lse[prow] = lse_v;
        if (r == 0 && hf == 0) p.seg_info[2 * range + sg.slot] = sg.unit_id;
      }
      tc_fence_before();
      warp_arrive(smem_u32(&sm.o_free));
      return true;
    };

    SegCursor cur = cur0;
    Segment sgA, nx;
    bool haveA = next_seg(cur, sgA);
    int tA = haveA ? sgA.tile_lo : 0;
    int nA = 0;
    bool ok = true;
    if (haveA) load_q(sgA);
    while (ok && haveA) {
      float cs[HC];
      bool gotA = false;
      Segment sgAc;
      int tAc = 0;
      int nAc = 0;
      if (haveA) {
        if (!wait_all(smem_u32(&sm.s_full), static_cast<uint32_t>(nA & 1), LKV_WAIT(W_SFULL))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < HC; c += 32) {
          uint32_t a[32];
          tmem_ld32(tm_addr(tbase, lb, S0 + c0 + c), a);
#pragma unroll
          for (int j = 0; j < 32; ++j) cs[c + j] = __uint_as_float(a[j]);
        }
        tmem_wait_ld();
        tc_fence_before();
        warp_arrive(smem_u32(&sm.s_free));
        const bool last = (tA == sgA.tile_hi - 1);
        bool have_nx = false;
        if (last) {
          // QK of this tile is done, so the query operands are free: stage the next unit's
          have_nx = next_seg(cur, nx);
          if (have_nx) load_q(nx);
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
      if (gotA) {
        int qi, qh;
        row_map(sgAc, qi, qh);
        uint32_t pw[HW];
        bool rescale;
        float alpha;
        if (!softmax_tile(cs, sgAc, tAc, qi, pw, rescale, alpha) || !finish_tile(pw, rescale, alpha, sgAc, tAc, nAc)) {
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
}

}  // namespace lkv
