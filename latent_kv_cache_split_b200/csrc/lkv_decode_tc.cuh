// Tensor-core (tcgen05 / TMEM) split-KV decode attention for sm_100a.
//
// One persistent CTA (MLA: one CTA pair, a thread-block cluster of 2) per work range
// (lkv_sched.cuh), 12 warps:
//   warp 0      TMA producer: streams key/value tiles of the cache (64 keys for MLA / GLA,
//               128 for GQLA) into rings of shared-memory stages (2-D boxes of tile rows x
//               64 bf16, 128-byte swizzle; the MLA RoPE halves 32 bf16 wide, 64-byte swizzle).
//   warp 1      TMEM owner and QK issuer (one thread): S = Q K^T into TMEM.  The non-RoPE part
//               of Q is an A operand in TMEM, the RoPE part one in shared memory; K is the B
//               operand in the stage.
//   warp 2      PV issuer (one thread): O += P V into TMEM, P an A operand in TMEM, V read
//               MN-major from the very same swizzled tile that served as K where K = V.
//   warp 3      MLA only: sender of the score messages to the peer CTA (st.async).
//   warps 4-11  softmax / epilogue.  Grouped modes: warp 4 + q + 4h owns TMEM lane quadrant q
//               and key-column half h of each tile; the two halves of a row agree on the
//               running max through a bounded shared-memory exchange.  MLA: warps 4-7 (score
//               warps) encode S as score codes and stage them, warps 8-11 (combine warps) add
//               both CTAs' codes, form P, rescale O and write the output, one tile behind the
//               score warps.
//
// TMEM columns: O [0, DV) | S [DV, DV+T) | P0, P1 [DV+T, DV+2T) | Q [DV+2T, ...) for T keys/tile.
// P is double buffered so the softmax of tile n+1 never waits for the PV of tile n.
//
// MLA absorbed path (h_q = 128 heads share the latent, GQLA explainer section 2): the
// 128 x 512 fp32 output accumulator alone fills a whole TMEM, so a CTA pair splits it:
// rank 0 owns value columns 0..255 and contracts latent columns 0..255 plus RoPE columns 0..31,
// rank 1 owns value columns 256..511 and contracts latent 256..511 plus RoPE 32..63.  Each CTA
// encodes its partial scores as 16-bit offsets below a per-row reference (its partial tile max)
// and sends them to the peer through distributed shared memory; both CTAs add the two codes of
// every key (an exact integer sum, so the full score is known to one code step), form the same
// P = 2^(score - m) and accumulate their own half of O.  Each CTA streams only the cache columns
// it needs, so the pair reads every cache byte once.
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

// Warps: 0 TMA producer, 1 QK issuer, 2 PV issuer, 3 MLA message sender, 4-11 softmax (roles in
// the file header).
constexpr int kTcThreads = 384;
// One MLA score message: 128 rows x 64 16-bit score codes, then the 128 rows' references (fp32).
constexpr int kMsgBytes = 128 * 128 + 128 * 4;
// Slot stride in shared memory: 1024-byte aligned, because the combine warps overwrite the
// peer's codes in a slot with P (same 128-byte-swizzled rows), the A operand of that tile's PV.
constexpr int kMsgStride = 17 * 1024;
// Incoming score messages in flight per CTA of the MLA pair.  A CTA sends message m only after
// it has read the peer's message m-1, which the peer sent after reading message m-2 (and so
// m-3) from this CTA, so with 3 slots the slot of message m is always free when it is written.
constexpr int kMsgSlots = 3;
constexpr int kTmemCols = 512;

// MLA pair score exchange.  A CTA holds only the partial score of each key over its half of the
// 576 contracted columns; the full score is the sum of both halves.  Each half is sent as a 16-bit
// code of (reference - partial score) in steps of 2^(e-10) log2 units, the reference being the
// row's partial tile max.  The step exponent e (0..5) is the smallest whose 65535 steps cover the
// row's partial scores in this tile; it travels in the low 3 bits of the fp32 reference, and the
// codes are taken against that very reference.  The receiving side adds the two halves, so the
// full score of every key is known to within half a step of each half.
constexpr int kStepBits = 3;                   // low mantissa bits of the reference carrying e
constexpr float kOffsetMagic = 8388608.f;      // 2^23: an fp32 sum there rounds to an integer
constexpr float kOffsetRefLimit = 16384.f;     // |reference| beyond this: report, outputs may drift

// 2^(e - 10): the code step of exponent e, in log2 units.
__device__ __forceinline__ float code_step(uint32_t e) { return __uint_as_float((117u + e) << 23); }
// 2^(10 - e): code steps per log2 unit.
__device__ __forceinline__ float code_inv_step(uint32_t e) { return __uint_as_float((137u - e) << 23); }

// Smallest e in [0, 5] whose 65535 steps of 2^(e-10) cover `range` log2 units.
__device__ __forceinline__ uint32_t code_exponent(float range) {
  uint32_t e = 0;
#pragma unroll
  for (int k = 0; k < 5; ++k) e += (range > 63.99f * static_cast<float>(1 << k)) ? 1u : 0u;
  return e;
}

// Codes of two raw scores s0, s1 (round((ref - s * sl2) / step), clamped to [0, 65535]), packed
// low / high.  nsl = -sl2 / step, refs = ref / step.
__device__ __forceinline__ uint32_t encode_offsets(float s0, float s1, float nsl, float refs) {
  const float a = fmaxf(fminf(fmaf(s0, nsl, refs) + kOffsetMagic, kOffsetMagic + 65535.f), kOffsetMagic);
  const float b = fmaxf(fminf(fmaf(s1, nsl, refs) + kOffsetMagic, kOffsetMagic + 65535.f), kOffsetMagic);
  return __byte_perm(__float_as_uint(a), __float_as_uint(b), 0x5410);
}
// -code * step for a 16-bit code (exact).
__device__ __forceinline__ float decode_offset(uint32_t code, float step) {
  return fmaf(__uint_as_float(0x4B000000u | code), -step, kOffsetMagic * step);
}
// Sum of the two bf16 values packed in w.
__device__ __forceinline__ float bf16x2_sum(uint32_t w) {
  return __uint_as_float(w << 16) + __uint_as_float(w & 0xffff0000u);
}

// MODE_GTA: grouped-tied attention, the GQLA shapes with K_j = V_j (one tied state per group).
enum DecodeMode { MODE_MLA = 0, MODE_GQLA = 1, MODE_GLA = 2, MODE_GTA = 3 };

// Wait sites (added to LKV_SITE_WAIT_BASE in the error word).
enum WaitSite {
  W_EMPTY = 1, W_FULL, W_SFREE, W_QREADY, W_PFULL, W_OFREE, W_SFULL, W_ODONE, W_XFREE, W_XFULL,
  W_DRAIN, W_XSTAGED, W_XCHG
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
  static constexpr bool kHead128 = (kMode == MODE_GQLA || kMode == MODE_GTA);  // d_h = 128 groups
  // Keys per tile.  GQLA runs 128-key tiles so that every QK UMMA is N = 128 (one issuing
  // thread then keeps the tensor pipe at full rate); MLA and GLA keep 64-key tiles because a
  // 128-column S tile would not fit next to their 256-column O accumulator and resident Q.
  static constexpr int kTile = kHead128 ? 128 : 64;
  static constexpr int kBoxBytes = kTile * 128;                 // one TMA box: kTile rows x 64 bf16
  // GQLA keeps K (+ k_rope) and V in separate rings: a K slot is refilled as soon as its QK
  // is done, while V waits for its PV.  Where K = V (MLA, GLA, GTA) one ring holds the tile.
  static constexpr bool kSplitKV = (kMode == MODE_GQLA);
  static constexpr int kKBoxes = kHead128 ? 2 : 4;  // 64-column boxes of the non-RoPE key per stage
  // MLA: each CTA of the pair contracts its 256 latent columns and one 32-column half of the
  // RoPE key (a 64-byte swizzled box); the other modes take the whole 64-column RoPE key.
  static constexpr int kRopeBoxBytes = kPair ? kTile * 64 : kBoxBytes;
  static constexpr int kStageBytes = kKBoxes * kBoxBytes + kRopeBoxBytes;  // K ring (or whole tile)
  static constexpr int kVStageBytes = 2 * kBoxBytes;                  // V ring (GQLA)
  static constexpr int kDV = kHead128 ? 128 : 256;  // value columns per CTA
  // GTA holds a stage from its load to its PV (K = V), so it gets the ring depth that GQLA
  // splits between its K ring (2) and V ring (3)
  static constexpr int kStages = (kMode == MODE_GQLA) ? 2 : (kMode == MODE_GTA ? 4 : (kPair ? 4 : 5));
  // L2 prefetch distance of the producer in tiles (0: off)
  static constexpr int kPrefetch = kPair ? kStages + 1 : 0;
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
  // (128-byte swizzle), or of the CTA's 32-column half in the MLA pair (64-byte swizzle).
  static constexpr int kQropeBytes = kPair ? 128 * 64 : 128 * 128;
  static constexpr int kRopeSteps = kPair ? 2 : 4;  // QK K-steps over the RoPE columns
  // MLA adds kMsgSlots incoming score messages and one outgoing staging copy
  static constexpr size_t kSmemBytes = 1024 + kRingBytes + kQropeBytes + (kPair ? (kMsgSlots + 1) * kMsgStride : 0);
};
static_assert(ModeCfg<MODE_MLA>::Q0 + 32 * ModeCfg<MODE_MLA>::kNope <= kTmemCols, "TMEM budget");
static_assert(ModeCfg<MODE_GLA>::Q0 + 32 * ModeCfg<MODE_GLA>::kNope <= kTmemCols, "TMEM budget");
static_assert(ModeCfg<MODE_GQLA>::Q0 + 32 * ModeCfg<MODE_GQLA>::kNope <= kTmemCols, "TMEM budget");
static_assert(ModeCfg<MODE_GTA>::Q0 + 32 * ModeCfg<MODE_GTA>::kNope <= kTmemCols, "TMEM budget");
static_assert(ModeCfg<MODE_MLA>::kTile == 64, "the score exchange rows hold 64 keys");
static_assert(ModeCfg<MODE_MLA>::kSmemBytes <= 232448, "shared memory budget");
static_assert(ModeCfg<MODE_GLA>::kSmemBytes <= 232448, "shared memory budget");
static_assert(ModeCfg<MODE_GQLA>::kSmemBytes <= 232448, "shared memory budget");
static_assert(ModeCfg<MODE_GTA>::kSmemBytes <= 232448, "shared memory budget");
static_assert(ModeCfg<MODE_GTA>::kStageBytes == 3 * ModeCfg<MODE_GTA>::kBoxBytes, "GTA stage: tied state + RoPE key");

// Advance a shared-memory descriptor by a byte offset (start-address field, 16-byte units).
__device__ __forceinline__ uint64_t desc_add(uint64_t d, uint32_t bytes) { return d + (bytes >> 4); }

template <int kStagesT, int kVStagesT>
struct __align__(16) TcSmem {
  uint64_t full[kStagesT];
  uint64_t empty[kStagesT];
  uint64_t vfull[kVStagesT];
  uint64_t vempty[kVStagesT];
  uint64_t s_full[2], s_free[2];  // per S buffer (MLA double-buffers S; grouped modes use [0])
  uint64_t o_free, q_ready, drain;
  uint64_t pvd[kMsgSlots];         // MLA: PV of a tile done, by message slot (for the sender)
  uint64_t p_full[2], o_done[2], x_full[kMsgSlots];
  uint64_t x_staged, x_stage_free;  // MLA: outgoing message staged by the softmax / read by the sender
  uint64_t x_consumed[2];           // MLA: incoming message of that parity read by the combine warps
  uint64_t own_read;                // MLA: the combine warps have read the staged message
  int n_armed;                      // MLA: incoming messages armed so far (for the abort drain)
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
  constexpr bool kPair = Cfg::kPair;
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
  uint8_t* rbuf = qrope_smem + Cfg::kQropeBytes;  // MLA only: kMsgSlots incoming messages
  uint8_t* sbuf = rbuf + kMsgSlots * kMsgStride;  // MLA only: the outgoing message being staged

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const uint32_t rank = kPair ? cluster_ctarank() : 0u;
  const int range = kPair ? (blockIdx.x >> 1) : blockIdx.x;
  const int n_row_warps = (p.R + 31) >> 5;  // lane quadrants holding valid rows
  const int n_sm_warps = 2 * n_row_warps;     // softmax warps: two column halves per quadrant
  const int n_sm_threads = n_sm_warps * 32;

  SchedArgs sa0;
  sa0.cu = p.cu;
  sa0.B = p.B;
  sa0.s_q = p.s_q;
  sa0.tile = TN;
  sa0.units_per_req = kPair ? p.s_q : p.G;
  sa0.per_query_units = kPair ? 1 : 0;
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
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(smem_u32(&sm.vfull[s]), 1);
      mbar_init(smem_u32(&sm.vempty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) mbar_init(smem_u32(&sm.s_full[b]), 1);
    // softmax-side barriers take one arrival per warp (lane 0, after a __syncwarp)
    // MLA: 4 score warps (S, Q, staging) and 4 combine warps (P, O); grouped: the softmax warps
    const int n_a = kPair ? 4 : n_sm_warps, n_b = kPair ? 4 : n_sm_warps;
    for (int b = 0; b < 2; ++b) mbar_init(smem_u32(&sm.s_free[b]), n_a);
    for (int b = 0; b < kMsgSlots; ++b) mbar_init(smem_u32(&sm.pvd[b]), 1);
    mbar_init(smem_u32(&sm.o_free), n_b);
    mbar_init(smem_u32(&sm.q_ready), n_a);
    mbar_init(smem_u32(&sm.drain), 2);  // one commit from each UMMA issuer
    for (int b = 0; b < kMsgSlots; ++b) mbar_init(smem_u32(&sm.x_full[b]), 1);  // armed here, filled by the peer
    mbar_init(smem_u32(&sm.x_staged), n_a);
    mbar_init(smem_u32(&sm.x_stage_free), 1);
    for (int b = 0; b < 2; ++b) mbar_init(smem_u32(&sm.x_consumed[b]), n_b);
    mbar_init(smem_u32(&sm.own_read), n_b);
    sm.n_armed = 0;
    for (int q = 0; q < 4; ++q)
      for (int b = 0; b < 2; ++b) mbar_init(smem_u32(&sm.xbar[q][b]), 2);
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&sm.p_full[b]), n_b);
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
      const uint32_t bytes = Cfg::kStageBytes;
      // L2 prefetch runs kPrefetch tiles ahead of the loads, so that a load issued when its ring
      // slot frees finds its rows in L2 instead of waiting for HBM.
      constexpr int kPrefetch = Cfg::kPrefetch;
      SegCursor pcur = cur0;
      Segment psg{};
      int pt = 0;
      bool pvalid = false;
      auto prefetch_next = [&]() {
        if (pvalid && pt + 1 < psg.tile_hi) {
          ++pt;
        } else {
          pvalid = next_seg(pcur, psg);
          if (!pvalid) return;
          pt = psg.tile_lo;
        }
        const int prow = psg.cu_b + pt * TN;
        if (kMode == MODE_MLA) {
          const int c0 = 256 * static_cast<int>(rank);
          for (int bx = 0; bx < 4; ++bx) tma_prefetch_l2_2d(&map_a, c0 + 64 * bx, prow);
          tma_prefetch_l2_2d(&map_r, 32 * static_cast<int>(rank), prow);
        } else if (kMode == MODE_GQLA) {
          const int c0 = 128 * psg.k;
          tma_prefetch_l2_2d(&map_a, c0, prow);
          tma_prefetch_l2_2d(&map_a, c0 + 64, prow);
          tma_prefetch_l2_2d(&map_r, 0, prow);
          tma_prefetch_l2_2d(&map_v, c0, prow);
          tma_prefetch_l2_2d(&map_v, c0 + 64, prow);
        } else if constexpr (kMode == MODE_GTA) {
          const int c0 = 128 * psg.k;
          tma_prefetch_l2_2d(&map_a, c0, prow);
          tma_prefetch_l2_2d(&map_a, c0 + 64, prow);
          tma_prefetch_l2_2d(&map_r, 0, prow);
        } else {
          const int c0 = 256 * psg.k;
          for (int bx = 0; bx < 4; ++bx) tma_prefetch_l2_2d(&map_a, c0 + 64 * bx, prow);
          tma_prefetch_l2_2d(&map_r, 0, prow);
        }
      };
      // the walker skips the tiles that the first loads fetch directly
      for (int i = 0; kPrefetch > 0 && i < kPrefetch && (i == 0 || pvalid); ++i) {
        if (pvalid && pt + 1 < psg.tile_hi) {
          ++pt;
        } else {
          pvalid = next_seg(pcur, psg);
          if (pvalid) pt = psg.tile_lo;
        }
      }
      SegCursor cur = cur0;
      Segment sg;
      int n = 0, nv = 0;   // K (or whole) tiles and V tiles issued (a CTA's tile count fits an int)
      bool ok = true;
      while (ok && next_seg(cur, sg)) {
        for (int t = sg.tile_lo; t < sg.tile_hi; ++t, ++n) {
          if (pvalid) prefetch_next();
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
          if (kMode == MODE_MLA) {
            const int c0 = 256 * static_cast<int>(rank);
            for (int bx = 0; bx < 4; ++bx) tma_load_2d(dst + bx * kBoxBytes, &map_a, fb, c0 + 64 * bx, row);
            tma_load_2d(dst + 4 * kBoxBytes, &map_r, fb, 32 * static_cast<int>(rank), row);  // RoPE half
          } else if (kMode == MODE_GQLA) {
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
        const uint64_t qrope_desc = kPair ? sdesc_sw64(qrope_base, 512) : sdesc_sw128(qrope_base, 16, 1024);
        while (ok && next_seg(cur, sg)) {
          for (int t = sg.tile_lo; t < sg.tile_hi; ++t, ++n) {
            const int st = static_cast<int>(n % KS);
            // MLA double-buffers S (buffer n % 2, last read for tile n-2); grouped modes have one
            const int sb = kPair ? (n & 1) : 0;
            const int prev = kPair ? n - 2 : n - 1;
            const uint32_t prev_par = static_cast<uint32_t>((kPair ? (prev >> 1) : prev) & 1);
            if (!mbar_wait(smem_u32(&sm.full[st]), static_cast<uint32_t>((n / KS) & 1), wc, LKV_WAIT(W_FULL)) ||
                (prev >= 0 && !mbar_wait(smem_u32(&sm.s_free[sb]), prev_par, wc, LKV_WAIT(W_SFREE))) ||
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
              umma_ts(tbase + S0 + TN * sb, tbase + Q0 + bx * 32 + kk * 8, desc_add(kdesc, bx * kBoxBytes + kk * 32),
                      id_qk, ks ? 1u : 0u);
            }
            const uint32_t rope_addr = stage_base + st * kStageBytes + Cfg::kRopeBox * kBoxBytes;
            const uint64_t rdesc = kPair ? sdesc_sw64(rope_addr, 512) : sdesc_sw128(rope_addr, 16, 1024);
#pragma unroll
            for (int kk = 0; kk < Cfg::kRopeSteps; ++kk)
              umma_ss(tbase + S0 + TN * sb, desc_add(qrope_desc, kk * 32), desc_add(rdesc, kk * 32), id_qk, 1u);
            umma_commit(smem_u32(&sm.s_full[sb]));
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
            if constexpr (kPair) {
              // P(n) was written over the peer's score codes in message slot n % 3 (K-major, 128-byte swizzle)
              const uint64_t pdesc = sdesc_sw128(smem_u32(rbuf + (n % kMsgSlots) * kMsgStride), 16, 1024);
#pragma unroll
              for (int kk = 0; kk < TN / 16; ++kk)
                umma_ss(tbase, desc_add(pdesc, kk * 32), desc_add(vdesc, kk * 2048), id_pv, (first && kk == 0) ? 0u : 1u);
            } else {
              const uint32_t pa = tbase + P0 + Cfg::kPCols * pb;
#pragma unroll
              for (int kk = 0; kk < TN / 16; ++kk)
                umma_ts(tbase, pa + kk * 8, desc_add(vdesc, kk * 2048), id_pv, (first && kk == 0) ? 0u : 1u);
            }
            umma_commit(smem_u32(&sm.o_done[pb]));
            umma_commit(kSplit ? smem_u32(&sm.vempty[n % VS]) : smem_u32(&sm.empty[n % KS]));
            if (kPair) umma_commit(smem_u32(&sm.pvd[n % kMsgSlots]));  // slot n % 3 readable again
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
  } else if (kPair && warp == 3) {
    // ============================================================ MLA message sender
    // Copies each staged score message into the peer's slot with st.async (each store completes
    // its bytes on the peer's x_full), so the softmax warps never wait on the cluster network.
    const int h = lane;
    const uint32_t peer = rank ^ 1u;
    uint32_t rrem[kMsgSlots], xrem[kMsgSlots];
#pragma unroll
    for (int b = 0; b < kMsgSlots; ++b) {
      rrem[b] = map_to_peer(smem_u32(rbuf + b * kMsgStride), peer);
      xrem[b] = map_to_peer(smem_u32(&sm.x_full[b]), peer);
    }
    SegCursor cur = cur0;
    Segment sg;
    int m = 0;
    bool ok = true;
    while (ok && next_seg(cur, sg)) {
      for (int t = sg.tile_lo; t < sg.tile_hi; ++t, ++m) {
        if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.x_staged), static_cast<uint32_t>(m & 1), wc,
                                                LKV_WAIT(W_XSTAGED)))) {
          ok = false;
          break;
        }
        // Two batches of 16-byte chunks: chunk lane + 32 i (a warp reads 512 contiguous bytes
        // per load), kC1 of them, then the remaining kC2.
        constexpr int kPer = kMsgBytes / 16 / 32;
        static_assert(kPer * 32 * 16 == kMsgBytes, "message chunking");
        constexpr int kC1 = (kPer + 1) / 2, kC2 = kPer - kC1;
        const uint4* src = reinterpret_cast<const uint4*>(sbuf);
        uint4 v[kC1];
#pragma unroll
        for (int i = 0; i < kC1; ++i) v[i] = src[h + 32 * i];
        // the peer's slot for message m is free once this CTA has read the peer's message m-1.
        // The staging copy is released only after this wait, and the combine warps read the
        // peer's message m+1 only after message m+1 was staged: so barrier x_consumed[(m-1) & 1]
        // never runs a phase ahead of the parity tested here.
        if (m >= 1 && !__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.x_consumed[(m - 1) & 1]),
                                                          static_cast<uint32_t>(((m - 1) >> 1) & 1), wc,
                                                          LKV_WAIT(W_XSTAGED)))) {
          ok = false;
          break;
        }
        const int xb = static_cast<int>(m % kMsgSlots);
        // The peer sends message m+1 into slot (m+1) % 3 after reading this message m; that slot
        // holds this CTA's P(m-2) until PV(m-2) is done.  Message m therefore goes only after
        // PV(m-2) (barrier pvd[(m-2) % 3]; its next phase needs PV(m+1), so no phase is skipped).
        if (m >= 2 && !__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.pvd[(m - 2) % kMsgSlots]),
                                                          static_cast<uint32_t>(((m - 2) / kMsgSlots) & 1), wc,
                                                          LKV_WAIT(W_ODONE)))) {
          ok = false;
          break;
        }
#pragma unroll
        for (int i = 0; i < kC1; ++i) st_async_v4(rrem[xb] + 16u * static_cast<uint32_t>(h + 32 * i), v[i], xrem[xb]);
#pragma unroll
        for (int i = 0; i < kC2; ++i) v[i] = src[h + 32 * (kC1 + i)];
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.x_stage_free));
#pragma unroll
        for (int i = 0; i < kC2; ++i)
          st_async_v4(rrem[xb] + 16u * static_cast<uint32_t>(h + 32 * (kC1 + i)), v[i], xrem[xb]);
      }
    }
  } else if (kPair && warp >= 4 && warp < 12) {
    // ============================================================ MLA softmax
    // Warps 4-7 (score warps) encode S as this CTA's score codes and stage them for the peer;
    // warps 8-11 (combine warps) form P from both CTAs' codes, publish it, rescale O and run
    // the epilogue.  The two run on different tiles at the same time (the score warps one tile
    // ahead), each warp owns TMEM lane quadrant q = warp % 4 and all 64 key columns.
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;            // row (head) == TMEM lane
    const uint32_t lb = static_cast<uint32_t>(q4 * 32);
    const int col_base = 256 * static_cast<int>(rank);
    auto wait_all = [&](uint32_t bar, uint32_t par, int site) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, par, wc, site)) != 0;
    };
    auto wait_all_cl = [&](uint32_t bar, uint32_t par, int site) -> bool {
      return __all_sync(0xffffffffu, mbar_wait<true>(bar, par, wc, site)) != 0;
    };
    auto warp_arrive = [&](uint32_t bar) {
      __syncwarp();
      if (lane == 0) mbar_arrive(bar);
    };
    SegCursor cur = cur0;
    Segment sg, nx;
    bool ok = true;
    int n = 0;
    if (warp < 8) {
      // ---------------------------------------------------------- score warps
      auto load_q = [&](const Segment& s) {
        const size_t qrow = (static_cast<size_t>(s.b) * p.s_q + s.k) * p.h_q + r;
#pragma unroll 1
        for (int bx = 0; bx < 4; ++bx) {
          uint32_t w[32];
          const uint4* src = reinterpret_cast<const uint4*>(p.q_nope + qrow * p.dq + col_base + 64 * bx);
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const uint4 x = __ldg(src + v);
            w[4 * v] = x.x;
            w[4 * v + 1] = x.y;
            w[4 * v + 2] = x.z;
            w[4 * v + 3] = x.w;
          }
          tmem_st32(tm_addr(tbase, lb, Q0 + bx * 32), w);
        }
        // this CTA's 32-column RoPE half, 64-byte swizzle: chunk c of row r at c ^ ((r / 2) % 4)
        const uint4* src = reinterpret_cast<const uint4*>(p.q_rope + qrow * 64 + 32 * rank);
#pragma unroll
        for (int c = 0; c < 4; ++c)
          *reinterpret_cast<uint4*>(qrope_smem + r * 64 + ((c ^ ((r >> 1) & 3)) << 4)) = __ldg(src + c);
        fence_proxy_async_smem();
        tmem_wait_st();
        tc_fence_before();
        warp_arrive(smem_u32(&sm.q_ready));
      };
      bool have = next_seg(cur, sg);
      if (have) load_q(sg);
      while (ok && have) {
        for (int t = sg.tile_lo; t < sg.tile_hi; ++t, ++n) {
          const int sb = n & 1;
          if (!wait_all(smem_u32(&sm.s_full[sb]), static_cast<uint32_t>((n >> 1) & 1), LKV_WAIT(W_SFULL))) {
            ok = false;
            break;
          }
          tc_fence_after();
          float cs[TN];
#pragma unroll
          for (int c = 0; c < TN; c += 32) {
            uint32_t a[32];
            tmem_ld32(tm_addr(tbase, lb, S0 + TN * sb + c), a);
#pragma unroll
            for (int j = 0; j < 32; ++j) cs[c + j] = __uint_as_float(a[j]);
          }
          tmem_wait_ld();
          tc_fence_before();
          warp_arrive(smem_u32(&sm.s_free[sb]));
          if (t == sg.tile_hi - 1 && (have = next_seg(cur, nx))) load_q(nx);  // QK(n) is done: Q is free
          const int xb = n % kMsgSlots;
          if (r == 0) {
            mbar_arrive_expect_tx(smem_u32(&sm.x_full[xb]), kMsgBytes);  // the peer's message n
            sm.n_armed = n + 1;
          }
          const int rem = sg.keys - t * TN;  // valid keys in this tile
          // row max and min of the partial scores over the valid keys (the scale is positive)
          float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
          float n4[4] = {INFINITY, INFINITY, INFINITY, INFINITY};
          if (rem < TN) {
#pragma unroll
            for (int c = 0; c < TN; ++c) {
              n4[c & 3] = (c < rem) ? fminf(n4[c & 3], cs[c]) : n4[c & 3];
              cs[c] = (c < rem) ? cs[c] : -INFINITY;
            }
          } else {
#pragma unroll
            for (int c = 0; c < TN; ++c) n4[c & 3] = fminf(n4[c & 3], cs[c]);
          }
#pragma unroll
          for (int c = 0; c < TN; ++c) m4[c & 3] = fmaxf(m4[c & 3], cs[c]);
          const float tcur = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * p.sl2;  // log2 units
          const float tmin = fminf(fminf(n4[0], n4[1]), fminf(n4[2], n4[3])) * p.sl2;
          const float tsub = (tcur == -INFINITY) ? 0.f : tcur;
          if (!(fabsf(tsub) < kOffsetRefLimit)) record_error(p.err, LKV_SITE_SCORE_RANGE);
          // The reference carries the step exponent in its low bits; codes are taken against it.
          const uint32_t ex = code_exponent(tsub - tmin);
          const float t_ref = __uint_as_float((__float_as_uint(tsub) & ~((1u << kStepBits) - 1u)) | ex);
          const float inv_step = code_inv_step(ex);
          uint32_t e[TN / 2];
#pragma unroll
          for (int c = 0; c < TN / 2; ++c)
            e[c] = encode_offsets(cs[2 * c], cs[2 * c + 1], -p.sl2 * inv_step, t_ref * inv_step);
          // the staging copy holds message n-1 until the sender and the combine warps read it
          if (n >= 1 &&
              (!wait_all(smem_u32(&sm.x_stage_free), static_cast<uint32_t>((n - 1) & 1), LKV_WAIT(W_XFREE)) ||
               !wait_all(smem_u32(&sm.own_read), static_cast<uint32_t>((n - 1) & 1), LKV_WAIT(W_XFREE)))) {
            ok = false;
            break;
          }
          // row r: 8 chunks of 16 bytes, XOR-swizzled by r so that readers avoid bank conflicts
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(sbuf + r * 128 + ((c ^ (r & 7)) << 4)) =
                make_uint4(e[4 * c], e[4 * c + 1], e[4 * c + 2], e[4 * c + 3]);
          reinterpret_cast<float*>(sbuf + 128 * 128)[r] = t_ref;
          warp_arrive(smem_u32(&sm.x_staged));
        }
        if (!ok) break;
        if (have) sg = nx;
      }
    } else {
      // ---------------------------------------------------------- combine warps
      float m_run = -INFINITY, l_run = 0.f, lb_run = 0.f;
      int nconsumed = 0;
      while (ok && next_seg(cur, sg)) {
        for (int t = sg.tile_lo; t < sg.tile_hi && ok; ++t, ++n) {
          const bool first = (t == sg.tile_lo), last = (t == sg.tile_hi - 1);
          if (!wait_all(smem_u32(&sm.x_staged), static_cast<uint32_t>(n & 1), LKV_WAIT(W_XSTAGED))) {
            ok = false;
            break;
          }
          uint32_t eo[32];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 x = *reinterpret_cast<const uint4*>(sbuf + r * 128 + ((c ^ (r & 7)) << 4));
            eo[4 * c] = x.x;
            eo[4 * c + 1] = x.y;
            eo[4 * c + 2] = x.z;
            eo[4 * c + 3] = x.w;
          }
          const float t_o = reinterpret_cast<const float*>(sbuf + 128 * 128)[r];
          warp_arrive(smem_u32(&sm.own_read));
          const int xb = n % kMsgSlots;
          if (!wait_all_cl(smem_u32(&sm.x_full[xb]), static_cast<uint32_t>((n / kMsgSlots) & 1), LKV_WAIT(W_XFULL))) {
            ok = false;
            break;
          }
          uint8_t* msg = rbuf + xb * kMsgStride;
          const float t_p = reinterpret_cast<const float*>(msg + 128 * 128)[r];
          const uint32_t e_o = __float_as_uint(t_o) & ((1u << kStepBits) - 1u);
          const uint32_t e_p = __float_as_uint(t_p) & ((1u << kStepBits) - 1u);
          const int rem = sg.keys - t * TN;  // valid keys in this tile (>= 1)
          // Both halves on one step (the usual case): per key the code sum, an exact integer in
          // common steps, saturated at 65535.  Otherwise each key's offset is formed in fp32.
          const bool same = __all_sync(0xffffffffu, e_o == e_p) != 0;
          const float st_o = code_step(e_o), st_p = code_step(e_p);
          float ybest;         // best key's offset below the reference sum (log2 units, <= 0)
          uint32_t smin2 = 0;  // same-step path: the best key's code sum in both halves of a word
          uint32_t nsat = 0;   // keys whose code saturated (the masked keys of a ragged tile excluded)
          if (same) {
            uint32_t mn2 = 0xffffffffu;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const uint4 x = *reinterpret_cast<const uint4*>(msg + r * 128 + ((c ^ (r & 7)) << 4));
              eo[4 * c] = __vaddus2(eo[4 * c], x.x);
              eo[4 * c + 1] = __vaddus2(eo[4 * c + 1], x.y);
              eo[4 * c + 2] = __vaddus2(eo[4 * c + 2], x.z);
              eo[4 * c + 3] = __vaddus2(eo[4 * c + 3], x.w);
              mn2 = __vminu2(mn2, __vminu2(__vminu2(eo[4 * c], eo[4 * c + 1]), __vminu2(eo[4 * c + 2], eo[4 * c + 3])));
              nsat += __popc(__vcmpeq2(eo[4 * c], 0xffffffffu)) + __popc(__vcmpeq2(eo[4 * c + 1], 0xffffffffu)) +
                      __popc(__vcmpeq2(eo[4 * c + 2], 0xffffffffu)) + __popc(__vcmpeq2(eo[4 * c + 3], 0xffffffffu));
            }
            // masked keys carry the top code on both sides, so the smallest sum is a valid key's
            const uint32_t smin = min(mn2 & 0xffffu, mn2 >> 16);
            smin2 = smin | (smin << 16);
            ybest = decode_offset(smin, st_o);
          } else {
            ybest = -INFINITY;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const uint4 x = *reinterpret_cast<const uint4*>(msg + r * 128 + ((c ^ (r & 7)) << 4));
              const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const uint32_t wo = eo[4 * c + j], wp = xw[j];
                const float y0 = decode_offset(wo & 0xffffu, st_o) + decode_offset(wp & 0xffffu, st_p);
                const float y1 = decode_offset(wo >> 16, st_o) + decode_offset(wp >> 16, st_p);
                const int k0 = 2 * (4 * c + j);
                ybest = fmaxf(ybest, fmaxf(k0 < rem ? y0 : -INFINITY, k0 + 1 < rem ? y1 : -INFINITY));
                nsat += __popc(__vcmpeq2(wo, 0xffffffffu) | __vcmpeq2(wp, 0xffffffffu));
              }
            }
          }
          nsat = nsat / 16 - (rem < TN ? static_cast<uint32_t>(TN - rem) : 0u);
          ++nconsumed;
          warp_arrive(smem_u32(&sm.x_consumed[n & 1]));
          // A saturated key's true offset exceeds its computed one, so its computed weight bounds its
          // true weight; both lie below 2^-(65535 steps + ...) of the best key.  Report the tile when
          // those keys together could carry more than 2^-12 of the best key's weight.
          if (nsat > 0) {
            const float gap = 65535.f * fminf(st_o, st_p) + ybest;  // log2 units between them, at least
            if (static_cast<float>(nsat) > ex2_approx(gap - 12.f)) record_error(p.err, LKV_SITE_SCORE_RANGE);
          }
          if (first) {
            m_run = -INFINITY;
            l_run = 0.f;
            lb_run = 0.f;
          }
          const float T = t_o + t_p;  // reference sum (log2 units)
          const float mx = T + ybest;  // this tile's row max
          bool rescale = false;
          float m_new = m_run;
          if (mx > m_run + 8.f) {  // lazy rescale: keep the running max unless it grows by 2^8
            m_new = mx;
            rescale = (m_run != -INFINITY);
          }
          const float alpha = rescale ? ex2_approx(m_run - m_new) : 1.f;
          // P = 2^(offset - ybest) (exact exponent, <= 0, centred on the tile max) times
          // f = 2^(mx - m_new) <= 2^8 in fp32
          const float f = ex2_approx(mx - m_new);
          float s4[4] = {0.f, 0.f, 0.f, 0.f}, b4[4] = {0.f, 0.f, 0.f, 0.f};
          uint32_t pw[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            float a0, a1;
            if (same) {
              const uint32_t dlt = __vsub2(eo[c], smin2);
              a0 = decode_offset(dlt & 0xffffu, st_o);
              a1 = decode_offset(dlt >> 16, st_o);
            } else {
              const uint32_t wp = *reinterpret_cast<const uint32_t*>(msg + r * 128 + (((c >> 2) ^ (r & 7)) << 4) + 4 * (c & 3));
              a0 = decode_offset(eo[c] & 0xffffu, st_o) + decode_offset(wp & 0xffffu, st_p) - ybest;
              a1 = decode_offset(eo[c] >> 16, st_o) + decode_offset(wp >> 16, st_p) - ybest;
            }
            if (rem < TN) {
              a0 = (2 * c < rem) ? a0 : -INFINITY;
              a1 = (2 * c + 1 < rem) ? a1 : -INFINITY;
            }
            const uint32_t pr = ex2_f16x2(a0, a1);
            const float e0 = f16_lo(pr) * f, e1 = f16_hi(pr) * f;
            s4[c & 3] += e0 + e1;
            pw[c] = pack_bf16x2(e0, e1);
            b4[c & 3] += bf16x2_sum(pw[c]);
          }
          // l_run (fp32 weights) gives the lse; lb_run sums the bf16 weights PV actually used, so
          // that the output is normalised by exactly the weights in O
          l_run = l_run * alpha + ((s4[0] + s4[1]) + (s4[2] + s4[3]));
          lb_run = lb_run * alpha + ((b4[0] + b4[1]) + (b4[2] + b4[3]));
          m_run = m_new;
          const int pb = n & 1;
          // P(n) replaces the peer's codes in slot xb: the same 128-byte swizzled rows are the
          // K-major A operand of PV(n) (the sender keeps the peer off this slot until PV(n) is done)
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(msg + r * 128 + ((c ^ (r & 7)) << 4)) =
                make_uint4(pw[4 * c], pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3]);
          fence_proxy_async_smem();
          if (__any_sync(0xffffffffu, rescale ? 1 : 0) && !first) {
            // O holds this segment's tiles up to n-1: wait for PV(n-1), then scale in place
            if (!wait_all(smem_u32(&sm.o_done[pb ^ 1]), static_cast<uint32_t>(((n - 1) >> 1) & 1),
                          LKV_WAIT(W_ODONE))) {
              ok = false;
              break;
            }
            tc_fence_after();
            tmem_scale_row(tm_addr(tbase, lb, 0), DV, alpha);
          }
          if (rem < TN) {
            // Rows past the unit's last key belong to another request or to unwritten cache:
            // their P is 0, but 0 * NaN would still poison O, so clear those V rows first.
            const int firstbad = rem;
            const int per_box = (TN - firstbad) * 8;  // 16-byte chunks per V box
            uint8_t* vb = dsm + (n % KS) * kStageBytes;
            for (int idx = r; idx < per_box * Cfg::kNV; idx += 128) {
              const int bx = idx / per_box, rem = idx % per_box;
              *reinterpret_cast<uint4*>(vb + bx * kBoxBytes + (firstbad + rem / 8) * 128 + (rem % 8) * 16) =
                  make_uint4(0u, 0u, 0u, 0u);
            }
            fence_proxy_async_smem();
          }
          tmem_wait_st();
          tc_fence_before();
          warp_arrive(smem_u32(&sm.p_full[pb]));
          if (!last) continue;
          // ---------------------------------------------------------- segment epilogue
          if (!wait_all(smem_u32(&sm.o_done[pb]), static_cast<uint32_t>((n >> 1) & 1), LKV_WAIT(W_ODONE))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float inv_l = lb_run > 0.f ? 1.f / lb_run : 0.f;
          const float lse_v = l_run > 0.f ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
          const size_t orow = (static_cast<size_t>(sg.b) * p.s_q + sg.k) * p.h_q + r;
          if (sg.complete) {
            tmem_row_to_bf16(tm_addr(tbase, lb, 0), DV, inv_l, p.out + orow * p.dv_total + col_base, true);
            if (rank == 0) p.lse[orow] = lse_v;
          } else {
            const size_t prow = static_cast<size_t>(2 * range + sg.slot) * p.rmax + r;
            tmem_row_to_f32(tm_addr(tbase, lb, 0), DV, inv_l, p.part_o + prow * p.dv_total + col_base, true);
            if (rank == 0) p.part_lse[prow] = lse_v;
            if (r == 0 && rank == 0) p.seg_info[2 * range + sg.slot] = sg.unit_id;
          }
          tc_fence_before();
          warp_arrive(smem_u32(&sm.o_free));
        }
      }
      if (!ok && r == 0) {
        // After giving up, the peer may still write messages into this CTA's shared memory: it
        // sends message m once it has read this CTA's message m-1, so at most up to message
        // n_armed (messages armed here bound those staged).  Let them land (bounded) before the
        // CTA can exit; every message is armed once.
        uint32_t zero = 0;
        const WaitCtl dc{&zero, p.err, p.wait_limit_ns};
        const int armed = *reinterpret_cast<volatile int*>(&sm.n_armed);
        for (int m = nconsumed; m <= armed && m < nconsumed + kMsgSlots; ++m) {
          if (m >= armed) mbar_arrive_expect_tx(smem_u32(&sm.x_full[m % kMsgSlots]), kMsgBytes);
          mbar_wait<true>(smem_u32(&sm.x_full[m % kMsgSlots]), static_cast<uint32_t>((m / kMsgSlots) & 1), dc,
                          LKV_WAIT(W_DRAIN));
        }
      }
    }
  } else if (!kPair && warp >= 4 && warp < 12 && ((warp - 4) & 3) < n_row_warps) {
   if constexpr (!kPair) {
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
      if (key0 + TN > sg.keys) {
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
        if (row_ok && rank == 0 && hf == 0) p.lse[orow] = lse_v;
      } else {
        const size_t prow = static_cast<size_t>(2 * range + sg.slot) * p.rmax + r;
        tmem_row_to_f32(tm_addr(tbase, lb, hf * (DV / 2)), DV / 2, inv_l, p.part_o + prow * p.dv_total + hf * (DV / 2),
                        row_ok);
        if (row_ok && rank == 0 && hf == 0) p.part_lse[prow] = lse_v;
        if (r == 0 && rank == 0 && hf == 0) p.seg_info[2 * range + sg.slot] = sg.unit_id;
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
        if (!wait_all(smem_u32(&sm.s_full[0]), static_cast<uint32_t>(nA & 1), LKV_WAIT(W_SFULL))) {
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
        warp_arrive(smem_u32(&sm.s_free[0]));
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
