// MLA absorbed decode on a CTA pair that shares one tensor-core MMA (tcgen05 cta_group::2).
//
// The absorbed path (GQLA explainer, section 2, "MQA absorbed path") has all h_q = 128 heads of a
// query token attend to one latent row per key: QK contracts the 512 latent columns plus the 64
// RoPE columns, PV multiplies by the same 512 latent columns.  The 128 x 512 fp32 output alone
// fills a whole TMEM, so the rows (heads) are split over the two CTAs of a cluster: CTA c owns
// heads 64c .. 64c+63 and holds, in its own TMEM, their full scores and their full output.
//
// One pair MMA of M = 128 rows takes its A rows from both CTAs (each its 64 heads) and its N
// columns of B half from each CTA; every CTA's TMEM receives its 64 rows for all N columns.  So:
//   QK:  S[128 heads, 256 keys] += Q[heads, 64 cols] K[keys, 64 cols]^T, per 64-column chunk.
//        CTA c streams keys 128c .. 128c+127 of the tile (all 576 columns); the pair reads every
//        key row once.
//   PV:  O[128 heads, 256 dims] += P[heads, 128 keys] V[128 keys, 256 dims], for the dims 0..255
//        and 256..511.  CTA c streams dims 256b + 128c .. +127 of the tile's keys (a second read
//        of latent rows the pair fetched for QK a moment before, served by L2).
// There is no score exchange between the CTAs: each has exact fp32 scores of its own heads.
//
// TMEM per CTA (512 columns, allocated for the pair): O dims block b at columns 128b .. 128b+127
// (lanes 0-63: dims 256b + col, lanes 64-127: dims 256b + 128 + col of heads 64c + lane % 64),
// S buffer sb at 256 + 128 sb (lanes 0-63: keys 0..127, lanes 64-127: keys 128..255).
//
// Warps (both CTAs): 0 TMA producer; 1 TMEM allocator and, in the even CTA, the MMA issuer;
// 2-9 softmax / epilogue: warp w reads TMEM lane quadrant w % 4 and key-column half (w - 2) / 4
// of its S lanes, so the four threads of a head (two lane halves x two column halves) agree on the
// row max through a bounded shared-memory exchange.
//
// Shared memory per CTA: Q (9 chunks of 64 heads x 64 columns), P for one 128-key value chunk
// (2 chunks of 64 heads x 64 keys) and a ring of four 32 KB stages that carries, in the MMA's
// order, the QK chunks of tile n+1 and then the PV chunks of tile n; every load is a 16 KB box of
// 128 rows x 64 columns.  P holds one value chunk at a time: the softmax threads of the tile's
// first chunk (in PV order) write theirs, the PV of that chunk runs, and only then do the threads
// of the second chunk write theirs over it.  Half a P buffer is what makes room for the fourth
// stage, and the ring's depth is what bounds this kernel (it fills ~41 GB/s per SM with three).  Ring stages are counted on the even CTA's barriers (the pair load
// form), released to both CTAs by the MMA's multicast commit.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "lkv_ptx.cuh"
#include "lkv_sched.cuh"
#include "../../include/lkv.h"

namespace lkv {

constexpr int kPairThreads = 320;          // 10 warps
constexpr int kPairTile = 256;             // keys per tile (N of the QK MMA)
// Ring of 32 KB stages.  The even CTA learns of every stage of both CTAs on one barrier and both
// CTAs learn of its release from one multicast commit; that hand-off has a fixed cost per stage, so
// stages carry 32 KB (measured: 16 KB stages stream at under half the rate of 32 KB ones, and
// three 32 KB stages already stream at HBM speed), in boxes of 16 KB (8 KB boxes stream at about
// two thirds of that rate).  Per 256-key tile a CTA fills 4 stages of two 64-column key chunks,
// 1 stage with the RoPE key chunk, and 1 stage per 128-key value chunk and dims block: this CTA's
// 128 dims of the block as two 64-dim boxes.
constexpr int kPairStages = 4;             // ring stages
constexpr int kPairStageBytes = 32768;
constexpr int kPairChunkBytes = 16384;     // one box: 128 keys x 64 columns
constexpr int kPairQBytes = 9 * 8192;      // 64 heads x (512 + 64) columns
constexpr int kPairPBytes = 2 * 8192;      // 64 heads x 128 keys (one value chunk)
constexpr int kPairQOff = 0;
constexpr int kPairPOff = kPairQBytes;
constexpr int kPairRingOff = kPairQBytes + kPairPBytes;
constexpr size_t kPairSmemBytes = 1024 + kPairRingOff + static_cast<size_t>(kPairStages) * kPairStageBytes;
constexpr uint32_t kPairS0 = 256;          // first S column
constexpr uint16_t kBothCtas = 3, kEvenCta = 1;  // multicast masks of a commit
static_assert(kPairSmemBytes <= 232448 - 4096, "shared memory budget");

// Wait sites of this kernel (added to LKV_SITE_WAIT_BASE in the error word; above the sites of
// the tensor-core kernel's four modes).
#define LKV_WAIT_BASE_PAIR(x) (LKV_SITE_WAIT_BASE + (x))
enum PairWaitSite {
  PW_EMPTY = 80, PW_FULL, PW_QFULL, PW_QFREE, PW_SFULL, PW_SFREE, PW_PFULL, PW_PVDONE, PW_OFREE, PW_VLAND,
  PW_XCHG, PW_DRAIN, PW_PLO, PW_PFULL2
};

struct __align__(16) PairSmem {
  uint64_t full[kPairStages];   // even CTA: both CTAs' bytes of a stage have landed
  uint64_t empty[kPairStages];  // each CTA: the MMA has consumed the stage (multicast commit)
  uint64_t q_full;              // even CTA: both CTAs' Q chunks landed
  uint64_t q_free;              // each CTA: the last QK of the current unit is done
  uint64_t s_full[2];           // each CTA: QK of the tile in S buffer b is done
  uint64_t s_free[2];           // even CTA: all 16 softmax warps read S buffer b
  uint64_t p_full;              // even CTA: all 16 softmax warps are done with the tile (P of its
                                // first value chunk written, O rescaled, rows past the end cleared)
  uint64_t p_lo_free;           // each CTA: the PV of the tile's first value chunk is done
  uint64_t p_full2;             // even CTA: the 8 warps of the second value chunk wrote its P
  uint64_t pv_done;             // each CTA: PV of the tile is done (P free, O settled)
  uint64_t o_free;              // even CTA: the epilogue of the last unit read O
  uint64_t vland;               // each CTA: the chunk to clear past the cache end has landed
  uint64_t drain;               // even CTA: every MMA issued is complete
  uint64_t xbar[2][2];          // row group (head rows 0-31 / 32-63) x buffer: 4 warps posted
  float xch[2][4][64];          // [buffer][lane half * 2 + column half][head row]
  uint32_t tmem_base;
  uint32_t abort;
  int vzero_stage[2];           // the two stages (dims blocks) of the chunk to clear
  int vzero_first;              // its first row to clear
  int peer_chunks, peer_units;  // odd CTA's producer counts, for the even CTA's drain
  int own_chunks, own_units;    // even CTA's producer counts
  int stage_bytes[kPairStages]; // even CTA: bytes per CTA of the last phase armed on each stage
  int peer_stage_bytes[kPairStages];  // the odd CTA's bytes of the last phase it loaded per stage
  long long t_begin, t_end, unit_t0;
  int b0, k0;
};

// Keys per tile of a unit (the last tile may be short) and its 64-key chunks.
__device__ __forceinline__ int pair_tile_keys(const Segment& sg, int t) {
  const int k = sg.keys - t * kPairTile;
  return k < kPairTile ? k : kPairTile;
}
// 128-key value chunks of tile t (1 or 2).
__device__ __forceinline__ int pair_pv_chunks(const Segment& sg, int t) { return (pair_tile_keys(sg, t) + 127) >> 7; }
// Does the PV of tile t read latent rows past the end of the last request (row T = cu[B])?  Those
// rows can hold anything, even NaN, and a zero weight times NaN is NaN: they are cleared first.
__device__ __forceinline__ bool pair_crosses_end(const Segment& sg, int t, int T) {
  const int r1 = sg.cu_b + t * kPairTile + 128 * pair_pv_chunks(sg, t);  // one past the last row PV reads
  return r1 > T;
}
// PV stage i (0 .. 2 nkc - 1) of a tile: value chunk (128 keys) i / 2 in processing order, dims block
// i % 2.  A tile that crosses the cache end takes its last chunk first (both blocks), so those two
// stages are resident before the softmax clears the rows past the end.
__device__ __forceinline__ int pair_pv_chunk(int i, int nkc, bool cross) {
  const int c = i >> 1;
  return cross ? (c == 0 ? nkc - 1 : c - 1) : c;
}
// Stages per tile for QK: 4 of two latent chunks, then 1 with the RoPE chunk.
constexpr int kPairQkStages = 5;

__global__ void __launch_bounds__(kPairThreads, 1)
    mla_pair_kernel(const __grid_constant__ CUtensorMap map_q,   // q_nope_abs [rows, 512], box 64 x 64
                    const __grid_constant__ CUtensorMap map_qr,  // q_rope [rows, 64], box 64 x 64
                    const __grid_constant__ CUtensorMap map_k,   // ckv [T, 512], box 64 x 128
                    const __grid_constant__ CUtensorMap map_kr,  // kpe [T, 64], box 64 x 128
                    const __grid_constant__ CUtensorMap map_v,   // ckv [T, 512], box 64 x 128
                    const TcParams p) {
  extern __shared__ __align__(1024) uint8_t pair_smem_raw[];
  __shared__ PairSmem sm;
  uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(pair_smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  const uint32_t q_base = smem_u32(dsm + kPairQOff);
  const uint32_t p_base = smem_u32(dsm + kPairPOff);
  const uint32_t ring_base = smem_u32(dsm + kPairRingOff);
  uint8_t* ring = dsm + kPairRingOff;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);
  const int range = blockIdx.x >> 1;
  constexpr int KS = kPairStages;

  SchedArgs sa;
  sa.cu = p.cu;
  sa.B = p.B;
  sa.s_q = p.s_q;
  sa.tile = kPairTile;
  sa.units_per_req = p.s_q;
  sa.per_query_units = 1;
  sa.P = p.P;
  const int T_end = __ldg(p.cu + p.B);  // end of the last request's rows

  // ---------------------------------------------------------------- set-up
  if (tid == 0) {
    for (int s = 0; s < KS; ++s) {
      mbar_init(smem_u32(&sm.full[s]), 1);
      mbar_init(smem_u32(&sm.empty[s]), 1);
    }
    mbar_init(smem_u32(&sm.q_full), 1);
    mbar_init(smem_u32(&sm.q_free), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&sm.s_full[b]), 1);
      mbar_init(smem_u32(&sm.s_free[b]), 16);
    }
    mbar_init(smem_u32(&sm.p_full), 16);
    mbar_init(smem_u32(&sm.p_lo_free), 1);
    mbar_init(smem_u32(&sm.p_full2), 8);
    mbar_init(smem_u32(&sm.pv_done), 1);
    mbar_init(smem_u32(&sm.o_free), 16);
    mbar_init(smem_u32(&sm.vland), 1);
    mbar_init(smem_u32(&sm.drain), 1);
    for (int g = 0; g < 2; ++g)
      for (int b = 0; b < 2; ++b) mbar_init(smem_u32(&sm.xbar[g][b]), 4);
    sm.abort = 0;
    sm.peer_chunks = 0;
    sm.peer_units = 0;
    sm.own_chunks = 0;
    sm.own_units = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    bool malformed = false;
    SegCursor c = locate_range(sa, range, &malformed);
    if (lane == 0) {
      if (malformed && range == 0 && leader) record_error(p.err, LKV_SITE_BAD_LENGTH);
      sm.t_begin = c.t_begin;
      sm.t_end = c.t_end;
      sm.unit_t0 = c.unit_t0;
      sm.b0 = c.b;
      sm.k0 = c.k;
      if (leader) {
        p.seg_info[2 * range] = -1;
        p.seg_info[2 * range + 1] = -1;
      }
      tma_prefetch_desc(&map_q);
      tma_prefetch_desc(&map_qr);
      tma_prefetch_desc(&map_k);
      tma_prefetch_desc(&map_kr);
      tma_prefetch_desc(&map_v);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(&sm.tmem_base), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any remote arrive or pair load
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

  // the even CTA's copy of a barrier (shared::cluster address)
  auto lead = [&](const uint64_t& bar) -> uint32_t { return map_to_peer(smem_u32(&bar), 0u); };

  if (warp == 0) {
    // ============================================================ TMA producer (both CTAs)
    if (lane == 0) {
      SegCursor cur = cur0;
      Segment sg, psg{};
      int pt = 0;
      bool have_prev = false, ok = true;
      int chunks = 0, units = 0;
      // one ring stage; `bytes` is what each CTA loads into it (the even CTA expects both CTAs')
      auto stage_acquire = [&](int& st, int bytes) -> bool {
        st = chunks % KS;
        if (!mbar_wait<true>(smem_u32(&sm.empty[st]), static_cast<uint32_t>(((chunks / KS) & 1) ^ 1), wc,
                             LKV_WAIT_BASE_PAIR(PW_EMPTY)))
          return false;
        if (leader) mbar_arrive_expect_tx(smem_u32(&sm.full[st]), 2 * bytes);
        sm.stage_bytes[st] = bytes;
        return true;
      };
      auto issue_pv = [&](const Segment& s, int t) -> bool {
        const int nkc = pair_pv_chunks(s, t);
        const bool cross = pair_crosses_end(s, t, T_end);
        for (int i = 0; i < 2 * nkc; ++i) {
          const int kc = pair_pv_chunk(i, nkc, cross);
          int st;
          if (!stage_acquire(st, kPairStageBytes)) return false;
          const uint32_t dst = ring_base + st * kPairStageBytes;
          const uint32_t fb = lead(sm.full[st]);
          const int row = s.cu_b + t * kPairTile + 128 * kc;
          // this CTA's 128 dims of dims block i % 2 as two 64-dim boxes
          const int x0 = 256 * (i & 1) + 128 * static_cast<int>(rank);
          tma_load_2d_pair(dst, &map_v, fb, x0, row);
          tma_load_2d_pair(dst + kPairChunkBytes, &map_v, fb, x0 + 64, row);
          ++chunks;
        }
        return true;
      };
      while (ok && cur.next(sa, sg)) {
        for (int t = sg.tile_lo; ok && t < sg.tile_hi; ++t) {
          if (t == sg.tile_lo) {
            // this unit's query rows (the previous unit's QKs must be done with the Q buffer)
            if (units > 0 && !mbar_wait<true>(smem_u32(&sm.q_free), static_cast<uint32_t>((units - 1) & 1), wc,
                                              LKV_WAIT_BASE_PAIR(PW_QFREE))) {
              ok = false;
              break;
            }
            if (leader) mbar_arrive_expect_tx(smem_u32(&sm.q_full), 2 * kPairQBytes);
            const uint32_t qb = lead(sm.q_full);
            const int qrow = (sg.b * p.s_q + sg.k) * 128 + 64 * static_cast<int>(rank);
            for (int j = 0; j < 8; ++j) tma_load_2d_pair(q_base + j * 8192, &map_q, qb, 64 * j, qrow);
            tma_load_2d_pair(q_base + 8 * 8192, &map_qr, qb, 0, qrow);
            ++units;
          }
          // QK chunks of this tile: this CTA's 128 keys, 64 columns per chunk
          const int krow = sg.cu_b + t * kPairTile + 128 * static_cast<int>(rank);
          for (int j = 0; j < kPairQkStages; ++j) {
            int st;
            if (!stage_acquire(st, j < 4 ? kPairStageBytes : kPairChunkBytes)) {
              ok = false;
              break;
            }
            const uint32_t dst = ring_base + st * kPairStageBytes;
            if (j < 4) {
              tma_load_2d_pair(dst, &map_k, lead(sm.full[st]), 128 * j, krow);
              tma_load_2d_pair(dst + kPairChunkBytes, &map_k, lead(sm.full[st]), 128 * j + 64, krow);
            } else {
              tma_load_2d_pair(dst, &map_kr, lead(sm.full[st]), 0, krow);
            }
            ++chunks;
          }
          if (!ok) break;
          // then the PV chunks of the previous tile
          if (have_prev && !issue_pv(psg, pt)) {
            ok = false;
            break;
          }
          psg = sg;
          pt = t;
          have_prev = true;
        }
      }
      if (ok && have_prev) issue_pv(psg, pt);
      // the counts the even CTA's drain needs
      if (!leader) {
        st_cluster_u32(map_to_peer(smem_u32(&sm.peer_chunks), 0u), static_cast<uint32_t>(chunks));
        st_cluster_u32(map_to_peer(smem_u32(&sm.peer_units), 0u), static_cast<uint32_t>(units));
        for (int s2 = 0; s2 < KS; ++s2)
          st_cluster_u32(map_to_peer(smem_u32(&sm.peer_stage_bytes[s2]), 0u), static_cast<uint32_t>(sm.stage_bytes[s2]));
      } else {
        sm.own_chunks = chunks;
        sm.own_units = units;
      }
    }
  } else if (warp == 1) {
    // ============================================================ MMA issuer (even CTA)
    if (leader && lane == 0) {
      const uint32_t id_qk = idesc_bf16(128, 256, 0, 0);
      const uint32_t id_pv = idesc_bf16(128, 256, 0, 1);
      SegCursor cur = cur0;
      Segment sg, psg{};
      int pt = 0, pn = 0, pseg = 0;
      bool have_prev = false, ok = true;
      int n = 0, ch = 0, seg = 0, n2 = 0;  // n2: tiles with two value chunks so far
      auto full_wait = [&](int c) -> bool {
        return mbar_wait<true>(smem_u32(&sm.full[c % KS]), static_cast<uint32_t>((c / KS) & 1), wc,
                               LKV_WAIT_BASE_PAIR(PW_FULL));
      };
      auto issue_pv = [&](const Segment& s, int t, int m, int sidx) -> bool {
        const bool first = (t == s.tile_lo);
        if (first && sidx > 0 &&
            !mbar_wait<true>(smem_u32(&sm.o_free), static_cast<uint32_t>((sidx - 1) & 1), wc,
                             LKV_WAIT_BASE_PAIR(PW_OFREE)))
          return false;
        const int nkc = pair_pv_chunks(s, t);
        const bool cross = pair_crosses_end(s, t, T_end);
        if (cross) {
          // the chunk past the cache end (its two stages) must be resident before the softmax
          // warps clear it
          if (!full_wait(ch) || !full_wait(ch + 1)) return false;
          const int first_bad = T_end - (s.cu_b + t * kPairTile + 128 * (nkc - 1));
          for (int b = 0; b < 2; ++b) {
            sm.vzero_stage[b] = (ch + b) % KS;
            st_cluster_u32(map_to_peer(smem_u32(&sm.vzero_stage[b]), 1u), static_cast<uint32_t>((ch + b) % KS));
          }
          sm.vzero_first = first_bad;
          st_cluster_u32(map_to_peer(smem_u32(&sm.vzero_first), 1u), static_cast<uint32_t>(first_bad));
          mbar_arrive_remote(lead(sm.vland));
          mbar_arrive_remote(map_to_peer(smem_u32(&sm.vland), 1u));
        }
        if (!mbar_wait<true>(smem_u32(&sm.p_full), static_cast<uint32_t>(m & 1), wc, LKV_WAIT_BASE_PAIR(PW_PFULL)))
          return false;
        tc_fence_after();
        for (int i = 0; i < 2 * nkc; ++i) {
          const int b = i & 1;
          if (i == 2) {
            // the first value chunk's PV must be done before its P is overwritten by the second's
            umma_pair_commit(smem_u32(&sm.p_lo_free), kBothCtas);
            if (!mbar_wait<true>(smem_u32(&sm.p_full2), static_cast<uint32_t>(n2 & 1), wc,
                                 LKV_WAIT_BASE_PAIR(PW_PFULL2)))
              return false;
            ++n2;
            tc_fence_after();
          }
          if (!full_wait(ch)) return false;
          tc_fence_after();
          // P keys 16 kk of the current value chunk: 64-key chunk kk / 4; V: two 64-dim boxes 16 KB apart
          const uint64_t vd = sdesc_sw128(ring_base + (ch % KS) * kPairStageBytes, kPairChunkBytes, 1024);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t pd = sdesc_sw128(p_base + (kk >> 2) * 8192, 16, 1024);
            umma_pair_ss(tbase + 128 * b, desc_add(pd, (kk & 3) * 32), desc_add(vd, kk * 2048), id_pv,
                         (first && i < 2 && kk == 0) ? 0u : 1u);
          }
          umma_pair_commit(smem_u32(&sm.empty[ch % KS]), kBothCtas);
          ++ch;
        }
        umma_pair_commit(smem_u32(&sm.pv_done), kBothCtas);
        return true;
      };
      while (ok && cur.next(sa, sg)) {
        for (int t = sg.tile_lo; ok && t < sg.tile_hi; ++t, ++n) {
          // ---- QK(n) into S buffer n % 2
          if ((t == sg.tile_lo &&
               !mbar_wait<true>(smem_u32(&sm.q_full), static_cast<uint32_t>(seg & 1), wc, LKV_WAIT_BASE_PAIR(PW_QFULL))) ||
              (n >= 2 && !mbar_wait<true>(smem_u32(&sm.s_free[n & 1]), static_cast<uint32_t>(((n - 2) >> 1) & 1), wc,
                                          LKV_WAIT_BASE_PAIR(PW_SFREE)))) {
            ok = false;
            break;
          }
          const uint32_t sacc = tbase + kPairS0 + 128 * (n & 1);
          for (int j = 0; j < kPairQkStages; ++j) {
            if (!full_wait(ch)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const int nc = j < 4 ? 2 : 1;  // key chunks in this stage (Q chunk 2j + h, or the RoPE chunk 8)
            for (int h = 0; h < nc; ++h) {
              const int qc = j < 4 ? 2 * j + h : 8;
              const uint64_t qd = sdesc_sw128(q_base + qc * 8192, 16, 1024);
              const uint64_t kd = sdesc_sw128(ring_base + (ch % KS) * kPairStageBytes + h * kPairChunkBytes, 16, 1024);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                umma_pair_ss(sacc, desc_add(qd, kk * 32), desc_add(kd, kk * 32), id_qk, (qc | kk) ? 1u : 0u);
            }
            umma_pair_commit(smem_u32(&sm.empty[ch % KS]), kBothCtas);
            ++ch;
          }
          if (!ok) break;
          umma_pair_commit(smem_u32(&sm.s_full[n & 1]), kBothCtas);
          if (t == sg.tile_hi - 1) umma_pair_commit(smem_u32(&sm.q_free), kBothCtas);
          // ---- PV(n - 1)
          if (have_prev && !issue_pv(psg, pt, pn, pseg)) {
            ok = false;
            break;
          }
          psg = sg;
          pt = t;
          pn = n;
          pseg = seg;
          have_prev = true;
          if (t == sg.tile_hi - 1) ++seg;
        }
      }
      if (ok && have_prev) issue_pv(psg, pt, pn, pseg);
      // every MMA complete before TMEM is released or a CTA exits
      umma_pair_commit(smem_u32(&sm.drain), kEvenCta);
      uint32_t zero = 0;
      const WaitCtl dc{&zero, p.err, p.wait_limit_ns};
      mbar_wait(smem_u32(&sm.drain), 0, dc, LKV_WAIT_BASE_PAIR(PW_DRAIN));
    }
  } else {
    // ============================================================ softmax / epilogue (warps 2-9)
    const int q4 = warp & 3;                  // TMEM lane quadrant
    const int chh = (warp - 2) >> 2;          // key-column half of the S lanes
    const int tl = 32 * q4 + lane;            // TMEM lane
    const int m = tl & 63;                    // head within this CTA
    const int kh = tl >> 6;                   // key half: lanes 64-127 hold keys 128..255
    const int grp = q4 & 1;                   // head rows 32 grp .. 32 grp + 31
    const int slot = kh * 2 + chh;
    const int head = 64 * static_cast<int>(rank) + m;
    const uint32_t trow = tbase + (static_cast<uint32_t>(32 * q4) << 16);
    auto wait_all = [&](uint32_t bar, uint32_t par, int site) -> bool {
      return __all_sync(0xffffffffu, mbar_wait<true>(bar, par, wc, site)) != 0;
    };
    auto arrive_lead = [&](const uint64_t& bar) {
      __syncwarp();
      if (lane == 0) mbar_arrive_pair(lead(bar));
    };
    // four-way exchange of one value per head row among the 4 warps of this row group
    int xc = 0;
    auto xchg4 = [&](float v, float (&o)[4]) -> bool {
      const int b = xc & 1;
      sm.xch[b][slot][m] = v;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.xbar[grp][b]));
      const bool okx = wait_all(smem_u32(&sm.xbar[grp][b]), static_cast<uint32_t>((xc >> 1) & 1),
                                LKV_WAIT_BASE_PAIR(PW_XCHG));
#pragma unroll
      for (int s = 0; s < 4; ++s) o[s] = sm.xch[b][s][m];
      ++xc;
      return okx;
    };
    float m_run = -INFINITY, l_run = 0.f, lb_run = 0.f;
    SegCursor cur = cur0;
    Segment sg;
    int n = 0, ncross = 0, n2s = 0;  // n2s: tiles with two value chunks so far
    bool ok = true;
    while (ok && cur.next(sa, sg)) {
      for (int t = sg.tile_lo; ok && t < sg.tile_hi; ++t, ++n) {
        const int sb = n & 1;
        if (!wait_all(smem_u32(&sm.s_full[sb]), static_cast<uint32_t>((n >> 1) & 1), LKV_WAIT_BASE_PAIR(PW_SFULL))) {
          ok = false;
          break;
        }
        tc_fence_after();
        float cs[64];
        {
          uint32_t a[32];
          tmem_ld32(trow + kPairS0 + 128 * sb + 64 * chh, a);
#pragma unroll
          for (int j = 0; j < 32; ++j) cs[j] = __uint_as_float(a[j]);
          tmem_ld32(trow + kPairS0 + 128 * sb + 64 * chh + 32, a);
#pragma unroll
          for (int j = 0; j < 32; ++j) cs[32 + j] = __uint_as_float(a[j]);
        }
        tmem_wait_ld();
        tc_fence_before();
        arrive_lead(sm.s_free[sb]);
        if (t == sg.tile_lo) {
          m_run = -INFINITY;
          l_run = 0.f;
          lb_run = 0.f;
        }
        // keys of this thread's 64 columns visible to the unit (the same for every head)
        const int rem = sg.keys - (t * kPairTile + 128 * kh + 64 * chh);
        if (rem < 64) {
#pragma unroll
          for (int c = 0; c < 64; ++c) cs[c] = (c < rem) ? cs[c] : -INFINITY;
        }
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < 64; ++c) m4[c & 3] = fmaxf(m4[c & 3], cs[c]);
        float mo[4];
        if (!xchg4(fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * p.sl2, mo)) {
          ok = false;
          break;
        }
        const float mx = fmaxf(fmaxf(mo[0], mo[1]), fmaxf(mo[2], mo[3]));  // this tile's row max
        bool rescale = false;
        float m_new = m_run;
        if (mx > m_run + 8.f) {  // lazy rescale: keep the running max unless it grows by 2^8
          m_new = mx;
          rescale = (m_run != -INFINITY);
        }
        const float alpha = rescale ? ex2_approx(m_run - m_new) : 1.f;
        // exponents centred on the tile max (<= 0), times f = 2^(mx - m_new) <= 2^8 in fp32
        const float msub = (mx == -INFINITY) ? 0.f : mx;
        const float f = (mx == -INFINITY) ? 0.f : ex2_approx(mx - m_new);
        float s4[4] = {0.f, 0.f, 0.f, 0.f}, b4[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t pw[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const uint32_t h = ex2_f16x2(fmaf(cs[2 * c], p.sl2, -msub), fmaf(cs[2 * c + 1], p.sl2, -msub));
          const float e0 = f16_lo(h) * f, e1 = f16_hi(h) * f;
          s4[c & 3] += e0 + e1;
          pw[c] = pack_bf16x2(e0, e1);
          b4[c & 3] += bf16x2_sum(pw[c]);
        }
        // l_run (fp32 weights) gives the lse; lb_run sums the bf16 weights PV uses
        l_run = l_run * alpha + ((s4[0] + s4[1]) + (s4[2] + s4[3]));
        lb_run = lb_run * alpha + ((b4[0] + b4[1]) + (b4[2] + b4[3]));
        m_run = m_new;
        // P is single-buffered and O holds the tiles so far: both wait for PV(n - 1)
        if (n >= 1 && !wait_all(smem_u32(&sm.pv_done), static_cast<uint32_t>((n - 1) & 1), LKV_WAIT_BASE_PAIR(PW_PVDONE))) {
          ok = false;
          break;
        }
        if (__any_sync(0xffffffffu, rescale ? 1 : 0) && t != sg.tile_lo) {
          tc_fence_after();
          tmem_scale_row(trow + 128 * chh, 128, alpha);  // this lane's 128 columns of dims block chh
        }
        // This thread's 64 keys of P belong to value chunk kh; the P buffer holds one chunk at a
        // time, the tile's first in PV order (the last chunk when the tile crosses the cache end)
        // now and the other after its PV.  Row m of 64-key chunk chh (K-major, 128-byte swizzle).
        const int nkc_t = pair_pv_chunks(sg, t);
        const int kc_first = pair_crosses_end(sg, t, T_end) ? nkc_t - 1 : 0;
        auto write_p = [&]() {
          uint8_t* prow = dsm + kPairPOff + chh * 8192 + m * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(prow + ((c ^ (m & 7)) << 4)) =
                make_uint4(pw[4 * c], pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3]);
        };
        if (kh == kc_first) write_p();
        fence_proxy_async_smem();
        if (pair_crosses_end(sg, t, T_end)) {
          // clear this CTA's latent rows past the cache end in the tile's last value chunk (two
          // stages, one per dims block, of two 64-dim boxes each) once the MMA issuer reports them
          // resident
          if (!wait_all(smem_u32(&sm.vland), static_cast<uint32_t>(ncross & 1), LKV_WAIT_BASE_PAIR(PW_VLAND))) {
            ok = false;
            break;
          }
          ++ncross;
          const int stz0 = *reinterpret_cast<volatile int*>(&sm.vzero_stage[0]);
          const int stz1 = *reinterpret_cast<volatile int*>(&sm.vzero_stage[1]);
          const int first = *reinterpret_cast<volatile int*>(&sm.vzero_first);
          const int rows = 128 - (first > 0 ? first : 0);
          const int per_box = rows * 8;  // 16-byte chunks
          const int sidx = (warp - 2) * 32 + lane;
          for (int idx = sidx; idx < 4 * per_box; idx += 256) {
            const int box = idx / per_box, r2 = idx % per_box;  // two stages x two 128-row, 64-dim boxes
            uint8_t* base = ring + ((box >> 1) ? stz1 : stz0) * kPairStageBytes + (box & 1) * kPairChunkBytes;
            *reinterpret_cast<uint4*>(base + (128 - rows + r2 / 8) * 128 + (r2 % 8) * 16) = make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
        }
        tmem_wait_st();
        tc_fence_before();
        arrive_lead(sm.p_full);
        if (nkc_t == 2) {
          // the second value chunk's threads: their P once the first chunk's PV is done
          if (kh != kc_first) {
            if (!wait_all(smem_u32(&sm.p_lo_free), static_cast<uint32_t>(n2s & 1), LKV_WAIT_BASE_PAIR(PW_PLO))) {
              ok = false;
              break;
            }
            write_p();
            fence_proxy_async_smem();
            arrive_lead(sm.p_full2);
          }
          ++n2s;
        }
        if (t != sg.tile_hi - 1) continue;
        // ---------------------------------------------------------- unit epilogue
        float lo[4], lbo[4];
        if (!xchg4(l_run, lo) || !xchg4(lb_run, lbo) ||
            !wait_all(smem_u32(&sm.pv_done), static_cast<uint32_t>(n & 1), LKV_WAIT_BASE_PAIR(PW_PVDONE))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float l_tot = (lo[0] + lo[1]) + (lo[2] + lo[3]);
        const float lb_tot = (lbo[0] + lbo[1]) + (lbo[2] + lbo[3]);
        const float inv_l = lb_tot > 0.f ? 1.f / lb_tot : 0.f;
        const float lse_v = l_tot > 0.f ? (m_run + __log2f(l_tot)) * 0.69314718055994531f : -INFINITY;
        const int d0 = 256 * chh + 128 * kh;  // the 128 dims of this thread's TMEM columns
        const size_t orow = (static_cast<size_t>(sg.b) * p.s_q + sg.k) * p.h_q + head;
        if (sg.complete) {
          tmem_row_to_bf16(trow + 128 * chh, 128, inv_l, p.out + orow * p.dv_total + d0, true);
          if (slot == 0) p.lse[orow] = lse_v;
        } else {
          const size_t prow = static_cast<size_t>(2 * range + sg.slot) * p.rmax + head;
          tmem_row_to_f32(trow + 128 * chh, 128, inv_l, p.part_o + prow * p.dv_total + d0, true);
          if (slot == 0) p.part_lse[prow] = lse_v;
          if (slot == 0 && head == 0) p.seg_info[2 * range + sg.slot] = sg.unit_id;
        }
        tc_fence_before();
        arrive_lead(sm.o_free);
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the odd CTA's producer counts are visible; every remote arrive has been made
  if (leader && warp == 0 && lane == 0) {
    // Drain: no copy may still be landing in either CTA when they exit.  Only the last KS ring
    // chunks and the last unit's Q can be outstanding; a phase one producer issued and the other
    // did not (after a wait gave up) is completed for the missing side here.
    uint32_t zero = 0;
    const WaitCtl dc{&zero, p.err, p.wait_limit_ns};
    const int nl = sm.own_chunks, np = sm.peer_chunks;
    const int nmax = nl > np ? nl : np;
    for (int i = (nmax > KS ? nmax - KS : 0); i < nmax; ++i) {
      const uint32_t fb = smem_u32(&sm.full[i % KS]);
      if (i < nl && i >= np) mbar_complete_tx(fb, static_cast<uint32_t>(sm.stage_bytes[i % KS]));
      if (i >= nl && i < np) mbar_arrive_expect_tx(fb, static_cast<uint32_t>(sm.peer_stage_bytes[i % KS]));
      mbar_wait(fb, static_cast<uint32_t>((i / KS) & 1), dc, LKV_WAIT_BASE_PAIR(PW_DRAIN));
    }
    const int ul = sm.own_units, up = sm.peer_units;
    const int umax = ul > up ? ul : up;
    if (umax > 0) {
      const uint32_t qb = smem_u32(&sm.q_full);
      if (ul == umax && up < umax) mbar_complete_tx(qb, kPairQBytes);
      if (up == umax && ul < umax) mbar_arrive_expect_tx(qb, kPairQBytes);
      mbar_wait(qb, static_cast<uint32_t>((umax - 1) & 1), dc, LKV_WAIT_BASE_PAIR(PW_DRAIN));
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tbase, 512);
  }
}

}  // namespace lkv
