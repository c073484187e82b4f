// Work partition shared by the decode kernels and the split combine.
//
// A "unit" is one query token of a request (MLA absorbed path: all h_q heads attend to the
// shared latent, one unit per new token) or one group of a request (GQLA / GLA: the rows of
// a unit are the group's heads for every new token).  Each unit needs ceil(keys / 64) key
// tiles (64 or 128 keys, per kernel).  All tiles of all units are laid end to end (request-major, then unit) and the
// sequence is cut into P equal ranges, one per persistent CTA (per CTA pair for MLA).  A
// range is processed as "segments": maximal runs of its tiles that belong to one unit.  A
// segment that covers its unit entirely writes the final output; the first or last segment
// of a range may cover only part of a unit and then writes an fp32 partial (slot 0 = first
// segment of the range, slot 1 = last), merged afterwards by the combine kernel.
//
// Lockstep variant for grouped units (G >= 4 groups per request, P a multiple of G): the
// requests' tiles (one unit per request, every group of a request has the same tiles) are cut
// into P / G equal blocks, and range p walks block p / G for group p % G.  The G ranges of a
// block then stream the same requests at the same pace, so the key rows they share (the RoPE
// key) are fetched from HBM once and served to the other groups from L2.  (With 2 groups the
// shared key is a tenth of the traffic, and measured no faster in lockstep.)
#pragma once
#include <cstdint>

#if defined(__CUDA_ARCH__)
#define LKV_LDG(p) __ldg(p)
#else
#define LKV_LDG(p) (*(p))
#endif

namespace lkv {

struct SchedArgs {
  const int* cu;         // [B+1]
  int B, s_q;
  int tile;              // keys per tile
  int units_per_req;     // MLA: s_q ; grouped: G
  int per_query_units;   // 1: unit k is query token k (MLA); 0: unit k is group k
  int P;                 // number of ranges
};

// Keys visible to unit k of a request of length L (0 if the request is malformed).
__host__ __device__ __forceinline__ int unit_keys(const SchedArgs& a, int L, int k) {
  if (L < a.s_q) return 0;
  return a.per_query_units ? (L - a.s_q + k + 1) : L;
}
__host__ __device__ __forceinline__ long long ceil_tiles(int keys, int tile) {
  return (static_cast<long long>(keys) + tile - 1) / tile;
}
__host__ __device__ __forceinline__ long long request_tiles(const SchedArgs& a, int b) {
  const int L = LKV_LDG(a.cu + b + 1) - LKV_LDG(a.cu + b);
  if (L < a.s_q) return 0;
  if (a.per_query_units) {
    long long t = 0;
    for (int k = 0; k < a.units_per_req; ++k) t += ceil_tiles(L - a.s_q + k + 1, a.tile);
    return t;
  }
  return a.units_per_req * ceil_tiles(L, a.tile);
}

struct Segment {
  int b, k;             // request, unit within request
  int cu_b, L;          // first cache row and length of request b
  int keys;             // keys visible to the unit (max over its rows)
  int tile_lo, tile_hi; // tiles [tile_lo, tile_hi) of the unit
  int complete;         // covers the whole unit
  int slot;             // partial slot (0 first segment of the range, 1 last); -1 if complete
  int unit_id;          // b * units_per_req + k
};

// Request-space arguments of the lockstep variant (see above), or `a` itself.
__host__ __device__ __forceinline__ bool lockstep_groups(const SchedArgs& a) {
  return !a.per_query_units && a.units_per_req >= 4 && a.P % a.units_per_req == 0;
}
__host__ __device__ __forceinline__ SchedArgs request_space(const SchedArgs& a) {
  SchedArgs r = a;
  if (lockstep_groups(a)) {
    r.units_per_req = 1;
    r.P = a.P / a.units_per_req;
  }
  return r;
}

// Cursor over the segments of one range.  Every role of a CTA runs its own copy from the
// same start state, so all roles see the same sequence.
struct SegCursor {
  long long t_begin, t_end;  // global tile range
  long long unit_t0;         // global index of the current unit's first tile
  int b, k;
  int produced;              // segments produced so far

  __host__ __device__ __forceinline__ bool next(const SchedArgs& a, Segment& s) {
    while (b < a.B && unit_t0 < t_end) {
      const int cu_b = LKV_LDG(a.cu + b);
      const int L = LKV_LDG(a.cu + b + 1) - cu_b;
      const int keys = unit_keys(a, L, k);
      const long long nt = ceil_tiles(keys, a.tile);
      const long long lo = (t_begin > unit_t0 ? t_begin : unit_t0) - unit_t0;
      const long long hi_g = unit_t0 + nt < t_end ? unit_t0 + nt : t_end;
      const long long hi = hi_g - unit_t0;
      const int cur_b = b, cur_k = k;
      unit_t0 += nt;
      if (++k == a.units_per_req) {
        k = 0;
        ++b;
      }
      if (nt == 0 || hi <= lo) continue;
      s.b = cur_b;
      s.k = cur_k;
      s.cu_b = cu_b;
      s.L = L;
      s.keys = keys;
      s.tile_lo = static_cast<int>(lo);
      s.tile_hi = static_cast<int>(hi);
      s.complete = (lo == 0 && hi == nt);
      s.slot = s.complete ? -1 : (produced == 0 ? 0 : 1);
      s.unit_id = cur_b * a.units_per_req + cur_k;
      ++produced;
      return true;
    }
    return false;
  }
};

__device__ __forceinline__ long long warp_sum_ll(long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Locate the start of range p.  Called by one full warp; returns the cursor in every lane.
// *malformed is set (all lanes) if some request holds fewer than s_q rows.
__device__ __forceinline__ SegCursor locate_range(const SchedArgs& a, int p, bool* malformed) {
  const int lane = threadIdx.x & 31;
  long long total = 0;
  bool bad = false;
  for (int b0 = 0; b0 < a.B; b0 += 32) {
    const int b = b0 + lane;
    total += warp_sum_ll(b < a.B ? request_tiles(a, b) : 0);
    if (b < a.B && (LKV_LDG(a.cu + b + 1) - LKV_LDG(a.cu + b)) < a.s_q) bad = true;
  }
  *malformed = __any_sync(0xffffffffu, bad) != 0;
  SegCursor c;
  c.t_begin = total * p / a.P;
  c.t_end = total * (p + 1) / a.P;
  c.produced = 0;
  // request containing t_begin
  long long acc = 0;
  int fb = a.B;
  long long facc = 0;
  for (int b0 = 0; b0 < a.B; b0 += 32) {
    const int b = b0 + lane;
    const long long t = b < a.B ? request_tiles(a, b) : 0;
    long long incl = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    const unsigned hit = __ballot_sync(0xffffffffu, b < a.B && acc + incl > c.t_begin);
    if (hit) {
      const int l0 = __ffs(hit) - 1;
      fb = b0 + l0;
      facc = acc + __shfl_sync(0xffffffffu, incl - t, l0);
      break;
    }
    acc += __shfl_sync(0xffffffffu, incl, 31);
  }
  c.b = fb;
  c.k = 0;
  c.unit_t0 = facc;
  if (fb < a.B) {
    // walk units inside the request until the one containing t_begin
    const int L = LKV_LDG(a.cu + fb + 1) - LKV_LDG(a.cu + fb);
    for (int k = 0; k < a.units_per_req; ++k) {
      const long long nt = ceil_tiles(unit_keys(a, L, k), a.tile);
      if (c.unit_t0 + nt > c.t_begin) {
        c.k = k;
        break;
      }
      c.unit_t0 += nt;
    }
  }
  return c;
}

// Host twin of locate_range, same arithmetic, sequential (used for CPU checks of the partition).
inline SegCursor locate_range_host(const SchedArgs& a, int p) {
  long long total = 0;
  for (int b = 0; b < a.B; ++b) total += request_tiles(a, b);
  SegCursor c;
  c.t_begin = total * p / a.P;
  c.t_end = total * (p + 1) / a.P;
  c.produced = 0;
  c.b = a.B;
  c.k = 0;
  c.unit_t0 = 0;
  long long acc = 0;
  for (int b = 0; b < a.B; ++b) {
    const long long t = request_tiles(a, b);
    if (acc + t > c.t_begin) {
      c.b = b;
      c.unit_t0 = acc;
      const int L = a.cu[b + 1] - a.cu[b];
      for (int k = 0; k < a.units_per_req; ++k) {
        const long long nt = ceil_tiles(unit_keys(a, L, k), a.tile);
        if (c.unit_t0 + nt > c.t_begin) {
          c.k = k;
          break;
        }
        c.unit_t0 += nt;
      }
      break;
    }
    acc += t;
  }
  return c;
}

}  // namespace lkv
