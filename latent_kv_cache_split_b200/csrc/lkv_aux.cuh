// CUDA-core kernels: fp32 decode (the fp32 storage path), cache append, split-KV combine,
// standalone partial merge, and the bounded-wait self test.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "lkv_ptx.cuh"
#include "lkv_sched.cuh"
#include "../../include/lkv.h"

namespace lkv {

// ------------------------------------------------------------------------------------------
// fp32 decode on CUDA cores.  One CTA per (request b, query token i, head h); exact fp32
// arithmetic with expf/logf (this path serves fp32 storage, where a tensor-core tf32 product
// could not hold a 1e-5 agreement).  Keys are visited in chunks of kSimtChunk with an online
// softmax, so any length works.
// ------------------------------------------------------------------------------------------
constexpr int kSimtThreads = 128;
constexpr int kSimtChunk = 256;
constexpr int kSimtMaxQ = 1024;  // d_k + d_R
constexpr int kSimtMaxV = 512;   // d_v

struct SimtParams {
  const float* q_nope;  // [B, s_q, h_q, dk]
  const float* q_rope;  // [B, s_q, h_q, dr]
  const float* k;       // row t, group j at k + t*k_rs + j*k_gs
  const float* v;
  const float* kr;      // row t at kr + t*kr_rs
  long long k_rs, k_gs, v_rs, v_gs, kr_rs;
  const int* cu;
  int B, s_q, h_q, G, dk, dv, dr;
  float scale;
  float* out;           // [B, s_q, h_q, dv]
  float* lse;           // [B, s_q, h_q]
  int* err;
};

__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float r = red[0];
  for (int i = 1; i < kSimtThreads / 32; ++i) r = fmaxf(r, red[i]);
  return r;
}
__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float r = 0.f;
  for (int i = 0; i < kSimtThreads / 32; ++i) r += red[i];
  return r;
}

__global__ void __launch_bounds__(kSimtThreads) decode_simt_fp32_kernel(const SimtParams p) {
  __shared__ float qs[kSimtMaxQ];
  __shared__ float ps[kSimtChunk];
  __shared__ float red[kSimtThreads / 32];
  const int h = blockIdx.x % p.h_q;
  const int i = (blockIdx.x / p.h_q) % p.s_q;
  const int b = blockIdx.x / (p.h_q * p.s_q);
  const int j = h / (p.h_q / p.G);
  const int tid = threadIdx.x;
  const int c0 = __ldg(p.cu + b);
  const int L = __ldg(p.cu + b + 1) - c0;
  const size_t qrow = (static_cast<size_t>(b) * p.s_q + i) * p.h_q + h;
  if (L < p.s_q) {
    if (tid == 0) record_error(p.err, LKV_SITE_BAD_LENGTH);
    return;
  }
  const int nvis = L - p.s_q + i + 1;
  for (int c = tid; c < p.dk; c += kSimtThreads) qs[c] = p.q_nope[qrow * p.dk + c];
  for (int c = tid; c < p.dr; c += kSimtThreads) qs[p.dk + c] = p.q_rope[qrow * p.dr + c];
  __syncthreads();
  float acc[kSimtMaxV / kSimtThreads];
#pragma unroll
  for (int a = 0; a < kSimtMaxV / kSimtThreads; ++a) acc[a] = 0.f;
  float m = -INFINITY, l = 0.f;
  for (int t0 = 0; t0 < nvis; t0 += kSimtChunk) {
    const int n = min(kSimtChunk, nvis - t0);
    float cmax = -INFINITY;
    for (int t = tid; t < n; t += kSimtThreads) {
      const long long row = c0 + t0 + t;
      const float* kp = p.k + row * p.k_rs + static_cast<long long>(j) * p.k_gs;
      const float* rp = p.kr + row * p.kr_rs;
      float s = 0.f;
      for (int c = 0; c < p.dk; ++c) s = fmaf(qs[c], __ldg(kp + c), s);
      for (int c = 0; c < p.dr; ++c) s = fmaf(qs[p.dk + c], __ldg(rp + c), s);
      s *= p.scale;
      ps[t] = s;
      cmax = fmaxf(cmax, s);
    }
    const float m_new = fmaxf(m, block_max(cmax, red));
    const float alpha = (m == -INFINITY) ? 0.f : expf(m - m_new);
    float csum = 0.f;
    for (int t = tid; t < n; t += kSimtThreads) {
      const float e = expf(ps[t] - m_new);
      ps[t] = e;
      csum += e;
    }
    l = l * alpha + block_sum(csum, red);  // block_sum's barriers also publish ps
    m = m_new;
#pragma unroll
    for (int a = 0; a < kSimtMaxV / kSimtThreads; ++a) {
      const int c = tid + a * kSimtThreads;
      if (c < p.dv) {
        float s = 0.f;
        const float* vp = p.v + static_cast<long long>(c0 + t0) * p.v_rs + static_cast<long long>(j) * p.v_gs + c;
        for (int t = 0; t < n; ++t) s = fmaf(ps[t], __ldg(vp + static_cast<long long>(t) * p.v_rs), s);
        acc[a] = acc[a] * alpha + s;
      }
    }
    __syncthreads();  // ps is rewritten by the next chunk
  }
  const float inv = 1.f / l;
#pragma unroll
  for (int a = 0; a < kSimtMaxV / kSimtThreads; ++a) {
    const int c = tid + a * kSimtThreads;
    if (c < p.dv) p.out[qrow * p.dv + c] = acc[a] * inv;
  }
  if (tid == 0) p.lse[qrow] = m + logf(l);
}

// ------------------------------------------------------------------------------------------
// Cache append: one warp per new row, 16-byte copies.
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) append_kernel(const uint8_t* src, long long src_rs,
                                                     uint8_t* cache, long long cache_rs,
                                                     long long cache_rows, long long row_bytes,
                                                     const int* cu, int B, int s_q, int* err) {
  const int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= B * s_q) return;
  const int b = w / s_q, i = w % s_q;
  const int c0 = __ldg(cu + b);
  const int L = __ldg(cu + b + 1) - c0;
  if (L < s_q) {
    if (lane == 0) record_error(err, LKV_SITE_BAD_LENGTH);
    return;
  }
  const long long dst_row = static_cast<long long>(c0) + L - s_q + i;
  if (dst_row < 0 || dst_row >= cache_rows) {
    if (lane == 0) record_error(err, LKV_SITE_BAD_ROW);
    return;
  }
  const uint4* s = reinterpret_cast<const uint4*>(src + static_cast<long long>(w) * src_rs);
  uint4* d = reinterpret_cast<uint4*>(cache + dst_row * cache_rs);
  for (long long c = lane; c < row_bytes / 16; c += 32) d[c] = s[c];
}

// ------------------------------------------------------------------------------------------
// Split-KV combine for the tensor-core decode: one warp per output row of a unit.  The
// pieces of unit u are the workspace slots whose record equals u (ranges are consecutive,
// so they form one run of slots in range order):
//   lse = ln sum_p exp(lse_p),  out = sum_p exp(lse_p - lse) o_p.
// Units processed whole by one range have no record and are left alone.
// ------------------------------------------------------------------------------------------
struct CombineParams {
  const int* seg_info;  // [2P]
  const float* part_lse;
  const float* part_o;
  int P, rmax, dv_total;
  int R;                // valid rows per unit
  int per_query_units;  // MLA: unit = (b, i), row = head; grouped: unit = (b, j)
  int units_per_req, s_q, h_q, hpg;
  __nv_bfloat16* out;
  float* lse;
};

constexpr int kCombineWarps = 4;

__global__ void __launch_bounds__(kCombineWarps * 32) combine_kernel(const CombineParams p) {
  griddep_wait();  // launched as a programmatic dependent of the decode kernel: its writes first
  __shared__ int lo, hi;
  const int u = blockIdx.x;
  const int tid = threadIdx.x;
  if (tid == 0) {
    lo = 1 << 30;
    hi = -1;
  }
  __syncthreads();
  for (int s = tid; s < 2 * p.P; s += blockDim.x) {
    if (p.seg_info[s] == u) {
      atomicMin(&lo, s);
      atomicMax(&hi, s);
    }
  }
  __syncthreads();
  if (hi < 0) return;
  const int warp = tid >> 5, lane = tid & 31;
  const int r = blockIdx.y * kCombineWarps + warp;
  if (r >= p.R) return;
  // global lse
  float mx = -INFINITY;
  for (int s = lo; s <= hi; ++s)
    if (p.seg_info[s] == u) mx = fmaxf(mx, p.part_lse[static_cast<size_t>(s) * p.rmax + r]);
  const float msafe = (mx == -INFINITY) ? 0.f : mx;
  float tot = 0.f;
  for (int s = lo; s <= hi; ++s)
    if (p.seg_info[s] == u) tot += expf(p.part_lse[static_cast<size_t>(s) * p.rmax + r] - msafe);
  const float lse = msafe + logf(tot);
  const float inv = tot > 0.f ? 1.f / tot : 0.f;
  int b, i, h;
  if (p.per_query_units) {
    b = u / p.units_per_req;
    i = u % p.units_per_req;
    h = r;
  } else {
    b = u / p.units_per_req;
    const int j = u % p.units_per_req;
    i = r / p.hpg;
    h = j * p.hpg + r % p.hpg;
  }
  const size_t orow = (static_cast<size_t>(b) * p.s_q + i) * p.h_q + h;
  for (int c = lane * 4; c < p.dv_total; c += 128) {
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = lo; s <= hi; ++s) {
      if (p.seg_info[s] != u) continue;
      const float lp = p.part_lse[static_cast<size_t>(s) * p.rmax + r];
      if (lp == -INFINITY) continue;
      const float w = expf(lp - msafe) * inv;
      const float4 o = *reinterpret_cast<const float4*>(p.part_o + (static_cast<size_t>(s) * p.rmax + r) * p.dv_total + c);
      a.x = fmaf(w, o.x, a.x);
      a.y = fmaf(w, o.y, a.y);
      a.z = fmaf(w, o.z, a.z);
      a.w = fmaf(w, o.w, a.w);
    }
    uint2 pk;
    pk.x = pack_bf16x2(a.x, a.y);
    pk.y = pack_bf16x2(a.z, a.w);
    *reinterpret_cast<uint2*>(p.out + orow * p.dv_total + c) = pk;
  }
  if (lane == 0) p.lse[orow] = lse;
}

// Standalone merge of n_parts partial results per row (lkv_merge_partials).
__global__ void __launch_bounds__(128) merge_kernel(const float* o_parts, const float* lse_parts,
                                                    int n_parts, long long rows, int d_v,
                                                    int out_fp32, void* out, float* lse) {
  const long long r = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  float mx = -INFINITY;
  for (int q = 0; q < n_parts; ++q) mx = fmaxf(mx, lse_parts[static_cast<long long>(q) * rows + r]);
  const float msafe = (mx == -INFINITY) ? 0.f : mx;
  float tot = 0.f;
  for (int q = 0; q < n_parts; ++q) tot += expf(lse_parts[static_cast<long long>(q) * rows + r] - msafe);
  const float inv = tot > 0.f ? 1.f / tot : 0.f;
  for (int c = lane * 4; c < d_v; c += 128) {
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int q = 0; q < n_parts; ++q) {
      const float lp = lse_parts[static_cast<long long>(q) * rows + r];
      if (lp == -INFINITY) continue;
      const float w = expf(lp - msafe) * inv;
      const float4 o = *reinterpret_cast<const float4*>(o_parts + (static_cast<long long>(q) * rows + r) * d_v + c);
      a.x = fmaf(w, o.x, a.x);
      a.y = fmaf(w, o.y, a.y);
      a.z = fmaf(w, o.z, a.z);
      a.w = fmaf(w, o.w, a.w);
    }
    if (out_fp32) {
      *reinterpret_cast<float4*>(static_cast<float*>(out) + r * d_v + c) = a;
    } else {
      uint2 pk;
      pk.x = pack_bf16x2(a.x, a.y);
      pk.y = pack_bf16x2(a.z, a.w);
      *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(out) + r * d_v + c) = pk;
    }
  }
  if (lane == 0 && lse) lse[r] = msafe + logf(tot);
}

// Bounded-wait self test: one thread waits on a barrier that nothing arrives at.
__global__ void selftest_wait_kernel(int* err, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitCtl wc{&abort_flag, err, limit_ns};
    mbar_wait(smem_u32(&bar), 0, wc, LKV_SITE_SELFTEST);
  }
}

}  // namespace lkv
