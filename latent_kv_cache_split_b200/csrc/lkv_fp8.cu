// FP8 (e4m3) latent cache rows: per-token quantisation of bf16 latent rows, in bulk or at append.
//
// The pages run the latent-attention models in FP8 for serving (Grouped Latent Attention article,
// section on the GLA-vs-MLA decoding test) but fix no cache format.  The format here: one row per
// token of row_bytes = r + 16 + 2 * d_rope bytes,
//   [0, r)            e4m3 codes of the latent c_KV[t, :]
//   [r, r + 4)        fp32 scale s_t: the smallest power of two with amax_t / s_t <= 448
//                     (amax_t = max |c_KV[t, :]|; 0 for a zero row)
//   [r + 4, r + 16)   zero
//   [r + 16, ...)     the bf16 RoPE key, unchanged
// so every field starts on a 16-byte boundary (TMA boxes can address each one) and the dequantised
// latent is e4m3(code) * s_t, exact in bf16 (a power of two times a 4-bit significand), so a decode
// can dequantise into bf16 tensor-core operands without rounding.  Codes: y = x / s_t (exact),
// rounded to the nearest e4m3 value with ties to even (OCP E4M3: bias 7, 3 mantissa bits, largest
// finite 448, no infinities).
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "../../include/lkv.h"

lkv_status lkv_internal_error_word(int** err);  // lkv_api.cu

namespace {

constexpr int kChunkElems = 8;                  // one 16-byte load of bf16 per lane and chunk
constexpr int kMaxChunks = 4;                   // r <= 32 lanes * 4 chunks * 8 = 1024
constexpr int kMaxLatent = 32 * kMaxChunks * kChunkElems;
constexpr float kE4m3Max = 448.f;

struct QuantArgs {
  const uint8_t* src;
  long long src_rs;      // bytes between source rows
  uint8_t* dst;
  long long dst_rs;      // bytes between cache rows
  long long dst_rows;
  long long n_rows;      // source rows
  int r, d_rope;
  const int* cu;         // append mode: destination from cu_seqlens (else row w -> row w)
  int B, s_q;
  int* err;
};

__device__ __forceinline__ void note_error(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

__device__ __forceinline__ float clamp_e4m3(float y) { return fminf(fmaxf(y, -kE4m3Max), kE4m3Max); }

// The smallest power of two s with amax / s <= 448, for a finite amax > 0: with amax = m * 2^E
// (m in [0.5, 1)), amax <= 448 * 2^e = 0.875 * 2^(9 + e) first holds at e = E - 9 when m <= 0.875,
// else at e = E - 8.  frexpf and ldexpf are exact.
__device__ __forceinline__ float pow2_scale(float amax) {
  int E;
  const float m = frexpf(amax, &E);
  return ldexpf(1.f, m <= 0.875f ? E - 9 : E - 8);
}

// Loads of one source row into registers: latent chunk lane + 32 k (8 bf16 each) and RoPE chunk
// `lane` (16 bytes); chunks past the row are left zero.
struct RowRegs {
  uint4 lat[kMaxChunks];
  uint4 rope;
};

__device__ __forceinline__ void load_row(const QuantArgs& a, long long w, int lane, RowRegs& v) {
  const uint8_t* srow = a.src + w * a.src_rs;
  const int nch = a.r / kChunkElems;
#pragma unroll
  for (int k = 0; k < kMaxChunks; ++k) {
    const int c = lane + 32 * k;
    v.lat[k] = c < nch ? *reinterpret_cast<const uint4*>(srow + 16 * c) : make_uint4(0u, 0u, 0u, 0u);
  }
  const int rope_chunks = a.d_rope * 2 / 16;
  v.rope = lane < rope_chunks ? reinterpret_cast<const uint4*>(srow + 2 * static_cast<long long>(a.r))[lane]
                              : make_uint4(0u, 0u, 0u, 0u);
}

// Quantise the row held in v (source row w) into its cache row.
__device__ __forceinline__ void store_row(const QuantArgs& a, long long w, int lane, const RowRegs& v) {
  long long dst_row = w;
  if (a.cu) {
    const int b = static_cast<int>(w / a.s_q), i = static_cast<int>(w % a.s_q);
    const int c0 = __ldg(a.cu + b);
    const int L = __ldg(a.cu + b + 1) - c0;
    if (L < a.s_q) {
      if (lane == 0) note_error(a.err, LKV_SITE_BAD_LENGTH);
      return;
    }
    dst_row = static_cast<long long>(c0) + L - a.s_q + i;
  }
  if (dst_row < 0 || dst_row >= a.dst_rows) {
    if (lane == 0) note_error(a.err, LKV_SITE_BAD_ROW);
    return;
  }
  uint8_t* drow = a.dst + dst_row * a.dst_rs;
  const int nch = a.r / kChunkElems;
  float amax = 0.f;  // chunks past the row are zero and do not change it
#pragma unroll
  for (int k = 0; k < kMaxChunks; ++k) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v.lat[k]);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h[e]);
      amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float scale = amax > 0.f ? pow2_scale(amax) : 0.f;
#pragma unroll
  for (int k = 0; k < kMaxChunks; ++k) {
    const int c = lane + 32 * k;
    if (c < nch) {
      uint32_t word[2] = {0u, 0u};
      if (scale > 0.f) {
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v.lat[k]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(h[e]);
          const float y0 = clamp_e4m3(__fdiv_rn(f.x, scale));
          const float y1 = clamp_e4m3(__fdiv_rn(f.y, scale));
          // .x lands in the low byte: element 2e at the lower address
          const uint32_t pair = __nv_cvt_float2_to_fp8x2(make_float2(y0, y1), __NV_SATFINITE, __NV_E4M3);
          word[e >> 1] |= (pair & 0xffffu) << (16 * (e & 1));
        }
      }
      *reinterpret_cast<uint2*>(drow + 8 * c) = make_uint2(word[0], word[1]);
    }
  }
  if (lane == 0) *reinterpret_cast<uint4*>(drow + a.r) = make_uint4(__float_as_uint(scale), 0u, 0u, 0u);
  const int rope_chunks = a.d_rope * 2 / 16;
  uint4* rd = reinterpret_cast<uint4*>(drow + a.r + 16);
  if (lane < rope_chunks) rd[lane] = v.rope;
  // RoPE keys wider than 32 chunks (d_rope > 256): the rest straight from the source row
  const uint4* rs = reinterpret_cast<const uint4*>(a.src + w * a.src_rs + 2 * static_cast<long long>(a.r));
  for (int c = 32 + lane; c < rope_chunks; c += 32) rd[c] = rs[c];
}

// Grid-stride over rows, one warp per row at a time: the next row's loads are issued before the
// current row is quantised, so every warp keeps two rows of loads in flight.
__global__ void __launch_bounds__(256, 3) quantize_fp8_kernel(QuantArgs a) {
  const int lane = threadIdx.x & 31;
  const long long n_warps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  long long w = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (w >= a.n_rows) return;
  RowRegs cur;
  load_row(a, w, lane, cur);
  while (true) {
    const long long wn = w + n_warps;
    const bool more = wn < a.n_rows;
    RowRegs nxt;
    if (more) load_row(a, wn, lane, nxt);
    store_row(a, w, lane, cur);
    if (!more) break;
    cur = nxt;
    w = wn;
  }
}

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t row_bytes_of(int r, int d_rope) {
  if (r <= 0 || r % 16 || r > kMaxLatent || d_rope < 0 || d_rope % 8) return 0;
  return static_cast<size_t>(r) + 16 + 2 * static_cast<size_t>(d_rope);
}

lkv_status launch(QuantArgs& a, lkv_stream_t stream) {
  if (a.n_rows * 32 >= (1LL << 31)) return LKV_ERR_UNSUPPORTED;
  int* err = nullptr;
  const lkv_status st = lkv_internal_error_word(&err);
  if (st != LKV_OK) return st;
  a.err = err;
  // enough 8-warp blocks for every row, at most the 3 per SM that are resident at once (80
  // registers a thread); the loop takes the rest
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      sms <= 0)
    return LKV_ERR_CUDA;
  const long long need = (a.n_rows + 7) / 8;
  const unsigned blocks = static_cast<unsigned>(need < 3LL * sms ? need : 3LL * sms);
  quantize_fp8_kernel<<<blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(a);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? LKV_OK : LKV_ERR_CUDA;
}

// Shared checks of the source rows (bf16, latent then RoPE key) and the cache rows.
lkv_status check_rows(const void* src, int64_t src_row_stride, const void* cache, int64_t cache_row_stride_bytes,
                      int r, int d_rope) {
  const size_t rb = row_bytes_of(r, d_rope);
  if (!src || !cache || rb == 0) return LKV_ERR_INVALID_ARG;
  if (!al16(src) || !al16(cache) || (src_row_stride * 2) % 16 || cache_row_stride_bytes % 16) return LKV_ERR_INVALID_ARG;
  if (src_row_stride < static_cast<int64_t>(r) + d_rope || cache_row_stride_bytes < static_cast<int64_t>(rb))
    return LKV_ERR_INVALID_ARG;
  return LKV_OK;
}

}  // namespace

extern "C" {

size_t lkv_fp8_cache_row_bytes(int r, int d_rope) { return row_bytes_of(r, d_rope); }

lkv_status lkv_quantize_latent_fp8(const void* src, int64_t src_row_stride, void* cache,
                                   int64_t cache_row_stride_bytes, int64_t n_rows, int r, int d_rope,
                                   lkv_stream_t stream) {
  lkv_status st = check_rows(src, src_row_stride, cache, cache_row_stride_bytes, r, d_rope);
  if (st != LKV_OK) return st;
  if (n_rows <= 0) return LKV_ERR_INVALID_ARG;
  QuantArgs a{};
  a.src = static_cast<const uint8_t*>(src);
  a.src_rs = src_row_stride * 2;
  a.dst = static_cast<uint8_t*>(cache);
  a.dst_rs = cache_row_stride_bytes;
  a.dst_rows = n_rows;
  a.n_rows = n_rows;
  a.r = r;
  a.d_rope = d_rope;
  return launch(a, stream);
}

lkv_status lkv_latent_cache_append_fp8(const void* new_rows, int64_t new_row_stride, void* cache,
                                       int64_t cache_row_stride_bytes, int64_t cache_rows, int r, int d_rope,
                                       const int32_t* cu_seqlens, int batch, int s_q, lkv_stream_t stream) {
  lkv_status st = check_rows(new_rows, new_row_stride, cache, cache_row_stride_bytes, r, d_rope);
  if (st != LKV_OK) return st;
  if (!cu_seqlens || batch <= 0 || s_q <= 0 || cache_rows <= 0) return LKV_ERR_INVALID_ARG;
  QuantArgs a{};
  a.src = static_cast<const uint8_t*>(new_rows);
  a.src_rs = new_row_stride * 2;
  a.dst = static_cast<uint8_t*>(cache);
  a.dst_rs = cache_row_stride_bytes;
  a.dst_rows = cache_rows;
  a.n_rows = static_cast<long long>(batch) * s_q;
  a.r = r;
  a.d_rope = d_rope;
  a.cu = cu_seqlens;
  a.B = batch;
  a.s_q = s_q;
  return launch(a, stream);
}

}  // extern "C"
