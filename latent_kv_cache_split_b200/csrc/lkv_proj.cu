// Projections either side of the decode path (GQLA explainer, section 2 "Methodology"):
//   absorbed path:  q_abs[t, h, :] = W_UK[j(h)] q[t, h, :]       (the query in latent space)
//                   out[t, h, :]   = W_UV[j(h)]^T o_lat[t, h, :]  (the output back in head space)
//   GQA path:       X[t, j, :]     = c_KV[t, :] W[j]              (expanded K_j or V_j of the cache)
// with j(h) = h / (h_q / G), and the output projection that follows attention,
//                   y[t, :]        = o[t, :] W_O                  (o = the heads' outputs side by side)
// which, with the heads split across GPUs along the group axis, gives each GPU a partial y to be summed
// (GQLA explainer, section 2, GQA path: tensor parallelism along the group axis).
//
// Each is one launch of the tensor-core GEMM of lkv_gemm.cuh (bf16 operands, fp32 accumulation in
// TMEM): the host describes the rows of A (which may gather the heads of one group across tokens),
// which B matrix a tile takes, and where each result row goes.
#include <climits>
#include <cstdint>
#include <mutex>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/lkv.h"
#include "lkv_gemm.cuh"
#include "lkv_tma_host.h"

lkv_status lkv_internal_device_info(int** err, int* num_sms, unsigned long long* wait_ns);  // lkv_api.cu

namespace {

using namespace lkv;

constexpr int kMaxDevices = 64;
constexpr int kNoColumnGroups = 1 << 30;  // nb when the column axis stays inside one B matrix

bool fits_int(long long v) { return v > 0 && v <= 0x7fffffffLL; }
bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
int cdiv(long long a, long long b) { return static_cast<int>((a + b - 1) / b); }

// Row tiling: a tile takes b1 consecutive rows of A's dim 1 (a power of two that divides
// rows_per_b, so one tile never spans two B matrices; 128 when rows do not select B) times b2 = 128 / b1
// rows of dim 2.
void set_rows(GemmParams& p, int n1, int n2, int rows_per_b) {
  int b1 = 128;
  if (rows_per_b) {
    b1 = 1;
    while (b1 < 128 && rows_per_b % (2 * b1) == 0) b1 *= 2;
  }
  p.b1 = b1;
  p.lg_b1 = 31 - __builtin_clz(static_cast<unsigned>(b1));
  p.b2 = 128 / b1;
  p.n1 = n1;
  p.n2 = n2;
  p.t1 = cdiv(n1, b1);
  p.t2 = cdiv(n2, p.b2);
  p.rows_per_b = rows_per_b;
}

// Column tiling: as few tiles of <= 256 columns as cover n, each a multiple of 64 wide.
void set_cols(GemmParams& p, int n) {
  p.n_tiles = cdiv(n, 256);
  p.tn = 64 * cdiv(cdiv(n, p.n_tiles), 64);
  p.b_bytes = p.tn * 128;
}

lkv_status launch(const CUtensorMap& ma, const CUtensorMap& mb, GemmParams& p, int k, cudaStream_t s) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LKV_ERR_CUDA;
  int num_sms = 0;
  lkv_status st = lkv_internal_device_info(&p.err, &num_sms, &p.wait_limit_ns);
  if (st != LKV_OK) return st;
  static std::mutex mu;
  static bool attr_set[kMaxDevices] = {};
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!attr_set[dev]) {
      if (cudaFuncSetAttribute(proj_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kGemmSmemBytes)) != cudaSuccess ||
          cudaFuncSetAttribute(proj_gemm_resident_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kResSmemBytes)) != cudaSuccess ||
          cudaFuncSetAttribute(proj_gemm_splitk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kGemmSmemBytes)) != cudaSuccess ||
          cudaFuncSetAttribute(proj_gemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kPgSmemBytes)) != cudaSuccess)
        return LKV_ERR_CUDA;
      attr_set[dev] = true;
    }
  }
  p.k_blocks = cdiv(k, 64);
  // CTA-pair weight-resident form: as the one-CTA form below, with A of one row dimension and at
  // least two 256-row tiles per pair.
  const int pg_n = cdiv(p.n_valid, kPgTn);
  const int pg_groups = pg_n <= num_sms / 2 ? (num_sms / 2) / pg_n : 0;
  const long long pg_m = (static_cast<long long>(p.t1) + 1) / 2;
  if (p.b_mn && p.rows_per_b == 0 && p.groups == 1 && p.n2 == 1 && p.k_blocks * 64 <= kResMaxK && pg_groups > 0 &&
      pg_m >= 2LL * pg_groups && pg_m <= INT_MAX) {
    p.tn = kPgTn;
    p.n_tiles = pg_n;
    p.m_tiles = static_cast<int>(pg_m);
    p.res_groups = pg_groups;
    p.total_tiles = static_cast<int>(pg_m * pg_n);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * pg_groups * pg_n));
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = kPgSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, proj_gemm_pair_kernel, ma, mb, p);
    if (e != cudaSuccess) cudaGetLastError();
    return e == cudaSuccess ? LKV_OK : LKV_ERR_CUDA;
  }
  // Weight-resident form: one B for every row (MN-major, not chosen per row or per column block),
  // K <= 512, at most one CTA per SM for each 128-column tile and at least two row tiles per CTA.
  const int res_n = cdiv(p.n_valid, kResTn);
  const long long res_m = static_cast<long long>(p.t1) * p.t2;
  const int res_groups = res_n <= num_sms ? num_sms / res_n : 0;
  if (p.b_mn && p.rows_per_b == 0 && p.groups == 1 && p.k_blocks * 64 <= kResMaxK && res_groups > 0 &&
      res_m >= 2LL * res_groups && res_m <= INT_MAX) {
    p.tn = kResTn;
    p.n_tiles = res_n;
    p.m_tiles = static_cast<int>(res_m);
    p.res_groups = res_groups;
    p.total_tiles = static_cast<int>(res_m * res_n);
    proj_gemm_resident_kernel<<<res_groups * res_n, kGemmThreads, kResSmemBytes, s>>>(ma, mb, p);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? LKV_OK : LKV_ERR_CUDA;
  }
  const long long tiles = static_cast<long long>(p.n_tiles) * p.t1 * p.t2 * p.groups;
  if (tiles <= 0 || tiles > INT_MAX) return LKV_ERR_INVALID_ARG;
  p.total_tiles = static_cast<int>(tiles);
  // Split-K form: fewer tiles than half the SMs over a long K (>= 2048; below that the cluster
  // reduction costs more than it saves: a 512-wide un-absorb measured 10.5 against 8.4 us) -- the S
  // CTAs of a cluster share a tile (S = 8, 4 or 2: the most that fit on the SMs with >= 4 K blocks
  // each).
  if (2 * tiles <= num_sms && p.k_blocks >= 32) {
    int splits = 0;
    for (int c = 8; c >= 2 && splits == 0; c >>= 1)
      if (tiles * c <= num_sms && p.k_blocks >= 4 * c) splits = c;
    if (splits) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(static_cast<unsigned>(tiles * splits));
      cfg.blockDim = dim3(kGemmThreads);
      cfg.dynamicSmemBytes = kGemmSmemBytes;
      cfg.stream = s;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = static_cast<unsigned>(splits);
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      const cudaError_t e = cudaLaunchKernelEx(&cfg, proj_gemm_splitk_kernel, ma, mb, p, splits);
      if (e != cudaSuccess) cudaGetLastError();
      return e == cudaSuccess ? LKV_OK : LKV_ERR_CUDA;
    }
  }
  const int grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
  proj_gemm_kernel<<<grid, kGemmThreads, kGemmSmemBytes, s>>>(ma, mb, p);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? LKV_OK : LKV_ERR_CUDA;
}

GemmParams base_params(void* out) {
  GemmParams p{};
  p.groups = 1;
  p.nb = kNoColumnGroups;
  p.out = out;
  return p;
}

}  // namespace

extern "C" {

lkv_status lkv_absorb_query(const void* q, const void* w_uk, void* q_abs, int n_tok, int h_q, int groups, int d_h,
                            int r, int dtype, lkv_stream_t stream) {
  if (!q || !w_uk || !q_abs || n_tok <= 0 || h_q <= 0 || groups <= 0 || d_h <= 0 || r <= 0 ||
      h_q % groups != 0 || !fits_int(static_cast<long long>(h_q) * r) || !fits_int(static_cast<long long>(h_q) * d_h))
    return LKV_ERR_INVALID_ARG;
  if (dtype != LKV_BF16) return LKV_ERR_UNSUPPORTED;
  if (d_h % 8 != 0 || !al16(q) || !al16(w_uk)) return LKV_ERR_INVALID_ARG;
  // rows (h, t) of q; B = W_UK[j] as [r, d_h] rows (K-major)
  GemmParams p = base_params(q_abs);
  set_rows(p, h_q, n_tok, h_q / groups);
  set_cols(p, r);
  p.n_valid = r;
  p.os1 = r;
  p.os2 = static_cast<long long>(h_q) * r;
  p.vec_ok = (r % 8 == 0) && al16(q_abs);
  CUtensorMap ma, mb;
  if (!make_tmap_bf16_3d(&ma, q, d_h, h_q, n_tok, 2ull * d_h, 2ull * d_h * h_q, p.b1, p.b2) ||
      !make_tmap_bf16_3d(&mb, w_uk, d_h, r, groups, 2ull * d_h, 2ull * d_h * r, p.tn, 1))
    return LKV_ERR_INVALID_ARG;
  return launch(ma, mb, p, d_h, static_cast<cudaStream_t>(stream));
}

lkv_status lkv_unabsorb_output(const void* o_lat, const void* w_uv, void* out, int n_tok, int h_q, int groups, int r,
                               int d_v, int dtype, lkv_stream_t stream) {
  if (!o_lat || !w_uv || !out || n_tok <= 0 || h_q <= 0 || groups <= 0 || r <= 0 || d_v <= 0 ||
      h_q % groups != 0 || !fits_int(static_cast<long long>(h_q) * r) || !fits_int(static_cast<long long>(h_q) * d_v))
    return LKV_ERR_INVALID_ARG;
  if (dtype != LKV_BF16) return LKV_ERR_UNSUPPORTED;
  if (r % 8 != 0 || d_v % 8 != 0 || !al16(o_lat) || !al16(w_uv)) return LKV_ERR_INVALID_ARG;
  // rows (h, t) of o_lat; B = W_UV[j] as [r, d_v] (MN-major)
  GemmParams p = base_params(out);
  set_rows(p, h_q, n_tok, h_q / groups);
  set_cols(p, d_v);
  p.b_mn = 1;
  p.n_valid = d_v;
  p.os1 = d_v;
  p.os2 = static_cast<long long>(h_q) * d_v;
  p.vec_ok = al16(out);
  CUtensorMap ma, mb;
  if (!make_tmap_bf16_3d(&ma, o_lat, r, h_q, n_tok, 2ull * r, 2ull * r * h_q, p.b1, p.b2) ||
      !make_tmap_bf16_3d(&mb, w_uv, d_v, r, groups, 2ull * d_v, 2ull * d_v * r, 64, 1))
    return LKV_ERR_INVALID_ARG;
  return launch(ma, mb, p, r, static_cast<cudaStream_t>(stream));
}

lkv_status lkv_expand_latent(const void* c, int64_t c_row_stride, const void* w, void* x, int64_t n_rows, int groups,
                             int r, int d, int dtype, lkv_stream_t stream) {
  if (!c || !w || !x || n_rows <= 0 || groups <= 0 || r <= 0 || d <= 0 || c_row_stride < r ||
      !fits_int(n_rows) || !fits_int(c_row_stride) || !fits_int(static_cast<long long>(groups) * d))
    return LKV_ERR_INVALID_ARG;
  if (dtype != LKV_BF16) return LKV_ERR_UNSUPPORTED;
  if (c_row_stride % 8 != 0 || d % 8 != 0 || !al16(c) || !al16(w)) return LKV_ERR_INVALID_ARG;
  // rows t of c; B = W[j] as [r, d] (MN-major).  With d a multiple of 64 the G matrices sit side by
  // side along the columns (one tile may span two groups: x[t] is [G, d] contiguous); else one
  // column block per group.
  GemmParams p = base_params(x);
  set_rows(p, static_cast<int>(n_rows), 1, 0);
  p.b_mn = 1;
  p.os1 = static_cast<long long>(groups) * d;
  if (d % 64 == 0) {
    set_cols(p, groups * d);
    p.nb = d;
    p.n_valid = groups * d;
  } else {
    set_cols(p, d);
    p.groups = groups;
    p.ocol = d;
    p.n_valid = d;
  }
  p.vec_ok = al16(x);
  const uint64_t cs = 2ull * static_cast<uint64_t>(c_row_stride);
  CUtensorMap ma, mb;
  if (!make_tmap_bf16_3d(&ma, c, r, n_rows, 1, cs, cs * static_cast<uint64_t>(n_rows), 128, 1) ||
      !make_tmap_bf16_3d(&mb, w, d, r, groups, 2ull * d, 2ull * d * r, 64, 1))
    return LKV_ERR_INVALID_ARG;
  return launch(ma, mb, p, r, static_cast<cudaStream_t>(stream));
}

lkv_status lkv_output_projection(const void* o, const void* w_o, void* y, int n_tok, int k, int d_model,
                                 int out_dtype, lkv_stream_t stream) {
  if (!o || !w_o || !y || n_tok <= 0 || k <= 0 || d_model <= 0) return LKV_ERR_INVALID_ARG;
  if (out_dtype != LKV_BF16 && out_dtype != LKV_FP32) return LKV_ERR_INVALID_ARG;
  if (k % 8 != 0 || d_model % 8 != 0 || !al16(o) || !al16(w_o)) return LKV_ERR_INVALID_ARG;
  // rows t of o; B = W_O as [k, d_model] (MN-major)
  GemmParams p = base_params(y);
  set_rows(p, n_tok, 1, 0);
  set_cols(p, d_model);
  p.b_mn = 1;
  p.out_fp32 = out_dtype == LKV_FP32;
  p.n_valid = d_model;
  p.os1 = d_model;
  p.vec_ok = al16(y);
  const uint64_t os = 2ull * static_cast<uint64_t>(k);
  CUtensorMap ma, mb;
  if (!make_tmap_bf16_3d(&ma, o, k, n_tok, 1, os, os * static_cast<uint64_t>(n_tok), 128, 1) ||
      !make_tmap_bf16_3d(&mb, w_o, d_model, k, 1, 2ull * d_model, 2ull * d_model * k, 64, 1))
    return LKV_ERR_INVALID_ARG;
  return launch(ma, mb, p, k, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
