// Projections either side of the decode path (GQLA explainer, section 2 "Methodology"):
//   absorbed path:  q_abs[t, h, :] = W_UK[j(h)] q[t, h, :]       (the query in latent space)
//                   out[t, h, :]   = W_UV[j(h)]^T o_lat[t, h, :]  (the output back in head space)
//   GQA path:       X[t, j, :]     = c_KV[t, :] W[j]              (expanded K_j or V_j of the cache)
// with j(h) = h / (h_q / G), and the output projection that follows attention,
//                   y[t, :]        = o[t, :] W_O                  (o = the heads' outputs side by side)
// which, with the heads split across GPUs along the group axis, gives each GPU a partial y to be summed
// (GQLA explainer, section 2, GQA path: tensor parallelism along the group axis).  These are plain GEMMs (bf16 operands, fp32 accumulation, bf16
// result), run by cuBLAS.  cuBLAS is opened at the first projection call (dlopen), so the decode path
// and the rest of the library never depend on it; each device gets one cuBLAS handle, created at its
// first projection call (cuBLAS allocates its own workspace then).
#include <cstdint>
#include <cstring>
#include <dlfcn.h>
#include <mutex>
#include <cublas_v2.h>
#include <cuda_runtime.h>

#include "../../include/lkv.h"

namespace {

// The C entry points used (32-bit sizes, 64-bit batch strides).
typedef cublasStatus_t (*CreateFn)(cublasHandle_t*);
typedef cublasStatus_t (*SetStreamFn)(cublasHandle_t, cudaStream_t);
typedef cublasStatus_t (*GemmFn)(cublasHandle_t, cublasOperation_t, cublasOperation_t, int, int, int, const void*,
                                 const void*, cudaDataType, int, long long, const void*, cudaDataType, int, long long,
                                 const void*, void*, cudaDataType, int, long long, int, cublasComputeType_t,
                                 cublasGemmAlgo_t);
struct CublasApi {
  CreateFn create = nullptr;
  SetStreamFn set_stream = nullptr;
  GemmFn gemm = nullptr;
  bool ok = false;
};

const CublasApi& cublas_api() {
  static CublasApi api;
  static std::once_flag once;
  std::call_once(once, [] {
    void* h = dlopen("libcublas.so.12", RTLD_NOW | RTLD_GLOBAL);
    if (!h) h = dlopen("libcublas.so", RTLD_NOW | RTLD_GLOBAL);
    if (!h) return;
    api.create = reinterpret_cast<decltype(api.create)>(dlsym(h, "cublasCreate_v2"));
    api.set_stream = reinterpret_cast<decltype(api.set_stream)>(dlsym(h, "cublasSetStream_v2"));
    api.gemm = reinterpret_cast<decltype(api.gemm)>(dlsym(h, "cublasGemmStridedBatchedEx"));
    api.ok = api.create && api.set_stream && api.gemm;
  });
  return api;
}

constexpr int kMaxDevices = 64;

// Serialises the projection calls of all host threads: a device's one handle is re-bound to the
// caller's stream at every call, so the binding and the GEMMs it enqueues must not interleave with
// another thread's.  Only the enqueueing is serialised, not the GPU work.
std::mutex& proj_mutex() {
  static std::mutex mu;
  return mu;
}

// The cuBLAS handle of the current device, bound to `stream`.  Call with proj_mutex() held.
lkv_status handle_for(cudaStream_t stream, cublasHandle_t* out) {
  const CublasApi& api = cublas_api();
  if (!api.ok) return LKV_ERR_UNSUPPORTED;
  static cublasHandle_t handles[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LKV_ERR_CUDA;
  if (!handles[dev] && api.create(&handles[dev]) != CUBLAS_STATUS_SUCCESS) {
    handles[dev] = nullptr;
    return LKV_ERR_CUDA;
  }
  if (api.set_stream(handles[dev], stream) != CUBLAS_STATUS_SUCCESS) return LKV_ERR_CUDA;
  *out = handles[dev];
  return LKV_OK;
}

// One strided-batched GEMM of bf16 operands in cuBLAS's column-major terms: C = op(A) op(B), fp32
// accumulate, C in bf16 (or fp32 when c_fp32).
lkv_status gemm(cublasHandle_t h, cublasOperation_t ta, int m, int n, int k, const void* A, int lda, long long sA,
                const void* B, int ldb, long long sB, void* C, int ldc, long long sC, int batch, bool c_fp32 = false) {
  const float one = 1.f, zero = 0.f;
  const cublasStatus_t s = cublas_api().gemm(h, ta, CUBLAS_OP_N, m, n, k, &one, A, CUDA_R_16BF, lda, sA, B, CUDA_R_16BF,
                                             ldb, sB, &zero, C, c_fp32 ? CUDA_R_32F : CUDA_R_16BF, ldc, sC, batch,
                                             CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT);
  return s == CUBLAS_STATUS_SUCCESS ? LKV_OK : LKV_ERR_CUDA;
}

bool fits_int(long long v) { return v > 0 && v <= 0x7fffffffLL; }

}  // namespace

extern "C" {

lkv_status lkv_absorb_query(const void* q, const void* w_uk, void* q_abs, int n_tok, int h_q, int groups, int d_h,
                            int r, int dtype, lkv_stream_t stream) {
  if (!q || !w_uk || !q_abs || n_tok <= 0 || h_q <= 0 || groups <= 0 || d_h <= 0 || r <= 0 ||
      h_q % groups != 0 || !fits_int(static_cast<long long>(h_q) * r) || !fits_int(static_cast<long long>(h_q) * d_h))
    return LKV_ERR_INVALID_ARG;
  if (dtype != LKV_BF16) return LKV_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(proj_mutex());
  cublasHandle_t h;
  lkv_status st = handle_for(static_cast<cudaStream_t>(stream), &h);
  if (st != LKV_OK) return st;
  const int hpg = h_q / groups;
  const auto* qb = static_cast<const uint16_t*>(q);
  const auto* wb = static_cast<const uint16_t*>(w_uk);
  auto* ob = static_cast<uint16_t*>(q_abs);
  if (groups == 1 && fits_int(static_cast<long long>(n_tok) * h_q))  // one shared W: a single GEMM over every (t, h)
    return gemm(h, CUBLAS_OP_T, r, n_tok * h_q, d_h, wb, d_h, 0, qb, d_h, 0, ob, r, 0, 1);
  for (int j = 0; j < groups && st == LKV_OK; ++j) {
    // per head of group j: (q_abs_h)^T [r x n] = W [r x d_h] * (q_h)^T [d_h x n]
    st = gemm(h, CUBLAS_OP_T, r, n_tok, d_h, wb + static_cast<size_t>(j) * r * d_h, d_h, 0,
              qb + static_cast<size_t>(j) * hpg * d_h, h_q * d_h, d_h, ob + static_cast<size_t>(j) * hpg * r, h_q * r, r,
              hpg);
  }
  return st;
}

lkv_status lkv_unabsorb_output(const void* o_lat, const void* w_uv, void* out, int n_tok, int h_q, int groups, int r,
                               int d_v, int dtype, lkv_stream_t stream) {
  if (!o_lat || !w_uv || !out || n_tok <= 0 || h_q <= 0 || groups <= 0 || r <= 0 || d_v <= 0 ||
      h_q % groups != 0 || !fits_int(static_cast<long long>(h_q) * r) || !fits_int(static_cast<long long>(h_q) * d_v))
    return LKV_ERR_INVALID_ARG;
  if (dtype != LKV_BF16) return LKV_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(proj_mutex());
  cublasHandle_t h;
  lkv_status st = handle_for(static_cast<cudaStream_t>(stream), &h);
  if (st != LKV_OK) return st;
  const int hpg = h_q / groups;
  const auto* ob = static_cast<const uint16_t*>(o_lat);
  const auto* wb = static_cast<const uint16_t*>(w_uv);
  auto* yb = static_cast<uint16_t*>(out);
  if (groups == 1 && fits_int(static_cast<long long>(n_tok) * h_q))
    return gemm(h, CUBLAS_OP_N, d_v, n_tok * h_q, r, wb, d_v, 0, ob, r, 0, yb, d_v, 0, 1);
  for (int j = 0; j < groups && st == LKV_OK; ++j) {
    // per head of group j: (out_h)^T [d_v x n] = W^T [d_v x r] * (o_h)^T [r x n]
    st = gemm(h, CUBLAS_OP_N, d_v, n_tok, r, wb + static_cast<size_t>(j) * r * d_v, d_v, 0,
              ob + static_cast<size_t>(j) * hpg * r, h_q * r, r, yb + static_cast<size_t>(j) * hpg * d_v, h_q * d_v, d_v,
              hpg);
  }
  return st;
}

lkv_status lkv_expand_latent(const void* c, int64_t c_row_stride, const void* w, void* x, int64_t n_rows, int groups,
                             int r, int d, int dtype, lkv_stream_t stream) {
  if (!c || !w || !x || n_rows <= 0 || groups <= 0 || r <= 0 || d <= 0 || c_row_stride < r ||
      !fits_int(n_rows) || !fits_int(c_row_stride) || !fits_int(static_cast<long long>(groups) * d))
    return LKV_ERR_INVALID_ARG;
  if (dtype != LKV_BF16) return LKV_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(proj_mutex());
  cublasHandle_t h;
  const lkv_status st = handle_for(static_cast<cudaStream_t>(stream), &h);
  if (st != LKV_OK) return st;
  // per group j: (X_j)^T [d x T] = W_j^T [d x r] * c^T [r x T]
  return gemm(h, CUBLAS_OP_N, d, static_cast<int>(n_rows), r, w, d, static_cast<long long>(r) * d, c,
              static_cast<int>(c_row_stride), 0, x, groups * d, d, groups);
}

lkv_status lkv_output_projection(const void* o, const void* w_o, void* y, int n_tok, int k, int d_model,
                                 int out_dtype, lkv_stream_t stream) {
  if (!o || !w_o || !y || n_tok <= 0 || k <= 0 || d_model <= 0) return LKV_ERR_INVALID_ARG;
  if (out_dtype != LKV_BF16 && out_dtype != LKV_FP32) return LKV_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(proj_mutex());
  cublasHandle_t h;
  const lkv_status st = handle_for(static_cast<cudaStream_t>(stream), &h);
  if (st != LKV_OK) return st;
  // y^T [d_model x n] = W_O^T [d_model x k] * o^T [k x n]
  return gemm(h, CUBLAS_OP_N, d_model, n_tok, k, w_o, d_model, 0, o, k, 0, y, d_model, 0, 1, out_dtype == LKV_FP32);
}

}  // extern "C"
