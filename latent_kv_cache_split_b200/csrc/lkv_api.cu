// Host side of the C ABI declared in include/lkv.h: argument validation (no CUDA call on
// the error paths), work planning, TMA descriptor construction and kernel launches.
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/lkv.h"
#include "lkv_aux.cuh"
#include "lkv_decode_tc.cuh"
#include "lkv_decode_swap.cuh"
#include "lkv_decode_swap_wide.cuh"
#include "lkv_mla_pair.cuh"
#include "lkv_ptx.cuh"
#include "lkv_tma_host.h"

namespace {

using namespace lkv;

// Device error word: every kernel of this library records failures here (first one wins).
__device__ int g_lkv_error_word = 0;

constexpr int kMaxDevices = 64;

struct DeviceState {
  bool ready = false;
  int num_sms = 0;
  int* err = nullptr;  // device address of g_lkv_error_word
};
DeviceState g_dev[kMaxDevices];

unsigned long long wait_limit_ns() {
  static unsigned long long v = [] {
    const char* e = std::getenv("LKV_WAIT_LIMIT_NS");
    unsigned long long x = e ? std::strtoull(e, nullptr, 10) : 0ull;
    return x ? x : 1000000000ull;  // 1 s: legitimate waits last microseconds
  }();
  return v;
}

constexpr size_t tc_smem_bytes(int mode) {
  return mode == MODE_GQLA   ? ModeCfg<MODE_GQLA>::kSmemBytes
         : mode == MODE_GTA  ? ModeCfg<MODE_GTA>::kSmemBytes
         : mode == MODE_GTA8 ? ModeCfg<MODE_GTA8>::kSmemBytes
                             : ModeCfg<MODE_GLA>::kSmemBytes;
}

// Per-device one-time set-up: SM count, error-word address, kernel attributes.
lkv_status device_state(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LKV_ERR_CUDA;
  DeviceState& d = g_dev[dev];
  if (!d.ready) {
    if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return LKV_ERR_CUDA;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_lkv_error_word) != cudaSuccess) return LKV_ERR_CUDA;
    d.err = static_cast<int*>(p);
    if (cudaFuncSetAttribute(decode_tc_kernel<MODE_GQLA>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(tc_smem_bytes(MODE_GQLA))) != cudaSuccess ||
        cudaFuncSetAttribute(decode_tc_kernel<MODE_GLA>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(tc_smem_bytes(MODE_GLA))) != cudaSuccess ||
        cudaFuncSetAttribute(decode_tc_kernel<MODE_GTA>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(tc_smem_bytes(MODE_GTA))) != cudaSuccess ||
        cudaFuncSetAttribute(decode_tc_kernel<MODE_GTA8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(tc_smem_bytes(MODE_GTA8))) != cudaSuccess ||
        cudaFuncSetAttribute(mla_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kPairSmemBytes)) != cudaSuccess ||
        cudaFuncSetAttribute(decode_swap_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(swap_smem_bytes(false))) != cudaSuccess ||
        cudaFuncSetAttribute(decode_swap_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(swap_smem_bytes(true))) != cudaSuccess ||
        cudaFuncSetAttribute(decode_swap_wide_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(WideCfg::kSmemBytes)) != cudaSuccess)
      return LKV_ERR_CUDA;
    d.ready = true;
  }
  *out = &d;
  return LKV_OK;
}

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool al4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
inline size_t up256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

int plan_ranges(int kind, int batch, int s_q, int groups, int num_sms) {
  if (batch <= 0 || s_q <= 0 || groups <= 0 || num_sms <= 0) return -1;
  const long long units = static_cast<long long>(batch) * (kind == 0 ? s_q : groups);
  const int pmax = kind == 0 ? num_sms / 2 : num_sms;
  if (pmax <= 0) return -1;
  // Grouped units run in lockstep (lkv_sched.cuh): G ranges per block of request tiles, as many
  // blocks as fit on the SMs.
  if (kind != 0 && groups >= 4) return groups * (num_sms / groups >= 1 ? num_sms / groups : 1);
  // One range per unit when the units alone nearly fill the machine: equal lengths then need
  // no split at all.  Otherwise one range per CTA (pair), cutting long units across SMs.
  if (units <= pmax && 4 * units >= 3LL * pmax) return static_cast<int>(units);
  return pmax;
}

struct WsLayout {
  size_t seg, lse, o, total;
};
WsLayout ws_layout(int P, int rmax, int dv_total) {
  WsLayout w;
  w.seg = 0;
  w.lse = up256(static_cast<size_t>(2 * P) * sizeof(int));
  w.o = w.lse + up256(static_cast<size_t>(2 * P) * rmax * sizeof(float));
  w.total = w.o + up256(static_cast<size_t>(2 * P) * rmax * dv_total * sizeof(float));
  return w;
}

lkv_status launch_err(cudaError_t e) {
  if (e == cudaSuccess) return LKV_OK;
  cudaGetLastError();  // a launch error is not sticky; clear it for the caller
  return LKV_ERR_CUDA;
}

// Merge the partial outputs of units split across ranges (units handled whole are left alone).
lkv_status launch_combine(const TcParams& p, int units_per_req, int per_query_units, cudaStream_t stream) {
  CombineParams c;
  c.seg_info = p.seg_info;
  c.part_lse = p.part_lse;
  c.part_o = p.part_o;
  c.P = p.P;
  c.rmax = p.rmax;
  c.dv_total = p.dv_total;
  c.R = p.R;
  c.per_query_units = per_query_units;
  c.units_per_req = units_per_req;
  c.s_q = p.s_q;
  c.h_q = p.h_q;
  c.hpg = p.hpg;
  c.out = p.out;
  c.lse = p.lse;
  // a programmatic dependent of the decode kernel: its launch overlaps the decode's run, and its
  // blocks wait (griddepcontrol.wait) for the decode's completion before reading the partials
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.B * units_per_req, (p.R + kCombineWarps - 1) / kCombineWarps);
  cfg.blockDim = dim3(kCombineWarps * 32);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return launch_err(cudaLaunchKernelEx(&cfg, combine_kernel, c));
}

// GLA units of at most 64 rows run the keys-in-M kernel (lkv_decode_swap_wide.cuh).
inline bool gla_keys_in_m(int mode, int R) { return mode == MODE_GLA && R <= kWideMaxRows; }

struct TcLaunch {
  int mode;
  CUtensorMap map_a, map_r, map_v;
  TcParams p;
  int units_per_req;
  int per_query_units;
};

// Grouped decode (one CTA per range), then the split combine.  GQLA and GTA units of at most 32
// rows and GLA units of at most 64 run with the keys in the MMA's M dimension (lkv_decode_swap.cuh,
// lkv_decode_swap_wide.cuh); the rest row-major.
lkv_status run_tc(TcLaunch& L, const DeviceState& d, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(L.p.P);
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = tc_smem_bytes(L.mode);
  cfg.stream = stream;
  cudaError_t e;
  const bool swap = (L.mode == MODE_GQLA || L.mode == MODE_GTA) && L.p.R <= kSwapMaxRows;
  if (gla_keys_in_m(L.mode, L.p.R)) {
    cfg.blockDim = dim3(kSwapThreads);
    cfg.dynamicSmemBytes = WideCfg::kSmemBytes;
    e = cudaLaunchKernelEx(&cfg, decode_swap_wide_kernel, L.map_a, L.map_r, L.p);
  } else if (swap) {
    cfg.blockDim = dim3(kSwapThreads);
    cfg.dynamicSmemBytes = swap_smem_bytes(L.mode == MODE_GTA);
    if (L.mode == MODE_GTA)
      e = cudaLaunchKernelEx(&cfg, decode_swap_kernel<true>, L.map_a, L.map_r, L.map_v, L.p);
    else
      e = cudaLaunchKernelEx(&cfg, decode_swap_kernel<false>, L.map_a, L.map_r, L.map_v, L.p);
  } else if (L.mode == MODE_GQLA) {
    e = cudaLaunchKernelEx(&cfg, decode_tc_kernel<MODE_GQLA>, L.map_a, L.map_r, L.map_v, L.p);
  } else if (L.mode == MODE_GTA) {
    e = cudaLaunchKernelEx(&cfg, decode_tc_kernel<MODE_GTA>, L.map_a, L.map_r, L.map_v, L.p);
  } else if (L.mode == MODE_GTA8) {
    e = cudaLaunchKernelEx(&cfg, decode_tc_kernel<MODE_GTA8>, L.map_a, L.map_r, L.map_v, L.p);
  } else {
    e = cudaLaunchKernelEx(&cfg, decode_tc_kernel<MODE_GLA>, L.map_a, L.map_r, L.map_v, L.p);
  }
  if (e != cudaSuccess) return launch_err(e);
  return launch_combine(L.p, L.units_per_req, L.per_query_units, stream);
}

// MLA absorbed decode on CTA pairs sharing one MMA (lkv_mla_pair.cuh), then the split combine.
lkv_status run_pair(const TcParams& p, const CUtensorMap (&maps)[5], cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * p.P);
  cfg.blockDim = dim3(kPairThreads);
  cfg.dynamicSmemBytes = kPairSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, mla_pair_kernel, maps[0], maps[1], maps[2], maps[3], maps[4], p);
  if (e != cudaSuccess) return launch_err(e);
  return launch_combine(p, p.s_q, 1, stream);
}

lkv_status run_simt(SimtParams& s, cudaStream_t stream) {
  const long long grid = static_cast<long long>(s.B) * s.s_q * s.h_q;
  if (grid > 0x7fffffffLL) return LKV_ERR_UNSUPPORTED;
  decode_simt_fp32_kernel<<<static_cast<unsigned>(grid), kSimtThreads, 0, stream>>>(s);
  return launch_err(cudaGetLastError());
}

// Checks shared by the three decode forms.
lkv_status common_checks(const void* q, const void* qr, const int32_t* cu, const void* out,
                         const float* lse, int batch, int s_q, int h_q, int groups, int d_rope,
                         int64_t cache_rows, int dtype, float scale) {
  if (!q || !qr || !cu || !out || !lse) return LKV_ERR_INVALID_ARG;
  if (batch <= 0 || h_q <= 0 || groups <= 0 || d_rope <= 0 || cache_rows <= 0)
    return LKV_ERR_INVALID_ARG;
  if (s_q != 1 && s_q != 2) return LKV_ERR_UNSUPPORTED;
  if (h_q % groups) return LKV_ERR_INVALID_ARG;
  if (dtype != LKV_BF16 && dtype != LKV_FP32) return LKV_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return LKV_ERR_INVALID_ARG;
  if (cache_rows >= (1LL << 31)) return LKV_ERR_UNSUPPORTED;
  if (static_cast<long long>(batch) * s_q * h_q >= (1LL << 31)) return LKV_ERR_UNSUPPORTED;
  return LKV_OK;
}

}  // namespace

// Device address of the error word of the current device, for the kernels of the other translation
// units (which cannot name the __device__ variable); sets the device up on first use.
lkv_status lkv_internal_error_word(int** err) {
  DeviceState* d;
  const lkv_status st = device_state(&d);
  if (st == LKV_OK) *err = d->err;
  return st;
}
// The same, with the device's SM count and the bounded-wait limit of the kernels.
lkv_status lkv_internal_device_info(int** err, int* num_sms, unsigned long long* wait_ns) {
  DeviceState* d;
  const lkv_status st = device_state(&d);
  if (st == LKV_OK) {
    *err = d->err;
    *num_sms = d->num_sms;
    *wait_ns = wait_limit_ns();
  }
  return st;
}

extern "C" {

int lkv_version(void) { return 100; }

const char* lkv_status_string(int s) {
  switch (s) {
    case LKV_OK: return "ok";
    case LKV_ERR_INVALID_ARG: return "invalid argument";
    case LKV_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case LKV_ERR_WORKSPACE: return "workspace missing or too small";
    case LKV_ERR_CUDA: return "CUDA runtime error";
    case LKV_ERR_DEVICE: return "device-side failure recorded";
    default: return "unknown status";
  }
}

int lkv_plan_ranges(int kind, int batch, int s_q, int groups, int num_sms) {
  if (kind == 3) kind = 1;  // GTA is partitioned like GQLA
  if (kind == 4) kind = 2;  // GLA with 128-key tiles: the same ranges
  if (kind < 0 || kind > 2) return -1;
  return plan_ranges(kind, batch, s_q, kind == 0 ? 1 : groups, num_sms);
}

static_assert(WideCfg::kTile == ModeCfg<MODE_GQLA>::kTile, "kind 4 describes the keys-in-M GLA tiles");

int lkv_plan_segments(int kind, const int32_t* cu_seqlens_host, int batch, int s_q, int groups,
                      int num_ranges, int32_t* out, int max_out) {
  if (kind == 3) kind = 1;
  // kind 4: GLA units of at most 64 rows, which the keys-in-M kernel walks in 128-key tiles
  const int tile = kind == 0 ? kPairTile
                 : (kind == 1 || kind == 4) ? ModeCfg<MODE_GQLA>::kTile
                                            : ModeCfg<MODE_GLA>::kTile;
  if (kind == 4) kind = 2;
  if (kind < 0 || kind > 2 || !cu_seqlens_host || batch <= 0 || s_q <= 0 || num_ranges <= 0 ||
      (kind != 0 && groups <= 0) || max_out < 0 || (max_out > 0 && !out))
    return -1;
  SchedArgs a;
  a.cu = cu_seqlens_host;
  a.B = batch;
  a.s_q = s_q;
  a.units_per_req = kind == 0 ? s_q : groups;
  a.per_query_units = kind == 0 ? 1 : 0;
  a.P = num_ranges;
  a.tile = tile;
  const bool lockstep = lockstep_groups(a);
  const SchedArgs ar = request_space(a);
  int n = 0;
  for (int p = 0; p < num_ranges; ++p) {
    SegCursor c = locate_range_host(ar, lockstep ? p / groups : p);
    Segment sg;
    while (c.next(ar, sg)) {
      if (lockstep) {
        sg.k = p % groups;
        sg.unit_id = sg.b * groups + sg.k;
      }
      if (n < max_out) {
        int32_t* r = out + 8 * n;
        r[0] = p;
        r[1] = sg.b;
        r[2] = sg.k;
        r[3] = sg.tile_lo;
        r[4] = sg.tile_hi;
        r[5] = sg.complete;
        r[6] = sg.slot;
        r[7] = sg.unit_id;
      }
      ++n;
    }
  }
  return n;
}

size_t lkv_mla_decode_workspace_size(int batch, int s_q, int h_q, int r_kv, int num_sms) {
  const int P = plan_ranges(0, batch, s_q, 1, num_sms);
  if (P <= 0 || h_q <= 0 || r_kv <= 0) return 0;
  return ws_layout(P, h_q, r_kv).total;
}

size_t lkv_group_decode_workspace_size(int kind, int batch, int s_q, int h_q, int groups, int d_v,
                                       int num_sms) {
  if (kind == 3) kind = 1;
  if (kind == 4) kind = 2;
  if (kind != 1 && kind != 2) return 0;
  const int P = plan_ranges(kind, batch, s_q, groups, num_sms);
  if (P <= 0 || h_q <= 0 || groups <= 0 || h_q % groups || d_v <= 0) return 0;
  return ws_layout(P, s_q * (h_q / groups), d_v).total;
}

lkv_status lkv_mla_absorbed_decode(const void* q_nope_abs, const void* q_rope, const void* ckv,
                                   int64_t ckv_row_stride, const void* kpe,
                                   int64_t kpe_row_stride, int64_t cache_rows,
                                   const int32_t* cu_seqlens, int batch, int s_q, int h_q,
                                   int r_kv, int d_rope, float scale, int dtype, void* out,
                                   float* lse, void* workspace, size_t workspace_bytes,
                                   lkv_stream_t stream) {
  lkv_status st = common_checks(q_nope_abs, q_rope, cu_seqlens, out, lse, batch, s_q, h_q, 1,
                                d_rope, cache_rows, dtype, scale);
  if (st != LKV_OK) return st;
  if (!ckv || !kpe || r_kv <= 0) return LKV_ERR_INVALID_ARG;
  if (ckv_row_stride < r_kv || kpe_row_stride < d_rope) return LKV_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == LKV_FP32) {
    if (r_kv + d_rope > kSimtMaxQ || r_kv > kSimtMaxV) return LKV_ERR_UNSUPPORTED;
    if (!al4(q_nope_abs) || !al4(q_rope) || !al4(ckv) || !al4(kpe) || !al4(out))
      return LKV_ERR_INVALID_ARG;
    DeviceState* d;
    if ((st = device_state(&d)) != LKV_OK) return st;
    SimtParams sp;
    sp.q_nope = static_cast<const float*>(q_nope_abs);
    sp.q_rope = static_cast<const float*>(q_rope);
    sp.k = static_cast<const float*>(ckv);
    sp.v = static_cast<const float*>(ckv);
    sp.kr = static_cast<const float*>(kpe);
    sp.k_rs = ckv_row_stride;
    sp.k_gs = 0;
    sp.v_rs = ckv_row_stride;
    sp.v_gs = 0;
    sp.kr_rs = kpe_row_stride;
    sp.cu = cu_seqlens;
    sp.B = batch;
    sp.s_q = s_q;
    sp.h_q = h_q;
    sp.G = 1;
    sp.dk = r_kv;
    sp.dv = r_kv;
    sp.dr = d_rope;
    sp.scale = scale;
    sp.out = static_cast<float*>(out);
    sp.lse = lse;
    sp.err = d->err;
    return run_simt(sp, s);
  }
  if (h_q != 128 || r_kv != 512 || d_rope != 64) return LKV_ERR_UNSUPPORTED;
  if (!al16(q_nope_abs) || !al16(q_rope) || !al16(ckv) || !al16(kpe) || !al16(out) ||
      (ckv_row_stride * 2) % 16 || (kpe_row_stride * 2) % 16)
    return LKV_ERR_INVALID_ARG;
  DeviceState* d;
  if ((st = device_state(&d)) != LKV_OK) return st;
  const int P = plan_ranges(0, batch, s_q, 1, d->num_sms);
  const WsLayout w = ws_layout(P, h_q, r_kv);
  if (!workspace || !al16(workspace) || workspace_bytes < w.total) return LKV_ERR_WORKSPACE;
  // Query rows (b, i, h) as 2-D [batch * s_q * h_q, width] maps in 64-row boxes (one CTA's heads);
  // cache rows in 128-row boxes for QK (one CTA's keys of a 256-key tile) and PV (a value chunk).
  const uint64_t qrows = static_cast<uint64_t>(batch) * s_q * h_q;
  CUtensorMap maps[5];
  if (!make_tmap_bf16(&maps[0], q_nope_abs, r_kv, qrows, static_cast<uint64_t>(r_kv) * 2, 64, 64) ||
      !make_tmap_bf16(&maps[1], q_rope, d_rope, qrows, static_cast<uint64_t>(d_rope) * 2, 64, 64) ||
      !make_tmap_bf16(&maps[2], ckv, r_kv, cache_rows, ckv_row_stride * 2, 64, 128) ||
      !make_tmap_bf16(&maps[3], kpe, d_rope, cache_rows, kpe_row_stride * 2, 64, 128) ||
      !make_tmap_bf16(&maps[4], ckv, r_kv, cache_rows, ckv_row_stride * 2, 64, 128))
    return LKV_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  TcParams p;
  p.q_nope = static_cast<const __nv_bfloat16*>(q_nope_abs);
  p.q_rope = static_cast<const __nv_bfloat16*>(q_rope);
  p.dq = r_kv;
  p.cu = cu_seqlens;
  p.B = batch;
  p.s_q = s_q;
  p.h_q = h_q;
  p.G = 1;
  p.hpg = h_q;
  p.R = h_q;
  p.sl2 = scale * 1.4426950408889634f;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.dv_total = r_kv;
  p.seg_info = reinterpret_cast<int*>(ws + w.seg);
  p.part_lse = reinterpret_cast<float*>(ws + w.lse);
  p.part_o = reinterpret_cast<float*>(ws + w.o);
  p.rmax = h_q;
  p.P = P;
  p.err = d->err;
  p.wait_limit_ns = wait_limit_ns();
  return run_pair(p, maps, s);
}

lkv_status lkv_gqla_group_decode(const void* q, const void* q_rope, const void* k,
                                 int64_t k_row_stride, const void* v, int64_t v_row_stride,
                                 const void* kpe, int64_t kpe_row_stride, int64_t cache_rows,
                                 const int32_t* cu_seqlens, int batch, int s_q, int h_q, int g,
                                 int d_h, int d_rope, float scale, int dtype, void* out,
                                 float* lse, void* workspace, size_t workspace_bytes,
                                 lkv_stream_t stream) {
  lkv_status st = common_checks(q, q_rope, cu_seqlens, out, lse, batch, s_q, h_q, g, d_rope,
                                cache_rows, dtype, scale);
  if (st != LKV_OK) return st;
  if (!k || !v || !kpe || d_h <= 0) return LKV_ERR_INVALID_ARG;
  if (k_row_stride < static_cast<int64_t>(g) * d_h || v_row_stride < static_cast<int64_t>(g) * d_h ||
      kpe_row_stride < d_rope)
    return LKV_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == LKV_FP32) {
    if (d_h + d_rope > kSimtMaxQ || d_h > kSimtMaxV) return LKV_ERR_UNSUPPORTED;
    if (!al4(q) || !al4(q_rope) || !al4(k) || !al4(v) || !al4(kpe) || !al4(out))
      return LKV_ERR_INVALID_ARG;
    DeviceState* d;
    if ((st = device_state(&d)) != LKV_OK) return st;
    SimtParams sp;
    sp.q_nope = static_cast<const float*>(q);
    sp.q_rope = static_cast<const float*>(q_rope);
    sp.k = static_cast<const float*>(k);
    sp.v = static_cast<const float*>(v);
    sp.kr = static_cast<const float*>(kpe);
    sp.k_rs = k_row_stride;
    sp.k_gs = d_h;
    sp.v_rs = v_row_stride;
    sp.v_gs = d_h;
    sp.kr_rs = kpe_row_stride;
    sp.cu = cu_seqlens;
    sp.B = batch;
    sp.s_q = s_q;
    sp.h_q = h_q;
    sp.G = g;
    sp.dk = d_h;
    sp.dv = d_h;
    sp.dr = d_rope;
    sp.scale = scale;
    sp.out = static_cast<float*>(out);
    sp.lse = lse;
    sp.err = d->err;
    return run_simt(sp, s);
  }
  const int hpg = h_q / g;
  if (d_h != 128 || d_rope != 64 || hpg > 64 || s_q * hpg > 128) return LKV_ERR_UNSUPPORTED;
  if (!al16(q) || !al16(q_rope) || !al16(k) || !al16(v) || !al16(kpe) || !al16(out) ||
      (k_row_stride * 2) % 16 || (v_row_stride * 2) % 16 || (kpe_row_stride * 2) % 16)
    return LKV_ERR_INVALID_ARG;
  DeviceState* d;
  if ((st = device_state(&d)) != LKV_OK) return st;
  const int P = plan_ranges(1, batch, s_q, g, d->num_sms);
  const int R = s_q * hpg;
  const WsLayout w = ws_layout(P, R, d_h);
  if (!workspace || !al16(workspace) || workspace_bytes < w.total) return LKV_ERR_WORKSPACE;
  TcLaunch L;
  L.mode = MODE_GQLA;
  const uint64_t width = static_cast<uint64_t>(g) * d_h;
  constexpr int TN = ModeCfg<MODE_GQLA>::kTile;
  if (!make_tmap_bf16(&L.map_a, k, width, cache_rows, k_row_stride * 2, 64, TN) ||
      !make_tmap_bf16(&L.map_v, v, width, cache_rows, v_row_stride * 2, 64, TN) ||
      !make_tmap_bf16(&L.map_r, kpe, d_rope, cache_rows, kpe_row_stride * 2, 64, TN))
    return LKV_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  TcParams& p = L.p;
  p.q_nope = static_cast<const __nv_bfloat16*>(q);
  p.q_rope = static_cast<const __nv_bfloat16*>(q_rope);
  p.dq = d_h;
  p.cu = cu_seqlens;
  p.B = batch;
  p.s_q = s_q;
  p.h_q = h_q;
  p.G = g;
  p.hpg = hpg;
  p.R = R;
  p.sl2 = scale * 1.4426950408889634f;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.dv_total = d_h;
  p.seg_info = reinterpret_cast<int*>(ws + w.seg);
  p.part_lse = reinterpret_cast<float*>(ws + w.lse);
  p.part_o = reinterpret_cast<float*>(ws + w.o);
  p.rmax = R;
  p.P = P;
  p.err = d->err;
  p.wait_limit_ns = wait_limit_ns();
  L.units_per_req = g;
  L.per_query_units = 0;
  return run_tc(L, *d, s);
}

lkv_status lkv_gta_group_decode(const void* q, const void* q_rope, const void* kv,
                                int64_t kv_row_stride, const void* kpe, int64_t kpe_row_stride,
                                int64_t cache_rows, const int32_t* cu_seqlens, int batch, int s_q,
                                int h_q, int g, int d_h, int d_rope, float scale, int dtype,
                                void* out, float* lse, void* workspace, size_t workspace_bytes,
                                lkv_stream_t stream) {
  // fp32 storage: the CUDA-core kernel of the GQA path with its value pointer on the tied rows
  if (dtype == LKV_FP32)
    return lkv_gqla_group_decode(q, q_rope, kv, kv_row_stride, kv, kv_row_stride, kpe, kpe_row_stride,
                                 cache_rows, cu_seqlens, batch, s_q, h_q, g, d_h, d_rope, scale, dtype,
                                 out, lse, workspace, workspace_bytes, stream);
  lkv_status st = common_checks(q, q_rope, cu_seqlens, out, lse, batch, s_q, h_q, g, d_rope,
                                cache_rows, dtype, scale);
  if (st != LKV_OK) return st;
  if (!kv || !kpe || d_h <= 0) return LKV_ERR_INVALID_ARG;
  if (kv_row_stride < static_cast<int64_t>(g) * d_h || kpe_row_stride < d_rope) return LKV_ERR_INVALID_ARG;
  const int hpg = h_q / g;
  if (d_h != 128 || d_rope != 64 || hpg > 64 || s_q * hpg > 128) return LKV_ERR_UNSUPPORTED;
  if (!al16(q) || !al16(q_rope) || !al16(kv) || !al16(kpe) || !al16(out) || (kv_row_stride * 2) % 16 ||
      (kpe_row_stride * 2) % 16)
    return LKV_ERR_INVALID_ARG;
  DeviceState* d;
  if ((st = device_state(&d)) != LKV_OK) return st;
  const int P = plan_ranges(1, batch, s_q, g, d->num_sms);
  const int R = s_q * hpg;
  const WsLayout w = ws_layout(P, R, d_h);
  if (!workspace || !al16(workspace) || workspace_bytes < w.total) return LKV_ERR_WORKSPACE;
  // One ring of whole tiles: the tied state is read once into shared memory and serves as the
  // key (with the RoPE key) and as the value.
  TcLaunch L;
  L.mode = MODE_GTA;
  constexpr int TN = ModeCfg<MODE_GTA>::kTile;
  if (!make_tmap_bf16(&L.map_a, kv, static_cast<uint64_t>(g) * d_h, cache_rows, kv_row_stride * 2, 64, TN) ||
      !make_tmap_bf16(&L.map_r, kpe, d_rope, cache_rows, kpe_row_stride * 2, 64, TN))
    return LKV_ERR_CUDA;
  L.map_v = L.map_a;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  TcParams& p = L.p;
  p.q_nope = static_cast<const __nv_bfloat16*>(q);
  p.q_rope = static_cast<const __nv_bfloat16*>(q_rope);
  p.dq = d_h;
  p.cu = cu_seqlens;
  p.B = batch;
  p.s_q = s_q;
  p.h_q = h_q;
  p.G = g;
  p.hpg = hpg;
  p.R = R;
  p.sl2 = scale * 1.4426950408889634f;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.dv_total = d_h;
  p.seg_info = reinterpret_cast<int*>(ws + w.seg);
  p.part_lse = reinterpret_cast<float*>(ws + w.lse);
  p.part_o = reinterpret_cast<float*>(ws + w.o);
  p.rmax = R;
  p.P = P;
  p.err = d->err;
  p.wait_limit_ns = wait_limit_ns();
  L.units_per_req = g;
  L.per_query_units = 0;
  return run_tc(L, *d, reinterpret_cast<cudaStream_t>(stream));
}

lkv_status lkv_gta_group_decode_fp8(const void* q, const void* q_rope, const void* cache,
                                    int64_t cache_row_stride_bytes, int64_t cache_rows,
                                    const int32_t* cu_seqlens, int batch, int s_q, int h_q, int g, int d_h,
                                    int d_rope, float scale, void* out, float* lse, void* workspace,
                                    size_t workspace_bytes, lkv_stream_t stream) {
  lkv_status st = common_checks(q, q_rope, cu_seqlens, out, lse, batch, s_q, h_q, g, d_rope,
                                cache_rows, LKV_BF16, scale);
  if (st != LKV_OK) return st;
  if (!cache || d_h <= 0) return LKV_ERR_INVALID_ARG;
  const int hpg = h_q / g;
  const int r = g * d_h;
  // the converter warps are the softmax slots a unit of <= 64 rows leaves free
  if (d_h != 128 || d_rope != 64 || r > 1024 || s_q * hpg > 64) return LKV_ERR_UNSUPPORTED;
  const size_t row_bytes = lkv_fp8_cache_row_bytes(r, d_rope);
  if (row_bytes == 0 || cache_row_stride_bytes < static_cast<int64_t>(row_bytes) || cache_row_stride_bytes % 16 ||
      !al16(q) || !al16(q_rope) || !al16(cache) || !al16(out))
    return LKV_ERR_INVALID_ARG;
  DeviceState* d;
  if ((st = device_state(&d)) != LKV_OK) return st;
  const int P = plan_ranges(1, batch, s_q, g, d->num_sms);
  const int R = s_q * hpg;
  const WsLayout w = ws_layout(P, R, d_h);
  if (!workspace || !al16(workspace) || workspace_bytes < w.total) return LKV_ERR_WORKSPACE;
  // The row's fields as three maps: the codes (bytes, 128 per group), the scale with its 12 zero
  // bytes (fp32, 4 per row) and the RoPE key (bf16, 64 per row), 128-row boxes.
  TcLaunch L;
  L.mode = MODE_GTA8;
  constexpr int TN = ModeCfg<MODE_GTA8>::kTile;
  const uint64_t rs = static_cast<uint64_t>(cache_row_stride_bytes);
  if (!make_tmap_2d(&L.map_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, cache, row_bytes, cache_rows, rs, 128, TN,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&L.map_v, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, cache, row_bytes / 4, cache_rows, rs, 4, TN,
                    CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tmap_bf16(&L.map_r, cache, row_bytes / 2, cache_rows, rs, 64, TN))
    return LKV_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  TcParams& p = L.p;
  p.q_nope = static_cast<const __nv_bfloat16*>(q);
  p.q_rope = static_cast<const __nv_bfloat16*>(q_rope);
  p.dq = d_h;
  p.cu = cu_seqlens;
  p.B = batch;
  p.s_q = s_q;
  p.h_q = h_q;
  p.G = g;
  p.hpg = hpg;
  p.R = R;
  p.sl2 = scale * 1.4426950408889634f;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.dv_total = d_h;
  p.seg_info = reinterpret_cast<int*>(ws + w.seg);
  p.part_lse = reinterpret_cast<float*>(ws + w.lse);
  p.part_o = reinterpret_cast<float*>(ws + w.o);
  p.rmax = R;
  p.P = P;
  p.err = d->err;
  p.wait_limit_ns = wait_limit_ns();
  p.fp8_scale_col = r / 4;
  p.fp8_rope_col = (r + 16) / 2;
  L.units_per_req = g;
  L.per_query_units = 0;
  return run_tc(L, *d, reinterpret_cast<cudaStream_t>(stream));
}

lkv_status lkv_gla_group_decode(const void* q, const void* q_rope, const void* clat,
                                int64_t clat_row_stride, const void* kpe, int64_t kpe_row_stride,
                                int64_t cache_rows, const int32_t* cu_seqlens, int batch, int s_q,
                                int h_q, int n_lat, int r_g, int d_rope, float scale, int dtype,
                                void* out, float* lse, void* workspace, size_t workspace_bytes,
                                lkv_stream_t stream) {
  lkv_status st = common_checks(q, q_rope, cu_seqlens, out, lse, batch, s_q, h_q, n_lat, d_rope,
                                cache_rows, dtype, scale);
  if (st != LKV_OK) return st;
  if (!clat || !kpe || r_g <= 0) return LKV_ERR_INVALID_ARG;
  if (clat_row_stride < static_cast<int64_t>(n_lat) * r_g || kpe_row_stride < d_rope)
    return LKV_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == LKV_FP32) {
    if (r_g + d_rope > kSimtMaxQ || r_g > kSimtMaxV) return LKV_ERR_UNSUPPORTED;
    if (!al4(q) || !al4(q_rope) || !al4(clat) || !al4(kpe) || !al4(out)) return LKV_ERR_INVALID_ARG;
    DeviceState* d;
    if ((st = device_state(&d)) != LKV_OK) return st;
    SimtParams sp;
    sp.q_nope = static_cast<const float*>(q);
    sp.q_rope = static_cast<const float*>(q_rope);
    sp.k = static_cast<const float*>(clat);
    sp.v = static_cast<const float*>(clat);
    sp.kr = static_cast<const float*>(kpe);
    sp.k_rs = clat_row_stride;
    sp.k_gs = r_g;
    sp.v_rs = clat_row_stride;
    sp.v_gs = r_g;
    sp.kr_rs = kpe_row_stride;
    sp.cu = cu_seqlens;
    sp.B = batch;
    sp.s_q = s_q;
    sp.h_q = h_q;
    sp.G = n_lat;
    sp.dk = r_g;
    sp.dv = r_g;
    sp.dr = d_rope;
    sp.scale = scale;
    sp.out = static_cast<float*>(out);
    sp.lse = lse;
    sp.err = d->err;
    return run_simt(sp, s);
  }
  const int hpg = h_q / n_lat;
  if (r_g != 256 || d_rope != 64 || s_q * hpg > 128) return LKV_ERR_UNSUPPORTED;
  if (!al16(q) || !al16(q_rope) || !al16(clat) || !al16(kpe) || !al16(out) ||
      (clat_row_stride * 2) % 16 || (kpe_row_stride * 2) % 16)
    return LKV_ERR_INVALID_ARG;
  DeviceState* d;
  if ((st = device_state(&d)) != LKV_OK) return st;
  const int P = plan_ranges(2, batch, s_q, n_lat, d->num_sms);
  const int R = s_q * hpg;
  const WsLayout w = ws_layout(P, R, r_g);
  if (!workspace || !al16(workspace) || workspace_bytes < w.total) return LKV_ERR_WORKSPACE;
  TcLaunch L;
  L.mode = MODE_GLA;
  // 128-key tiles for the keys-in-M kernel, 64-key tiles for the rows-in-M one
  const uint32_t box_rows = gla_keys_in_m(MODE_GLA, R) ? WideCfg::kTile : ModeCfg<MODE_GLA>::kTile;
  if (!make_tmap_bf16(&L.map_a, clat, static_cast<uint64_t>(n_lat) * r_g, cache_rows,
                      clat_row_stride * 2, 64, box_rows) ||
      !make_tmap_bf16(&L.map_r, kpe, d_rope, cache_rows, kpe_row_stride * 2, 64, box_rows))
    return LKV_ERR_CUDA;
  L.map_v = L.map_a;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  TcParams& p = L.p;
  p.q_nope = static_cast<const __nv_bfloat16*>(q);
  p.q_rope = static_cast<const __nv_bfloat16*>(q_rope);
  p.dq = r_g;
  p.cu = cu_seqlens;
  p.B = batch;
  p.s_q = s_q;
  p.h_q = h_q;
  p.G = n_lat;
  p.hpg = hpg;
  p.R = R;
  p.sl2 = scale * 1.4426950408889634f;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.dv_total = r_g;
  p.seg_info = reinterpret_cast<int*>(ws + w.seg);
  p.part_lse = reinterpret_cast<float*>(ws + w.lse);
  p.part_o = reinterpret_cast<float*>(ws + w.o);
  p.rmax = R;
  p.P = P;
  p.err = d->err;
  p.wait_limit_ns = wait_limit_ns();
  L.units_per_req = n_lat;
  L.per_query_units = 0;
  return run_tc(L, *d, s);
}

// Fixed scratch for lkv_gqla_group_decode_noalloc.  In host code this name is only a
// stand-in for the device symbol; its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_lkv_static_scratch[LKV_STATIC_SCRATCH_BYTES];
static void* g_static_scratch_addr[kMaxDevices] = {};

lkv_status lkv_gqla_group_decode_noalloc(const void* q, const void* q_rope, const void* k,
                                         int64_t k_row_stride, const void* v,
                                         int64_t v_row_stride, const void* kpe,
                                         int64_t kpe_row_stride, int64_t cache_rows,
                                         const int32_t* cu_seqlens, int batch, int s_q, int h_q,
                                         int g, int d_h, int d_rope, float scale, int dtype,
                                         void* out, float* lse, lkv_stream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LKV_ERR_CUDA;
  if (!g_static_scratch_addr[dev]) {
    // once per device, with that device current (first call; before any stream capture)
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_lkv_static_scratch) != cudaSuccess || !ptr) return LKV_ERR_CUDA;
    g_static_scratch_addr[dev] = ptr;
  }
  // the regular entry point rejects a shape whose workspace exceeds the array (LKV_ERR_WORKSPACE)
  return lkv_gqla_group_decode(q, q_rope, k, k_row_stride, v, v_row_stride, kpe, kpe_row_stride,
                               cache_rows, cu_seqlens, batch, s_q, h_q, g, d_h, d_rope, scale, dtype,
                               out, lse, g_static_scratch_addr[dev], LKV_STATIC_SCRATCH_BYTES, stream);
}

lkv_status lkv_latent_cache_append(const void* new_rows, int64_t new_row_stride_bytes,
                                   void* cache, int64_t cache_row_stride_bytes,
                                   int64_t cache_rows, int64_t row_bytes,
                                   const int32_t* cu_seqlens, int batch, int s_q,
                                   lkv_stream_t stream) {
  if (!new_rows || !cache || !cu_seqlens) return LKV_ERR_INVALID_ARG;
  if (batch <= 0 || s_q <= 0 || cache_rows <= 0 || row_bytes <= 0) return LKV_ERR_INVALID_ARG;
  if (row_bytes % 16 || new_row_stride_bytes % 16 || cache_row_stride_bytes % 16 ||
      !al16(new_rows) || !al16(cache))
    return LKV_ERR_INVALID_ARG;
  if (new_row_stride_bytes < row_bytes || cache_row_stride_bytes < row_bytes)
    return LKV_ERR_INVALID_ARG;
  if (static_cast<long long>(batch) * s_q * 32 >= (1LL << 31)) return LKV_ERR_UNSUPPORTED;
  DeviceState* d;
  lkv_status st = device_state(&d);
  if (st != LKV_OK) return st;
  const long long threads = static_cast<long long>(batch) * s_q * 32;
  const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
  append_kernel<<<blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(new_rows), new_row_stride_bytes, static_cast<uint8_t*>(cache),
      cache_row_stride_bytes, cache_rows, row_bytes, cu_seqlens, batch, s_q, d->err);
  return launch_err(cudaGetLastError());
}

lkv_status lkv_merge_partials(const float* o_parts, const float* lse_parts, int n_parts,
                              int64_t rows, int d_v, int out_dtype, void* out, float* lse,
                              lkv_stream_t stream) {
  if (!o_parts || !lse_parts || !out) return LKV_ERR_INVALID_ARG;
  if (n_parts <= 0 || rows <= 0 || d_v <= 0 || d_v % 4 || d_v > 1024) return LKV_ERR_INVALID_ARG;
  if (out_dtype != LKV_BF16 && out_dtype != LKV_FP32) return LKV_ERR_INVALID_ARG;
  if (!al16(o_parts) || !al16(out) || !al4(lse_parts)) return LKV_ERR_INVALID_ARG;
  if (rows * 32 / 128 + 1 >= (1LL << 31)) return LKV_ERR_UNSUPPORTED;
  DeviceState* d;
  lkv_status st = device_state(&d);
  if (st != LKV_OK) return st;
  const unsigned blocks = static_cast<unsigned>((rows * 32 + 127) / 128);
  merge_kernel<<<blocks, 128, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      o_parts, lse_parts, n_parts, rows, d_v, out_dtype == LKV_FP32, out, lse);
  return launch_err(cudaGetLastError());
}

lkv_status lkv_check_device(int32_t* code_out, int clear) {
  DeviceState* d;
  lkv_status st = device_state(&d);
  if (st != LKV_OK) return st;
  if (cudaDeviceSynchronize() != cudaSuccess) return LKV_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_lkv_error_word, sizeof(int)) != cudaSuccess) return LKV_ERR_CUDA;
  if (code_out) *code_out = v;
  if (clear && v) {
    const int z = 0;
    if (cudaMemcpyToSymbol(g_lkv_error_word, &z, sizeof(int)) != cudaSuccess) return LKV_ERR_CUDA;
  }
  return v ? LKV_ERR_DEVICE : LKV_OK;
}

lkv_status lkv_check_stream(lkv_stream_t stream, int32_t* code_out, int clear) {
  DeviceState* d;
  lkv_status st = device_state(&d);
  if (st != LKV_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int v = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return LKV_ERR_CUDA;
  if (cudaMemcpyFromSymbolAsync(&v, g_lkv_error_word, sizeof(int), 0, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return LKV_ERR_CUDA;
  if (code_out) *code_out = v;
  if (clear && v) {
    static const int z = 0;
    if (cudaMemcpyToSymbolAsync(g_lkv_error_word, &z, sizeof(int), 0, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
      return LKV_ERR_CUDA;
  }
  return v ? LKV_ERR_DEVICE : LKV_OK;
}

lkv_status lkv_selftest_wait_timeout(uint64_t limit_ns, lkv_stream_t stream) {
  if (limit_ns == 0 || limit_ns > 10000000000ull) return LKV_ERR_INVALID_ARG;
  DeviceState* d;
  lkv_status st = device_state(&d);
  if (st != LKV_OK) return st;
  selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(d->err, limit_ns);
  return launch_err(cudaGetLastError());
}

}  // extern "C"
