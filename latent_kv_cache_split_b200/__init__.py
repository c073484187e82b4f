"""Python binding for liblkv.so: B200 (sm_100a) decode attention over a latent / grouped KV cache.

Argument marshalling only: every function passes device pointers, sizes and the current
CUDA stream to the C ABI (include/lkv.h) and raises on a non-OK status.  PyTorch supplies
device memory and streams; all computation runs in the library's CUDA kernels.  There is no
fallback: if liblkv.so is missing the import fails.

Functions (same names as the C entry points without the ``lkv_`` prefix):
    mla_absorbed_decode, gqla_group_decode, gla_group_decode, latent_cache_append,
    merge_partials, check_device, selftest_wait_timeout, plan_ranges,
    mla_decode_workspace_size, group_decode_workspace_size,
    absorb_query, unabsorb_output, expand_latent (the projections either side of the path),
    gta_group_decode, fp8_cache_row_bytes, quantize_latent_fp8, latent_cache_append_fp8
    (and fp8_cache_fields: views of the fields of FP8 cache rows)
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblkv.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python latent_kv_cache_split_b200/build.py` "
        "(the CUDA library is required; there is no fallback)")
_lib = ctypes.CDLL(LIB_PATH)

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_DEVICE = range(6)
BF16, FP32 = 0, 1
KIND_MLA, KIND_GQLA, KIND_GLA, KIND_GTA = 0, 1, 2, 3
SITE_SELFTEST, SITE_BAD_LENGTH, SITE_BAD_ROW, SITE_WAIT_BASE = 1, 2, 3, 100   # device error word

_vp, _i64, _i32, _f32, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_size_t


def _sig(name, res, *args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = list(args)
    return f


_lib_version = _sig("lkv_version", _i32)
_status_string = _sig("lkv_status_string", ctypes.c_char_p, _i32)
_plan = _sig("lkv_plan_ranges", _i32, _i32, _i32, _i32, _i32, _i32)
_mla_ws = _sig("lkv_mla_decode_workspace_size", _sz, _i32, _i32, _i32, _i32, _i32)
_grp_ws = _sig("lkv_group_decode_workspace_size", _sz, _i32, _i32, _i32, _i32, _i32, _i32, _i32)
_mla = _sig("lkv_mla_absorbed_decode", _i32, _vp, _vp, _vp, _i64, _vp, _i64, _i64, _vp,
            _i32, _i32, _i32, _i32, _i32, _f32, _i32, _vp, _vp, _vp, _sz, _vp)
_gqla = _sig("lkv_gqla_group_decode", _i32, _vp, _vp, _vp, _i64, _vp, _i64, _vp, _i64, _i64,
             _vp, _i32, _i32, _i32, _i32, _i32, _i32, _f32, _i32, _vp, _vp, _vp, _sz, _vp)
_gla = _sig("lkv_gla_group_decode", _i32, _vp, _vp, _vp, _i64, _vp, _i64, _i64, _vp,
            _i32, _i32, _i32, _i32, _i32, _i32, _f32, _i32, _vp, _vp, _vp, _sz, _vp)
_gta = _sig("lkv_gta_group_decode", _i32, _vp, _vp, _vp, _i64, _vp, _i64, _i64, _vp,
            _i32, _i32, _i32, _i32, _i32, _i32, _f32, _i32, _vp, _vp, _vp, _sz, _vp)
_gta_fp8 = _sig("lkv_gta_group_decode_fp8", _i32, _vp, _vp, _vp, _i64, _i64, _vp, _i32, _i32, _i32, _i32,
                _i32, _i32, _f32, _vp, _vp, _vp, _sz, _vp)
_fp8_row_bytes = _sig("lkv_fp8_cache_row_bytes", _sz, _i32, _i32)
_quant_fp8 = _sig("lkv_quantize_latent_fp8", _i32, _vp, _i64, _vp, _i64, _i64, _i32, _i32, _vp)
_append_fp8 = _sig("lkv_latent_cache_append_fp8", _i32, _vp, _i64, _vp, _i64, _i64, _i32, _i32, _vp,
                   _i32, _i32, _vp)
_gqla_noalloc = _sig("lkv_gqla_group_decode_noalloc", _i32, _vp, _vp, _vp, _i64, _vp, _i64, _vp, _i64,
                     _i64, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _f32, _i32, _vp, _vp, _vp)
_append = _sig("lkv_latent_cache_append", _i32, _vp, _i64, _vp, _i64, _i64, _i64, _vp,
               _i32, _i32, _vp)
_merge = _sig("lkv_merge_partials", _i32, _vp, _vp, _i32, _i64, _i32, _i32, _vp, _vp, _vp)
_check = _sig("lkv_check_device", _i32, ctypes.POINTER(ctypes.c_int32), _i32)
_check_stream = _sig("lkv_check_stream", _i32, _vp, ctypes.POINTER(ctypes.c_int32), _i32)
_selftest = _sig("lkv_selftest_wait_timeout", _i32, ctypes.c_uint64, _vp)
_segments = _sig("lkv_plan_segments", _i32, _i32, _vp, _i32, _i32, _i32, _i32, _vp, _i32)
_absorb = _sig("lkv_absorb_query", _i32, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _vp)
_unabsorb = _sig("lkv_unabsorb_output", _i32, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _vp)
_expand = _sig("lkv_expand_latent", _i32, _vp, _i64, _vp, _vp, _i64, _i32, _i32, _i32, _i32, _vp)
_oproj = _sig("lkv_output_projection", _i32, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp)

EXPORTED = ["lkv_version", "lkv_status_string", "lkv_plan_ranges", "lkv_mla_decode_workspace_size",
            "lkv_group_decode_workspace_size", "lkv_mla_absorbed_decode", "lkv_gqla_group_decode",
            "lkv_gla_group_decode", "lkv_latent_cache_append", "lkv_merge_partials",
            "lkv_check_device", "lkv_selftest_wait_timeout", "lkv_plan_segments",
            "lkv_gqla_group_decode_noalloc", "lkv_absorb_query", "lkv_unabsorb_output",
            "lkv_expand_latent", "lkv_gta_group_decode", "lkv_fp8_cache_row_bytes",
            "lkv_quantize_latent_fp8", "lkv_latent_cache_append_fp8", "lkv_output_projection",
            "lkv_check_stream", "lkv_gta_group_decode_fp8"]


class LkvError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_status_string(status).decode()} (status {status})")


def _ck(status: int, where: str):
    if status != OK:
        raise LkvError(status, where)


def version() -> int:
    return _lib_version()


def status_string(status: int) -> str:
    return _status_string(status).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("query / output tensors must be contiguous")


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _same_dtype(ref: torch.Tensor, **named):
    """The C ABI takes one storage type per call: every tensor given must have ref's dtype."""
    for name, t in named.items():
        if t is not None and t.dtype != ref.dtype:
            raise TypeError(f"{name} is {t.dtype}, expected {ref.dtype}")


def _row_stride(t: torch.Tensor) -> int:
    if t.dim() < 2 or t.stride(-1) != 1:
        raise ValueError("cache rows must have unit stride in the last dimension")
    return t.stride(0)


def _num_sms(device) -> int:
    return torch.cuda.get_device_properties(device).multi_processor_count


def plan_ranges(kind: int, batch: int, s_q: int, groups: int, num_sms: int) -> int:
    return _plan(kind, batch, s_q, groups, num_sms)


def plan_segments(kind: int, cu_seqlens_host, s_q: int, groups: int, num_ranges: int):
    """Segments the decode kernels process, as a list of
    (range, request, unit, tile_lo, tile_hi, complete, slot, unit_id) tuples (host only)."""
    import numpy as np
    cu = np.ascontiguousarray(np.asarray(cu_seqlens_host, dtype=np.int32))
    B = cu.size - 1
    n = _segments(kind, cu.ctypes.data, B, s_q, groups, num_ranges, None, 0)
    if n < 0:
        raise ValueError("bad partition arguments")
    buf = np.zeros((max(n, 1), 8), dtype=np.int32)
    _segments(kind, cu.ctypes.data, B, s_q, groups, num_ranges, buf.ctypes.data, n)
    return [tuple(int(x) for x in row) for row in buf[:n]]


def mla_decode_workspace_size(batch, s_q, h_q, r_kv, num_sms) -> int:
    return _mla_ws(batch, s_q, h_q, r_kv, num_sms)


def group_decode_workspace_size(kind, batch, s_q, h_q, groups, d_v, num_sms) -> int:
    return _grp_ws(kind, batch, s_q, h_q, groups, d_v, num_sms)


def _alloc_ws(nbytes, device):
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def mla_absorbed_decode(q_nope_abs, q_rope, ckv, kpe, cu_seqlens, scale, out=None, lse=None,
                        workspace=None, stream=None):
    """MLA absorbed decode.  q_nope_abs [B,s_q,h_q,r_kv], q_rope [B,s_q,h_q,d_R], ckv [rows,r_kv]
    and kpe [rows,d_R] (unit inner stride; may be column slices of one interleaved cache),
    cu_seqlens int32 [B+1].  Returns (out [B,s_q,h_q,r_kv], lse [B,s_q,h_q] fp32)."""
    B, s_q, h_q, r_kv = q_nope_abs.shape
    d_r = q_rope.shape[-1]
    dev = q_nope_abs.device
    _same_dtype(q_nope_abs, q_rope=q_rope, ckv=ckv, kpe=kpe, out=out)
    if out is None:
        out = torch.empty((B, s_q, h_q, r_kv), dtype=q_nope_abs.dtype, device=dev)
    if lse is None:
        lse = torch.empty((B, s_q, h_q), dtype=torch.float32, device=dev)
    if workspace is None and q_nope_abs.dtype == torch.bfloat16:
        workspace = _alloc_ws(mla_decode_workspace_size(B, s_q, h_q, r_kv, _num_sms(dev)), dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _contig(q_nope_abs, q_rope, out, lse)
    _ck(_mla(_ptr(q_nope_abs), _ptr(q_rope), _ptr(ckv), _row_stride(ckv),
             _ptr(kpe), _row_stride(kpe), ckv.shape[0], _ptr(cu_seqlens), B, s_q, h_q, r_kv, d_r,
             float(scale), _dtype_code(q_nope_abs), _ptr(out), _ptr(lse), _ptr(workspace),
             ws_bytes, _stream(stream)), "lkv_mla_absorbed_decode")
    return out, lse


def gqla_group_decode(q, q_rope, k, v, kpe, cu_seqlens, scale, out=None, lse=None,
                      workspace=None, stream=None):
    """GQLA grouped decode.  q [B,s_q,h_q,d_h], k / v [rows,g,d_h], kpe [rows,d_R]."""
    _same_dtype(q, q_rope=q_rope, k=k, v=v, kpe=kpe, out=out)
    B, s_q, h_q, d_h = q.shape
    g = k.shape[1]
    d_r = q_rope.shape[-1]
    dev = q.device
    if out is None:
        out = torch.empty((B, s_q, h_q, d_h), dtype=q.dtype, device=dev)
    if lse is None:
        lse = torch.empty((B, s_q, h_q), dtype=torch.float32, device=dev)
    if workspace is None and q.dtype == torch.bfloat16:
        workspace = _alloc_ws(group_decode_workspace_size(KIND_GQLA, B, s_q, h_q, g, d_h, _num_sms(dev)), dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if k.stride(2) != 1 or k.stride(1) != d_h or v.stride(2) != 1 or v.stride(1) != d_h:
        raise ValueError("k and v must be [rows, g, d_h] with contiguous groups")
    _contig(q, q_rope, out, lse)
    _ck(_gqla(_ptr(q), _ptr(q_rope), _ptr(k), k.stride(0), _ptr(v),
              v.stride(0), _ptr(kpe), _row_stride(kpe), k.shape[0], _ptr(cu_seqlens), B, s_q, h_q,
              g, d_h, d_r, float(scale), _dtype_code(q), _ptr(out), _ptr(lse), _ptr(workspace),
              ws_bytes, _stream(stream)), "lkv_gqla_group_decode")
    return out, lse


def gqla_group_decode_noalloc(q, q_rope, k, v, kpe, cu_seqlens, scale, out=None, lse=None,
                              stream=None):
    """GQLA grouped decode without a workspace: for callers that cannot allocate device memory
    per call.  The library keeps one fixed 8 MiB device scratch array per GPU instead; calls
    that overlap on the GPU race on it, and shapes needing more scratch raise LkvError
    (ERR_WORKSPACE).  `out` and `lse` are still caller-provided (allocated here if omitted)."""
    _same_dtype(q, q_rope=q_rope, k=k, v=v, kpe=kpe, out=out)
    B, s_q, h_q, d_h = q.shape
    g = k.shape[1]
    d_r = q_rope.shape[-1]
    dev = q.device
    if out is None:
        out = torch.empty((B, s_q, h_q, d_h), dtype=q.dtype, device=dev)
    if lse is None:
        lse = torch.empty((B, s_q, h_q), dtype=torch.float32, device=dev)
    if k.stride(2) != 1 or k.stride(1) != d_h or v.stride(2) != 1 or v.stride(1) != d_h:
        raise ValueError("k and v must be [rows, g, d_h] with contiguous groups")
    _contig(q, q_rope, out, lse)
    _ck(_gqla_noalloc(_ptr(q), _ptr(q_rope), _ptr(k), k.stride(0), _ptr(v), v.stride(0), _ptr(kpe),
                      _row_stride(kpe), k.shape[0], _ptr(cu_seqlens), B, s_q, h_q, g, d_h, d_r,
                      float(scale), _dtype_code(q), _ptr(out), _ptr(lse), _stream(stream)),
        "lkv_gqla_group_decode_noalloc")
    return out, lse


def gta_group_decode(q, q_rope, kv, kpe, g, cu_seqlens, scale, out=None, lse=None,
                     workspace=None, stream=None):
    """GTA decode over tied groups.  q [B,s_q,h_q,d_h], kv [rows, g*d_h] (tied key/value state
    of each group, contiguous within a row), kpe [rows,d_R]."""
    _same_dtype(q, q_rope=q_rope, kv=kv, kpe=kpe, out=out)
    B, s_q, h_q, d_h = q.shape
    d_r = q_rope.shape[-1]
    dev = q.device
    if kv.shape[-1] != g * d_h:
        raise ValueError("kv rows must hold g * d_h elements")
    if out is None:
        out = torch.empty((B, s_q, h_q, d_h), dtype=q.dtype, device=dev)
    if lse is None:
        lse = torch.empty((B, s_q, h_q), dtype=torch.float32, device=dev)
    if workspace is None and q.dtype == torch.bfloat16:
        workspace = _alloc_ws(group_decode_workspace_size(KIND_GTA, B, s_q, h_q, g, d_h, _num_sms(dev)), dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _contig(q, q_rope, out, lse)
    _ck(_gta(_ptr(q), _ptr(q_rope), _ptr(kv), _row_stride(kv), _ptr(kpe), _row_stride(kpe), kv.shape[0],
             _ptr(cu_seqlens), B, s_q, h_q, g, d_h, d_r, float(scale), _dtype_code(q), _ptr(out), _ptr(lse),
             _ptr(workspace), ws_bytes, _stream(stream)), "lkv_gta_group_decode")
    return out, lse


def gta_group_decode_fp8(q, q_rope, cache, g, cu_seqlens, scale, out=None, lse=None, workspace=None,
                         stream=None):
    """GTA decode over FP8 cache rows.  q [B,s_q,h_q,d_h] and q_rope [B,s_q,h_q,d_R] bf16; cache
    [rows, >= fp8_cache_row_bytes(g*d_h, d_R)] uint8 (row stride a multiple of 16 bytes)."""
    _same_dtype(q, q_rope=q_rope, out=out)
    if q.dtype != torch.bfloat16 or cache.dtype != torch.uint8:
        raise TypeError("gta_group_decode_fp8 takes a bf16 query and a uint8 FP8 cache")
    B, s_q, h_q, d_h = q.shape
    d_r = q_rope.shape[-1]
    dev = q.device
    if cache.stride(-1) != 1:
        raise ValueError("cache rows must be contiguous")
    if out is None:
        out = torch.empty((B, s_q, h_q, d_h), dtype=q.dtype, device=dev)
    if lse is None:
        lse = torch.empty((B, s_q, h_q), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = _alloc_ws(group_decode_workspace_size(KIND_GTA, B, s_q, h_q, g, d_h, _num_sms(dev)), dev)
    ws_bytes = workspace.numel() * workspace.element_size()
    _contig(q, q_rope, out, lse)
    _ck(_gta_fp8(_ptr(q), _ptr(q_rope), _ptr(cache), cache.stride(0), cache.shape[0], _ptr(cu_seqlens), B, s_q,
                 h_q, g, d_h, d_r, float(scale), _ptr(out), _ptr(lse), _ptr(workspace), ws_bytes, _stream(stream)),
        "lkv_gta_group_decode_fp8")
    return out, lse


def gla_group_decode(q, q_rope, clat, kpe, n_lat, cu_seqlens, scale, out=None, lse=None,
                     workspace=None, stream=None):
    """GLA decode.  q [B,s_q,h_q,r_g], clat [rows, n_lat*r_g], kpe [rows,d_R]."""
    _same_dtype(q, q_rope=q_rope, clat=clat, kpe=kpe, out=out)
    B, s_q, h_q, r_g = q.shape
    d_r = q_rope.shape[-1]
    dev = q.device
    if out is None:
        out = torch.empty((B, s_q, h_q, r_g), dtype=q.dtype, device=dev)
    if lse is None:
        lse = torch.empty((B, s_q, h_q), dtype=torch.float32, device=dev)
    if workspace is None and q.dtype == torch.bfloat16:
        workspace = _alloc_ws(group_decode_workspace_size(KIND_GLA, B, s_q, h_q, n_lat, r_g, _num_sms(dev)), dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _contig(q, q_rope, out, lse)
    _ck(_gla(_ptr(q), _ptr(q_rope), _ptr(clat), _row_stride(clat),
             _ptr(kpe), _row_stride(kpe), clat.shape[0], _ptr(cu_seqlens), B, s_q, h_q, n_lat, r_g,
             d_r, float(scale), _dtype_code(q), _ptr(out), _ptr(lse), _ptr(workspace), ws_bytes,
             _stream(stream)), "lkv_gla_group_decode")
    return out, lse


def latent_cache_append(new_rows, cache, cu_seqlens, s_q, stream=None):
    """Write row b*s_q+i of new_rows [B*s_q, ...] to cache row cu[b] + L_b - s_q + i."""
    n = new_rows.shape[0]
    B = cu_seqlens.numel() - 1
    if n != B * s_q:
        raise ValueError("new_rows must hold batch * s_q rows")
    row_bytes = new_rows[0].numel() * new_rows.element_size()
    _ck(_append(_ptr(new_rows), new_rows.stride(0) * new_rows.element_size(), _ptr(cache),
                cache.stride(0) * cache.element_size(), cache.shape[0], row_bytes,
                _ptr(cu_seqlens), B, s_q, _stream(stream)), "lkv_latent_cache_append")
    return cache


def fp8_cache_row_bytes(r: int, d_rope: int) -> int:
    """Bytes of one FP8 cache row (e4m3 latent, fp32 scale + pad, bf16 RoPE key); 0 if unsupported."""
    return _fp8_row_bytes(r, d_rope)


def fp8_cache_fields(cache, r: int, d_rope: int):
    """Views of the fields of FP8 cache rows cache [rows, >= row_bytes] uint8 (row stride and
    start 16-byte aligned): (codes uint8 [rows, r], scales fp32 [rows], k_rope bf16 [rows, d_rope])."""
    rb = fp8_cache_row_bytes(r, d_rope)
    if (rb == 0 or cache.dtype != torch.uint8 or cache.dim() != 2 or cache.shape[1] < rb
            or cache.stride(1) != 1 or cache.stride(0) % 16 or cache.storage_offset() % 16):
        raise ValueError("cache must be [rows, >= row_bytes] uint8 rows on 16-byte boundaries")
    rows, rs, off = cache.shape[0], cache.stride(0), cache.storage_offset()
    st = cache.untyped_storage()
    scales = torch.empty(0, dtype=torch.float32, device=cache.device).set_(st, (off + r) // 4, (rows,), (rs // 4,))
    kpe = torch.empty(0, dtype=torch.bfloat16, device=cache.device).set_(st, (off + r + 16) // 2, (rows, d_rope),
                                                                           (rs // 2, 1))
    return cache[:, :r], scales, kpe


def quantize_latent_fp8(rows, r: int, cache=None, stream=None):
    """Quantise bf16 rows [n, >= r + d_rope] (latent then RoPE key) into FP8 cache rows, row i to
    row i.  Returns the cache [n, row_bytes] uint8 (allocated if not given)."""
    if rows.dtype != torch.bfloat16 or (cache is not None and cache.dtype != torch.uint8):
        raise TypeError("quantize_latent_fp8 takes bf16 rows and a uint8 cache")
    n, width = rows.shape
    d_rope = width - r
    rb = fp8_cache_row_bytes(r, d_rope)
    if rb == 0:
        raise ValueError("unsupported r / d_rope for the FP8 cache")
    if cache is None:
        cache = torch.empty((n, rb), dtype=torch.uint8, device=rows.device)
    _ck(_quant_fp8(_ptr(rows), _row_stride(rows), _ptr(cache), cache.stride(0), n, r, d_rope,
                   _stream(stream)), "lkv_quantize_latent_fp8")
    return cache


def latent_cache_append_fp8(new_rows, cache, cu_seqlens, s_q, r: int, stream=None):
    """Quantise row b*s_q+i of the bf16 new_rows [B*s_q, r + d_rope] into FP8 cache row
    cu[b] + L_b - s_q + i of cache [rows, row_bytes] uint8."""
    if new_rows.dtype != torch.bfloat16 or cache.dtype != torch.uint8:
        raise TypeError("latent_cache_append_fp8 takes bf16 rows and a uint8 cache")
    n, width = new_rows.shape
    B = cu_seqlens.numel() - 1
    if n != B * s_q:
        raise ValueError("new_rows must hold batch * s_q rows")
    _ck(_append_fp8(_ptr(new_rows), _row_stride(new_rows), _ptr(cache), cache.stride(0), cache.shape[0], r,
                    width - r, _ptr(cu_seqlens), B, s_q, _stream(stream)), "lkv_latent_cache_append_fp8")
    return cache


def merge_partials(o_parts, lse_parts, out_dtype=torch.bfloat16, out=None, lse=None, stream=None):
    """Merge [n_parts, rows, d_v] fp32 partial outputs with their [n_parts, rows] lse."""
    n, rows, d_v = o_parts.shape
    dev = o_parts.device
    if out is None:
        out = torch.empty((rows, d_v), dtype=out_dtype, device=dev)
    if lse is None:
        lse = torch.empty((rows,), dtype=torch.float32, device=dev)
    _contig(o_parts, lse_parts, out, lse)
    _ck(_merge(_ptr(o_parts), _ptr(lse_parts), n, rows, d_v,
               _dtype_code(out), _ptr(out), _ptr(lse), _stream(stream)), "lkv_merge_partials")
    return out, lse


def check_device(clear: bool = True) -> int:
    """Synchronise and return the device error word (0 = no failure recorded)."""
    code = ctypes.c_int32(0)
    st = _check(ctypes.byref(code), 1 if clear else 0)
    if st not in (OK, ERR_DEVICE):
        raise LkvError(st, "lkv_check_device")
    return code.value


def check_stream(stream=None, clear: bool = True) -> int:
    """Wait for the work queued on `stream` (not the whole device) and return the device error
    word (0 = no failure recorded)."""
    code = ctypes.c_int32(0)
    st = _check_stream(_stream(stream), ctypes.byref(code), 1 if clear else 0)
    if st not in (OK, ERR_DEVICE):
        raise LkvError(st, "lkv_check_stream")
    return code.value


def selftest_wait_timeout(limit_ns: int, stream=None):
    _ck(_selftest(int(limit_ns), _stream(stream)), "lkv_selftest_wait_timeout")


def absorb_query(q, w_uk, out=None, stream=None):
    """q_abs[..., h, :] = w_uk[j(h)] @ q[..., h, :].  q [..., h_q, d_h], w_uk [G, r, d_h] (bf16,
    contiguous) -> [..., h_q, r] bf16."""
    _same_dtype(q, w_uk=w_uk, out=out)
    G, r, d_h = w_uk.shape
    h_q = q.shape[-2]
    if q.shape[-1] != d_h:
        raise ValueError("q and w_uk disagree on d_h")
    n_tok = q.numel() // (h_q * d_h)
    if out is None:
        out = torch.empty(q.shape[:-1] + (r,), dtype=q.dtype, device=q.device)
    _contig(q, w_uk, out)
    _ck(_absorb(_ptr(q), _ptr(w_uk), _ptr(out), n_tok, h_q, G, d_h, r, _dtype_code(q), _stream(stream)),
        "lkv_absorb_query")
    return out


def unabsorb_output(o_lat, w_uv, out=None, stream=None):
    """out[..., h, :] = w_uv[j(h)]^T @ o_lat[..., h, :].  o_lat [..., h_q, r], w_uv [G, r, d_v]
    (bf16, contiguous) -> [..., h_q, d_v] bf16."""
    _same_dtype(o_lat, w_uv=w_uv, out=out)
    G, r, d_v = w_uv.shape
    h_q = o_lat.shape[-2]
    if o_lat.shape[-1] != r:
        raise ValueError("o_lat and w_uv disagree on r")
    n_tok = o_lat.numel() // (h_q * r)
    if out is None:
        out = torch.empty(o_lat.shape[:-1] + (d_v,), dtype=o_lat.dtype, device=o_lat.device)
    _contig(o_lat, w_uv, out)
    _ck(_unabsorb(_ptr(o_lat), _ptr(w_uv), _ptr(out), n_tok, h_q, G, r, d_v, _dtype_code(o_lat), _stream(stream)),
        "lkv_unabsorb_output")
    return out


def expand_latent(c, w, out=None, stream=None):
    """x[t, j, :] = c[t, :] @ w[j].  c [T, r] (unit inner stride; may be a column slice of the
    cache), w [G, r, d] contiguous (bf16) -> x [T, G, d] bf16."""
    _same_dtype(c, w=w, out=out)
    G, r, d = w.shape
    T = c.shape[0]
    if c.shape[1] != r:
        raise ValueError("c and w disagree on r")
    if out is None:
        out = torch.empty((T, G, d), dtype=c.dtype, device=c.device)
    _contig(w, out)
    _ck(_expand(_ptr(c), _row_stride(c), _ptr(w), _ptr(out), T, G, r, d, _dtype_code(c), _stream(stream)),
        "lkv_expand_latent")
    return out


def output_projection(o, w_o, out_dtype=torch.float32, out=None, stream=None):
    """y = o @ w_o.  o [n_tok, k] (or [n_tok, heads, d_v], flattened) bf16 contiguous, w_o [k, d_model]
    bf16 contiguous -> y [n_tok, d_model] in out_dtype (fp32 by default: a partial sum to reduce)."""
    n = o.shape[0]
    o2 = o.reshape(n, -1)
    k, d_model = w_o.shape
    if o2.shape[1] != k:
        raise ValueError("o and w_o disagree on k")
    if o2.dtype != torch.bfloat16 or w_o.dtype != torch.bfloat16:
        raise TypeError("output_projection takes bf16 operands")
    if out is None:
        out = torch.empty((n, d_model), dtype=out_dtype, device=o.device)
    _contig(o2, w_o, out)
    _ck(_oproj(_ptr(o2), _ptr(w_o), _ptr(out), n, k, d_model, _dtype_code(out), _stream(stream)),
        "lkv_output_projection")
    return out
