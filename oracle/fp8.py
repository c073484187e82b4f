"""FP8 (e4m3) latent cache: encoding, per-token quantisation and decode over the dequantised cache.

TEST INFRASTRUCTURE ONLY, like the rest of oracle/: the library never imports it.

What the pages fix and what is read into them:
* The serving comparison in the Grouped Latent Attention article (news page, section on the
  GLA-vs-MLA decoding test) runs DeepSeek-Coder-V2 in FP8; the pages give no cache format.
* Reading: the latent part of each cached token is stored as e4m3 codes with one fp32 scale per
  token, s_t = the smallest power of two with amax_t / s_t <= 448 (amax_t = max |c_KV[t, :]|), so
  that the largest entry lands in the top binade of e4m3 (224, 448]; the RoPE key stays bf16.
  Dequantised value = e4m3(code) * s_t.  A power of two (as in the OCP microscaling formats' shared
  scales) makes the dequantised value exact in bf16: a decode may dequantise into bf16 operands and
  still compute on exactly the values this oracle reads.
* e4m3 is the OCP 8-bit floating-point E4M3 format: 1 sign bit, 4 exponent bits with bias 7,
  3 mantissa bits; exponent field 0 holds subnormals m * 2^-9; fields 1..15 hold
  (1 + m/8) * 2^(e-7); the all-ones pattern S.1111.111 is NaN; there are no infinities, so the
  largest finite magnitude is 1.75 * 2^8 = 448.

Quantisation arithmetic (the same steps the CUDA kernel takes, so that the codes, which floating
point decides, come out identical): amax in fp32 (exact: a max of stored bf16 values), s the
power of two above (exact), y = x / s (exact: a power-of-two division), y clamped to [-448, 448]
(a no-op), code = y rounded to the nearest e4m3 value with ties to the even code.  A row whose
amax is 0 gets s = 0 and all codes 0.
"""
from __future__ import annotations

import numpy as np

__all__ = ["E4M3_MAX", "e4m3_decode", "e4m3_encode", "pow2_scale", "quantize_rows", "dequantize_rows",
           "mla_absorbed_decode_fp8", "gta_group_decode_fp8"]

E4M3_MAX = 448.0


def _decode_one(code: int) -> float:
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * m * 2.0 ** -9
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


# every code's value, straight from the field definitions
_TABLE = np.array([_decode_one(c) for c in range(256)], dtype=np.float64)


def e4m3_decode(codes) -> np.ndarray:
    """float64 value of each uint8 e4m3 code (NaN for the two NaN codes)."""
    return _TABLE[np.asarray(codes, dtype=np.uint8)]


# the non-negative finite values in code order 0x00 .. 0x7E (increasing with the code)
_POS = _TABLE[:0x7F]


def e4m3_encode(y) -> np.ndarray:
    """Nearest e4m3 code of each value (ties to the even code); |y| must be <= 448.

    The sign bit is the sign of y (so -0.0 and negative values that round to zero give 0x80)."""
    y = np.asarray(y, dtype=np.float64)
    a = np.abs(y)
    if np.any(~np.isfinite(a)) or np.any(a > E4M3_MAX):
        raise ValueError("e4m3_encode takes finite values with |y| <= 448")
    hi = np.searchsorted(_POS, a, side="left")          # first code whose value >= a
    hi = np.minimum(hi, 0x7E)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - _POS[lo]
    d_hi = _POS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    mag = np.where(pick_hi, hi, lo).astype(np.uint8)
    return np.where(np.signbit(y), mag | 0x80, mag).astype(np.uint8)


def pow2_scale(amax) -> np.ndarray:
    """Per-token scale: the smallest power of two s with amax / s <= 448 (0 where amax is 0).

    With amax = m * 2^E (m in [0.5, 1), numpy's frexp), amax <= 448 * 2^e = 0.875 * 2^(9 + e) holds
    for e = E - 9 when m <= 0.875 and first for e = E - 8 otherwise."""
    a = np.asarray(amax, dtype=np.float64)
    m, E = np.frexp(a)
    e = np.where(m <= 0.875, E - 9, E - 8)
    return np.where(a > 0, np.ldexp(1.0, e), 0.0).astype(np.float32)


def quantize_rows(x):
    """Per-row e4m3 quantisation of stored latent rows x [n, r] (bf16 or fp32 values).

    Returns (codes uint8 [n, r], scales float32 [n])."""
    x32 = np.asarray(x, dtype=np.float32)
    if x32.ndim != 2:
        raise ValueError("x must be [n, r]")
    amax = np.abs(x32).max(axis=1)                        # exact in fp32
    scales = pow2_scale(amax)
    codes = np.zeros(x32.shape, dtype=np.uint8)
    nz = scales > 0
    if np.any(nz):
        y = (x32[nz] / scales[nz, None]).astype(np.float32)   # exact: division by a power of two
        y = np.clip(y, -E4M3_MAX, E4M3_MAX)
        codes[nz] = e4m3_encode(y)
    return codes, scales


def dequantize_rows(codes, scales) -> np.ndarray:
    """float64 [n, r]: e4m3(code) * scale of the code's row."""
    return e4m3_decode(codes) * np.asarray(scales, dtype=np.float64)[:, None]


def mla_absorbed_decode_fp8(q_nope_abs, q_rope, codes, scales, kpe, cu_seqlens, scale, requests=None):
    """MLA absorbed decode over an FP8 latent cache: the plain absorbed-path attention over the
    dequantised latent (codes [T, r_kv], scales [T]) and the bf16 RoPE key kpe [T, d_R]."""
    from .attend import mla_absorbed_decode
    return mla_absorbed_decode(q_nope_abs, q_rope, dequantize_rows(codes, scales), kpe, cu_seqlens, scale,
                               requests=requests)


def gta_group_decode_fp8(q, q_rope, codes, scales, kpe, g, cu_seqlens, scale, requests=None):
    """GTA decode over FP8 rows: the tied states of the g groups are one latent-shaped row per token
    (codes [T, g*d_h] with one scale per token), dequantised and read as K_j = V_j of group j; the
    bf16 RoPE key kpe [T, d_R] is shared by all groups."""
    from .attend import gta_group_decode
    return gta_group_decode(q, q_rope, dequantize_rows(codes, scales), kpe, g, cu_seqlens, scale,
                            requests=requests)
