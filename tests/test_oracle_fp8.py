"""Pin the FP8 (e4m3) oracle: every code against torch's float8_e4m3fn conversion (an independent
library routine), closed-form values of the format, round-to-nearest-even ties, the error bound of a
3-bit mantissa, and the per-token power-of-two scale (its defining property and closed forms)."""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import fp8


def _torch_decode_all():
    return torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).float().double().numpy()


def test_decode_every_code_matches_library():
    ours = fp8.e4m3_decode(np.arange(256))
    lib = _torch_decode_all()
    nan = np.isnan(lib)
    assert np.array_equal(np.isnan(ours), nan)
    assert nan.sum() == 2
    np.testing.assert_array_equal(ours[~nan], lib[~nan])
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(lib[~nan]))


def test_decode_closed_forms():
    d = fp8.e4m3_decode
    assert d(0x7E) == 448.0 and d(0xFE) == -448.0          # 1.75 * 2^8, the largest finite
    assert d(0x01) == 2.0 ** -9                             # smallest subnormal
    assert d(0x07) == 7 * 2.0 ** -9                         # largest subnormal
    assert d(0x08) == 2.0 ** -6                             # smallest normal
    assert d(0x38) == 1.0 and d(0xB8) == -1.0               # exponent field 7 = bias
    assert d(0x3C) == 1.5
    assert math.isnan(d(0x7F)) and math.isnan(d(0xFF))


def test_encode_round_trips_every_finite_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    np.testing.assert_array_equal(fp8.e4m3_encode(fp8.e4m3_decode(codes)), codes)


def test_encode_matches_library_on_midpoints_and_random_values():
    pos = fp8.e4m3_decode(np.arange(0x7F))
    mids = (pos[:-1] + pos[1:]) / 2                          # every tie
    rng = np.random.default_rng(0)
    rand = np.concatenate([rng.uniform(-448, 448, 20000), rng.standard_normal(20000) * 1e-2,
                           rng.standard_normal(5000) * 1e-3])
    vals = np.concatenate([pos, mids, -mids, mids * (1 + 1e-6), mids * (1 - 1e-6), rand]).astype(np.float32)
    ours = fp8.e4m3_encode(vals)
    lib = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(ours, lib)


def test_ties_go_to_the_even_code():
    # 1.0625 lies halfway between 1.0 (0x38) and 1.125 (0x39): even code 0x38
    assert fp8.e4m3_encode([1.0625])[0] == 0x38
    # 1.1875 lies between 1.125 (0x39) and 1.25 (0x3A): even code 0x3A
    assert fp8.e4m3_encode([1.1875])[0] == 0x3A
    # 2^-10 lies between 0 and 2^-9: even code 0;  -2^-10 keeps the sign bit
    assert fp8.e4m3_encode([2.0 ** -10])[0] == 0x00
    assert fp8.e4m3_encode([-(2.0 ** -10)])[0] == 0x80
    with pytest.raises(ValueError):
        fp8.e4m3_encode([449.0])


def test_quantize_rows_scale_and_error_bound():
    rng = np.random.default_rng(1)
    x = torch.from_numpy(rng.standard_normal((64, 512)).astype(np.float32) / 24).bfloat16().float().numpy()
    x[3] *= 1e-30                                            # tiny row: scale still exact in fp32
    x[5] *= 2.0 ** 40
    codes, scales = fp8.quantize_rows(x)
    amax = np.abs(x).max(axis=1).astype(np.float64)
    s64 = scales.astype(np.float64)
    # the scale's defining property, checked directly: a power of two, the smallest one that
    # brings amax within 448
    m, _ = np.frexp(s64)
    assert (m == 0.5).all()
    assert (amax / s64 <= 448).all() and (amax / (s64 / 2) > 448).all()
    # the largest entry of every row lands in the top binade of e4m3, (224, 448]
    mag = codes & 0x7F
    assert ((mag.max(axis=1) >= 0x70) & (mag.max(axis=1) <= 0x7E)).all()
    deq = fp8.dequantize_rows(codes, scales)
    # 3 mantissa bits: half an ulp is 2^-4 relative for normals, 2^-10 * s absolute below 2^-6 * s
    bound = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * s64[:, None]) * (1 + 1e-6)
    assert (np.abs(deq - x) <= bound + 1e-300).all()
    # and the dequantised values are exact in bf16 (a power-of-two scale times a 4-bit significand)
    assert np.array_equal(torch.from_numpy(deq).bfloat16().double().numpy(), deq)


def test_pow2_scale_closed_forms():
    assert fp8.pow2_scale([448.0])[0] == 1.0                  # 448 / 1 fits, 448 / 0.5 does not
    assert fp8.pow2_scale([449.0])[0] == 2.0
    assert fp8.pow2_scale([1.0])[0] == 2.0 ** -8              # 1 / 2^-8 = 256 <= 448 < 512
    assert fp8.pow2_scale([1.75])[0] == 2.0 ** -8             # 1.75 * 2^8 = 448 exactly
    assert fp8.pow2_scale([1.76])[0] == 2.0 ** -7
    assert fp8.pow2_scale([0.0])[0] == 0.0


def test_zero_row_and_exactly_representable_row():
    x = np.zeros((2, 16), dtype=np.float32)
    x[1] = fp8.e4m3_decode(np.arange(0x6F, 0x7F)) * 2.0 ** -8  # amax 448 * 2^-8: the scale is 2^-8
    codes, scales = fp8.quantize_rows(x)
    assert scales[0] == 0 and (codes[0] == 0).all()
    assert scales[1] == 2.0 ** -8
    np.testing.assert_array_equal(fp8.dequantize_rows(codes, scales)[1], x[1])


def test_fp8_decode_equals_decode_over_dequantised_latent():
    """With power-of-two scales the dequantised latent is exact in bf16, so the FP8 decode equals the
    plain absorbed decode over that bf16 latent; a mixed-up scale row or a dropped scale fails."""
    rng = np.random.default_rng(2)
    B, S, H, r, dr = 2, 2, 4, 16, 4
    cu = np.array([0, 5, 12])
    T = 12
    codes = rng.integers(0, 0x7E, size=(T, r), dtype=np.uint8) | (rng.integers(0, 2, size=(T, r), dtype=np.uint8) << 7)
    scales = (2.0 ** rng.integers(-8, -2, size=T)).astype(np.float32)
    lat = fp8.e4m3_decode(codes) * scales[:, None].astype(np.float64)
    assert np.array_equal(torch.from_numpy(lat).bfloat16().double().numpy(), lat)
    q = rng.standard_normal((B, S, H, r))
    qr = rng.standard_normal((B, S, H, dr))
    kpe = rng.standard_normal((T, dr))
    out, lse = fp8.mla_absorbed_decode_fp8(q, qr, codes, scales, kpe, cu, 0.3)
    ref_out, ref_lse = oracle.mla_absorbed_decode(q, qr, lat, kpe, cu, 0.3)
    np.testing.assert_allclose(out, ref_out, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, atol=1e-12)
    # scales matter per row: swapping two rows' scales changes the result
    sw = scales.copy()
    sw[[0, 1]] = sw[[1, 0]]
    if sw[0] != sw[1]:
        o2, _ = fp8.mla_absorbed_decode_fp8(q, qr, codes, sw, kpe, cu, 0.3)
        assert np.abs(o2 - out).max() > 1e-6


def test_gta_fp8_decode_equals_gta_decode_over_dequantised_states():
    """Power-of-two scales keep the dequantised tied states exact in bf16: the FP8 GTA decode equals
    the GTA decode over them; scales are per token across all groups of the row."""
    rng = np.random.default_rng(3)
    B, S, H, g, d, dr = 2, 2, 8, 4, 8, 4
    cu = np.array([0, 6, 13])
    T = 13
    codes = rng.integers(0, 0x7E, size=(T, g * d), dtype=np.uint8) | (rng.integers(0, 2, size=(T, g * d), dtype=np.uint8) << 7)
    scales = (2.0 ** rng.integers(-8, -2, size=T)).astype(np.float32)
    tied = fp8.e4m3_decode(codes) * scales[:, None].astype(np.float64)
    q = rng.standard_normal((B, S, H, d))
    qr = rng.standard_normal((B, S, H, dr))
    kpe = rng.standard_normal((T, dr))
    out, lse = fp8.gta_group_decode_fp8(q, qr, codes, scales, kpe, g, cu, 0.35)
    ref_out, ref_lse = oracle.gta_group_decode(q, qr, tied, kpe, g, cu, 0.35)
    np.testing.assert_allclose(out, ref_out, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, atol=1e-12)
    # one scale for the whole row: doubling a token's scale doubles its key and value in every group
    s2 = scales.copy()
    s2[7] *= 2
    out2, _ = fp8.gta_group_decode_fp8(q, qr, codes, s2, kpe, g, cu, 0.35)
    tied2 = tied.copy()
    tied2[7] *= 2
    ref2, _ = oracle.gta_group_decode(q, qr, tied2, kpe, g, cu, 0.35)
    np.testing.assert_allclose(out2, ref2, atol=1e-12)
