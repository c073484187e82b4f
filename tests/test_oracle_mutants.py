"""Plant plausible mistakes in a copy of the oracle and check that the pins catch each one.

Each mutant is the oracle's source with one edit (a dropped term, an index or
sign error, an off-by-one); the brute-force and closed-form checks must reject it.
Mutants are built on the CPU from the source text; the real oracle is untouched.
"""
import importlib.util
import os
import types

import numpy as np
import pytest

from test_oracle_bruteforce import _brute, _case

SRC = open(os.path.join(os.path.dirname(__file__), "..", "oracle", "attend.py")).read()

MUTANTS = {
    "drop_rope_term": ("qn @ kj[:n].T + qr @ kr[:n].T", "qn @ kj[:n].T"),
    "causal_off_by_one": ("return length - s_q + i + 1", "return length - s_q + i"),
    "see_all_keys": ("return length - s_q + i + 1", "return length"),
    "strided_group_map": ("hs = slice(j * hpg, (j + 1) * hpg)", "hs = slice(j, H, G)"),
    "scale_only_nope": ("s = scale * (qn @ kj[:n].T + qr @ kr[:n].T)",
                        "s = scale * (qn @ kj[:n].T) + qr @ kr[:n].T"),
    "v_uses_k": ("out[b, i, hs], lse[b, i, hs] = _softmax_attend(s, vj[:n])",
                 "out[b, i, hs], lse[b, i, hs] = _softmax_attend(s, kj[:n, :vj.shape[1]])"),
    "lse_drops_max": ("lse = m[:, 0] + np.log(denom[:, 0])", "lse = np.log(denom[:, 0])"),
    "every_request_from_row_0": ("c0, c1 = int(cu[b]), int(cu[b + 1])",
                                 "c0, c1 = 0, int(cu[b + 1]) - int(cu[b])"),
}


def _load(src):
    mod = types.ModuleType("oracle_mutant")
    exec(compile(src, "oracle_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    old, new = MUTANTS[name]
    assert old in SRC, f"mutation site for {name} not found"
    mod = _load(SRC.replace(old, new))
    caught = False
    for S, H, G, lengths in [(2, 4, 2, [3, 6]), (1, 4, 1, [2, 5]), (2, 2, 2, [4, 4])]:
        rng = np.random.default_rng(S * 100 + H * 10 + G)
        q, qr, k, v, kr, cu = _case(rng, len(lengths), S, H, G, 4, 3, 2, lengths)
        try:
            out, lse = mod.grouped_decode(q, qr, k, v, kr, cu, 0.7)
        except Exception:
            caught = True
            break
        bo, bl = _brute(q, qr, k, v, kr, cu, 0.7)
        if not (np.allclose(out, bo, atol=1e-9) and np.allclose(lse, bl, atol=1e-9)):
            caught = True
            break
    assert caught, f"mutant {name} survived the brute-force pin"


def test_unmutated_source_passes():
    mod = _load(SRC)
    rng = np.random.default_rng(1)
    q, qr, k, v, kr, cu = _case(rng, 2, 2, 4, 2, 4, 3, 2, [3, 6])
    out, lse = mod.grouped_decode(q, qr, k, v, kr, cu, 0.7)
    bo, bl = _brute(q, qr, k, v, kr, cu, 0.7)
    np.testing.assert_allclose(out, bo, atol=1e-12)
    np.testing.assert_allclose(lse, bl, atol=1e-12)


# ---------------------------------------------------------------------------------------------
# FP8 (e4m3) oracle: each mutant must fail at least one of the pins in test_oracle_fp8.py
# (run against the mutant in place of oracle.fp8).
FP8_SRC = open(os.path.join(os.path.dirname(__file__), "..", "oracle", "fp8.py")).read()

FP8_MUTANTS = {
    "exponent_bias_8": ("return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)", "return sign * (1.0 + m / 8.0) * 2.0 ** (e - 8)"),
    "subnormals_flushed": ("return sign * m * 2.0 ** -9", "return sign * 0.0"),
    "nan_code_finite": ("if e == 0xF and m == 0x7:", "if False:"),
    "ties_away_from_zero": ("pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))", "pick_hi = d_hi <= d_lo"),
    "ties_toward_zero": ("pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))", "pick_hi = d_hi < d_lo"),
    "sign_dropped": ("return np.where(np.signbit(y), mag | 0x80, mag).astype(np.uint8)", "return mag"),
    "scale_per_column": ("amax = np.abs(x32).max(axis=1)", "amax = np.abs(x32).max(axis=0)"),
    "scale_from_row_sum": ("amax = np.abs(x32).max(axis=1)", "amax = np.abs(x32).sum(axis=1) / 8"),
    "dequant_divides": ("return e4m3_decode(codes) * np.asarray(scales, dtype=np.float64)[:, None]",
                        "return e4m3_decode(codes) / np.asarray(scales, dtype=np.float64)[:, None]"),
    "y_off_by_one_percent": ("y = np.clip(y, -E4M3_MAX, E4M3_MAX)", "y = y * np.float32(1.01)"),
    "scale_one_binade_high": ("e = np.where(m <= 0.875, E - 9, E - 8)", "e = np.where(m <= 0.875, E - 8, E - 7)"),
    "scale_threshold_strict": ("e = np.where(m <= 0.875, E - 9, E - 8)", "e = np.where(m < 0.875, E - 9, E - 8)"),
    "scale_not_power_of_two": ("scales = pow2_scale(amax)", "scales = (amax / np.float32(E4M3_MAX)).astype(np.float32)"),
}


def _fp8_pins_pass(mod) -> bool:
    import test_oracle_fp8 as T
    saved = T.fp8
    T.fp8 = mod
    try:
        for name in sorted(dir(T)):
            if name.startswith("test_"):
                getattr(T, name)()
        return True
    except Exception:
        return False
    finally:
        T.fp8 = saved


def _load_fp8(src):
    mod = types.ModuleType("oracle.fp8_mutant")
    mod.__dict__["__package__"] = "oracle"
    exec(compile(src, "oracle_fp8_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(FP8_MUTANTS))
def test_fp8_mutant_is_caught(name):
    old, new = FP8_MUTANTS[name]
    assert old in FP8_SRC, f"mutation site for {name} not found"
    assert not _fp8_pins_pass(_load_fp8(FP8_SRC.replace(old, new))), f"fp8 mutant {name} survived the pins"


def test_fp8_unmutated_source_passes_the_pins():
    assert _fp8_pins_pass(_load_fp8(FP8_SRC))


# GTA and the output projection (attend.py): the brute-force / identity pins catch these.
def test_gta_block_map_mutant_is_caught():
    import test_oracle_bruteforce as TB
    old, new = "tied = kv.reshape(T, g, -1)", "tied = kv.reshape(T, -1, g).transpose(0, 2, 1)"
    assert old in SRC
    mod = _load(SRC.replace(old, new))
    import oracle
    saved = oracle.gta_group_decode
    oracle.gta_group_decode = mod.gta_group_decode
    try:
        with pytest.raises(AssertionError):
            TB.test_gta_instance_matches_brute_force()
    finally:
        oracle.gta_group_decode = saved


def test_output_projection_mutant_is_caught():
    import test_oracle_identities as TI
    old, new = "return o.reshape(o.shape[0], -1) @ w", "return o.transpose(0, 2, 1).reshape(o.shape[0], -1) @ w"
    assert old in SRC
    mod = _load(SRC.replace(old, new))
    import oracle
    saved = oracle.output_projection
    oracle.output_projection = mod.output_projection
    try:
        with pytest.raises(AssertionError):
            TI.test_output_projection_identity_and_head_blocks()
    finally:
        oracle.output_projection = saved
