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
