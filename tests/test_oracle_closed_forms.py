"""Closed forms, invariants and special cases that fix the oracle independently of its code."""
import math

import numpy as np
import pytest

import oracle


def _rand(seed, B=1, S=1, H=4, G=1, dk=5, dv=5, dr=3, L=7):
    rng = np.random.default_rng(seed)
    lengths = np.full(B, L)
    cu = np.concatenate([[0], np.cumsum(lengths)])
    T = int(cu[-1])
    return (rng.standard_normal((B, S, H, dk)), rng.standard_normal((B, S, H, dr)),
            rng.standard_normal((T, G, dk)), rng.standard_normal((T, G, dv)),
            rng.standard_normal((T, dr)), cu)


def test_single_key_returns_that_value_and_its_score():
    q, qr, k, v, kr, cu = _rand(1, L=1)
    out, lse = oracle.grouped_decode(q, qr, k, v, kr, cu, 0.3)
    s0 = 0.3 * (q[0, 0] @ k[0, 0] + qr[0, 0] @ kr[0])
    np.testing.assert_array_equal(out[0, 0], np.broadcast_to(v[0, 0], out[0, 0].shape))
    np.testing.assert_allclose(lse[0, 0], s0, atol=1e-13)


@pytest.mark.parametrize("S", [1, 2])
def test_zero_query_is_uniform_mean(S):
    q, qr, k, v, kr, cu = _rand(2, S=S, L=9)
    q[:] = 0
    qr[:] = 0
    out, lse = oracle.grouped_decode(q, qr, k, v, kr, cu, 1.0)
    for i in range(S):
        n = 9 - S + i + 1
        np.testing.assert_allclose(out[0, i], np.broadcast_to(v[:n, 0].mean(0), out[0, i].shape),
                                   atol=1e-14)
        np.testing.assert_allclose(lse[0, i], math.log(n), atol=1e-14)


def test_two_keys_logistic():
    q, qr, k, v, kr, cu = _rand(3, L=2, H=1)
    out, lse = oracle.grouped_decode(q, qr, k, v, kr, cu, 0.8)
    s = [0.8 * (q[0, 0, 0] @ k[t, 0] + qr[0, 0, 0] @ kr[t]) for t in range(2)]
    w1 = 1.0 / (1.0 + math.exp(s[0] - s[1]))
    w0 = 1.0 / (1.0 + math.exp(s[1] - s[0]))
    np.testing.assert_allclose(out[0, 0, 0], w0 * v[0, 0] + w1 * v[1, 0], atol=1e-14)
    np.testing.assert_allclose(lse[0, 0, 0], max(s) + math.log1p(math.exp(-abs(s[0] - s[1]))),
                               atol=1e-14)


def test_dominant_key_selects_its_value():
    q, qr, k, v, kr, cu = _rand(4, L=6, H=1, dr=1)
    qr[:] = 1.0
    kr[:] = 0.0
    kr[3] = 50.0                     # score of key 3 is 50 above its neighbours' rope part
    q[:] *= 1e-3
    out, _ = oracle.grouped_decode(q, qr, k, v, kr, cu, 1.0)
    assert np.max(np.abs(out[0, 0, 0] - v[3, 0])) < 1e-18 + 10 * math.exp(-49.0) * np.abs(v).max()


def test_key_permutation_invariance():
    q, qr, k, v, kr, cu = _rand(5, L=8, H=2)
    perm = np.random.default_rng(0).permutation(8)
    a = oracle.grouped_decode(q, qr, k, v, kr, cu, 0.6)
    b = oracle.grouped_decode(q, qr, k[perm], v[perm], kr[perm], cu, 0.6)
    np.testing.assert_allclose(a[0], b[0], atol=1e-13)
    np.testing.assert_allclose(a[1], b[1], atol=1e-13)


def test_constant_score_shift_moves_only_lse():
    """Identical k_rope rows add the same c to every score of a head: out fixed, lse + c."""
    q, qr, k, v, kr, cu = _rand(6, L=7, H=3)
    kr[:] = np.array([0.25, -1.5, 2.0])
    scale = 0.45
    shifted = oracle.grouped_decode(q, qr, k, v, kr, cu, scale)
    base = oracle.grouped_decode(q, np.zeros_like(qr), k, v, kr, cu, scale)
    c = scale * (qr[0, 0] @ kr[0])       # per head
    np.testing.assert_allclose(shifted[0], base[0], atol=1e-13)
    np.testing.assert_allclose(shifted[1][0, 0], base[1][0, 0] + c, atol=1e-13)


def test_causal_mtp_equals_single_token_runs():
    """With s_q = 2, query 0 equals an s_q = 1 decode over L-1 rows; query 1 over all L rows."""
    q, qr, k, v, kr, cu = _rand(7, S=2, L=6, H=2)
    out, lse = oracle.grouped_decode(q, qr, k, v, kr, cu, 0.5)
    o0, l0 = oracle.grouped_decode(q[:, :1], qr[:, :1], k[:5], v[:5], kr[:5], np.array([0, 5]), 0.5)
    o1, l1 = oracle.grouped_decode(q[:, 1:], qr[:, 1:], k, v, kr, cu, 0.5)
    np.testing.assert_array_equal(out[:, 0], o0[:, 0])
    np.testing.assert_array_equal(lse[:, 0], l0[:, 0])
    np.testing.assert_array_equal(out[:, 1], o1[:, 0])


def test_varlen_requests_are_independent():
    rng = np.random.default_rng(8)
    lengths = [3, 9, 1, 4]
    cu = np.concatenate([[0], np.cumsum(lengths)])
    T = int(cu[-1])
    q = rng.standard_normal((4, 1, 2, 3))
    qr = rng.standard_normal((4, 1, 2, 2))
    k = rng.standard_normal((T, 1, 3))
    v = rng.standard_normal((T, 1, 4))
    kr = rng.standard_normal((T, 2))
    full = oracle.grouped_decode(q, qr, k, v, kr, cu, 1.0)
    for b in range(4):
        sl = slice(cu[b], cu[b + 1])
        one = oracle.grouped_decode(q[b:b + 1], qr[b:b + 1], k[sl], v[sl], kr[sl],
                                    np.array([0, lengths[b]]), 1.0)
        np.testing.assert_array_equal(full[0][b], one[0][0])


@pytest.mark.parametrize("cuts", [[3], [1, 5], [2, 3, 7], [6]])
def test_merge_of_partitions_equals_unsplit(cuts):
    q, qr, k, v, kr, cu = _rand(9, L=8, H=3, G=1)
    full_o, full_l = oracle.grouped_decode(q, qr, k, v, kr, cu, 0.7)
    edges = [0] + cuts + [8]
    parts_o, parts_l = [], []
    for a, b in zip(edges[:-1], edges[1:]):
        o, l = oracle.grouped_decode(q, qr, k[a:b], v[a:b], kr[a:b], np.array([0, b - a]), 0.7)
        parts_o.append(o)
        parts_l.append(l)
    mo, ml = oracle.merge_partials(np.stack(parts_o), np.stack(parts_l))
    np.testing.assert_allclose(mo, full_o, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(ml, full_l, rtol=1e-12, atol=1e-13)


def test_merge_ignores_empty_parts():
    o = np.array([[1.0, 2.0], [np.nan, np.nan], [3.0, 5.0]])[:, None, :]
    l = np.array([0.0, -np.inf, math.log(3.0)])[:, None]
    mo, ml = oracle.merge_partials(o, l)
    np.testing.assert_allclose(ml, [math.log(4.0)], atol=1e-15)
    np.testing.assert_allclose(mo[0], [(1 * 1 + 3 * 3) / 4, (2 * 1 + 5 * 3) / 4], atol=1e-15)


def test_short_request_rejected():
    q, qr, k, v, kr, cu = _rand(10, S=2, L=1)
    with pytest.raises(ValueError):
        oracle.grouped_decode(q, qr, k, v, kr, cu, 1.0)


def test_append_destinations_hand_example():
    # lengths 3 and 4 (new tokens already counted), s_q = 2: rows 1,2 and 5,6.
    np.testing.assert_array_equal(oracle.append_destinations([0, 3, 7], 2), [1, 2, 5, 6])
    np.testing.assert_array_equal(oracle.append_destinations([0, 3, 7], 1), [2, 6])
    cache = np.zeros((8, 2))
    new = np.arange(8).reshape(4, 2) + 1.0
    got = oracle.append_rows(cache, new, [0, 3, 7], 2)
    assert got[1].tolist() == [1, 2] and got[2].tolist() == [3, 4]
    assert got[5].tolist() == [5, 6] and got[6].tolist() == [7, 8]
    assert not got[[0, 3, 4, 7]].any()
