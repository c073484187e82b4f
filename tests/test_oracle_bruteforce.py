"""Pin the oracle against a pure-Python brute force on tiny inputs.

The brute force evaluates the softmax straight from its definition --
exp(s_t) / sum_u exp(s_u) with no max shift, sums with math.fsum, the group
map j(h) = h // (h_q/G) and the causal limit L - s_q + i written out as loops.
A dropped term, a wrong index, a transposed operand, a wrong group map or an
off-by-one in the causal limit in the oracle makes these fail.
"""
import math
import random

import numpy as np
import pytest

import oracle


def _brute(q, qr, k, v, kr, cu, scale):
    B, S, H, _ = q.shape
    G = k.shape[1]
    hpg = H // G
    d_v = v.shape[2]
    out = np.zeros((B, S, H, d_v))
    lse = np.zeros((B, S, H))
    for b in range(B):
        c0 = int(cu[b])
        L = int(cu[b + 1]) - c0
        for i in range(S):
            last = L - S + i          # query i sees rows 0..last
            for h in range(H):
                j = h // hpg
                sc = []
                for t in range(last + 1):
                    terms = [float(q[b, i, h, c]) * float(k[c0 + t, j, c]) for c in range(q.shape[3])]
                    terms += [float(qr[b, i, h, c]) * float(kr[c0 + t, c]) for c in range(qr.shape[3])]
                    sc.append(scale * math.fsum(terms))
                ex = [math.exp(x) for x in sc]
                z = math.fsum(ex)
                lse[b, i, h] = math.log(z)
                for c in range(d_v):
                    out[b, i, h, c] = math.fsum(ex[t] / z * float(v[c0 + t, j, c])
                                                for t in range(last + 1))
    return out, lse


def _case(rng, B, S, H, G, dk, dv, dr, lengths):
    cu = np.concatenate([[0], np.cumsum(lengths)])
    T = int(cu[-1])
    q = rng.standard_normal((B, S, H, dk))
    qr = rng.standard_normal((B, S, H, dr))
    k = rng.standard_normal((T, G, dk))
    v = rng.standard_normal((T, G, dv))
    kr = rng.standard_normal((T, dr))
    return q, qr, k, v, kr, cu


@pytest.mark.parametrize("S", [1, 2])
@pytest.mark.parametrize("H,G", [(1, 1), (4, 1), (4, 2), (4, 4)])
def test_grouped_decode_matches_brute_force(S, H, G):
    rng = np.random.default_rng(100 + 10 * S + H + G)
    lengths = [3, 6] if S == 2 else [1, 5]
    dk, dv, dr = 4, 3, 2
    q, qr, k, v, kr, cu = _case(rng, 2, S, H, G, dk, dv, dr, lengths)
    scale = 0.7
    out, lse = oracle.grouped_decode(q, qr, k, v, kr, cu, scale)
    bo, bl = _brute(q, qr, k, v, kr, cu, scale)
    np.testing.assert_allclose(out, bo, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, bl, rtol=0, atol=1e-12)


def test_mla_and_gla_instances_match_brute_force():
    rng = np.random.default_rng(7)
    B, S, H, r, dr = 2, 2, 4, 6, 2
    lengths = [4, 5]
    cu = np.concatenate([[0], np.cumsum(lengths)])
    T = int(cu[-1])
    q = rng.standard_normal((B, S, H, r))
    qr = rng.standard_normal((B, S, H, dr))
    c = rng.standard_normal((T, r))
    kr = rng.standard_normal((T, dr))
    out, lse = oracle.mla_absorbed_decode(q, qr, c, kr, cu, 0.5)
    bo, bl = _brute(q, qr, c[:, None, :], c[:, None, :], kr, cu, 0.5)
    np.testing.assert_allclose(out, bo, atol=1e-12)
    np.testing.assert_allclose(lse, bl, atol=1e-12)
    # GLA-2: heads 0,1 use latent columns 0..2, heads 2,3 use columns 3..5.
    qg = rng.standard_normal((B, S, H, r // 2))
    out, lse = oracle.gla_group_decode(qg, qr, c, kr, 2, cu, 0.5)
    lat = c.reshape(T, 2, r // 2)
    bo, bl = _brute(qg, qr, lat, lat, kr, cu, 0.5)
    np.testing.assert_allclose(out, bo, atol=1e-12)
    np.testing.assert_allclose(lse, bl, atol=1e-12)


def test_gta_instance_matches_brute_force():
    """GTA, g = 2 tied groups of width 3: heads 0, 1 read columns 0..2 as key and value,
    heads 2, 3 read columns 3..5; the RoPE key is shared."""
    rng = np.random.default_rng(11)
    B, S, H, g, d, dr = 2, 2, 4, 2, 3, 2
    lengths = [3, 6]
    cu = np.concatenate([[0], np.cumsum(lengths)])
    T = int(cu[-1])
    q = rng.standard_normal((B, S, H, d))
    qr = rng.standard_normal((B, S, H, dr))
    kv = rng.standard_normal((T, g * d))
    kr = rng.standard_normal((T, dr))
    out, lse = oracle.gta_group_decode(q, qr, kv, kr, g, cu, 0.6)
    tied = np.stack([kv[:, :d], kv[:, d:]], axis=1)
    bo, bl = _brute(q, qr, tied, tied, kr, cu, 0.6)
    np.testing.assert_allclose(out, bo, atol=1e-12)
    np.testing.assert_allclose(lse, bl, atol=1e-12)


def test_brute_force_itself_on_hand_example():
    """One key pair worked by hand: s = scale*(q.k + qr.kr) for two keys, then a 2-way softmax."""
    q = np.array([[[[1.0, 2.0]]]])          # B=1,S=1,H=1,dk=2
    qr = np.array([[[[0.5]]]])
    k = np.array([[[1.0, 0.0]], [[0.0, 1.0]]])  # T=2, G=1
    v = np.array([[[10.0]], [[20.0]]])
    kr = np.array([[2.0], [0.0]])
    cu = np.array([0, 2])
    # s0 = 1*(1 + 1) = 2, s1 = 1*(2 + 0) = 2 -> equal weights
    for fn in (_brute, oracle.grouped_decode):
        out, lse = fn(q, qr, k, v, kr, cu, 1.0)
        assert abs(out[0, 0, 0, 0] - 15.0) < 1e-12
        assert abs(lse[0, 0, 0] - (2.0 + math.log(2.0))) < 1e-12


def test_random_shapes_fuzz():
    rnd = random.Random(5)
    for trial in range(6):
        S = rnd.choice([1, 2])
        G = rnd.choice([1, 2])
        H = G * rnd.choice([1, 2])
        lengths = [rnd.randint(S, 6) for _ in range(rnd.randint(1, 2))]
        rng = np.random.default_rng(trial)
        q, qr, k, v, kr, cu = _case(rng, len(lengths), S, H, G, 3, 2, 2, lengths)
        out, lse = oracle.grouped_decode(q, qr, k, v, kr, cu, 0.9)
        bo, bl = _brute(q, qr, k, v, kr, cu, 0.9)
        np.testing.assert_allclose(out, bo, atol=1e-12)
        np.testing.assert_allclose(lse, bl, atol=1e-12)
