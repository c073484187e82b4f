"""Algebraic identities the pages fix between the decode forms, checked on the oracle.

* Absorbed = expanded: folding W_UK into the query and W_UV into the output lets
  every head read the latent directly -- GQLA explainer, section 2 ("MQA absorbed
  path"); MLA-vs-GQA post ("absorb trick" paragraph).
* GQLA exposes two algebraically equivalent paths on the same weights: the
  absorbed path with per-group up-projections, and GQA over K_j = C W_UK[j],
  V_j = C W_UV[j] -- GQLA explainer, section 2 "Architecture" and section 5.
* "Mixing can learn copying": MLA with selector up-projections is GQA -- MLA-vs-GQA post.
* GQA with one head per group is MHA; GQA equals MHA over per-head replicated K/V.
"""
import numpy as np
import pytest

import oracle


def _setup(seed, B=2, S=2, H=4, G=2, r=6, dh=3, dv=4, dr=2, lengths=(5, 7)):
    rng = np.random.default_rng(seed)
    cu = np.concatenate([[0], np.cumsum(lengths)])
    T = int(cu[-1])
    return dict(rng=rng, cu=cu, T=T, q=rng.standard_normal((B, S, H, dh)),
                qr=rng.standard_normal((B, S, H, dr)), C=rng.standard_normal((T, r)),
                kr=rng.standard_normal((T, dr)), w_uk=rng.standard_normal((G, r, dh)),
                w_uv=rng.standard_normal((G, r, dv)), H=H, G=G)


@pytest.mark.parametrize("G", [1, 2, 4])
def test_absorbed_path_equals_expanded_path(G):
    d = _setup(11 + G, G=G)
    q_abs = oracle.absorb_query(d["q"], d["w_uk"], G)
    o_lat, lse_a = oracle.mla_absorbed_decode(q_abs, d["qr"], d["C"], d["kr"], d["cu"], 0.4)
    out_a = oracle.unabsorb_output(o_lat, d["w_uv"], G)
    K = oracle.expand_latent(d["C"], d["w_uk"])
    V = oracle.expand_latent(d["C"], d["w_uv"])
    out_e, lse_e = oracle.grouped_decode(d["q"], d["qr"], K, V, d["kr"], d["cu"], 0.4)
    np.testing.assert_allclose(out_a, out_e, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(lse_a, lse_e, rtol=1e-10, atol=1e-10)


def test_per_head_expansion_is_mha():
    """MLA with per-head up-projections (G = h_q) equals MHA over expanded per-head K/V."""
    d = _setup(21, G=4, H=4)
    q_abs = oracle.absorb_query(d["q"], d["w_uk"], 4)
    o_lat, lse_a = oracle.mla_absorbed_decode(q_abs, d["qr"], d["C"], d["kr"], d["cu"], 1.1)
    out_a = oracle.unabsorb_output(o_lat, d["w_uv"], 4)
    K = oracle.expand_latent(d["C"], d["w_uk"])
    V = oracle.expand_latent(d["C"], d["w_uv"])
    out_m, lse_m = oracle.grouped_decode(d["q"], d["qr"], K, V, d["kr"], d["cu"], 1.1)
    np.testing.assert_allclose(out_a, out_m, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(lse_a, lse_m, rtol=1e-10, atol=1e-10)


@pytest.mark.parametrize("H,G", [(4, 2), (8, 2), (8, 4)])
def test_gqa_equals_mha_with_replicated_groups(H, G):
    """Pins the head->group map: GQA(G) == MHA over K/V replicated to each head of its block."""
    rng = np.random.default_rng(H * 10 + G)
    lengths = [6, 4]
    cu = np.concatenate([[0], np.cumsum(lengths)])
    T = int(cu[-1])
    q = rng.standard_normal((2, 2, H, 3))
    qr = rng.standard_normal((2, 2, H, 2))
    k = rng.standard_normal((T, G, 3))
    v = rng.standard_normal((T, G, 5))
    kr = rng.standard_normal((T, 2))
    hpg = H // G
    rep = np.array([h // hpg for h in range(H)])
    out_g, lse_g = oracle.grouped_decode(q, qr, k, v, kr, cu, 0.5)
    out_m, lse_m = oracle.grouped_decode(q, qr, k[:, rep], v[:, rep], kr, cu, 0.5)
    np.testing.assert_allclose(out_g, out_m, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(lse_g, lse_m, rtol=1e-13, atol=1e-13)
    # a strided (h % G) assignment gives a different result: the map is observable
    rep_bad = np.array([h % G for h in range(H)])
    out_b, _ = oracle.grouped_decode(q, qr, k[:, rep_bad], v[:, rep_bad], kr, cu, 0.5)
    assert np.abs(out_b - out_g).max() > 1e-3


def test_mixing_can_copy():
    """MLA whose up-projections select block j of C = [K_0..K_{G-1}, V_0..V_{G-1}] is GQA."""
    rng = np.random.default_rng(31)
    G, H, dh, dv, dr = 2, 4, 3, 3, 2
    lengths = [5, 6]
    cu = np.concatenate([[0], np.cumsum(lengths)])
    T = int(cu[-1])
    k = rng.standard_normal((T, G, dh))
    v = rng.standard_normal((T, G, dv))
    kr = rng.standard_normal((T, dr))
    q = rng.standard_normal((2, 1, H, dh))
    qr = rng.standard_normal((2, 1, H, dr))
    C = np.concatenate([k.reshape(T, -1), v.reshape(T, -1)], axis=1)     # r = G*(dh+dv)
    r = C.shape[1]
    w_uk = np.zeros((G, r, dh))
    w_uv = np.zeros((G, r, dv))
    for j in range(G):
        w_uk[j, j * dh:(j + 1) * dh, :] = np.eye(dh)
        w_uv[j, G * dh + j * dv:G * dh + (j + 1) * dv, :] = np.eye(dv)
    q_abs = oracle.absorb_query(q, w_uk, G)
    o_lat, lse_a = oracle.mla_absorbed_decode(q_abs, qr, C, kr, cu, 0.9)
    out_a = oracle.unabsorb_output(o_lat, w_uv, G)
    out_g, lse_g = oracle.gqla_group_decode(q, qr, k, v, kr, cu, 0.9)
    np.testing.assert_allclose(out_a, out_g, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse_a, lse_g, rtol=1e-12, atol=1e-12)


def test_gla_is_block_diagonal_mla():
    """GLA-2 equals MLA over the full latent with each head's query zero outside its block."""
    rng = np.random.default_rng(41)
    H, rg, dr = 4, 3, 2
    lengths = [4, 7]
    cu = np.concatenate([[0], np.cumsum(lengths)])
    T = int(cu[-1])
    clat = rng.standard_normal((T, 2 * rg))
    kr = rng.standard_normal((T, dr))
    q = rng.standard_normal((2, 1, H, rg))
    qr = rng.standard_normal((2, 1, H, dr))
    out_g, lse_g = oracle.gla_group_decode(q, qr, clat, kr, 2, cu, 0.8)
    qfull = np.zeros((2, 1, H, 2 * rg))
    for h in range(H):
        j = h // (H // 2)
        qfull[:, :, h, j * rg:(j + 1) * rg] = q[:, :, h]
    out_m, lse_m = oracle.mla_absorbed_decode(qfull, qr, clat, kr, cu, 0.8)
    np.testing.assert_allclose(lse_g, lse_m, atol=1e-13)
    for h in range(H):
        j = h // (H // 2)
        np.testing.assert_allclose(out_g[:, :, h], out_m[:, :, h, j * rg:(j + 1) * rg], atol=1e-13)


def test_output_projection_identity_and_head_blocks():
    """y = o W_O: with W_O = I the heads come back side by side, and splitting the heads into blocks
    (the group-axis split) and summing the blocks' products gives the full projection."""
    rng = np.random.default_rng(41)
    o = rng.standard_normal((3, 4, 5))
    y = oracle.output_projection(o, np.eye(20))
    np.testing.assert_array_equal(y, o.reshape(3, 20))
    w = rng.standard_normal((20, 7))
    full = oracle.output_projection(o, w)
    parts = sum(oracle.output_projection(o[:, h0:h0 + 2], w[h0 * 5:(h0 + 2) * 5]) for h0 in (0, 2))
    np.testing.assert_allclose(parts, full, atol=1e-12)
    # brute force on one entry
    t, c = 2, 6
    assert abs(full[t, c] - sum(o[t, h, e] * w[h * 5 + e, c] for h in range(4) for e in range(5))) < 1e-12
