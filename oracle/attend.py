"""fp64 CPU oracle for single-step decode attention over a latent / grouped KV cache.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this module:
only tests/, the smoke check in __graft_entry__ and the CPU-baseline leg of
bench.py call it.  It shares no code with the CUDA kernels.

What it computes (all arithmetic in float64, inputs read from their stored
bf16 / fp32 values):

For request b, new token i in [0, s_q), query head h in group j = floor(h / (h_q/G))
and visible keys t in [0, L_b - s_q + i]:

    s[t]  = scale * ( q[b,i,h,:] . K[cu_b + t, j, :]  +  q_rope[b,i,h,:] . k_rope[cu_b + t, :] )
    lse   = log( sum_t exp(s[t]) )                       (natural log)
    out   = sum_t exp(s[t] - lse) * V[cu_b + t, j, :]

Sources:
* Decode reads the whole cached key/value history for every generated token,
  which is the bandwidth problem the method targets -- GQLA explainer
  ("GQLA: Group-Query Latent Attention for Hardware-Adaptive Large Language
  Model Decoding"), section 1 "Problem statement".
* MQA absorbed path: the key/value up-projections are folded into the query
  and the output, so every head attends directly to the latent c_KV (width
  r_kv) plus one shared RoPE key (width d_R); the cache holds only those two
  -- same page, section 2, "MQA absorbed path".  Instance: G = 1, K = V = c_KV.
* GQA path: the latent is expanded once into g key/value groups (2*g*d_h per
  token plus the shared RoPE key) and decode is native grouped-query attention
  -- same page, section 2, "GQA path".  Instance: G = g, separate K_j, V_j.
* GLA: query heads are split into groups and each group shares its own latent
  -- "Grouped Latent Attention" article (Tri Dao et al. news page), section
  "GLA".  Instance: G = n_lat, K_j = V_j = latent group j, one shared RoPE key.
* GTA (grouped-tied attention): the heads of a group share one tied key/value
  state, so the group's cached state is read as its key and as its value --
  same article, section "GTA".  Instance: G = g, K_j = V_j = tied state j (width
  d_h), with the one shared RoPE key of the other forms (a reading: the article
  does not say where RoPE goes).
* MHA: G = h_q.

Readings where the pages are silent (listed again in the design notes):
* heads map to groups in contiguous blocks, j(h) = floor(h*G/h_q);
* the s_q new tokens are already the last s_q rows of each request's cache;
  query i sees rows 0 .. L_b - s_q + i (causal inside the new tokens);
* the softmax scale is passed in (1/sqrt(d_k + d_R) for the workloads).
"""
from __future__ import annotations

import numpy as np

__all__ = ["grouped_decode", "mla_absorbed_decode", "gqla_group_decode", "gla_group_decode",
           "gta_group_decode", "merge_partials", "append_rows", "append_destinations", "visible_keys",
           "absorb_query", "unabsorb_output", "expand_latent", "output_projection"]


def _f64(x) -> np.ndarray:
    """Stored values (numpy, or a torch CPU tensor of bf16/fp32) as float64."""
    if hasattr(x, "detach"):
        x = x.detach()
        if str(x.dtype) == "torch.bfloat16":
            x = x.float()
        x = x.numpy()
    return np.asarray(x, dtype=np.float64)


def visible_keys(length: int, s_q: int, i: int) -> int:
    """Number of cache rows query i (of s_q new tokens) may attend to: L - s_q + i + 1."""
    if length < s_q:
        raise ValueError("a request's cache must already hold its s_q new tokens")
    return length - s_q + i + 1


def _softmax_attend(s: np.ndarray, v: np.ndarray):
    """Stable softmax over the last axis of scores s [rows, n] and the weighted sum of v [n, d]."""
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    denom = e.sum(axis=1, keepdims=True)
    lse = m[:, 0] + np.log(denom[:, 0])
    return (e / denom) @ v, lse


def grouped_decode(q, q_rope, k, v, k_rope, cu_seqlens, scale, s_q=None, requests=None):
    """The general definition above.

    q [B, s_q, h_q, d_k], q_rope [B, s_q, h_q, d_R], k [T, G, d_k], v [T, G, d_v],
    k_rope [T, d_R], cu_seqlens [B+1] (exclusive prefix of the cache lengths).
    `requests` optionally restricts the work to a subset of b (other rows stay NaN).
    Returns out [B, s_q, h_q, d_v] and lse [B, s_q, h_q] (float64).
    """
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    B, S, H, _ = q.shape
    if s_q is not None:
        assert S == s_q
    G, d_v = k.shape[1], v.shape[2]
    if H % G:
        raise ValueError("h_q must be a multiple of the group count")
    hpg = H // G
    out = np.full((B, S, H, d_v), np.nan)
    lse = np.full((B, S, H), np.nan)
    for b in (range(B) if requests is None else requests):
        c0, c1 = int(cu[b]), int(cu[b + 1])
        length = c1 - c0
        kr = _f64(k_rope[c0:c1])
        for j in range(G):
            kj = _f64(k[c0:c1, j, :])
            vj = _f64(v[c0:c1, j, :])
            hs = slice(j * hpg, (j + 1) * hpg)
            for i in range(S):
                n = visible_keys(length, S, i)
                qn = _f64(q[b, i, hs, :])
                qr = _f64(q_rope[b, i, hs, :])
                s = scale * (qn @ kj[:n].T + qr @ kr[:n].T)
                out[b, i, hs], lse[b, i, hs] = _softmax_attend(s, vj[:n])
    return out, lse


def mla_absorbed_decode(q_nope_abs, q_rope, ckv, kpe, cu_seqlens, scale, requests=None):
    """MQA absorbed path: every head attends to the shared latent; V is the latent itself.

    q_nope_abs [B, s_q, h_q, r_kv] (query with W_UK already folded in), ckv [T, r_kv],
    kpe [T, d_R].  Output lives in latent space: out [B, s_q, h_q, r_kv].
    """
    lat = ckv[:, None, :]
    return grouped_decode(q_nope_abs, q_rope, lat, lat, kpe, cu_seqlens, scale,
                          requests=requests)


def gqla_group_decode(q, q_rope, k, v, kpe, cu_seqlens, scale, requests=None):
    """GQA path of GQLA: g expanded key/value groups k, v [T, g, d_h] plus the shared k_rope."""
    return grouped_decode(q, q_rope, k, v, kpe, cu_seqlens, scale, requests=requests)


def gla_group_decode(q, q_rope, clat, kpe, n_lat, cu_seqlens, scale, requests=None):
    """GLA: n_lat latent groups clat [T, n_lat*r_g]; group j's heads use latent group j as K and V."""
    T = clat.shape[0]
    lat = clat.reshape(T, n_lat, -1)
    return grouped_decode(q, q_rope, lat, lat, kpe, cu_seqlens, scale, requests=requests)


def gta_group_decode(q, q_rope, kv, kpe, g, cu_seqlens, scale, requests=None):
    """GTA: g tied groups kv [T, g*d_h]; group j's heads read tied state j as both key and value,
    plus the shared k_rope kpe [T, d_R].  Output out [B, s_q, h_q, d_h]."""
    T = kv.shape[0]
    tied = kv.reshape(T, g, -1)
    return grouped_decode(q, q_rope, tied, tied, kpe, cu_seqlens, scale, requests=requests)


def merge_partials(o_parts, lse_parts):
    """Combine attention over disjoint key sets from their (normalised out, lse) pairs.

    For parts p with lse_p = log sum_{t in p} exp(s_t) and o_p = sum_{t in p} exp(s_t - lse_p) v_t:
        lse = log sum_p exp(lse_p),   out = sum_p exp(lse_p - lse) o_p.
    A part with no keys carries lse = -inf and contributes nothing.
    o_parts [n, ..., d], lse_parts [n, ...].
    """
    o = _f64(o_parts)
    l = _f64(lse_parts)
    m = l.max(axis=0)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    w = np.exp(l - m_safe)
    tot = w.sum(axis=0)
    lse = m_safe + np.log(tot)
    out = (w[..., None] * np.where(np.isfinite(l)[..., None], o, 0.0)).sum(axis=0) / tot[..., None]
    return out, lse


def append_destinations(cu_seqlens, s_q):
    """Cache row of new token i of request b: cu_b + L_b - s_q + i (the new tokens are the tail)."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    B = len(cu) - 1
    dst = np.empty(B * s_q, dtype=np.int64)
    for b in range(B):
        length = int(cu[b + 1] - cu[b])
        if length < s_q:
            raise ValueError("cache length below s_q")
        for i in range(s_q):
            dst[b * s_q + i] = cu[b] + length - s_q + i
    return dst


def append_rows(cache, new_rows, cu_seqlens, s_q):
    """Return a copy of `cache` with new_rows[b*s_q + i] written at its destination row."""
    out = np.array(cache, copy=True)
    dst = append_destinations(cu_seqlens, s_q)
    out[dst] = np.asarray(new_rows)
    return out


def absorb_query(q, w_uk, groups):
    """Fold W_UK into the query: q_abs[..., h, :] = W_UK[j(h)] @ q[..., h, :].

    q [..., h_q, d_h], w_uk [G, r, d_h]  ->  [..., h_q, r].
    """
    q = _f64(q)
    w = _f64(w_uk)
    H = q.shape[-2]
    hpg = H // groups
    out = np.empty(q.shape[:-1] + (w.shape[1],))
    for h in range(H):
        out[..., h, :] = q[..., h, :] @ w[h // hpg].T
    return out


def unabsorb_output(o_lat, w_uv, groups):
    """Apply W_UV after attention in latent space: out[..., h, :] = W_UV[j(h)]^T @ o_lat[..., h, :].

    o_lat [..., h_q, r], w_uv [G, r, d_v]  ->  [..., h_q, d_v].
    """
    o = _f64(o_lat)
    w = _f64(w_uv)
    H = o.shape[-2]
    hpg = H // groups
    out = np.empty(o.shape[:-1] + (w.shape[2],))
    for h in range(H):
        out[..., h, :] = o[..., h, :] @ w[h // hpg]
    return out


def expand_latent(c, w):
    """Expanded per-group keys or values: X[t, j, :] = c[t, :] @ W[j]  (c [T, r], W [G, r, d])."""
    c = _f64(c)
    w = _f64(w)
    return np.einsum("tr,grd->tgd", c, w)


def output_projection(o, w_o):
    """Output projection after attention: y[t, :] = sum over heads h and columns c of
    o[t, h, c] * W_O[h*d_v + c, :]  (o [n, h, d_v] or [n, h*d_v], W_O [h*d_v, d_model])."""
    o = _f64(o)
    w = _f64(w_o)
    return o.reshape(o.shape[0], -1) @ w
