"""Byte and FLOP accounting for decode attention (test infrastructure, like the rest of oracle/).

Algorithmic cost of one decode step, counting every cache row once and every
query/output/lse element once; work on padding or split partials is not counted.

* Cache bytes per token: the absorbed path stores the latent plus the shared
  RoPE key, r_kv + d_R elements; the GQA path stores 2*g*d_h + d_R -- GQLA
  explainer, section 2 ("MQA absorbed path" / "GQA path", cache lines).
* GTA stores one tied key/value state per group plus the shared RoPE key,
  g*d_h + d_R per token; the article on GTA/GLA puts the saving against GQA at
  about half of the KV cache ("Grouped Latent Attention" article, section "GTA").
* FLOPs: per visible (query row, key) pair, 2*(d_k + d_R) for q.k and 2*d_v
  for p.v, over h_q heads.
* Arithmetic intensity = FLOPs / cache bytes per token; the page gives about
  242 FLOPs/byte for the absorbed path at s_q = 1 and about 37 for the GQA
  path at (g=8, s_q=2) or (g=4, s_q=1) -- same page, section 2 and "Path selection".
"""
from __future__ import annotations

import numpy as np

__all__ = ["cache_row_elems", "cache_bytes_per_token", "flops_per_token",
           "intensity_per_token", "step_bytes", "step_flops"]


def cache_row_elems(kind, groups, d_k, d_v, d_rope):
    """Elements stored per cached token: latent(s) + RoPE key, or expanded K and V + RoPE key."""
    if kind in ("mla", "gla", "gta"):
        return groups * d_k + d_rope
    if kind == "gqla":
        return groups * (d_k + d_v) + d_rope
    raise ValueError(kind)


def cache_bytes_per_token(kind, groups, d_k, d_v, d_rope, elem_bytes=2):
    return cache_row_elems(kind, groups, d_k, d_v, d_rope) * elem_bytes


def flops_per_token(h_q, s_q, d_k, d_v, d_rope):
    """FLOPs spent per cached token when all s_q queries see it: 2*s_q*h_q*(d_k + d_R + d_v)."""
    return 2 * s_q * h_q * (d_k + d_rope + d_v)


def intensity_per_token(kind, h_q, s_q, groups, d_k, d_v, d_rope, elem_bytes=2):
    return (flops_per_token(h_q, s_q, d_k, d_v, d_rope)
            / cache_bytes_per_token(kind, groups, d_k, d_v, d_rope, elem_bytes))


def step_bytes(kind, lengths, s_q, h_q, groups, d_k, d_v, d_rope, elem_bytes=2):
    """Algorithmic bytes of one step: cache rows once, q and q_rope, out, fp32 lse."""
    lengths = np.asarray(lengths, dtype=np.int64)
    B = len(lengths)
    cache = int(lengths.sum()) * cache_bytes_per_token(kind, groups, d_k, d_v, d_rope, elem_bytes)
    q = B * s_q * h_q * (d_k + d_rope) * elem_bytes
    out = B * s_q * h_q * d_v * elem_bytes
    lse = B * s_q * h_q * 4
    return cache + q + out + lse


def step_flops(lengths, s_q, h_q, d_k, d_v, d_rope):
    """sum_b sum_i (L_b - s_q + i + 1) * 2*h_q*(d_k + d_R + d_v): only visible pairs count."""
    lengths = np.asarray(lengths, dtype=np.int64)
    vis = sum(int((lengths - s_q + i + 1).sum()) for i in range(s_q))
    return vis * 2 * h_q * (d_k + d_rope + d_v)
