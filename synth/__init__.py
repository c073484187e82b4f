"""Seeded synthetic inputs for the decode-attention workloads.

This module is shared by the CUDA path (tests, bench) and by the oracle's tests.
It holds shapes, seeds, random draws and storage rounding only: no attention
arithmetic lives here.  Every tensor is built on the CPU with numpy's PCG64
generator so that both sides see bit-identical inputs.

Workload shapes follow the decode settings the pages discuss: the MLA absorbed
path with a 512-wide latent plus a 64-wide shared RoPE key and 128 query heads
(GQLA explainer, section 2 "MQA absorbed path"), the GQLA grouped path with
g = 8 groups of d_h = 128 and s_q = 2 multi-token prediction (same page,
section 2 "GQA path" and "Path selection"), and GLA with two latent groups
(Grouped Latent Attention article, section "GLA").
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import numpy as np
import torch

__all__ = ["Workload", "WORKLOADS", "workload", "make_inputs", "new_token_rows", "draw_lengths",
           "prefix_offsets", "to_bf16"]


@dataclass(frozen=True)
class Workload:
    """One decode workload: shapes, storage type, seed and value distribution.

    kind    "mla"  -- all h_q heads share one latent (G = 1, K = V = latent).
            "gqla" -- G = g expanded key/value groups, separate K_j and V_j.
            "gla"  -- G = n_lat latent groups, K_j = V_j = latent group j.
            "gta"  -- G = g tied groups, K_j = V_j = tied state j (same layout as "gla").
    d_k     width of the non-RoPE part of each key (r_kv, d_h or r_g).
    d_v     width of each value row (equals d_k for "mla" and "gla").
    seqlen  uniform per-request cache length, or None for log-uniform lengths
            in [len_lo, len_hi].
    input_std  standard deviation of every Gaussian input entry before the
            storage rounding.
    q_std   standard deviation of the query entries (q and q_rope) when it differs
            from input_std (None: input_std).  Widening only the query widens the
            score range while the cached values keep their size.
    """
    name: str
    kind: str
    dtype: str
    batch: int
    s_q: int
    h_q: int
    groups: int
    d_k: int
    d_v: int
    d_rope: int
    seqlen: int | None
    seed: int
    input_std: float
    len_lo: int = 0
    len_hi: int = 0
    q_std: float | None = None

    @property
    def scale(self) -> float:
        """Softmax scale 1/sqrt(d_k + d_R) (the tiny fp32 workload states it)."""
        return 1.0 / math.sqrt(self.d_k + self.d_rope)

    @property
    def heads_per_group(self) -> int:
        return self.h_q // self.groups

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


def _std(d):
    return 1.0 / math.sqrt(d)


WORKLOADS = {
    # fp32 toy: B=2, 16 heads, r_kv=64, d_R=16, L=256, N(0,1), seed 0.
    "tiny_fp32_mla": Workload("tiny_fp32_mla", "mla", "fp32", 2, 1, 16, 1, 64, 64, 16,
                              256, 0, 1.0),
    # MLA absorbed, B=64, 128 heads, r_kv=512, d_R=64, L=4096, inputs N(0,1)/sqrt(576).
    "mla_b64_l4096": Workload("mla_b64_l4096", "mla", "bf16", 64, 1, 128, 1, 512, 512, 64,
                              4096, 1, _std(576)),
    # GQLA grouped GQA path, g=8, d_h=128, d_R=64, s_q=2 causal, L=8192, N(0,1)/sqrt(192).
    "gqla_g8_sq2_l8192": Workload("gqla_g8_sq2_l8192", "gqla", "bf16", 64, 2, 128, 8, 128, 128,
                                  64, 8192, 2, _std(192)),
    # Varlen MLA, B=128, lengths log-uniform in [1024, 65536] (seed 3), s_q = 1 and 2.
    "varlen_mla_sq1": Workload("varlen_mla_sq1", "mla", "bf16", 128, 1, 128, 1, 512, 512, 64,
                               None, 3, _std(576), 1024, 65536),
    "varlen_mla_sq2": Workload("varlen_mla_sq2", "mla", "bf16", 128, 2, 128, 1, 512, 512, 64,
                               None, 3, _std(576), 1024, 65536),
    # Long context, B=8, L=131072: GLA-2 (2 x (64 heads, r=256)) + d_R=64, and the same
    # shapes through the MLA absorbed path and the g=8 GQLA path.
    "long_gla2": Workload("long_gla2", "gla", "bf16", 8, 1, 128, 2, 256, 256, 64,
                          131072, 4, _std(320)),
    "long_mla": Workload("long_mla", "mla", "bf16", 8, 1, 128, 1, 512, 512, 64,
                         131072, 4, _std(576)),
    "long_gqla_g8": Workload("long_gqla_g8", "gqla", "bf16", 8, 1, 128, 8, 128, 128, 64,
                             131072, 4, _std(192)),
    # GTA: the GQLA shapes (g=8, d_h=128, d_R=64, s_q=2, L=8192) with K and V tied per group.
    "gta_g8_sq2_l8192": Workload("gta_g8_sq2_l8192", "gta", "bf16", 64, 2, 128, 8, 128, 128, 64,
                                 8192, 5, _std(192)),
    # GQA-2: two K/V groups of 64 heads each (the group size the VHA fold gives), s_q=2, L=8192.
    "gqa2_sq2_l8192": Workload("gqa2_sq2_l8192", "gqla", "bf16", 64, 2, 128, 2, 128, 128, 64,
                               8192, 6, _std(192)),
}


def workload(name: str, **overrides) -> Workload:
    w = WORKLOADS[name]
    return w.with_(**overrides) if overrides else w


def draw_lengths(rng: np.random.Generator, batch: int, lo: int, hi: int) -> np.ndarray:
    """Per-request lengths, log-uniform in [lo, hi]: floor(exp(U(ln lo, ln hi))), clamped."""
    u = rng.uniform(math.log(lo), math.log(hi), size=batch)
    return np.clip(np.floor(np.exp(u)).astype(np.int64), lo, hi)


def prefix_offsets(lengths) -> np.ndarray:
    """Exclusive prefix sum [0, L0, L0+L1, ...] as int64 (the cu_seqlens layout)."""
    lengths = np.asarray(lengths, dtype=np.int64)
    out = np.zeros(len(lengths) + 1, dtype=np.int64)
    np.cumsum(lengths, out=out[1:])
    return out


def to_bf16(x: np.ndarray) -> torch.Tensor:
    """Round fp32 values to bf16 with round-to-nearest-even (torch's cast)."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


_CHUNK = 1 << 22  # elements drawn per call; bounds host memory for the 4 GB caches


def _normal(rng: np.random.Generator, shape, std: float, dtype: str) -> torch.Tensor:
    """Gaussian tensor N(0, std^2) in the storage dtype, drawn row-chunk by row-chunk."""
    shape = tuple(int(s) for s in shape)
    rows = shape[0]
    inner = int(np.prod(shape[1:])) if len(shape) > 1 else 1
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    out = torch.empty((rows, inner), dtype=tdt)
    step = max(1, _CHUNK // max(inner, 1))
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        x = rng.standard_normal((r1 - r0, inner), dtype=np.float32)
        if std != 1.0:
            x *= np.float32(std)
        out[r0:r1] = torch.from_numpy(x).to(tdt)
    return out.view(shape)


def make_inputs(w: Workload, extra_rows: int = 0, lengths=None) -> dict:
    """Build the seeded inputs of workload `w` on the CPU.

    Draw order: lengths (varlen only), then q (non-RoPE part), q_rope, the key
    cache (latent / K), V (GQLA only), k_rope.  Returns a dict with
      lengths     int64 numpy [B]
      cu_seqlens  int32 torch [B+1]
      q, q_rope   [B, s_q, h_q, d_k], [B, s_q, h_q, d_R]
      mla / gla / gta:  cache [T + extra_rows, G*d_k + d_R] with the latent (tied state) in the
                  first G*d_k columns and k_rope in the last d_R (one row per token)
      gqla:       k, v [T + extra_rows, g, d_h]; kpe [T + extra_rows, d_R]
    Rows past T (extra_rows) are zero; tests poison them to check masking.
    """
    rng = np.random.default_rng(w.seed)
    if lengths is None:
        if w.seqlen is None:
            lengths = draw_lengths(rng, w.batch, w.len_lo, w.len_hi)
        else:
            lengths = np.full(w.batch, w.seqlen, dtype=np.int64)
    lengths = np.asarray(lengths, dtype=np.int64)
    assert lengths.shape == (w.batch,)
    cu = prefix_offsets(lengths)
    total = int(cu[-1])
    rows = total + extra_rows
    B, S, H, G = w.batch, w.s_q, w.h_q, w.groups
    std = w.input_std
    qs = std if w.q_std is None else w.q_std
    q = _normal(rng, (B, S, H, w.d_k), qs, w.dtype)
    q_rope = _normal(rng, (B, S, H, w.d_rope), qs, w.dtype)
    res = {"lengths": lengths, "cu_seqlens": torch.from_numpy(cu.astype(np.int32)),
           "q": q, "q_rope": q_rope, "workload": w}
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    if w.kind in ("mla", "gla", "gta"):
        width = G * w.d_k
        cache = torch.zeros((rows, width + w.d_rope), dtype=tdt)
        cache[:total, :width] = _normal(rng, (total, width), std, w.dtype)
        cache[:total, width:] = _normal(rng, (total, w.d_rope), std, w.dtype)
        res["cache"] = cache
    elif w.kind == "gqla":
        k = torch.zeros((rows, G, w.d_k), dtype=tdt)
        v = torch.zeros((rows, G, w.d_v), dtype=tdt)
        kpe = torch.zeros((rows, w.d_rope), dtype=tdt)
        k[:total] = _normal(rng, (total, G, w.d_k), std, w.dtype)
        v[:total] = _normal(rng, (total, G, w.d_v), std, w.dtype)
        kpe[:total] = _normal(rng, (total, w.d_rope), std, w.dtype)
        res.update(k=k, v=v, kpe=kpe)
    else:
        raise ValueError(w.kind)
    return res


def new_token_rows(w: Workload, seed_offset: int = 1000) -> dict:
    """Rows for the s_q new tokens of every request (the cache-append input).

    mla/gla/gta: [B*s_q, G*d_k + d_R];  gqla: k/v [B*s_q, g, d_h] and kpe [B*s_q, d_R].
    """
    rng = np.random.default_rng(w.seed + seed_offset)
    n = w.batch * w.s_q
    if w.kind in ("mla", "gla", "gta"):
        return {"rows": _normal(rng, (n, w.groups * w.d_k + w.d_rope), w.input_std, w.dtype)}
    return {"k": _normal(rng, (n, w.groups, w.d_k), w.input_std, w.dtype),
            "v": _normal(rng, (n, w.groups, w.d_v), w.input_std, w.dtype),
            "kpe": _normal(rng, (n, w.d_rope), w.input_std, w.dtype)}
