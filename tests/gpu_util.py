"""Helpers shared by the GPU parity tests: run the library through its C ABI and the oracle on
the same seeded inputs, and apply the numeric gates.

Gates (against the fp64 oracle on the identical bf16-rounded inputs):
  bf16 storage: out max-abs <= 1e-2 and rel-L2 <= 5e-3; lse max-abs <= 1e-3
  fp32 storage: out max-abs <= 1e-5 and rel-L2 <= 1e-5; lse max-abs <= 1e-5
"""
import numpy as np
import torch

import oracle
import synth

GATE_BF16 = dict(max_abs=1e-2, rel_l2=5e-3, lse=1e-3)
GATE_FP32 = dict(max_abs=1e-5, rel_l2=1e-5, lse=1e-5)


def to_dev(inputs, dev):
    d = dict(inputs)
    for k in ("q", "q_rope", "cache", "k", "v", "kpe", "cu_seqlens"):
        if k in d:
            d[k] = d[k].to(dev)
    return d


def run_lib(L, d):
    """Call the library entry point for the workload in d (device tensors)."""
    w = d["workload"]
    if w.kind == "mla":
        c = d["cache"]
        return L.mla_absorbed_decode(d["q"], d["q_rope"], c[:, :w.d_k], c[:, w.d_k:],
                                     d["cu_seqlens"], w.scale)
    if w.kind == "gqla":
        return L.gqla_group_decode(d["q"], d["q_rope"], d["k"], d["v"], d["kpe"],
                                   d["cu_seqlens"], w.scale)
    c = d["cache"]
    if w.kind == "gta":
        return L.gta_group_decode(d["q"], d["q_rope"], c[:, :w.groups * w.d_k], c[:, w.groups * w.d_k:],
                                  w.groups, d["cu_seqlens"], w.scale)
    return L.gla_group_decode(d["q"], d["q_rope"], c[:, :w.groups * w.d_k], c[:, w.groups * w.d_k:],
                              w.groups, d["cu_seqlens"], w.scale)


def run_oracle(d, requests=None):
    """Oracle on CPU tensors (the same storage values the GPU saw)."""
    w = d["workload"]
    cu = d["cu_seqlens"].cpu().numpy().astype(np.int64)
    if w.kind == "mla":
        c = d["cache"]
        return oracle.mla_absorbed_decode(d["q"], d["q_rope"], c[:, :w.d_k], c[:, w.d_k:], cu, w.scale,
                                          requests=requests)
    if w.kind == "gqla":
        return oracle.gqla_group_decode(d["q"], d["q_rope"], d["k"], d["v"], d["kpe"], cu, w.scale,
                                        requests=requests)
    c = d["cache"]
    width = w.groups * w.d_k
    if w.kind == "gta":
        return oracle.gta_group_decode(d["q"], d["q_rope"], c[:, :width].contiguous(), c[:, width:], w.groups,
                                       cu, w.scale, requests=requests)
    return oracle.gla_group_decode(d["q"], d["q_rope"], c[:, :width].contiguous(), c[:, width:], w.groups,
                                   cu, w.scale, requests=requests)


def compare(out, lse, ref_out, ref_lse, fp32=False, requests=None, label=""):
    """Apply the gate on the requests given (all by default); returns the measured errors."""
    g = GATE_FP32 if fp32 else GATE_BF16
    o = out.detach().float().cpu().numpy().astype(np.float64)
    l = lse.detach().cpu().numpy().astype(np.float64)
    if requests is not None:
        o, l = o[requests], l[requests]
        ref_out, ref_lse = ref_out[requests], ref_lse[requests]
    assert np.isfinite(o).all(), f"{label}: non-finite output"
    diff = o - ref_out
    max_abs = float(np.abs(diff).max())
    rel = float(np.linalg.norm(diff) / max(np.linalg.norm(ref_out), 1e-300))
    lerr = float(np.abs(l - ref_lse).max())
    msg = f"{label}: max_abs={max_abs:.3e} rel_l2={rel:.3e} lse={lerr:.3e}"
    assert max_abs <= g["max_abs"], msg
    assert rel <= g["rel_l2"], msg
    assert lerr <= g["lse"], msg
    return dict(max_abs=max_abs, rel_l2=rel, lse=lerr)
