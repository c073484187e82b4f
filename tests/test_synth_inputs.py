"""The seeded input module: determinism, shapes, storage rounding, length recipe."""
import math

import numpy as np
import torch

import synth


def test_bf16_rounding_is_nearest_even():
    vals = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -9, -2.0 - 2.0 ** -7],
                    dtype=np.float32)
    got = synth.to_bf16(vals).float().numpy()
    # bf16 keeps 8 significant bits: ties go to the even mantissa
    assert got.tolist() == [1.0, 1.0 + 2.0 ** -6, 1.0, -2.0]


def test_inputs_are_deterministic_and_shaped():
    w = synth.workload("tiny_fp32_mla")
    a = synth.make_inputs(w)
    b = synth.make_inputs(w)
    assert torch.equal(a["q"], b["q"]) and torch.equal(a["cache"], b["cache"])
    assert a["q"].shape == (2, 1, 16, 64) and a["q_rope"].shape == (2, 1, 16, 16)
    assert a["cache"].shape == (512, 80) and a["cache"].dtype == torch.float32
    assert a["cu_seqlens"].tolist() == [0, 256, 512]
    assert abs(w.scale - 1 / math.sqrt(80)) < 1e-15


def test_gqla_layout_and_extra_rows():
    w = synth.workload("gqla_g8_sq2_l8192", batch=2, seqlen=40)
    d = synth.make_inputs(w, extra_rows=5)
    assert d["k"].shape == (85, 8, 128) and d["v"].shape == (85, 8, 128)
    assert d["kpe"].shape == (85, 64) and d["k"].dtype == torch.bfloat16
    assert not d["k"][80:].any()
    assert d["q"].shape == (2, 2, 128, 128)


def test_varlen_lengths_recipe():
    w = synth.workload("varlen_mla_sq1")
    rng = np.random.default_rng(w.seed)
    L = synth.draw_lengths(rng, w.batch, w.len_lo, w.len_hi)
    assert L.min() >= 1024 and L.max() <= 65536 and len(L) == 128
    # log-uniform: the median of log2(L) sits near the middle of [10, 16]
    assert 12 < np.median(np.log2(L)) < 14
    cu = synth.prefix_offsets(L)
    assert cu[0] == 0 and cu[-1] == L.sum()


def test_scaled_inputs_have_stated_std():
    w = synth.workload("mla_b64_l4096", batch=2, seqlen=2048)
    d = synth.make_inputs(w)
    std = d["cache"][:, :512].float().std().item()
    assert abs(std - 1 / 24) < 1e-3
