"""Pin the byte/FLOP accounting to the figures the pages print (tests/golden/page_figures.json)."""
import json
import os

import numpy as np
import pytest

from oracle import accounting as acc

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")))


def _close(got, entry):
    want = entry["value"]
    tol = entry["rel_tol"]
    assert abs(got - want) <= tol * abs(want) + 1e-15, (got, want, entry["cite"])


def test_absorbed_cache_fraction():
    e = GOLD["absorbed_cache_fraction_vs_llama3_8b_gqa"]
    s = e["setting"]
    mla = acc.cache_bytes_per_token("mla", 1, s["r_kv"], s["r_kv"], s["d_rope"])
    # LLaMA-3-8B GQA: K and V for 8 KV heads of 128, no separate RoPE key.
    gqa = acc.cache_bytes_per_token("gqla", s["gqa_kv_heads"], s["d_h"], s["d_h"], 0)
    _close(mla / gqa, e)


def test_absorbed_intensity():
    e = GOLD["absorbed_path_intensity_sq1"]
    s = e["setting"]
    ai = acc.intensity_per_token("mla", s["h_q"], s["s_q"], 1, s["r_kv"], s["r_kv"], s["d_rope"])
    _close(ai, e)


@pytest.mark.parametrize("key", ["gqa_path_intensity_g8_sq2", "gqa_path_intensity_g4_sq1"])
def test_gqa_intensity(key):
    e = GOLD[key]
    s = e["setting"]
    ai = acc.intensity_per_token("gqla", s["h_q"], s["s_q"], s["g"], s["d_h"], s["d_h"], s["d_rope"])
    _close(ai, e)


def test_gta_cache_fraction():
    """Tied groups store g*d_h + d_R per token against GQA's 2*g*d_h + d_R."""
    e = GOLD["gta_cache_fraction_vs_gqa"]
    s = e["setting"]
    gta = acc.cache_bytes_per_token("gta", s["g"], s["d_h"], s["d_h"], s["d_rope"])
    gqa = acc.cache_bytes_per_token("gqla", s["g"], s["d_h"], s["d_h"], s["d_rope"])
    assert gta == 2 * (s["g"] * s["d_h"] + s["d_rope"])
    _close(1 - gta / gqa, e)


def test_heads_per_group():
    e = GOLD["gqla_heads_per_group"]
    _close(e["setting"]["h_q"] // e["setting"]["g"], e)


def test_step_flops_counts_only_visible_pairs():
    # lengths 4 and 2, s_q = 2: visible pairs (3 + 4) + (1 + 2) = 10 per head
    f = acc.step_flops([4, 2], 2, 3, 5, 7, 2)
    assert f == 10 * 2 * 3 * (5 + 2 + 7)


def test_step_bytes_components():
    b = acc.step_bytes("mla", [10, 20], 1, 4, 1, 8, 8, 2)
    cache = 30 * (8 + 2) * 2
    q = 2 * 1 * 4 * (8 + 2) * 2
    out = 2 * 1 * 4 * 8 * 2
    lse = 2 * 1 * 4 * 4
    assert b == cache + q + out + lse
