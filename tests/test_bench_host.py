"""bench.py on the CPU: the reference arm's JSON line, the CPU baseline, and the algorithmic
bytes and FLOPs behind every roofline fraction (checked against the pinned accounting oracle)."""
import argparse
import os

import numpy as np
import pytest

import bench
import synth
from oracle import accounting as acc


def test_reference_line_keeps_the_contract(monkeypatch):
    calls = []

    def fake_baseline(w, budget, one_thread=True):
        calls.append(budget)
        return {"value": 12.5, "unit": "tokens/s", "cores": 4, "kind": "oracle",
                "sample": f"1 of {w.batch} requests of {w.name} (fp64 numpy oracle)", "seconds": 0.1}

    monkeypatch.setattr(bench, "cpu_baseline", fake_baseline)
    args = argparse.Namespace(steps=2, warmup=3, workload="mla_b64_l4096")
    res = bench.bench_reference(args, 0, 1)
    assert len(calls) == 5                                   # W untimed + K timed samples
    assert res["impl"] == "reference" and res["metric"] == bench.METRIC
    assert res["unit"] == "tokens/s" and res["higher_is_better"] is True and res["value"] == 12.5
    assert res["steps"] == 2 and res["warmup"] == 3 and res["n_gpus"] == 1
    assert res["config"]["workload"] == "mla_b64_l4096"
    assert res["e2e"] == {"value": 12.5, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert res["cpu_baseline"]["kind"] == "oracle" and res["cpu_baseline"]["value"] == 12.5
    assert res["ms_per_step"] == pytest.approx(1e3 * 64 / 12.5)
    assert bench.bench_reference(args, 1, 2) is None          # only rank 0 runs it


def test_cpu_baseline_runs_the_oracle_on_a_bounded_sample():
    cb = bench.cpu_baseline(synth.workload("tiny_fp32_mla"), 0.2)
    assert cb["kind"] == "oracle" and cb["unit"] == "tokens/s" and cb["value"] > 0
    assert cb["cores"] == os.cpu_count()
    assert "of 2 requests of tiny_fp32_mla" in cb["sample"]


@pytest.mark.parametrize("name", ["mla_b64_l4096", "gqla_g8_sq2_l8192", "long_gla2", "gta_g8_sq2_l8192",
                                  "gqa2_sq2_l8192", "tiny_fp32_mla"])
def test_roofline_accounting_matches_the_pinned_oracle(name):
    w = synth.workload(name)
    lengths = np.full(w.batch, w.seqlen, dtype=np.int64)
    cache_bytes, io_bytes, flops = bench.workload_accounting(w, lengths)
    elem = 2 if w.dtype == "bf16" else 4
    want_bytes = acc.step_bytes(w.kind, lengths, w.s_q, w.h_q, w.groups, w.d_k, w.d_v, w.d_rope, elem_bytes=elem)
    assert cache_bytes + io_bytes == want_bytes
    assert flops == acc.step_flops(lengths, w.s_q, w.h_q, w.d_k, w.d_v, w.d_rope)


def test_source_hash_covers_only_the_decode_kernel_sources():
    h = bench.kernel_source_hash("mla")
    assert len(h) == 16
    for f in ("lkv_proj.cu", "lkv_fp8.cu", "lkv_api.cu", "lkv_gemm.cuh"):
        assert f not in bench.DECODE_SOURCES
    assert "lkv_mla_pair.cuh" not in bench.KERNEL_SOURCES["grouped"]
    assert bench.kernel_source_hash("mla") == h                   # deterministic
    assert bench.kernel_source_hash("gqla") == bench.kernel_source_hash("gta") != h
    assert "lkv_decode_swap.cuh" in bench.KERNEL_SOURCES["grouped"]
    assert "lkv_decode_swap.cuh" not in bench.KERNEL_SOURCES["mla"]
    assert "lkv_decode_swap_wide.cuh" in bench.KERNEL_SOURCES["gla"]
    assert "lkv_decode_swap_wide.cuh" not in bench.KERNEL_SOURCES["grouped"]
    assert bench.kernel_source_hash("gla") not in (h, bench.kernel_source_hash("gqla"))


def test_decode_kernel_name_follows_the_launch_rule():
    """GQLA / GTA units of at most 32 query rows and GLA units of at most 64 run keys-in-M."""
    names = {n: bench.decode_kernel_name(synth.workload(n)) for n in synth.WORKLOADS}
    assert names["mla_b64_l4096"] == "mla_pair_kernel"
    assert names["gqla_g8_sq2_l8192"] == "decode_swap_kernel<false>"    # 16 heads x 2 queries
    assert names["long_gqla_g8"] == "decode_swap_kernel<false>"
    assert names["gta_g8_sq2_l8192"] == "decode_swap_kernel<true>"
    assert names["gqa2_sq2_l8192"] == "decode_tc_kernel<MODE_GQLA>"     # 64 heads x 2 queries
    assert names["long_gla2"] == "decode_swap_wide_kernel"              # 64 heads x 1 query


def test_roofline_entry_is_the_slower_of_bytes_and_flops():
    w = synth.workload("mla_b64_l4096")
    lengths = np.full(w.batch, w.seqlen, dtype=np.int64)
    peaks = {"hbm_gbs": 1000.0, "bf16_tflops": 100.0}
    cache_bytes, io_bytes, flops = bench.workload_accounting(w, lengths)
    t_hbm, t_tc = (cache_bytes + io_bytes) / 1e12, flops / 1e14
    r = bench.roofline_entry(w, lengths, 2e3 * max(t_hbm, t_tc), peaks, "test")
    assert r["bound"] == ("hbm" if t_hbm >= t_tc else "tensor")
    assert r["frac"] == pytest.approx(0.5)                  # twice the roofline time
    assert r["roofline_ms"] == pytest.approx(1e3 * max(t_hbm, t_tc))
    assert r["algorithmic_bytes"] == cache_bytes + io_bytes and r["algorithmic_flops"] == flops


@pytest.mark.parametrize("name,kw", [("tiny_fp32_mla", {}),
                                     ("gqla_g8_sq2_l8192", dict(batch=2, seqlen=130)),
                                     ("gta_g8_sq2_l8192", dict(batch=2, seqlen=70)),
                                     ("varlen_mla_sq1", dict(batch=3, len_lo=8, len_hi=64))])
def test_device_inputs_match_the_synth_layout(name, kw):
    import torch
    w = synth.workload(name, **kw)
    d = bench.device_inputs(w, torch.device("cpu"))
    ref = synth.make_inputs(w)
    assert np.array_equal(d["lengths"], ref["lengths"])      # the same length draw
    assert torch.equal(d["cu_seqlens"], ref["cu_seqlens"])
    for k in ("q", "q_rope", "cache", "k", "v", "kpe"):
        if k in ref:
            assert d[k].shape == ref[k][:int(ref["lengths"].sum())].shape if k not in ("q", "q_rope") \
                else d[k].shape == ref[k].shape
            assert d[k].dtype == ref[k].dtype
    x = d["cache"] if "cache" in d else d["k"]
    assert abs(float(x.float().std()) - w.input_std) < 0.1 * w.input_std


def test_cpu_baseline_on_device_inputs_is_bounded():
    import torch
    w = synth.workload("gqla_g8_sq2_l8192", batch=3, seqlen=None, len_lo=16, len_hi=64)
    d = bench.device_inputs(w, torch.device("cpu"))
    cb = bench.cpu_baseline_device(w, d, 0.0)                # budget spent after the first request
    assert cb["kind"] == "oracle" and cb["value"] > 0 and cb["cores"] == os.cpu_count()
    assert cb["sample"].startswith("1 of 3 requests")


@pytest.mark.parametrize("world,rank", [(1, 0), (2, 1), (8, 7)])
def test_tp_local_inputs_hold_one_ranks_groups_and_heads(world, rank):
    """The group-axis TP workload's per-rank inputs: g / world groups of K_j and V_j, the heads of
    those groups, the full RoPE key and the matching h_q / world * d_v rows of W_O."""
    import torch
    from latent_kv_cache_split_b200.tp import group_shard
    w = synth.workload(bench.TP_WORKLOAD, batch=2, seqlen=40)
    sh = group_shard(w.groups, w.h_q, world, rank)
    d = bench.tp_local_inputs(w, sh, torch.device("cpu"), 64)
    T = 2 * 40
    assert d["q"].shape == (2, w.s_q, w.h_q // world, w.d_k)
    assert d["q_rope"].shape == (2, w.s_q, w.h_q // world, w.d_rope)
    assert d["k"].shape == (T, w.groups // world, w.d_k) and d["v"].shape == (T, w.groups // world, w.d_v)
    assert d["kpe"].shape == (T, w.d_rope)
    assert d["w_o"].shape == (w.h_q // world * w.d_v, 64)
    assert d["cu_seqlens"].tolist() == [0, 40, 80]
    assert all(t.dtype == torch.bfloat16 for k, t in d.items() if k not in ("lengths", "cu_seqlens"))


def test_fp8_accounting_counts_the_fp8_rows(lkv_built):
    """The FP8 GTA entry's roofline counts one FP8 row per token (codes, 16-byte scale field, bf16
    RoPE key), the size the library's own row-size call gives, and the bf16 query / output bytes."""
    lkv = lkv_built
    assert bench.fp8_row_bytes(512, 64) == 656 == lkv.fp8_cache_row_bytes(512, 64)
    assert bench.fp8_row_bytes(1024, 64) == 1168 == lkv.fp8_cache_row_bytes(1024, 64)
    w = synth.workload(bench.FP8_BASE)
    lengths = np.full(w.batch, w.seqlen, dtype=np.int64)
    c16, io16, f16 = bench.workload_accounting(w, lengths)
    c8, io8, f8 = bench.workload_accounting(w, lengths, fp8=True)
    assert c8 == int(lengths.sum()) * 1168 and c16 == int(lengths.sum()) * 2176
    assert (io8, f8) == (io16, f16)
    r = bench.roofline_entry(w, lengths, 1.0, {"hbm_gbs": 1000.0, "bf16_tflops": 100.0}, "test", fp8=True)
    assert r["algorithmic_bytes"] == c8 + io8 and r["traffic"] is None
    with pytest.raises(ValueError):
        bench.workload_accounting(synth.workload("gqla_g8_sq2_l8192"), lengths, fp8=True)


def test_cpu_baseline_fp8_reads_the_rows_fields(lkv_built):
    """The FP8 entry's CPU baseline splits the rows into codes, scales and RoPE key with the
    library's field views and runs the oracle's FP8 GTA decode on them: the same result as the
    oracle on the quantised fields it was built from."""
    import torch
    from oracle import fp8
    lkv = lkv_built
    w = synth.workload(bench.FP8_BASE, batch=2, seqlen=None, len_lo=20, len_hi=40)
    d = bench.device_inputs(w, torch.device("cpu"))
    width = w.groups * w.d_k
    codes, scales = fp8.quantize_rows(d["cache"][:, :width].float().numpy())
    rows = torch.zeros((codes.shape[0], bench.fp8_row_bytes(width, w.d_rope)), dtype=torch.uint8)
    rows[:, :width] = torch.from_numpy(codes)
    rows[:, width:width + 4] = torch.from_numpy(scales.view(np.uint8).reshape(-1, 4))
    rows[:, width + 16:width + 16 + 2 * w.d_rope] = d["cache"][:, width:].contiguous().view(torch.uint8)
    c_v, s_v, k_v = lkv.fp8_cache_fields(rows, width, w.d_rope)
    assert np.array_equal(c_v.numpy(), codes) and np.array_equal(s_v.numpy(), scales)
    assert torch.equal(k_v, d["cache"][:, width:])
    cb = bench.cpu_baseline_fp8(w, d, rows, lkv, 0.0)       # budget spent after the first request
    assert cb["kind"] == "oracle" and cb["value"] > 0 and cb["sample"].startswith("1 of 2 requests")


def test_a_failing_guarded_entry_is_recorded_not_raised():
    side = {"x": {"decode_ms": 1.0}}

    def boom():
        raise RuntimeError("device error while timing gta_g8_sq2_l8192_fp8")

    r = bench.add_guarded(side, bench.FP8_NAME, boom)
    assert r == side[bench.FP8_NAME] and r["error"].startswith("RuntimeError: device error")
    assert bench.add_guarded(side, "y", lambda: {"decode_ms": 2.0}) == {"decode_ms": 2.0}
    assert side["x"] == {"decode_ms": 1.0}
