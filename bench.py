"""Benchmark: decode-attention tokens/s on one B200 (or N, data parallel) through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one whole decode step of the hot path on one batch: append the s_q new cache rows
of every request, then decode attention over the full cache (range planning, tensor-core
split-KV kernel, split combine).  Inputs are seeded synthetic tensors resident in HBM before
the timed region; the cache (0.30 GB for the default workload) is larger than the 126 MB L2,
so the timed steps run back to back with no flush.  Timing: CUDA events on the launching stream
over exactly K steps, bracketed by a barrier and a device synchronise, max over ranks.  Rank 0
prints one JSON line.

The same line carries, under "workloads", every other decode workload of the build timed on its
own (the decode call alone, CUDA events, a 256 MB L2-flushing write before each call and outside
its events), with its roofline fraction and a bounded sample of the CPU oracle on the same
inputs; and, for the headline workload, the decode call timed the same flushed way.

`--impl reference` times the fp64 CPU oracle (the correctness reference) on the host cores,
on a bounded sample of the same workload; under torchrun only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "decode attn tokens/s; KV-cache GB/s & TFLOPS as fraction of B200 roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Datasheet figures (HGX B200, dense bf16), reported beside the measured-peak fraction: the fraction
# of the roofline time max(bytes / HBM, FLOPs / tensor) that the decode call achieves.
NOMINAL_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}


# The sources the decode kernels and their launch are built from (the projections' translation unit
# and the header's declarations do not change what a decode launch reads or writes).
# Device sources of each decode kernel: a traffic figure measured with ncu is only reported while the
# kernel it was measured on is unchanged (host code and the other kernels do not count).
KERNEL_SOURCES = {
    "mla": ("lkv_mla_pair.cuh", "lkv_decode_tc.cuh", "lkv_ptx.cuh", "lkv_sched.cuh"),  # with the shared TMEM row helpers
    "grouped": ("lkv_decode_swap.cuh", "lkv_decode_tc.cuh", "lkv_ptx.cuh", "lkv_sched.cuh"),
    "gla": ("lkv_decode_swap_wide.cuh", "lkv_decode_swap.cuh", "lkv_decode_tc.cuh", "lkv_ptx.cuh", "lkv_sched.cuh"),
}
DECODE_SOURCES = tuple(sorted({f for v in KERNEL_SOURCES.values() for f in v}))


def kernel_source_hash(kind: str = "mla") -> str:
    """Hash of the CUDA sources of the decode kernel that a workload of this kind launches
    ("mla" for the CTA-pair kernel, "gla" for the GLA kernels, anything else for the grouped one)."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kind if kind in ("mla", "gla") else "grouped"]:
        h.update(f.encode())
        with open(os.path.join(ROOT, "latent_kv_cache_split_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


SWAP_MAX_ROWS = 32  # GQLA / GTA units of at most this many query rows run keys-in-M
WIDE_MAX_ROWS = 64  # GLA units of at most this many query rows run keys-in-M


def decode_kernel_name(w) -> str:
    """The tensor-core kernel a bf16 decode call of this workload launches."""
    if w.kind == "mla":
        return "mla_pair_kernel"
    rows = (w.h_q // w.groups) * w.s_q
    if w.kind in ("gqla", "gta") and rows <= SWAP_MAX_ROWS:
        return "decode_swap_kernel<%s>" % ("true" if w.kind == "gta" else "false")
    if w.kind == "gla" and rows <= WIDE_MAX_ROWS:
        return "decode_swap_wide_kernel"
    return {"gqla": "decode_tc_kernel<MODE_GQLA>", "gla": "decode_tc_kernel<MODE_GLA>",
            "gta": "decode_tc_kernel<MODE_GTA>"}.get(w.kind, "decode_tc_kernel")


def measured_traffic(workload: str):
    """DRAM bytes (read + write) per decode-kernel launch from an ncu capture recorded in
    profiles/traffic.json, or None when absent or taken on other kernel sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    entry = json.load(open(p)).get(workload)
    if not entry or entry.get("kernel_hash") != kernel_source_hash(synth.workload(workload).kind):
        return None
    return entry.get("dram_bytes_per_launch")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def shard_requests(batch: int, rank: int, world: int):
    """Weak scaling: every rank decodes its own full batch; returns the global request ids of
    this rank (disjoint across ranks)."""
    return list(range(rank * batch, (rank + 1) * batch))


def reduce_max(x: float, world: int, device) -> float:
    """Max of x over ranks (the job's time is its slowest rank's time)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, ms_this_rank: float, world: int, device):
    """Whole-job tokens/s: all ranks' tokens over the slowest rank's time."""
    ms = reduce_max(ms_this_rank, world, device)
    return tokens_per_rank * world / (ms * 1e-3), ms


def fp8_row_bytes(width: int, d_rope: int) -> int:
    """Bytes of one FP8 cache row: width e4m3 codes, the fp32 scale padded to 16 bytes, the bf16
    RoPE key, rounded up to 16 bytes (656 for the 512-wide MLA latent, 1168 for GTA's 8 x 128)."""
    return 16 * ((width + 16 + 2 * d_rope + 15) // 16)


def workload_accounting(w, lengths, fp8: bool = False):
    """Algorithmic bytes (cache rows once, q, out, lse) and FLOPs (visible query-key pairs).
    fp8: the latent / tied-state rows are FP8 cache rows (fp8_row_bytes per token)."""
    lengths = np.asarray(lengths, dtype=np.int64)
    elem = 2 if w.dtype == "bf16" else 4
    if fp8:
        if w.kind not in ("mla", "gla", "gta"):
            raise ValueError("FP8 rows hold a latent or tied-state cache")
        cache_bytes = int(lengths.sum()) * fp8_row_bytes(w.groups * w.d_k, w.d_rope)
    else:
        row = (w.groups * w.d_k if w.kind in ("mla", "gla", "gta") else w.groups * (w.d_k + w.d_v)) + w.d_rope
        cache_bytes = int(lengths.sum()) * row * elem
    io_bytes = w.batch * w.s_q * w.h_q * ((w.d_k + w.d_rope) * elem + w.d_v * elem + 4)
    vis = sum(int((lengths - w.s_q + i + 1).sum()) for i in range(w.s_q))
    flops = vis * 2 * w.h_q * (w.d_k + w.d_rope + w.d_v)
    return cache_bytes, io_bytes, flops


# The other workloads timed beside the headline: the five configurations' remaining shapes and the
# tied / narrow-group variants.
SIDE_WORKLOADS = ("tiny_fp32_mla", "gqla_g8_sq2_l8192", "varlen_mla_sq1", "varlen_mla_sq2", "long_gla2",
                  "long_mla", "long_gqla_g8", "gta_g8_sq2_l8192", "gqa2_sq2_l8192")
L2_FLUSH_BYTES = 256 << 20   # twice the 126 MB L2


def roofline_entry(w, lengths, dec_ms, peaks, how, fp8: bool = False):
    """Algorithmic bytes / FLOPs of one decode call and the fraction of the roofline time
    max(bytes / HBM peak, FLOPs / tensor peak) that a call of dec_ms milliseconds achieves.
    fp8: the cache is FP8 rows (no ncu traffic figure is recorded for that kernel)."""
    cache_bytes, io_bytes, flops = workload_accounting(w, lengths, fp8=fp8)
    alg_bytes = cache_bytes + io_bytes
    dec_s = dec_ms * 1e-3
    gbs = alg_bytes / dec_s / 1e9
    tfl = flops / dec_s / 1e12
    t_hbm = alg_bytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    bound = "hbm" if t_hbm >= t_tc else "tensor"
    achieved = gbs if bound == "hbm" else tfl
    peak = peaks["hbm_gbs"] if bound == "hbm" else peaks["bf16_tflops"]
    nominal = max(alg_bytes / (NOMINAL_PEAKS["hbm_gbs"] * 1e9), flops / (NOMINAL_PEAKS["bf16_tflops"] * 1e12)) / dec_s
    return {"bound": bound, "achieved": achieved, "peak": peak, "unit": "GB/s" if bound == "hbm" else "TFLOP/s",
            "frac": achieved / peak, "traffic": None if fp8 else measured_traffic(w.name),
            "peak_source": f"{how} (MEASURED_PEAKS.json burst)", "nominal": {"frac": nominal},
            "roofline_ms": max(t_hbm, t_tc) * 1e3, "algorithmic_bytes": alg_bytes, "algorithmic_flops": flops,
            "kv_gbs": gbs, "tflops": tfl}


def device_inputs(w, dev):
    """Seeded synthetic inputs of workload w drawn on the device (torch's generator seeded with the
    workload's seed): the shapes, layout and value distribution of synth.make_inputs, without the
    host draw and copy of multi-GB caches.  Lengths come from synth (the same draw)."""
    g = torch.Generator(device=dev)
    g.manual_seed(1000 + w.seed)
    if w.seqlen is None:
        lengths = synth.draw_lengths(np.random.default_rng(w.seed), w.batch, w.len_lo, w.len_hi)
    else:
        lengths = np.full(w.batch, w.seqlen, dtype=np.int64)
    cu = synth.prefix_offsets(lengths)
    T = int(cu[-1])
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    def randn(*shape, std):
        return torch.randn(*shape, generator=g, device=dev, dtype=dt).mul_(std)

    qs = w.input_std if w.q_std is None else w.q_std
    d = {"workload": w, "lengths": lengths, "cu_seqlens": torch.from_numpy(cu.astype(np.int32)).to(dev),
         "q": randn(w.batch, w.s_q, w.h_q, w.d_k, std=qs), "q_rope": randn(w.batch, w.s_q, w.h_q, w.d_rope, std=qs)}
    if w.kind == "gqla":
        d["k"] = randn(T, w.groups, w.d_k, std=w.input_std)
        d["v"] = randn(T, w.groups, w.d_v, std=w.input_std)
        d["kpe"] = randn(T, w.d_rope, std=w.input_std)
    else:
        d["cache"] = randn(T, w.groups * w.d_k + w.d_rope, std=w.input_std)
    return d


def make_decoder(lkv, w, d, nsm):
    """decode(q, q_rope, out, lse) for workload w over the cache tensors in d, workspace allocated here."""
    dev = d["q"].device
    B, S = w.batch, w.s_q
    if w.kind == "mla":
        ws = torch.empty(lkv.mla_decode_workspace_size(B, S, w.h_q, w.d_k, nsm), dtype=torch.uint8, device=dev)
    else:
        kind = {"gqla": lkv.KIND_GQLA, "gla": lkv.KIND_GLA, "gta": lkv.KIND_GTA}[w.kind]
        ws = torch.empty(lkv.group_decode_workspace_size(kind, B, S, w.h_q, w.groups, w.d_v, nsm),
                         dtype=torch.uint8, device=dev)
    cu = d["cu_seqlens"]
    if w.kind == "gqla":
        k, v, kpe = d["k"], d["v"], d["kpe"]
    else:
        width = w.groups * w.d_k
        lat, kpe = d["cache"][:, :width], d["cache"][:, width:]

    def decode(qq, qqr, o, l):
        if w.kind == "mla":
            lkv.mla_absorbed_decode(qq, qqr, lat, kpe, cu, w.scale, out=o, lse=l, workspace=ws)
        elif w.kind == "gqla":
            lkv.gqla_group_decode(qq, qqr, k, v, kpe, cu, w.scale, out=o, lse=l, workspace=ws)
        elif w.kind == "gta":
            lkv.gta_group_decode(qq, qqr, lat, kpe, w.groups, cu, w.scale, out=o, lse=l, workspace=ws)
        else:
            lkv.gla_group_decode(qq, qqr, lat, kpe, w.groups, cu, w.scale, out=o, lse=l, workspace=ws)
    return decode


TP_WORKLOAD = "gqla_g8_sq2_l8192"
TP_D_MODEL = 7168   # model width the output projection maps the heads' outputs back to


def tp_local_inputs(w, sh, dev, d_model: int):
    """One rank's share of the group-axis TP step, drawn on the device (seeded by workload and rank):
    the query heads of its groups, the expanded K_j, V_j of its groups, the RoPE key every rank
    keeps, and the rows of W_O [h_q * d_v, d_model] that multiply its heads."""
    g = torch.Generator(device=dev)
    g.manual_seed(2000 + 17 * w.seed + sh.rank)
    lengths = np.full(w.batch, w.seqlen, dtype=np.int64)
    cu = synth.prefix_offsets(lengths)
    T = int(cu[-1])

    def randn(*shape, std):
        return torch.randn(*shape, generator=g, device=dev, dtype=torch.bfloat16).mul_(std)

    return {"lengths": lengths, "cu_seqlens": torch.from_numpy(cu.astype(np.int32)).to(dev),
            "q": randn(w.batch, w.s_q, sh.heads, w.d_k, std=w.input_std),
            "q_rope": randn(w.batch, w.s_q, sh.heads, w.d_rope, std=w.input_std),
            "k": randn(T, sh.groups, w.d_k, std=w.input_std), "v": randn(T, sh.groups, w.d_v, std=w.input_std),
            "kpe": randn(T, w.d_rope, std=w.input_std),
            "w_o": randn(sh.heads * w.d_v, d_model, std=(w.h_q * w.d_v) ** -0.5)}


def bench_tp(lkv, dev, rank: int, world: int, steps: int, warmup: int):
    """Group-axis tensor parallelism of the GQA path (GQLA explainer, section 2): the GQLA decode
    step of one fixed batch with its g groups split over the ranks, each rank's heads projected by
    its rows of W_O and the partial outputs summed by one NCCL all-reduce.  Total work is fixed
    (strong scaling).  Times are device times, the max over ranks: the whole step, and the decode,
    the projection and the all-reduce each timed alone."""
    from latent_kv_cache_split_b200.tp import GroupAxisTP, group_shard
    w = synth.workload(TP_WORKLOAD)
    if w.groups % world:
        return {"workload": w.name, "tp": world, "skipped": f"{world} ranks do not divide g = {w.groups}"}
    sh = group_shard(w.groups, w.h_q, world, rank)
    d = tp_local_inputs(w, sh, dev, TP_D_MODEL)
    B, S = w.batch, w.s_q
    nsm = torch.cuda.get_device_properties(dev).multi_processor_count
    ws = torch.empty(lkv.group_decode_workspace_size(lkv.KIND_GQLA, B, S, sh.heads, sh.groups, w.d_v, nsm),
                     dtype=torch.uint8, device=dev)
    out = torch.empty((B, S, sh.heads, w.d_v), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, S, sh.heads), dtype=torch.float32, device=dev)
    y = torch.empty((B * S, TP_D_MODEL), dtype=torch.float32, device=dev)

    def decode_fn(q, qr, k, v, kpe, cu, scale):
        lkv.gqla_group_decode(q, qr, k, v, kpe, cu, scale, out=out, lse=lse, workspace=ws)
        return out, lse

    def proj_fn(o, w_o):
        return lkv.output_projection(o, w_o, out=y)

    tp = GroupAxisTP(sh, decode_fn=decode_fn, proj_fn=proj_fn)
    args_ = (d["q"], d["q_rope"], d["k"], d["v"], d["kpe"], d["cu_seqlens"], w.scale, d["w_o"])
    stream = torch.cuda.current_stream(dev)

    def sync_all():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize(dev)

    def timed(fn, n):
        sync_all()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        sync_all()
        return reduce_max(e0.elapsed_time(e1) / n, world, dev)

    for _ in range(warmup):
        tp.step(*args_)
    step_ms = timed(lambda: tp.step(*args_), steps)
    dec_ms = timed(lambda: decode_fn(*args_[:7]), steps)
    o2 = out.reshape(B * S, sh.heads * w.d_v)
    proj_ms = timed(lambda: proj_fn(o2, d["w_o"]), steps)
    ar_ms = timed(lambda: tp.allreduce_fn(y), steps)
    if lkv.check_device() != 0:
        raise RuntimeError("device error in the group-axis TP step")
    return {"workload": w.name, "tp": world, "groups_per_rank": sh.groups, "heads_per_rank": sh.heads,
            "d_model": TP_D_MODEL, "scaling": "strong", "steps": steps,
            "tokens_per_s": B * S / (step_ms * 1e-3), "ms_per_step": step_ms,
            "decode_ms": dec_ms, "projection_ms": proj_ms, "allreduce_ms": ar_ms,
            "allreduce_bytes": B * S * TP_D_MODEL * 4,
            "collective": "torch.distributed all_reduce (NCCL) of the fp32 partial projection" if world > 1
            else "none (one rank)"}


def time_flushed(decode, args_, stream, flush, iters: int):
    """Per-call decode times (ms): each call preceded by an L2-flushing write outside its events."""
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
    for e0, e1 in ev:
        flush.zero_()
        e0.record(stream)
        decode(*args_)
        e1.record(stream)
    torch.cuda.synchronize()
    return [e0.elapsed_time(e1) for e0, e1 in ev]


def cpu_baseline_device(w, d, budget_s: float):
    """The oracle as it stands on the host cores, on a bounded sample (whole requests, shortest
    first) of the device-drawn inputs d, copied to the host request by request."""
    import oracle
    cu = d["cu_seqlens"].cpu().numpy().astype(np.int64)
    order = [int(b) for b in np.argsort(d["lengths"], kind="stable")]
    t0 = time.perf_counter()
    done = keys = 0
    for b in order:
        c0, c1 = int(cu[b]), int(cu[b + 1])
        one = np.array([0, c1 - c0], dtype=np.int64)
        q, qr = d["q"][b:b + 1].cpu(), d["q_rope"][b:b + 1].cpu()
        if w.kind == "gqla":
            oracle.gqla_group_decode(q, qr, d["k"][c0:c1].cpu(), d["v"][c0:c1].cpu(), d["kpe"][c0:c1].cpu(), one,
                                     w.scale)
        else:
            c = d["cache"][c0:c1].cpu()
            width = w.groups * w.d_k
            if w.kind == "mla":
                oracle.mla_absorbed_decode(q, qr, c[:, :width], c[:, width:], one, w.scale)
            elif w.kind == "gta":
                oracle.gta_group_decode(q, qr, c[:, :width], c[:, width:], w.groups, one, w.scale)
            else:
                oracle.gla_group_decode(q, qr, c[:, :width], c[:, width:], w.groups, one, w.scale)
        done += 1
        keys += c1 - c0
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": done * w.s_q / dt, "unit": "tokens/s", "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{done} of {w.batch} requests ({keys} cached tokens) of {w.name}, shortest first "
                      "(fp64 numpy oracle)", "seconds": dt}


def bench_side_workloads(lkv, dev, names, iters: int, cpu_budget: float):
    """Decode time, roofline fraction and a bounded CPU-oracle sample for each workload in names."""
    peaks, how = load_peaks()
    nsm = torch.cuda.get_device_properties(dev).multi_processor_count
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    res = {}
    for name in names:
        w = synth.workload(name)
        d = device_inputs(w, dev)
        out = torch.empty((w.batch, w.s_q, w.h_q, w.d_v), dtype=d["q"].dtype, device=dev)
        lse = torch.empty((w.batch, w.s_q, w.h_q), dtype=torch.float32, device=dev)
        decode = make_decoder(lkv, w, d, nsm)
        for _ in range(3):
            decode(d["q"], d["q_rope"], out, lse)
        if lkv.check_device() != 0:
            raise RuntimeError(f"device error during warm-up of {name}")
        ms = time_flushed(decode, (d["q"], d["q_rope"], out, lse), stream, flush, iters)
        if lkv.check_device() != 0:
            raise RuntimeError(f"device error while timing {name}")
        med = float(np.median(ms))
        entry = {"decode_ms": med, "decode_ms_min": float(min(ms)), "decode_ms_max": float(max(ms)),
                 "calls": iters, "tokens_per_s": w.batch * w.s_q / (med * 1e-3), "dtype": w.dtype,
                 "shape": {"kind": w.kind, "batch": w.batch, "s_q": w.s_q, "h_q": w.h_q, "groups": w.groups,
                           "d_k": w.d_k, "d_v": w.d_v, "d_rope": w.d_rope, "seqlen": w.seqlen,
                           "total_cached_tokens": int(d["lengths"].sum())},
                 "roofline": roofline_entry(w, d["lengths"], med, peaks, how),
                 "cpu_baseline": cpu_baseline_device(w, d, cpu_budget)}
        if w.dtype == "fp32":
            entry["roofline"]["note"] = "latency-bound CUDA-core fp32 path (0.18 MB); not gated on the roofline"
        res[name] = entry
        del d, out, lse, decode
        torch.cuda.empty_cache()
    return res


# The GTA workload with its tied states stored as FP8 cache rows (e4m3 codes, a power-of-two fp32
# scale per token, the bf16 RoPE key), quantised on the device by the library before timing.
FP8_BASE = "gta_g8_sq2_l8192"
FP8_NAME = "gta_g8_sq2_l8192_fp8"


def cpu_baseline_fp8(w, d, rows, lkv, budget_s: float):
    """The oracle's FP8 GTA decode (dequantise, then the plain attention) on the host cores, on a
    bounded sample (whole requests) of the device-quantised rows."""
    import oracle
    width = w.groups * w.d_k
    codes_v, scales_v, kpe_v = lkv.fp8_cache_fields(rows, width, w.d_rope)
    cu = d["cu_seqlens"].cpu().numpy().astype(np.int64)
    t0 = time.perf_counter()
    done = keys = 0
    for b in range(w.batch):
        c0, c1 = int(cu[b]), int(cu[b + 1])
        one = np.array([0, c1 - c0], dtype=np.int64)
        oracle.fp8.gta_group_decode_fp8(d["q"][b:b + 1].cpu(), d["q_rope"][b:b + 1].cpu(),
                                        codes_v[c0:c1].contiguous().cpu().numpy(),
                                        scales_v[c0:c1].contiguous().cpu().numpy(),
                                        kpe_v[c0:c1].contiguous().cpu(), w.groups, one, w.scale)
        done += 1
        keys += c1 - c0
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": done * w.s_q / dt, "unit": "tokens/s", "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{done} of {w.batch} requests ({keys} cached tokens) of {FP8_NAME} (fp64 numpy oracle "
                      "over the dequantised rows)", "seconds": dt}


def add_guarded(side: dict, name: str, fn):
    """side[name] = fn(); an exception is recorded there as {"error": "<type>: <message>"} instead of
    ending the run (the entry is reported, not hidden)."""
    try:
        side[name] = fn()
    except Exception as e:  # noqa: BLE001
        side[name] = {"error": f"{type(e).__name__}: {e}"[:300]}
    return side[name]


def bench_fp8_gta(lkv, dev, iters: int, cpu_budget: float):
    """lkv_gta_group_decode_fp8 on the GTA workload's shape (64 requests of 8192 keys, s_q = 2,
    g = 8): the device-drawn bf16 tied states and RoPE key quantised into FP8 rows by
    lkv_quantize_latent_fp8, then each decode call timed after an L2 flush like the other workloads.
    The roofline counts the FP8 rows' bytes (1168 per token against 2176 in bf16)."""
    w = synth.workload(FP8_BASE)
    peaks, how = load_peaks()
    nsm = torch.cuda.get_device_properties(dev).multi_processor_count
    stream = torch.cuda.current_stream(dev)
    d = device_inputs(w, dev)
    width = w.groups * w.d_k
    rows = lkv.quantize_latent_fp8(d.pop("cache"), width)
    torch.cuda.empty_cache()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    ws = torch.empty(lkv.group_decode_workspace_size(lkv.KIND_GTA, w.batch, w.s_q, w.h_q, w.groups, w.d_v, nsm),
                     dtype=torch.uint8, device=dev)
    out = torch.empty((w.batch, w.s_q, w.h_q, w.d_v), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.batch, w.s_q, w.h_q), dtype=torch.float32, device=dev)
    cu = d["cu_seqlens"]

    def decode(qq, qqr, o, l):
        lkv.gta_group_decode_fp8(qq, qqr, rows, w.groups, cu, w.scale, out=o, lse=l, workspace=ws)

    for _ in range(3):
        decode(d["q"], d["q_rope"], out, lse)
    if lkv.check_device() != 0:
        raise RuntimeError(f"device error during warm-up of {FP8_NAME}")
    ms = time_flushed(decode, (d["q"], d["q_rope"], out, lse), stream, flush, iters)
    if lkv.check_device() != 0:
        raise RuntimeError(f"device error while timing {FP8_NAME}")
    med = float(np.median(ms))
    return {"decode_ms": med, "decode_ms_min": float(min(ms)), "decode_ms_max": float(max(ms)), "calls": iters,
            "tokens_per_s": w.batch * w.s_q / (med * 1e-3),
            "dtype": "bf16 (cache rows e4m3 + power-of-two scale, dequantised in shared memory)",
            "kernel": "decode_tc_kernel<MODE_GTA8> + split combine (one lkv_gta_group_decode_fp8 call)",
            "shape": {"kind": "gta", "batch": w.batch, "s_q": w.s_q, "h_q": w.h_q, "groups": w.groups,
                      "d_k": w.d_k, "d_v": w.d_v, "d_rope": w.d_rope, "seqlen": w.seqlen,
                      "fp8_row_bytes": fp8_row_bytes(width, w.d_rope),
                      "total_cached_tokens": int(d["lengths"].sum())},
            "roofline": roofline_entry(w, d["lengths"], med, peaks, how, fp8=True),
            "cpu_baseline": cpu_baseline_fp8(w, d, rows, lkv, cpu_budget)}


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the GPU works (200 ms period)."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.rows = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.rows.append(parts)

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=2)

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in self.rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in self.rows if num(r[2]) is not None]
        load = [s for s in sm if mx and s > 0.5 * max(mx)] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(load) if load else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(self.rows)}


def bench_gpu(args, rank, world, local_rank):
    import latent_kv_cache_split_b200 as lkv
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    w = synth.workload(args.workload)
    d = synth.make_inputs(w)
    new = synth.new_token_rows(w)
    lengths = d["lengths"]
    cu = d["cu_seqlens"].to(dev)
    q = d["q"].to(dev)
    qr = d["q_rope"].to(dev)
    B, S = w.batch, w.s_q
    if w.kind in ("mla", "gla", "gta"):
        cache = d["cache"].to(dev)
        width = w.groups * w.d_k
        lat, kpe = cache[:, :width], cache[:, width:]
        new_rows = new["rows"].to(dev)
    else:
        k, v, kpe = d["k"].to(dev), d["v"].to(dev), d["kpe"].to(dev)
        new_k, new_v, new_kpe = new["k"].to(dev), new["v"].to(dev), new["kpe"].to(dev)
    out = torch.empty((B, S, w.h_q, w.d_v), dtype=q.dtype, device=dev)
    lse = torch.empty((B, S, w.h_q), dtype=torch.float32, device=dev)
    nsm = torch.cuda.get_device_properties(dev).multi_processor_count
    if w.kind == "mla":
        ws = torch.empty(lkv.mla_decode_workspace_size(B, S, w.h_q, w.d_k, nsm), dtype=torch.uint8, device=dev)
    else:
        kind = {"gqla": lkv.KIND_GQLA, "gla": lkv.KIND_GLA, "gta": lkv.KIND_GTA}[w.kind]
        ws = torch.empty(lkv.group_decode_workspace_size(kind, B, S, w.h_q, w.groups, w.d_v, nsm),
                         dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    launches_per_step = 3 if w.kind != "gqla" else 5   # append(s) + decode + combine

    def append():
        if w.kind in ("mla", "gla", "gta"):
            lkv.latent_cache_append(new_rows, cache, cu, S)
        else:
            lkv.latent_cache_append(new_k, k, cu, S)
            lkv.latent_cache_append(new_v, v, cu, S)
            lkv.latent_cache_append(new_kpe, kpe, cu, S)

    def decode(qq, qqr, o, l):
        if w.kind == "mla":
            lkv.mla_absorbed_decode(qq, qqr, lat, kpe, cu, w.scale, out=o, lse=l, workspace=ws)
        elif w.kind == "gqla":
            lkv.gqla_group_decode(qq, qqr, k, v, kpe, cu, w.scale, out=o, lse=l, workspace=ws)
        elif w.kind == "gta":
            lkv.gta_group_decode(qq, qqr, lat, kpe, w.groups, cu, w.scale, out=o, lse=l, workspace=ws)
        else:
            lkv.gla_group_decode(qq, qqr, lat, kpe, w.groups, cu, w.scale, out=o, lse=l, workspace=ws)

    def step():
        append()
        decode(q, qr, out, lse)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize(dev)

    sampler = ClockSampler(dev.index if dev.index is not None else 0) if rank == 0 else None
    for _ in range(args.warmup):
        step()
    if lkv.check_device() != 0:
        raise RuntimeError("device error during warm-up")
    if sampler:
        sampler.start()
        time.sleep(0.3)
    # ---- timed region: exactly K steps, per-step events around the decode call as well
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ev_d = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    barrier()
    t0.record(stream)
    for i in range(args.steps):
        ev_s[i].record(stream)
        append()
        ev_d[i].record(stream)
        decode(q, qr, out, lse)
        ev_e[i].record(stream)
    t1.record(stream)
    barrier()
    total_ms = t0.elapsed_time(t1)
    dec_ms = [ev_d[i].elapsed_time(ev_e[i]) for i in range(args.steps)]
    if sampler:
        time.sleep(0.2)
        sampler.stop()
    err = lkv.check_device()
    if err != 0:
        raise RuntimeError(f"device error word {err} after the timed region")
    value, total_ms = job_throughput(B * S * args.steps, total_ms, world, dev)
    dec_avg_ms = reduce_max(float(np.mean(dec_ms)), world, dev)

    # ---- end to end through the public API: host inputs in, host result out, every step
    q_h = d["q"].pin_memory()
    qr_h = d["q_rope"].pin_memory()
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    lse_h = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    q_d = torch.empty_like(q)
    qr_d = torch.empty_like(qr)
    if w.kind in ("mla", "gla", "gta"):
        rows_h = new["rows"].pin_memory()
        step_in = [(rows_h, new_rows)]
    else:
        step_in = [(new["k"].pin_memory(), new_k), (new["v"].pin_memory(), new_v),
                   (new["kpe"].pin_memory(), new_kpe)]
    h2d = (q_h.numel() * q_h.element_size() + qr_h.numel() * qr_h.element_size()
           + sum(h.numel() * h.element_size() for h, _ in step_in))
    d2h = out_h.numel() * out_h.element_size() + lse_h.numel() * lse_h.element_size()
    e2e_steps = max(3, min(args.steps, 200))

    def e2e_step():
        q_d.copy_(q_h, non_blocking=True)
        qr_d.copy_(qr_h, non_blocking=True)
        for h, dd in step_in:
            dd.copy_(h, non_blocking=True)
        append()
        decode(q_d, qr_d, out, lse)
        out_h.copy_(out, non_blocking=True)
        lse_h.copy_(lse, non_blocking=True)

    def time_e2e(step_fn, tail_stream=None):
        for n in range(2):
            step_fn(n)
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for n in range(e2e_steps):
            step_fn(n)
        if tail_stream is not None:
            stream.wait_stream(tail_stream)
        e1.record(stream)
        barrier()
        return reduce_max(e0.elapsed_time(e1), world, dev) / e2e_steps

    e2e_serial_ms = time_e2e(lambda n: e2e_step())

    # Pipelined: step n copies its inputs in on s_in, appends and decodes on the compute stream and
    # copies its result out on s_out, so the copies of neighbouring steps overlap its compute (two
    # buffer sets alternate; every step still moves its own h2d and d2h bytes).
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)
    sets = []
    for _ in range(2):
        sets.append({"q": torch.empty_like(q), "qr": torch.empty_like(qr),
                     "rows": [torch.empty_like(dd) for _, dd in step_in],
                     "out": torch.empty_like(out), "lse": torch.empty_like(lse),
                     "out_h": torch.empty(out.shape, dtype=out.dtype).pin_memory(),
                     "lse_h": torch.empty(lse.shape, dtype=lse.dtype).pin_memory(),
                     "ev_in": torch.cuda.Event(), "ev_comp": torch.cuda.Event(), "ev_out": torch.cuda.Event()})

    def append_rows(rows):
        if w.kind in ("mla", "gla", "gta"):
            lkv.latent_cache_append(rows[0], cache, cu, S)
        else:
            lkv.latent_cache_append(rows[0], k, cu, S)
            lkv.latent_cache_append(rows[1], v, cu, S)
            lkv.latent_cache_append(rows[2], kpe, cu, S)

    def e2e_step_pipelined(n):
        st = sets[n % 2]
        if n == 0:
            s_in.wait_stream(stream)            # the timed region starts after everything before it
        s_in.wait_event(st["ev_comp"])          # the set's inputs were consumed by step n - 2
        with torch.cuda.stream(s_in):
            st["q"].copy_(q_h, non_blocking=True)
            st["qr"].copy_(qr_h, non_blocking=True)
            for (h, _), dd in zip(step_in, st["rows"]):
                dd.copy_(h, non_blocking=True)
            st["ev_in"].record(s_in)
        stream.wait_event(st["ev_in"])
        stream.wait_event(st["ev_out"])         # the set's result was copied out by step n - 2
        append_rows(st["rows"])
        decode(st["q"], st["qr"], st["out"], st["lse"])
        st["ev_comp"].record(stream)
        s_out.wait_event(st["ev_comp"])
        with torch.cuda.stream(s_out):
            st["out_h"].copy_(st["out"], non_blocking=True)
            st["lse_h"].copy_(st["lse"], non_blocking=True)
            st["ev_out"].record(s_out)

    e2e_ms = time_e2e(e2e_step_pipelined, tail_stream=s_out)
    torch.cuda.synchronize(dev)

    # The headline decode call once more, each call after an L2-flushing write (outside its events),
    # then every other workload the same way (single process only: they hold up to 4.4 GB each).
    flushed_ms = None
    side = None
    if world == 1 and args.side_iters > 0:
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        flushed_ms = time_flushed(decode, (q, qr, out, lse), stream, flush, args.side_iters)
        del flush
        if lkv.check_device() != 0:
            raise RuntimeError("device error while timing the flushed decode calls")
        names = [n for n in SIDE_WORKLOADS if n != w.name]
        side = bench_side_workloads(lkv, dev, names, args.side_iters, args.side_cpu_budget)

    # Group-axis TP of the GQLA step over all ranks (every rank takes the same collective steps).
    del d
    tp_res = bench_tp(lkv, dev, rank, world, args.tp_steps, 3) if args.tp_steps > 0 else None

    # The FP8 GTA decode last, its failure recorded in the line rather than ending the run.
    if side is not None:
        add_guarded(side, FP8_NAME, lambda: bench_fp8_gta(lkv, dev, args.side_iters, args.side_cpu_budget))

    tokens = B * S * world
    cache_bytes, io_bytes, flops = workload_accounting(w, lengths)
    res = None
    if rank == 0:
        peaks, how = load_peaks()
        ms = total_ms / args.steps
        alg_bytes = cache_bytes + io_bytes
        dec_s = dec_avg_ms * 1e-3
        gbs = alg_bytes / dec_s / 1e9
        tfl = flops / dec_s / 1e12
        t_hbm = alg_bytes / (peaks["hbm_gbs"] * 1e9)
        t_tc = flops / (peaks["bf16_tflops"] * 1e12)
        bound = "hbm" if t_hbm >= t_tc else "tensor"
        achieved = gbs if bound == "hbm" else tfl
        peak = peaks["hbm_gbs"] if bound == "hbm" else peaks["bf16_tflops"]
        res = {
            "metric": METRIC,
            "value": value,
            "unit": "tokens/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": w.dtype,
            "data": "synthetic (seeded Gaussian, shapes of the pages' MLA/GQLA decode workloads)",
            "config": {"workload": w.name, "kind": w.kind, "batch_per_gpu": B, "s_q": S, "h_q": w.h_q,
                       "groups": w.groups, "d_k": w.d_k, "d_v": w.d_v, "d_rope": w.d_rope,
                       "seqlen": w.seqlen, "cache_gb_per_gpu": round(cache_bytes / 1e9, 4),
                       "l2": "inputs larger than L2 (cache >> 126 MB); no flush",
                       "parallelism": f"dp{world}"},
            "decode_kernel_ms": dec_avg_ms,
            "decode_ms_per_step": {"min": float(np.min(dec_ms)), "median": float(np.median(dec_ms)),
                                   "max": float(np.max(dec_ms))},
            "decode_ms_l2_flushed": (None if flushed_ms is None else
                                     {"median": float(np.median(flushed_ms)), "min": float(np.min(flushed_ms)),
                                      "calls": len(flushed_ms),
                                      "frac": roofline_entry(w, lengths, float(np.median(flushed_ms)),
                                                             *load_peaks())["frac"]}),
            "kv_gbs": gbs,
            "tflops": tfl,
            "roofline": {"bound": bound, "achieved": achieved, "peak": peak,
                         "unit": "GB/s" if bound == "hbm" else "TFLOP/s", "frac": achieved / peak,
                         "traffic": measured_traffic(w.name), "kernel_source_hash": kernel_source_hash(w.kind),
                         "peak_source": f"{how} (MEASURED_PEAKS.json burst)",
                         "nominal": {"hbm_gbs": NOMINAL_PEAKS["hbm_gbs"], "bf16_tflops": NOMINAL_PEAKS["bf16_tflops"],
                                     "frac": max(alg_bytes / (NOMINAL_PEAKS["hbm_gbs"] * 1e9),
                                                 flops / (NOMINAL_PEAKS["bf16_tflops"] * 1e12)) / dec_s},
                         "roofline_ms": max(t_hbm, t_tc) * 1e3,
                         "frac_of_step_roofline": max(t_hbm, t_tc) * 1e3 / ms,
                         "kernel": decode_kernel_name(w) + " + split combine (one lkv_*_decode call)",
                         "algorithmic_bytes": alg_bytes, "algorithmic_flops": flops},
            "e2e": {"value": tokens / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": int(h2d),
                    "d2h_bytes_per_step": int(d2h), "ms_per_step": e2e_ms,
                    "pipeline": "h2d, append + decode and d2h of neighbouring steps on three streams, two buffer sets",
                    "serial": {"value": tokens / (e2e_serial_ms * 1e-3), "ms_per_step": e2e_serial_ms}},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": sampler.summary() if sampler else None,
            "workloads": side,
            "tp": tp_res,
        }
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return res


_INPUT_CACHE = {}


def cpu_baseline(w, budget_s: float, one_thread: bool = True):
    """The oracle as it stands on the host cores, on a bounded sample of the workload; with
    one_thread, also its time on one core (BLAS limited to one thread) on a smaller sample."""
    import oracle
    if w.name not in _INPUT_CACHE:
        _INPUT_CACHE[w.name] = synth.make_inputs(w)
    d = _INPUT_CACHE[w.name]
    cu = d["cu_seqlens"].numpy().astype(np.int64)
    order = list(range(w.batch))
    single = None
    if one_thread:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            single = cpu_baseline(w, max(0.5, budget_s / 4), one_thread=False)
        single = {k: single[k] for k in ("value", "sample", "seconds")}
    t0 = time.perf_counter()
    done = 0
    for b in order:
        if w.kind == "mla":
            c = d["cache"]
            oracle.mla_absorbed_decode(d["q"], d["q_rope"], c[:, :w.d_k], c[:, w.d_k:], cu, w.scale, requests=[b])
        elif w.kind == "gqla":
            oracle.gqla_group_decode(d["q"], d["q_rope"], d["k"], d["v"], d["kpe"], cu, w.scale, requests=[b])
        elif w.kind == "gta":
            width = w.groups * w.d_k
            c = d["cache"]
            oracle.gta_group_decode(d["q"], d["q_rope"], c[:, :width], c[:, width:], w.groups, cu, w.scale,
                                    requests=[b])
        else:
            width = w.groups * w.d_k
            c = d["cache"]
            oracle.gla_group_decode(d["q"], d["q_rope"], c[:, :width], c[:, width:], w.groups, cu, w.scale,
                                    requests=[b])
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    res = {"value": done * w.s_q / dt, "unit": "tokens/s", "cores": os.cpu_count(),
           "kind": "oracle", "sample": f"{done} of {w.batch} requests of {w.name} (fp64 numpy oracle)",
           "seconds": dt}
    if single is not None:
        res["one_thread"] = single
    return res


def bench_reference(args, rank, world):
    if rank != 0:
        return None
    w = synth.workload(args.workload)
    budget = max(1.0, 150.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_baseline(w, budget, one_thread=False)
    vals = [cpu_baseline(w, budget, one_thread=(i == args.steps - 1)) for i in range(args.steps)]
    v = float(np.mean([x["value"] for x in vals]))
    cb = dict(vals[-1])
    cb["value"] = v
    return {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * w.batch * w.s_q / v,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": w.name, "batch_per_gpu": w.batch, "s_q": w.s_q,
                                        "seqlen": w.seqlen, "parallelism": f"dp{world}"},
        "cpu_baseline": cb,
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="mla_b64_l4096", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="lkv", choices=["lkv", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--side-iters", type=int, default=50,
                    help="calls per workload for the flushed per-workload timings (0: skip them)")
    ap.add_argument("--side-cpu-budget", type=float, default=1.5,
                    help="seconds of CPU-oracle work per side workload")
    ap.add_argument("--tp-steps", type=int, default=20,
                    help="timed steps of the group-axis TP workload on all ranks (0: skip it)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", str(args.gpus)))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus and "WORLD_SIZE" in os.environ:
        raise SystemExit("--gpus must match the launcher's world size")
    if args.impl == "reference":
        res = bench_reference(args, rank, world)
    else:
        res = bench_gpu(args, rank, world, local_rank)
        if rank == 0 and world == 1:
            res["cpu_baseline"] = cpu_baseline(synth.workload(args.workload), args.cpu_budget)
        elif rank == 0:
            res["cpu_baseline"] = None
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
