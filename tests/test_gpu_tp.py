"""GPU tests for the output projection and the group-axis TP runner.  One GPU only: the shards of a
2- and 4-way split run one after another with the library's kernels, each with an identity
all-reduce, and the host sums their partials (no kernel waits on another).  Gate: the fp64 oracle
on the same bf16 inputs (decode + projection), rel-L2 <= 5e-3."""
import numpy as np
import pytest
import torch

import oracle
import synth
from latent_kv_cache_split_b200.tp import GroupAxisTP, group_shard

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L(gpu):
    import latent_kv_cache_split_b200 as lib
    lib.check_device(clear=True)
    return lib


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def _rel(a, b):
    return np.linalg.norm(a - b) / np.linalg.norm(b)


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_output_projection(L, gpu, out_dtype):
    rng = np.random.default_rng(3)
    o = torch.from_numpy(rng.standard_normal((130, 16, 128)).astype(np.float32)).bfloat16().to(gpu)
    w = torch.from_numpy(rng.standard_normal((16 * 128, 1024)).astype(np.float32) / 45).bfloat16().to(gpu)
    y = L.output_projection(o, w, out_dtype=out_dtype)
    ref = oracle.output_projection(_f64(o), _f64(w))
    assert y.dtype == out_dtype and y.shape == (130, 1024)
    assert _rel(_f64(y), ref) <= (1e-5 if out_dtype == torch.float32 else 5e-3)


@pytest.mark.parametrize("world", [1, 2, 4])
def test_group_axis_shards_sum_to_full_projection(L, gpu, world):
    w = synth.workload("gqla_g8_sq2_l8192", batch=3, seqlen=None)
    d = synth.make_inputs(w, lengths=[700, 2, 129])
    rng = np.random.default_rng(5)
    d_model = 512
    w_o = torch.from_numpy(rng.standard_normal((w.h_q * w.d_v, d_model)).astype(np.float32) / 128).bfloat16()
    dev = {k: d[k].to(gpu) for k in ("q", "q_rope", "k", "v", "kpe", "cu_seqlens")}
    w_o_d = w_o.to(gpu)
    total = None
    for rank in range(world):
        sh = group_shard(w.groups, w.h_q, world, rank)
        tp = GroupAxisTP(sh, allreduce_fn=lambda y: y)
        y, _, _ = tp.step(tp.local_query(dev["q"]), tp.local_query(dev["q_rope"]), tp.local_cache(dev["k"]),
                          tp.local_cache(dev["v"]), dev["kpe"], dev["cu_seqlens"], w.scale,
                          w_o_d[sh.w_o_rows(w.d_v)].contiguous())
        total = y.clone() if total is None else total + y
    torch.cuda.synchronize()
    assert L.check_device() == 0
    cu = d["cu_seqlens"].numpy().astype(np.int64)
    out, _ = oracle.gqla_group_decode(d["q"], d["q_rope"], d["k"], d["v"], d["kpe"], cu, w.scale)
    ref = oracle.output_projection(out.reshape(w.batch * w.s_q, w.h_q, w.d_v), _f64(w_o))
    assert _rel(_f64(total), ref) <= 5e-3
