"""GPU parity of the keys-in-M decode kernels (GQLA / GTA units of at most 32 rows, GLA units of at
most 64) on the unit shapes the benchmark workloads do not reach: two queries per unit with the
second starting inside a softmax warp's rows, and padding rows (fewer live rows than the MMA's N).
(The entry points take s_q = 1 or 2.)  Each case against the fp64 oracle with the usual bf16
gates, ragged lengths that span several 128-key tiles, a request shorter than a tile and one of
exactly s_q keys."""
import pytest
import torch

import synth
from gpu_util import compare, run_lib, run_oracle, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L(gpu):
    import latent_kv_cache_split_b200 as lib
    return lib


def _run(L, gpu, w, lengths):
    d = synth.make_inputs(w, lengths=lengths)
    out, lse = run_lib(L, to_dev(d, gpu))
    torch.cuda.synchronize()
    assert L.check_device() == 0
    ref_out, ref_lse = run_oracle(d)
    return compare(out, lse, ref_out, ref_lse, label=f"{w.name} g={w.groups} h_q={w.h_q} s_q={w.s_q}")


@pytest.mark.parametrize("groups,s_q,lengths", [
    (4, 2, [300, 2, 129]),     # 32 heads x 2 queries = 64 rows: query 1 starts at row 32
    (8, 2, [257, 2, 130]),     # 16 heads x 2 queries = 32 rows: half of every warp's rows padding
    (4, 1, [200, 65, 1]),      # 32 heads x 1 query: rows 32..63 padding
])
def test_gla_keys_in_m_unit_shapes(L, gpu, groups, s_q, lengths):
    w = synth.workload("long_gla2", batch=len(lengths), s_q=s_q, seqlen=None, groups=groups)
    _run(L, gpu, w, lengths)


@pytest.mark.parametrize("kind,groups,s_q,lengths", [
    ("gqla", 16, 2, [130, 2, 260]),   # 8 heads x 2 queries = 16 rows: query 1 from row 8, rows 16..31 padding
    ("gqla", 32, 1, [129, 3, 64]),    # 4 rows
    ("gta", 16, 2, [200, 2, 129]),
    ("gta", 32, 2, [131, 2, 70]),     # 4 heads x 2 queries = 8 rows
])
def test_grouped_keys_in_m_unit_shapes(L, gpu, kind, groups, s_q, lengths):
    base = {"gqla": "gqla_g8_sq2_l8192", "gta": "gta_g8_sq2_l8192"}[kind]
    w = synth.workload(base, batch=len(lengths), s_q=s_q, seqlen=None, groups=groups)
    _run(L, gpu, w, lengths)
