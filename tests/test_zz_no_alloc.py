"""The allocation-free GQLA decode entry point (fixed library-owned scratch) against the
regular entry point that takes a caller workspace, and against the fp64 oracle.

Some callers cannot allocate device memory on the decode path (no allocator of their own, or
all memory reserved up front); lkv_gqla_group_decode_noalloc serves them with a fixed 8 MiB
device array inside the library.  The array keeps whatever the previous call left in it, so the
calls below change shape between calls (groups, new tokens per request, batch): the partial
slots, the rows per unit and the number of work ranges all differ from one call to the next, and
stale partials of an earlier layout would show up as a mismatch.

This file is collected last so that a failure here leaves every other test already run; it must
pass alone in a fresh process and after the others."""
import numpy as np
import pytest
import torch

import synth
from gpu_util import GATE_BF16, compare, run_oracle, to_dev

pytestmark = pytest.mark.gpu


def _regular(L, d, w):
    return L.gqla_group_decode(d["q"], d["q_rope"], d["k"], d["v"], d["kpe"], d["cu_seqlens"], w.scale)


def _noalloc(L, d, w):
    return L.gqla_group_decode_noalloc(d["q"], d["q_rope"], d["k"], d["v"], d["kpe"], d["cu_seqlens"],
                                       w.scale)


# (workload, overrides, lengths), all inside the 8 MiB array: g = 8 at s_q = 2 (32 rows per unit,
# 144 ranges), g = 4 at s_q = 1 (32 rows per unit, 148 ranges), g = 8 at s_q = 1 (16 rows per
# unit, 144 ranges) with another batch
SHAPES = [
    ("gqla_g8_sq2_l8192", dict(batch=5, seqlen=None), [700, 65, 3000, 2, 1500]),
    ("gqla_g8_sq2_l8192", dict(batch=3, seqlen=None, s_q=1, groups=4), [2049, 1, 333]),
    ("gqla_g8_sq2_l8192", dict(batch=2, seqlen=None, s_q=1), [4100, 129]),
]


def _against_regular(out, lse, ref_out, ref_lse, label):
    o = out.float().cpu().numpy().astype(np.float64)
    r = ref_out.float().cpu().numpy().astype(np.float64)
    diff = o - r
    assert np.isfinite(o).all(), label
    assert np.abs(diff).max() <= GATE_BF16["max_abs"], label
    assert np.linalg.norm(diff) / np.linalg.norm(r) <= GATE_BF16["rel_l2"], label
    assert np.abs(lse.cpu().numpy() - ref_lse.cpu().numpy()).max() <= GATE_BF16["lse"], label


def test_noalloc_matches_regular_entry_point_on_two_calls(gpu):
    import latent_kv_cache_split_b200 as L
    L.check_device(clear=True)
    w = synth.workload("gqla_g8_sq2_l8192", batch=5, seqlen=None)
    d = to_dev(synth.make_inputs(w, lengths=[700, 65, 3000, 2, 1500]), gpu)
    ref_out, ref_lse = (t.clone() for t in _regular(L, d, w))
    for call in range(2):
        out, lse = _noalloc(L, d, w)
        torch.cuda.synchronize()
        assert L.check_device() == 0
        _against_regular(out, lse, ref_out, ref_lse, f"call {call}")


def test_noalloc_across_changing_shapes_against_regular_and_oracle(gpu):
    import latent_kv_cache_split_b200 as L
    L.check_device(clear=True)
    cases = []
    for name, kw, lengths in SHAPES:
        w = synth.workload(name, **kw)
        host = synth.make_inputs(w, lengths=lengths)
        cases.append((w, host, to_dev(host, gpu), run_oracle(host)))
    # every shape after every other: A, B, C, A, C, B
    for idx in (0, 1, 2, 0, 2, 1):
        w, host, d, (o_ref, l_ref) = cases[idx]
        out, lse = _noalloc(L, d, w)
        torch.cuda.synchronize()
        assert L.check_device() == 0
        ref_out, ref_lse = _regular(L, d, w)
        torch.cuda.synchronize()
        _against_regular(out, lse, ref_out, ref_lse, f"shape {idx}")
        compare(out, lse, o_ref, l_ref, label=f"shape {idx} vs oracle")


def test_noalloc_rejects_shapes_beyond_its_scratch(gpu):
    import latent_kv_cache_split_b200 as L
    # 512 heads in 8 groups with s_q = 2: 128 rows per unit needs ~19 MB of partials > 8 MiB
    w = synth.workload("gqla_g8_sq2_l8192", batch=1, seqlen=70, h_q=512)
    d = to_dev(synth.make_inputs(w), gpu)
    with pytest.raises(L.LkvError) as e:
        _noalloc(L, d, w)
    assert e.value.status == L.ERR_WORKSPACE
    assert L.check_device() == 0
