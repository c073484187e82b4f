"""The allocation-free GQLA decode entry point (fixed library-owned scratch) against the
regular entry point that takes a caller workspace.

Some callers cannot allocate device memory on the decode path (no allocator of their own, or
all memory reserved up front); lkv_gqla_group_decode_noalloc serves them with a fixed 8 MiB
device array inside the library.  This file is collected last so that a failure here leaves
every other test already run; it must pass alone in a fresh process and after the others."""
import numpy as np
import pytest
import torch

import synth
from gpu_util import GATE_BF16, to_dev

pytestmark = pytest.mark.gpu


def _regular(L, d, w):
    return L.gqla_group_decode(d["q"], d["q_rope"], d["k"], d["v"], d["kpe"], d["cu_seqlens"], w.scale)


def _noalloc(L, d, w):
    return L.gqla_group_decode_noalloc(d["q"], d["q_rope"], d["k"], d["v"], d["kpe"], d["cu_seqlens"],
                                       w.scale)


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
        o = out.float().cpu().numpy().astype(np.float64)
        r = ref_out.float().cpu().numpy().astype(np.float64)
        diff = o - r
        assert np.isfinite(o).all()
        assert np.abs(diff).max() <= GATE_BF16["max_abs"], call
        assert np.linalg.norm(diff) / np.linalg.norm(r) <= GATE_BF16["rel_l2"], call
        assert np.abs(lse.cpu().numpy() - ref_lse.cpu().numpy()).max() <= GATE_BF16["lse"], call


def test_noalloc_rejects_shapes_beyond_its_scratch(gpu):
    import latent_kv_cache_split_b200 as L
    # 512 heads in 8 groups with s_q = 2: 128 rows per unit needs ~19 MB of partials > 8 MiB
    w = synth.workload("gqla_g8_sq2_l8192", batch=1, seqlen=70, h_q=512)
    d = to_dev(synth.make_inputs(w), gpu)
    with pytest.raises(L.LkvError) as e:
        _noalloc(L, d, w)
    assert e.value.status == L.ERR_WORKSPACE
    assert L.check_device() == 0
