"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle, element by element, on
identical seeded inputs.  Small cases span several 64-key tiles, ragged tails, single-key
requests and range splits; the full-size cases use the benchmark's own launch configuration
and check every output of every request."""
import numpy as np
import pytest
import torch

import synth
from gpu_util import compare, run_lib, run_oracle, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L(gpu):
    import latent_kv_cache_split_b200 as lib
    return lib


def _run(L, gpu, w, lengths=None, requests=None, extra_rows=0):
    d = synth.make_inputs(w, extra_rows=extra_rows, lengths=lengths)
    out, lse = run_lib(L, to_dev(d, gpu))
    torch.cuda.synchronize()
    assert L.check_device() == 0
    ref_out, ref_lse = run_oracle(d, requests=requests)
    return compare(out, lse, ref_out, ref_lse, fp32=(w.dtype == "fp32"), requests=requests,
                   label=w.name)


def test_tiny_fp32_mla_full(L, gpu):
    _run(L, gpu, synth.workload("tiny_fp32_mla"))


@pytest.mark.parametrize("kind", ["mla", "gqla", "gla"])
def test_fp32_path_all_forms(L, gpu, kind):
    base = {"mla": "tiny_fp32_mla", "gqla": "gqla_g8_sq2_l8192", "gla": "long_gla2"}[kind]
    w = synth.workload(base, dtype="fp32", batch=2, seqlen=None, len_lo=0, len_hi=0, input_std=1.0)
    if kind == "gqla":
        w = w.with_(h_q=16, groups=4, d_k=32, d_v=32, d_rope=16)
    if kind == "gla":
        w = w.with_(h_q=8, groups=2, d_k=48, d_v=48, d_rope=16)
    _run(L, gpu, w, lengths=[77, 300])


@pytest.mark.parametrize("s_q,lengths", [(1, [130, 64, 1]), (2, [2, 65, 200]), (1, [4096, 63, 129, 5000])])
def test_mla_small_ragged(L, gpu, s_q, lengths):
    w = synth.workload("mla_b64_l4096", batch=len(lengths), s_q=s_q, seqlen=None)
    _run(L, gpu, w, lengths=lengths)


def test_mla_b64_l4096_full(L, gpu):
    """The benchmark workload, every output checked."""
    _run(L, gpu, synth.workload("mla_b64_l4096"))


@pytest.mark.parametrize("s_q", [1, 2])
def test_mla_unscaled_stress(L, gpu, s_q):
    w = synth.workload("mla_b64_l4096", batch=4, s_q=s_q, seqlen=1000, input_std=1.0)
    _run(L, gpu, w)


@pytest.mark.parametrize("s_q,lengths", [(2, [130, 7]), (1, [1, 200, 64]), (2, [8192, 2])])
def test_gqla_small(L, gpu, s_q, lengths):
    w = synth.workload("gqla_g8_sq2_l8192", batch=len(lengths), s_q=s_q, seqlen=None)
    _run(L, gpu, w, lengths=lengths)


def test_gqla_b64_l8192_full(L, gpu):
    _run(L, gpu, synth.workload("gqla_g8_sq2_l8192"))


def test_gqla_unscaled_stress(L, gpu):
    w = synth.workload("gqla_g8_sq2_l8192", batch=3, seqlen=700, input_std=1.0)
    _run(L, gpu, w)


@pytest.mark.parametrize("s_q,lengths", [(1, [300, 65]), (2, [129, 64, 3])])
def test_gla_small(L, gpu, s_q, lengths):
    w = synth.workload("long_gla2", batch=len(lengths), s_q=s_q, seqlen=None)
    _run(L, gpu, w, lengths=lengths)


@pytest.mark.parametrize("s_q,lengths", [(2, [130, 7]), (1, [1, 200, 64]), (2, [8192, 2, 129])])
def test_gta_small(L, gpu, s_q, lengths):
    """Tied groups (K_j = V_j) through the grouped kernel: ragged tails, one-key requests, splits."""
    w = synth.workload("gta_g8_sq2_l8192", batch=len(lengths), s_q=s_q, seqlen=None)
    _run(L, gpu, w, lengths=lengths)


def test_gta_b64_l8192_full(L, gpu):
    _run(L, gpu, synth.workload("gta_g8_sq2_l8192"))


def test_gta_unscaled_stress(L, gpu):
    w = synth.workload("gta_g8_sq2_l8192", batch=3, seqlen=700, input_std=1.0)
    _run(L, gpu, w)


@pytest.mark.parametrize("s_q,lengths", [(2, [130, 7]), (1, [1, 300, 64]), (2, [4097, 2])])
def test_gqa2_small(L, gpu, s_q, lengths):
    """Two K/V groups of 64 heads: 128 score rows per unit at s_q = 2 (the full M of one UMMA)."""
    w = synth.workload("gqa2_sq2_l8192", batch=len(lengths), s_q=s_q, seqlen=None)
    _run(L, gpu, w, lengths=lengths)


def test_gqa2_b64_l8192_full(L, gpu):
    _run(L, gpu, synth.workload("gqa2_sq2_l8192"))


@pytest.mark.parametrize("name", ["long_gla2", "long_mla", "long_gqla_g8"])
def test_long_context_full(L, gpu, name):
    """B = 8 requests of 131072 keys through each path, every output checked."""
    _run(L, gpu, synth.workload(name))


@pytest.mark.parametrize("name", ["varlen_mla_sq1", "varlen_mla_sq2"])
def test_varlen_full(L, gpu, name):
    """All 128 log-uniform lengths in [1024, 65536], every output checked."""
    _run(L, gpu, synth.workload(name))
