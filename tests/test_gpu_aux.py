"""GPU tests for the rest of the boundary: bit-exact cache append, the partial merge, bitwise
masking properties, failure reporting, and the same-weights agreement of the decode forms."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import compare, run_lib, run_oracle, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L(gpu):
    import latent_kv_cache_split_b200 as lib
    lib.check_device(clear=True)
    return lib


@pytest.mark.parametrize("row_elems,s_q", [(576, 1), (576, 2), (2048, 2), (64, 1)])
def test_append_bit_exact(L, gpu, row_elems, s_q):
    rng = np.random.default_rng(row_elems + s_q)
    lengths = rng.integers(s_q, 300, size=9)
    cu = synth.prefix_offsets(lengths)
    rows = int(cu[-1]) + 5
    cache = torch.from_numpy(rng.standard_normal((rows, row_elems)).astype(np.float32)).bfloat16()
    new = torch.from_numpy(rng.standard_normal((9 * s_q, row_elems)).astype(np.float32)).bfloat16()
    want = oracle.append_rows(cache.view(torch.int16).numpy(), new.view(torch.int16).numpy(), cu, s_q)
    dc = cache.to(gpu)
    L.latent_cache_append(new.to(gpu), dc, torch.from_numpy(cu.astype(np.int32)).to(gpu), s_q)
    got = dc.cpu().view(torch.int16).numpy()
    assert L.check_device() == 0
    np.testing.assert_array_equal(got, want)


def test_append_rejects_short_request_on_device(L, gpu):
    cu = torch.tensor([0, 1, 5], dtype=torch.int32, device=gpu)   # request 0 has L = 1 < s_q = 2
    cache = torch.zeros((8, 64), dtype=torch.bfloat16, device=gpu)
    new = torch.ones((4, 64), dtype=torch.bfloat16, device=gpu)
    L.latent_cache_append(new, cache, cu, 2)
    assert L.check_device(clear=True) == 2          # LKV_SITE_BAD_LENGTH
    assert cache[:1].abs().sum().item() == 0         # nothing written for the bad request
    assert cache[3:5].float().sum().item() == 128    # the good request's rows 3, 4
    assert L.check_device() == 0


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_merge_partials(L, gpu, out_dtype):
    rng = np.random.default_rng(3)
    n, rows, d = 5, 300, 512
    o = rng.standard_normal((n, rows, d)).astype(np.float32)
    l = (rng.standard_normal((n, rows)) * 3).astype(np.float32)
    l[1, :40] = -np.inf                                  # empty parts
    ref_o, ref_l = oracle.merge_partials(o, l)
    out, lse = L.merge_partials(torch.from_numpy(o).to(gpu), torch.from_numpy(l).to(gpu), out_dtype=out_dtype)
    got = out.float().cpu().numpy()
    tol = 1e-5 if out_dtype == torch.float32 else 8e-3
    np.testing.assert_allclose(got, ref_o, atol=tol, rtol=tol)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_l, atol=2e-6, rtol=1e-6)


@pytest.mark.parametrize("name", ["mla_b64_l4096", "gqla_g8_sq2_l8192", "long_gla2"])
def test_rows_past_the_cache_do_not_leak(L, gpu, name):
    """NaN in cache rows after the last request gives bitwise the same result as zeros there."""
    w = synth.workload(name, batch=3, seqlen=None)
    lengths = [100, 37, 129]
    d = to_dev(synth.make_inputs(w, extra_rows=70, lengths=lengths), gpu)
    out0, lse0 = (t.clone() for t in run_lib(L, d))
    T = sum(lengths)
    for key in ("cache", "k", "v", "kpe"):
        if key in d:
            d[key][T:] = float("nan")
    out1, lse1 = run_lib(L, d)
    torch.cuda.synchronize()
    assert torch.isfinite(out1.float()).all()
    assert torch.equal(out0, out1) and torch.equal(lse0, lse1)


@pytest.mark.parametrize("name", ["mla_b64_l4096", "gqla_g8_sq2_l8192"])
def test_mtp_query0_ignores_the_newest_row(L, gpu, name):
    """With s_q = 2, query 0 may not see row L-1: changing it leaves query 0 bitwise unchanged."""
    w = synth.workload(name, batch=2, s_q=2, seqlen=None)
    d = to_dev(synth.make_inputs(w, lengths=[130, 64]), gpu)
    out0, lse0 = (t.clone() for t in run_lib(L, d))
    last = int(d["cu_seqlens"][1].item()) - 1       # newest row of request 0
    for key in ("cache", "k", "v", "kpe"):
        if key in d:
            d[key][last] = d[key][last] * 3 + 1
    out1, lse1 = run_lib(L, d)
    torch.cuda.synchronize()
    assert torch.equal(out0[:, 0], out1[:, 0]) and torch.equal(lse0[:, 0], lse1[:, 0])
    assert not torch.equal(out0[0, 1], out1[0, 1])   # query 1 does see it
    assert torch.equal(out0[1], out1[1])


def test_requests_are_independent(L, gpu):
    """Changing one request's cache rows leaves the other requests' outputs bitwise unchanged."""
    w = synth.workload("varlen_mla_sq1", batch=6)
    lengths = [1500, 64, 3000, 1, 900, 4100]
    d = to_dev(synth.make_inputs(w, lengths=lengths), gpu)
    out0, lse0 = (t.clone() for t in run_lib(L, d))
    cu = d["cu_seqlens"].tolist()
    d["cache"][cu[2]:cu[3]] = -d["cache"][cu[2]:cu[3]]
    out1, lse1 = run_lib(L, d)
    torch.cuda.synchronize()
    for b in range(6):
        same = torch.equal(out0[b], out1[b]) and torch.equal(lse0[b], lse1[b])
        assert same == (b != 2), b


def test_bad_length_is_reported_not_trapped(L, gpu):
    w = synth.workload("gqla_g8_sq2_l8192", batch=2, seqlen=None)
    d = to_dev(synth.make_inputs(w, lengths=[1, 90]), gpu)   # request 0 shorter than s_q = 2
    run_lib(L, d)
    assert L.check_device(clear=True) == 2
    assert L.check_device() == 0


def test_workspace_too_small(L, gpu):
    w = synth.workload("mla_b64_l4096", batch=2, seqlen=128)
    d = to_dev(synth.make_inputs(w), gpu)
    c = d["cache"]
    ws = torch.empty(1024, dtype=torch.uint8, device=gpu)
    with pytest.raises(L.LkvError) as e:
        L.mla_absorbed_decode(d["q"], d["q_rope"], c[:, :512], c[:, 512:], d["cu_seqlens"], w.scale,
                              workspace=ws)
    assert e.value.status == L.ERR_WORKSPACE


def test_bounded_wait_gives_up_and_context_survives(L, gpu):
    L.selftest_wait_timeout(2_000_000)     # 2 ms on a barrier nothing arrives at
    assert L.check_device(clear=True) == 1  # LKV_SITE_SELFTEST
    assert L.check_device() == 0
    x = torch.arange(10, device=gpu, dtype=torch.float32).sum().item()
    assert x == 45.0
    _ = run_lib(L, to_dev(synth.make_inputs(synth.workload("mla_b64_l4096", batch=1, seqlen=70)), gpu))
    assert L.check_device() == 0


def test_absorbed_and_grouped_paths_agree_on_same_weights(L, gpu):
    """GQLA explainer, section 2: the MQA-absorbed path and the GQA path are algebraically
    equivalent on the same trained weights.  Diagnostic on the GPU: both runs take bf16 inputs
    derived from one set of fp64 weights (latent C, per-group W_UK / W_UV), so they differ by
    bf16 rounding of those inputs only; the gate is rel-L2 <= 2e-2 between the two outputs."""
    rng = np.random.default_rng(77)
    B, H, G, dh, r, dr, Lk = 2, 128, 8, 128, 512, 64, 300
    cu = synth.prefix_offsets([Lk, Lk - 40])
    T = int(cu[-1])
    C = rng.standard_normal((T, r)) / math.sqrt(r)
    kr = rng.standard_normal((T, dr)) / 8
    w_uk = rng.standard_normal((G, r, dh)) / math.sqrt(r) * 2
    w_uv = rng.standard_normal((G, r, dh)) / math.sqrt(r)
    q = rng.standard_normal((B, 1, H, dh)) / math.sqrt(dh) * 4
    qr = rng.standard_normal((B, 1, H, dr)) / 8
    scale = 1 / math.sqrt(dh + dr)
    bf = lambda a: torch.from_numpy(np.asarray(a, dtype=np.float32)).bfloat16().to(gpu)
    cu_d = torch.from_numpy(cu.astype(np.int32)).to(gpu)
    # absorbed: q_abs = W_UK q (latent space), out = W_UV^T o_lat
    q_abs = oracle.absorb_query(q, w_uk, G)
    cache = torch.cat([bf(C), bf(kr)], dim=1)
    o_lat, lse_a = L.mla_absorbed_decode(bf(q_abs), bf(qr), cache[:, :r], cache[:, r:], cu_d, scale)
    out_a = oracle.unabsorb_output(o_lat.float().cpu().numpy(), w_uv, G)
    # GQA path on the expanded cache K_j = C W_UK[j], V_j = C W_UV[j]
    K = oracle.expand_latent(C, w_uk)
    V = oracle.expand_latent(C, w_uv)
    out_g, lse_g = L.gqla_group_decode(bf(q), bf(qr), bf(K), bf(V), bf(kr), cu_d, scale)
    og = out_g.float().cpu().numpy()
    rel = np.linalg.norm(out_a - og) / np.linalg.norm(og)
    assert rel < 2e-2, rel
    assert np.abs(lse_a.cpu().numpy() - lse_g.cpu().numpy()).max() < 2e-2
    # and the exact identity holds in the oracle on these very weights
    ref_a, _ = oracle.mla_absorbed_decode(q_abs, qr, C, kr, cu, scale)
    ref_g, _ = oracle.gqla_group_decode(q, qr, K, V, kr, cu, scale)
    np.testing.assert_allclose(oracle.unabsorb_output(ref_a, w_uv, G), ref_g, atol=1e-10)
