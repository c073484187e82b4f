"""GPU tests for the projections either side of the decode path (GQLA explainer, section 2
"Methodology": W_UK folded into the query and W_UV applied after attention on the absorbed path,
the latent expanded into per-group keys and values on the GQA path), against the fp64 oracle on
the same bf16 inputs, and the same-weights agreement of the two decode forms with every step on
the GPU."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

# bf16 results of fp32-accumulated products of bf16 inputs: the output rounding alone gives a
# relative error of up to 2^-9 per element
GATE = dict(rel_l2=5e-3, max_rel=1e-2)


@pytest.fixture(scope="module")
def L(gpu):
    import latent_kv_cache_split_b200 as lib
    lib.check_device(clear=True)
    return lib


def _bf(a, dev):
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).bfloat16().to(dev)


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def _check(got, ref):
    got = _f64(got)
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    max_rel = np.abs(got - ref).max() / np.abs(ref).max()
    assert rel <= GATE["rel_l2"] and max_rel <= GATE["max_rel"], (rel, max_rel)


@pytest.mark.parametrize("n_tok,h_q,G,d_h,r", [(64, 128, 1, 128, 512), (128, 128, 8, 128, 512), (5, 32, 4, 64, 96)])
def test_absorb_query(L, gpu, n_tok, h_q, G, d_h, r):
    rng = np.random.default_rng(n_tok + G)
    q = _bf(rng.standard_normal((n_tok, h_q, d_h)), gpu)
    w = _bf(rng.standard_normal((G, r, d_h)) / math.sqrt(d_h), gpu)
    _check(L.absorb_query(q, w), oracle.absorb_query(_f64(q), _f64(w), G))


@pytest.mark.parametrize("n_tok,h_q,G,r,d_v", [(64, 128, 1, 512, 128), (128, 128, 8, 512, 128), (7, 16, 2, 64, 32)])
def test_unabsorb_output(L, gpu, n_tok, h_q, G, r, d_v):
    rng = np.random.default_rng(n_tok + 3 * G)
    o = _bf(rng.standard_normal((n_tok, h_q, r)), gpu)
    w = _bf(rng.standard_normal((G, r, d_v)) / math.sqrt(r), gpu)
    _check(L.unabsorb_output(o, w), oracle.unabsorb_output(_f64(o), _f64(w), G))


@pytest.mark.parametrize("T,G,r,d", [(300, 8, 512, 128), (1, 2, 256, 64), (4099, 8, 512, 128)])
def test_expand_latent_from_interleaved_cache(L, gpu, T, G, r, d):
    """The latent is a column slice of the interleaved [T, r + 64] cache (row stride r + 64)."""
    rng = np.random.default_rng(T + G)
    cache = _bf(rng.standard_normal((T, r + 64)), gpu)
    w = _bf(rng.standard_normal((G, r, d)) / math.sqrt(r), gpu)
    c = cache[:, :r]
    _check(L.expand_latent(c, w), oracle.expand_latent(_f64(c), _f64(w)))


def _nan_out(shape, gpu, dtype=torch.bfloat16):
    return torch.full(shape, float("nan"), dtype=dtype, device=gpu)


@pytest.mark.parametrize("n_tok,h_q,G,d_h,r", [(9, 12, 2, 64, 520), (3, 24, 8, 128, 64), (200, 4, 1, 32, 256)])
def test_absorb_every_element_written_once(L, gpu, n_tok, h_q, G, d_h, r):
    """Odd heads per group (6, 3: tiles of 2 and 1 head rows x tokens), r over several column tiles,
    a NaN-filled output: every element is written, by the right group's weights."""
    rng = np.random.default_rng(h_q + r)
    q = _bf(rng.standard_normal((n_tok, h_q, d_h)), gpu)
    w = _bf(rng.standard_normal((G, r, d_h)) / math.sqrt(d_h), gpu)
    out = L.absorb_query(q, w, out=_nan_out((n_tok, h_q, r), gpu))
    assert not torch.isnan(out).any()
    _check(out, oracle.absorb_query(_f64(q), _f64(w), G))


@pytest.mark.parametrize("n_tok,h_q,G,r,d_v", [(5, 12, 3, 136, 200), (33, 128, 8, 512, 128), (2, 2, 2, 64, 8)])
def test_unabsorb_every_element_written_once(L, gpu, n_tok, h_q, G, r, d_v):
    rng = np.random.default_rng(h_q + d_v)
    o = _bf(rng.standard_normal((n_tok, h_q, r)), gpu)
    w = _bf(rng.standard_normal((G, r, d_v)) / math.sqrt(r), gpu)
    out = L.unabsorb_output(o, w, out=_nan_out((n_tok, h_q, d_v), gpu))
    assert not torch.isnan(out).any()
    _check(out, oracle.unabsorb_output(_f64(o), _f64(w), G))


@pytest.mark.parametrize("T,G,r,d", [(130, 3, 64, 40), (257, 5, 128, 64), (129, 1, 512, 512)])
def test_expand_every_element_written_once(L, gpu, T, G, r, d):
    """d not a multiple of 64 (one column block per group), groups side by side across a tile edge
    (5 x 64 columns in tiles of 192), one wide group over two column tiles."""
    rng = np.random.default_rng(T + d)
    c = _bf(rng.standard_normal((T, r)), gpu)
    w = _bf(rng.standard_normal((G, r, d)) / math.sqrt(r), gpu)
    x = L.expand_latent(c, w, out=_nan_out((T, G, d), gpu))
    assert not torch.isnan(x).any()
    _check(x, oracle.expand_latent(_f64(c), _f64(w)))


def test_expand_full_cache_sampled_rows(L, gpu):
    """The expansion of a long cache (65536 rows of the interleaved [T, 576] cache into 8 groups of
    128): 512 sampled rows against the oracle, and no row left unwritten."""
    rng = np.random.default_rng(17)
    T, G, r, d = 65536, 8, 512, 128
    cache = torch.randn((T, r + 64), generator=torch.Generator(device=gpu).manual_seed(3), device=gpu).bfloat16()
    w = _bf(rng.standard_normal((G, r, d)) / math.sqrt(r), gpu)
    x = L.expand_latent(cache[:, :r], w, out=_nan_out((T, G, d), gpu))
    assert not torch.isnan(x).any()
    rows = np.sort(rng.choice(T, 512, replace=False))
    rows[-1] = T - 1
    rows_t = torch.from_numpy(rows).to(gpu)
    _check(x[rows_t], oracle.expand_latent(_f64(cache[rows_t, :r]), _f64(w)))


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_output_projection_weight_resident(L, gpu, out_dtype):
    """An output projection with K <= 512 and >= one 128-column tile per SM runs the weight-resident
    form (B kept in shared memory per column tile, tiles split in contiguous ranges): every element
    against the oracle."""
    rng = np.random.default_rng(21)
    o = _bf(rng.standard_normal((8193, 384)), gpu)
    w = _bf(rng.standard_normal((384, 1000)) / 20, gpu)
    y = L.output_projection(o, w, out_dtype=out_dtype, out=torch.full((8193, 1000), float("nan"), dtype=out_dtype,
                                                                      device=gpu))
    assert not torch.isnan(y).any()
    _check(y, oracle.output_projection(_f64(o), _f64(w)))


@pytest.mark.parametrize("T,G,r,d", [(9300, 8, 512, 128), (9301, 16, 320, 64)])
def test_expand_cta_pair_form(L, gpu, T, G, r, d):
    """Enough 256-row tiles for the CTA-pair form (two CTAs share each tile's MMAs, each holding half
    of the column tile's weights): every element against the oracle, an odd number of 128-row
    tiles, K not a multiple of 128 (a last stage of one K block)."""
    rng = np.random.default_rng(T + r)
    c = _bf(rng.standard_normal((T, r)), gpu)
    w = _bf(rng.standard_normal((G, r, d)) / math.sqrt(r), gpu)
    x = L.expand_latent(c, w, out=_nan_out((T, G, d), gpu))
    torch.cuda.synchronize()
    assert L.check_device() == 0
    assert not torch.isnan(x).any()
    _check(x, oracle.expand_latent(_f64(c), _f64(w)))


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_output_projection_cta_pair_form(L, gpu, out_dtype):
    rng = np.random.default_rng(31)
    o = _bf(rng.standard_normal((9300, 256)), gpu)
    w = _bf(rng.standard_normal((256, 2048)) / 16, gpu)
    y = L.output_projection(o, w, out_dtype=out_dtype, out=torch.full((9300, 2048), float("nan"), dtype=out_dtype,
                                                                      device=gpu))
    torch.cuda.synchronize()
    assert L.check_device() == 0
    assert not torch.isnan(y).any()
    _check(y, oracle.output_projection(_f64(o), _f64(w)))


def test_projection_argument_errors(L, gpu):
    q = torch.zeros((4, 6, 8), dtype=torch.bfloat16, device=gpu)
    w = torch.zeros((4, 16, 8), dtype=torch.bfloat16, device=gpu)
    with pytest.raises(L.LkvError) as e:
        L.absorb_query(q, w)  # 6 heads do not split into 4 groups
    assert e.value.status == L.ERR_INVALID_ARG
    q8 = torch.zeros((4, 8, 8), dtype=torch.float32, device=gpu)
    with pytest.raises(L.LkvError) as e:
        L.absorb_query(q8, w.float())  # fp32 operands: only bf16 is implemented
    assert e.value.status == L.ERR_UNSUPPORTED


def test_same_weights_agreement_all_on_gpu(L, gpu):
    """GQLA explainer, section 2: absorbed path (q -> W_UK q on the GPU, MLA decode over the latent,
    W_UV^T o_lat on the GPU) against the GQA path (K_j = C W_UK[j], V_j = C W_UV[j] expanded on the
    GPU, GQLA decode).  Exact in real arithmetic; bf16 rounding of the intermediate tensors bounds
    the difference (gate rel-L2 <= 2e-2, as for the oracle-projected diagnostic)."""
    rng = np.random.default_rng(78)
    B, H, G, dh, r, dr, Lk = 3, 128, 8, 128, 512, 64, 700
    cu = synth.prefix_offsets([Lk, Lk - 40, 129])
    T = int(cu[-1])
    cache = _bf(np.concatenate([rng.standard_normal((T, r)) / math.sqrt(r), rng.standard_normal((T, dr)) / 8], 1), gpu)
    C, kr = cache[:, :r], cache[:, r:]
    w_uk = _bf(rng.standard_normal((G, r, dh)) / math.sqrt(r) * 2, gpu)
    w_uv = _bf(rng.standard_normal((G, r, dh)) / math.sqrt(r), gpu)
    q = _bf(rng.standard_normal((B, 1, H, dh)) / math.sqrt(dh) * 4, gpu)
    qr = _bf(rng.standard_normal((B, 1, H, dr)) / 8, gpu)
    scale = 1 / math.sqrt(dh + dr)
    cu_d = torch.from_numpy(cu.astype(np.int32)).to(gpu)
    q_abs = L.absorb_query(q, w_uk)
    o_lat, lse_a = L.mla_absorbed_decode(q_abs, qr, C, kr, cu_d, scale)
    out_a = L.unabsorb_output(o_lat, w_uv)
    K = L.expand_latent(C, w_uk)
    V = L.expand_latent(C, w_uv)
    out_g, lse_g = L.gqla_group_decode(q, qr, K, V, kr.contiguous(), cu_d, scale)
    a, g = _f64(out_a), _f64(out_g)
    rel = np.linalg.norm(a - g) / np.linalg.norm(g)
    assert rel < 2e-2, rel
    assert np.abs(lse_a.cpu().numpy() - lse_g.cpu().numpy()).max() < 2e-2
    # and each side matches the fp64 oracle on its own GPU-produced bf16 operands
    ref_a, _ = oracle.mla_absorbed_decode(_f64(q_abs), _f64(qr), _f64(C), _f64(kr), cu, scale)
    rel_a = np.linalg.norm(_f64(o_lat) - ref_a) / np.linalg.norm(ref_a)
    assert rel_a < 5e-3, rel_a


def test_projection_throughput(L, gpu):
    """Measurement (printed with -s): the projections of one decode step of the MLA B=64 workload
    (absorb for 64 tokens x 128 heads, unabsorb) and the GQLA expansion of 4096 new cache rows,
    as TFLOP/s of the plain GEMMs (bf16, fp32 accumulation)."""
    rng = np.random.default_rng(5)
    cases = []
    q = _bf(rng.standard_normal((64, 128, 128)), gpu)
    wk = _bf(rng.standard_normal((8, 512, 128)) / 11, gpu)
    wk1 = wk[:1].contiguous()
    cases.append(("absorb 64 tok x 128 heads, g=1", lambda: L.absorb_query(q, wk1), 2 * 64 * 128 * 128 * 512))
    cases.append(("absorb 64 tok x 128 heads, g=8", lambda: L.absorb_query(q, wk), 2 * 64 * 128 * 128 * 512))
    o = _bf(rng.standard_normal((64, 128, 512)), gpu)
    wv = _bf(rng.standard_normal((8, 512, 128)) / 22, gpu)
    wv1 = wv[:1].contiguous()
    cases.append(("unabsorb 64 tok x 128 heads, g=1", lambda: L.unabsorb_output(o, wv1), 2 * 64 * 128 * 512 * 128))
    cases.append(("unabsorb 64 tok x 128 heads, g=8", lambda: L.unabsorb_output(o, wv), 2 * 64 * 128 * 512 * 128))
    c = _bf(rng.standard_normal((4096, 512)), gpu)
    cases.append(("expand 4096 rows to g=8 x 128", lambda: L.expand_latent(c, wk), 2 * 4096 * 512 * 8 * 128))
    cl = torch.randn((65536, 512), device=gpu).bfloat16()
    cases.append(("expand 65536 rows to g=8 x 128", lambda: L.expand_latent(cl, wk), 2 * 65536 * 512 * 8 * 128))
    ob = _bf(rng.standard_normal((64, 128 * 128)), gpu)
    wo = _bf(rng.standard_normal((128 * 128, 7168)) / 128, gpu)
    cases.append(("output projection 64 tok, 16384 -> 7168", lambda: L.output_projection(ob, wo),
                  2 * 64 * 16384 * 7168))
    # Device time per call: 20 calls captured in one CUDA graph (the host cost of a call -- tensor
    # maps, argument marshalling -- is then outside the timed replay).
    s = torch.cuda.Stream()
    for name, fn, flops in cases:
        with torch.cuda.stream(s):
            for _ in range(3):
                fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for _ in range(20):
                fn()
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        assert L.check_device() == 0
        ms = e0.elapsed_time(e1) / 20
        print(f"{name}: {ms * 1e3:.1f} us, {flops / ms / 1e9:.1f} TFLOP/s")
