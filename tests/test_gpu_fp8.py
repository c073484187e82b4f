"""GPU tests for FP8 (e4m3) latent cache rows: the quantisation kernel against the oracle's steps,
bit for bit (the codes are integers that floating point decides; the power-of-two scale makes the
division exact on both sides, and both round to nearest even), in bulk and at append; and the GTA
decode over FP8 rows against the oracle's decode over the dequantised states (rows built on the
host by the oracle's quantiser, so no input comes from the GPU path)."""
import numpy as np
import pytest
import torch

import synth
from oracle import fp8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L(gpu):
    import latent_kv_cache_split_b200 as lib
    lib.check_device(clear=True)
    return lib


def _rows(rng, n, r, d_rope, std):
    x = rng.standard_normal((n, r + d_rope)).astype(np.float32) * np.float32(std)
    return torch.from_numpy(x).bfloat16()


def _check_rows(L, cache_rows, src_rows, r, d_rope):
    """cache_rows: [n, row_bytes] uint8 on the CPU; src_rows: the bf16 rows they came from."""
    codes, scales, kpe = L.fp8_cache_fields(cache_rows, r, d_rope)
    want_codes, want_scales = fp8.quantize_rows(src_rows[:, :r].float().numpy())
    got_codes = codes.numpy()
    bad = np.argwhere(got_codes != want_codes)
    assert bad.size == 0, f"{len(bad)} codes differ, first at {bad[:3].tolist()}"
    np.testing.assert_array_equal(scales.numpy().view(np.uint32), want_scales.view(np.uint32))
    assert torch.equal(kpe.view(torch.int16), src_rows[:, r:].contiguous().view(torch.int16))
    assert (cache_rows[:, r + 4:r + 16] == 0).all()


@pytest.mark.parametrize("r,d_rope,n", [(512, 64, 5000), (256, 64, 777), (16, 0, 33), (1024, 8, 65)])
def test_quantize_bit_exact(L, gpu, r, d_rope, n):
    rng = np.random.default_rng(r + n)
    src = _rows(rng, n, r, d_rope, 1 / 24)
    src[1] = 0                                         # zero row: scale 0, codes 0
    src[2] *= 1e-20                                    # tiny values, normal fp32 scale
    src[3, : r // 2] *= 300                            # wide range inside one row (many subnormal codes)
    cache = L.quantize_latent_fp8(src.to(gpu), r)
    torch.cuda.synchronize()
    assert L.check_device() == 0
    _check_rows(L, cache.cpu(), src, r, d_rope)


def test_quantize_from_interleaved_cache_slice(L, gpu):
    """Source rows are the bf16 MLA cache itself ([T, 576]: latent then RoPE key, row stride 576)."""
    w = synth.workload("mla_b64_l4096", batch=3, seqlen=None)
    d = synth.make_inputs(w, lengths=[300, 1, 129])
    src = d["cache"]
    rb = L.fp8_cache_row_bytes(512, 64)
    big = torch.full((src.shape[0], rb + 48), 0xAB, dtype=torch.uint8, device=gpu)   # padded rows
    L.quantize_latent_fp8(src.to(gpu), 512, cache=big)
    torch.cuda.synchronize()
    out = big.cpu()
    _check_rows(L, out, src, 512, 64)
    assert (out[:, rb:] == 0xAB).all()


def test_append_fp8_bit_exact_and_leaves_other_rows(L, gpu):
    rng = np.random.default_rng(9)
    lengths = [5, 130, 2, 64]
    s_q = 2
    cu = synth.prefix_offsets(lengths)
    T = int(cu[-1])
    r, d_rope = 512, 64
    rb = L.fp8_cache_row_bytes(r, d_rope)
    cache = torch.full((T + 3, rb), 0x5A, dtype=torch.uint8, device=gpu)
    new = _rows(rng, len(lengths) * s_q, r, d_rope, 0.05)
    cu_d = torch.from_numpy(cu.astype(np.int32)).to(gpu)
    L.latent_cache_append_fp8(new.to(gpu), cache, cu_d, s_q, r)
    torch.cuda.synchronize()
    assert L.check_device() == 0
    got = cache.cpu()
    dst = [int(cu[b]) + lengths[b] - s_q + i for b in range(len(lengths)) for i in range(s_q)]
    _check_rows(L, got[dst], new, r, d_rope)
    rest = sorted(set(range(T + 3)) - set(dst))
    assert (got[rest] == 0x5A).all()


def test_append_fp8_short_request_is_recorded(L, gpu):
    """A request shorter than s_q is skipped and reported in the device error word (no fault)."""
    r, d_rope = 64, 0
    rb = L.fp8_cache_row_bytes(r, d_rope)
    cache = torch.zeros((10, rb), dtype=torch.uint8, device=gpu)
    cu = torch.tensor([0, 1, 10], dtype=torch.int32, device=gpu)
    new = torch.ones((4, r), dtype=torch.bfloat16, device=gpu)
    L.latent_cache_append_fp8(new, cache, cu, 2, r)
    torch.cuda.synchronize()
    assert L.check_device(clear=True) == L.SITE_BAD_LENGTH
    # request 0 (L = 1) is skipped; request 1 (L = 9) writes rows 1 + 9 - 2 + i = 8, 9
    # ones: scale 2^-8 (the smallest power of two with 1 / s <= 448), code of 256 = 0x78
    assert (cache[:8] == 0).all() and (cache[8:10, :r] == 0x78).all()


def test_fp8_argument_errors(L, gpu):
    src = torch.zeros((4, 576), dtype=torch.bfloat16, device=gpu)
    with pytest.raises(ValueError):
        L.quantize_latent_fp8(src, 500)              # r not a multiple of 16
    cache = torch.zeros((4, 100), dtype=torch.uint8, device=gpu)
    with pytest.raises(L.LkvError) as e:
        L.quantize_latent_fp8(src, 512, cache=cache)  # rows shorter than the FP8 row size
    assert e.value.status == L.ERR_INVALID_ARG


def test_quantize_throughput(L, gpu):
    """Measurement (printed with -s): quantising the whole MLA B=64, L=4096 cache (262144 rows)."""
    T, r, d_rope = 64 * 4096, 512, 64
    src = torch.randn((T, r + d_rope), device=gpu).bfloat16()
    cache = torch.empty((T, L.fp8_cache_row_bytes(r, d_rope)), dtype=torch.uint8, device=gpu)
    for _ in range(3):
        L.quantize_latent_fp8(src, r, cache=cache)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(20):
        L.quantize_latent_fp8(src, r, cache=cache)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / 20
    moved = T * ((r + d_rope) * 2 + cache.shape[1])
    print(f"quantize {T} rows: {ms * 1e3:.1f} us, {moved / ms / 1e6:.0f} GB/s (bytes read + written)")


# ---------------------------------------------------------------------------------------------
# GTA decode over FP8 rows
import math  # noqa: E402

from gpu_util import compare  # noqa: E402


def _fp8_gta_case(lengths, s_q=2, groups=8, h_q=128, seed=0, extra_rows=0, std=None, q_std=None):
    """bf16 GTA inputs of the given shape, their tied states quantised into FP8 rows by the oracle."""
    kw = {} if std is None else {"input_std": std}
    if q_std is not None:
        kw["q_std"] = q_std
    w = synth.workload("gta_g8_sq2_l8192", batch=len(lengths), s_q=s_q, seqlen=None, groups=groups, h_q=h_q,
                       seed=seed, **kw)
    d = synth.make_inputs(w, lengths=lengths, extra_rows=extra_rows)
    width = w.groups * w.d_k
    tied = d["cache"][:, :width].float().numpy()
    kpe = d["cache"][:, width:].contiguous()
    codes, scales = fp8.quantize_rows(tied)
    rb = 16 * ((width + 16 + 2 * w.d_rope + 15) // 16)
    rows = np.zeros((tied.shape[0], rb), dtype=np.uint8)
    rows[:, :width] = codes
    rows[:, width:width + 4] = scales.view(np.uint8).reshape(-1, 4)
    rows[:, width + 16:width + 16 + 2 * w.d_rope] = kpe.view(torch.uint8).numpy()
    return w, d, torch.from_numpy(rows), codes, scales, kpe


def _run_fp8_gta(L, gpu, w, d, rows):
    return L.gta_group_decode_fp8(d["q"].to(gpu), d["q_rope"].to(gpu), rows.to(gpu), w.groups,
                                  d["cu_seqlens"].to(gpu), w.scale)


def _oracle_fp8_gta(w, d, codes, scales, kpe, requests=None):
    cu = d["cu_seqlens"].numpy().astype(np.int64)
    return fp8.gta_group_decode_fp8(d["q"], d["q_rope"], codes, scales, kpe, w.groups, cu, w.scale,
                                    requests=requests)


@pytest.mark.parametrize("lengths,s_q,groups", [([900, 130, 2, 1500], 2, 8), ([257, 1, 128, 129], 1, 8),
                                                ([700, 64, 3], 2, 4), ([1, 2, 3, 4000], 1, 2)])
def test_gta_fp8_decode_parity(L, gpu, lengths, s_q, groups):
    """Ragged lengths over several 128-key tiles and a tail, s_q 1 and 2, 8 / 4 / 2 groups (units of
    32, 64 and 64 rows)."""
    w, d, rows, codes, scales, kpe = _fp8_gta_case(lengths, s_q=s_q, groups=groups, h_q=128 if groups > 2 else 64)
    out, lse = _run_fp8_gta(L, gpu, w, d, rows)
    torch.cuda.synchronize()
    assert L.check_device() == 0
    ref_out, ref_lse = _oracle_fp8_gta(w, d, codes, scales, kpe)
    compare(out, lse, ref_out, ref_lse, label=f"gta fp8 {lengths} s_q={s_q} g={groups}")


@pytest.mark.parametrize("spread", [4.0, 16.0])
def test_gta_fp8_decode_wide_score_spread(L, gpu, spread):
    w, d, rows, codes, scales, kpe = _fp8_gta_case([900, 130, 2, 1500], std=0.5, q_std=2.0 * spread, seed=5)
    out, lse = _run_fp8_gta(L, gpu, w, d, rows)
    ref_out, ref_lse = _oracle_fp8_gta(w, d, codes, scales, kpe)
    compare(out, lse, ref_out, ref_lse, label=f"gta fp8 spread {spread}")


def test_gta_fp8_decode_full_size_sampled(L, gpu):
    """The GTA workload at full size (64 requests of 8192 keys, s_q = 2) in FP8: eight requests
    against the oracle."""
    w, d, rows, codes, scales, kpe = _fp8_gta_case([8192] * 64, seed=2)
    out, lse = _run_fp8_gta(L, gpu, w, d, rows)
    torch.cuda.synchronize()
    assert L.check_device() == 0
    req = [0, 9, 18, 27, 36, 45, 54, 63]
    ref_out, ref_lse = _oracle_fp8_gta(w, d, codes, scales, kpe, requests=req)
    compare(out, lse, ref_out, ref_lse, requests=req, label="gta fp8 full size")


def test_gta_fp8_rows_past_the_cache_do_not_leak(L, gpu):
    """NaN codes and an infinite scale in the rows after the last request give bitwise the result of
    zero rows there."""
    lengths = [100, 37, 129]
    w, d, rows, codes, scales, kpe = _fp8_gta_case(lengths, extra_rows=70)
    out0, lse0 = (t.clone() for t in _run_fp8_gta(L, gpu, w, d, rows))
    T = sum(lengths)
    bad = rows.clone()
    width = w.groups * w.d_k
    bad[T:, :width] = 0x7F                                    # e4m3 NaN
    bad[T:, width:width + 4] = torch.tensor(np.array([np.inf], dtype=np.float32).view(np.uint8))
    out1, lse1 = _run_fp8_gta(L, gpu, w, d, bad)
    torch.cuda.synchronize()
    assert torch.isfinite(out1.float()).all()
    assert torch.equal(out0, out1) and torch.equal(lse0, lse1)


def test_gta_fp8_agrees_with_bf16_gta_on_the_dequantised_states(L, gpu):
    """The FP8 decode and the bf16 GTA decode over the dequantised (bf16-exact) states compute on
    the same values.  The two run different kernels (the FP8 rows row-major, bf16 GTA with the keys
    in the MMA's M dimension), whose fp32 sums are taken in different orders, so they agree within
    the bf16 parity gates rather than bit for bit."""
    w, d, rows, codes, scales, kpe = _fp8_gta_case([700, 64, 3], seed=7)
    deq = torch.from_numpy(fp8.dequantize_rows(codes, scales)).bfloat16()
    assert torch.equal(deq.double(), torch.from_numpy(fp8.dequantize_rows(codes, scales)))
    out8, lse8 = _run_fp8_gta(L, gpu, w, d, rows)
    cache = torch.cat([deq, kpe], 1).to(gpu)
    width = w.groups * w.d_k
    out16, lse16 = L.gta_group_decode(d["q"].to(gpu), d["q_rope"].to(gpu), cache[:, :width], cache[:, width:],
                                      w.groups, d["cu_seqlens"].to(gpu), w.scale)
    torch.cuda.synchronize()
    compare(out8, lse8, out16.double().cpu().numpy(), lse16.double().cpu().numpy(), label="fp8 vs bf16 GTA")


def test_gta_fp8_argument_errors(L, gpu):
    w, d, rows, codes, scales, kpe = _fp8_gta_case([40, 50])
    q, qr, cu = d["q"].to(gpu), d["q_rope"].to(gpu), d["cu_seqlens"].to(gpu)
    short = torch.zeros((rows.shape[0], 1152), dtype=torch.uint8, device=gpu)
    with pytest.raises(L.LkvError) as e:   # rows shorter than the 1168-byte FP8 row
        L.gta_group_decode_fp8(q, qr, short, w.groups, cu, w.scale)
    assert e.value.status == L.ERR_INVALID_ARG
    with pytest.raises(L.LkvError) as e:   # one group: 256 rows per unit, more than the converters leave room for
        L.gta_group_decode_fp8(q, qr, rows.to(gpu), 1, cu, w.scale)
    assert e.value.status == L.ERR_UNSUPPORTED
