"""GPU tests for FP8 (e4m3) latent cache rows: the quantisation kernel against the oracle's fp32
steps, bit for bit (the codes are integers that floating point decides, and both sides take the
same IEEE fp32 division and round-to-nearest-even), in bulk and at append."""
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
    assert (cache[:8] == 0).all() and (cache[8:10, :r] == 0x7E).all()   # ones quantise to 448


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
