"""The C-ABI library on the CPU: it loads, exports every symbol include/lkv.h declares, and its
host-only logic (planning, workspace sizing, argument validation) behaves -- no GPU needed."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lkv():
    import importlib.util
    spec = importlib.util.spec_from_file_location("lkv_build", os.path.join(ROOT, "latent_kv_cache_split_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    import latent_kv_cache_split_b200 as L
    return L


def _declared():
    src = open(os.path.join(ROOT, "include", "lkv.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(lkv_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(lkv):
    names = _declared()
    assert len(names) >= 12
    lib = ctypes.CDLL(lkv.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(lkv.EXPORTED) == names


def test_version_and_status_strings(lkv):
    assert lkv.version() >= 100
    for s in range(6):
        assert lkv.status_string(s)
    assert lkv.status_string(99) == "unknown status"


@pytest.mark.parametrize("kind,B,s_q,G,want", [
    (0, 64, 1, 1, 64),      # MLA B=64: one range per request, no split
    (0, 128, 1, 1, 74),     # varlen MLA: one range per CTA pair
    (0, 128, 2, 1, 74),
    (0, 8, 1, 1, 74),       # long context: split across every pair
    (1, 64, 2, 8, 144),     # GQLA 512 units: 8 groups in lockstep x 18 blocks
    (2, 8, 1, 2, 148),      # GLA-2 long context: one range per SM (no lockstep for 2 groups)
    (1, 8, 1, 8, 144),
    (1, 1, 1, 8, 144),      # one request: every block is a slice of it
    (3, 64, 2, 8, 144),     # GTA runs the GQLA kernel and partition
    (1, 64, 2, 2, 128),     # GQA-2: 128 equal units nearly fill 148 SMs: one range per unit
    (4, 8, 1, 2, 148),      # GLA units of 64 rows: the ranges of kind 2
])
def test_plan_ranges(lkv, kind, B, s_q, G, want):
    assert lkv.plan_ranges(kind, B, s_q, G, 148) == want


def test_plan_rejects_bad_input(lkv):
    assert lkv.plan_ranges(5, 1, 1, 1, 148) == -1
    assert lkv.plan_ranges(0, 0, 1, 1, 148) == -1
    assert lkv.plan_ranges(0, 1, 1, 1, 1) == -1


def test_workspace_sizes(lkv):
    mla = lkv.mla_decode_workspace_size(64, 1, 128, 512, 148)
    P = 64
    assert mla >= 2 * P * 128 * 512 * 4 + 2 * P * 128 * 4 + 2 * P * 4
    g = lkv.group_decode_workspace_size(1, 64, 2, 128, 8, 128, 148)
    assert g >= 2 * 144 * 32 * 128 * 4
    assert lkv.group_decode_workspace_size(3, 64, 2, 128, 8, 128, 148) == g   # GTA: the GQLA layout
    assert lkv.group_decode_workspace_size(4, 8, 1, 128, 2, 256, 148) == lkv.group_decode_workspace_size(2, 8, 1, 128, 2, 256, 148) > 0
    assert lkv.group_decode_workspace_size(5, 1, 1, 128, 8, 128, 148) == 0
    assert lkv.group_decode_workspace_size(1, 1, 1, 128, 7, 128, 148) == 0


def _check_partition(segs, cu, kind, s_q, G, P):
    """Every tile of every unit is covered exactly once; slot rules hold."""
    B = len(cu) - 1
    T = {0: 256, 1: 128, 2: 64, 3: 128, 4: 128}[kind]   # keys per tile: MLA pair, GQLA, GLA, GTA, GLA keys-in-M
    upr = s_q if kind == 0 else G
    covered = {}
    by_range = {}
    for (p, b, k, lo, hi, complete, slot, uid) in segs:
        assert uid == b * upr + k
        L = cu[b + 1] - cu[b]
        keys = (L - s_q + k + 1) if kind == 0 else L
        nt = -(-keys // T)
        assert 0 <= lo < hi <= nt
        assert complete == int(lo == 0 and hi == nt)
        for t in range(lo, hi):
            assert (b, k, t) not in covered
            covered[(b, k, t)] = p
        by_range.setdefault(p, []).append((b, k, lo, hi, complete, slot))
    for b in range(B):
        L = cu[b + 1] - cu[b]
        for k in range(upr):
            keys = (L - s_q + k + 1) if kind == 0 else L
            for t in range(-(-keys // T)):
                assert (b, k, t) in covered
    sizes = []
    for p, lst in by_range.items():
        sizes.append(sum(hi - lo for (_, _, lo, hi, _, _) in lst))
        for idx, (b, k, lo, hi, complete, slot) in enumerate(lst):
            if complete:
                assert slot == -1
            else:
                assert slot == (0 if idx == 0 else 1)
                assert idx in (0, len(lst) - 1)
    assert max(sizes) - min(sizes) <= 1 if len(sizes) == P else True


@pytest.mark.parametrize("kind,s_q,G,P", [(0, 1, 1, 74), (0, 2, 1, 74), (1, 2, 8, 148), (2, 1, 2, 148),
                                         (0, 1, 1, 3), (1, 1, 4, 5), (1, 2, 8, 144), (1, 1, 4, 8),
                                         (4, 1, 2, 148), (4, 2, 4, 148), (3, 2, 8, 144), (3, 1, 4, 148)])
def test_partition_covers_every_tile_once(lkv, kind, s_q, G, P):
    rng = np.random.default_rng(kind * 10 + s_q + P)
    for trial in range(4):
        B = int(rng.integers(1, 40))
        lengths = rng.integers(s_q, 3000, size=B)
        cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
        segs = lkv.plan_segments(kind, cu, s_q, G, P)
        _check_partition(segs, cu.tolist(), kind, s_q, G, P)


def test_lockstep_ranges_share_requests(lkv):
    """With P a multiple of G, the G ranges of a block walk the same requests and tiles, one
    group each (the RoPE key rows they share are then read at the same time)."""
    rng = np.random.default_rng(7)
    lengths = rng.integers(2, 5000, size=23)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    G, P = 8, 144
    segs = lkv.plan_segments(1, cu, 2, G, P)
    _check_partition(segs, cu.tolist(), 1, 2, G, P)
    by_range = {}
    for (p, b, k, lo, hi, complete, slot, uid) in segs:
        assert k == p % G
        by_range.setdefault(p, []).append((b, lo, hi))
    for j in range(P // G):
        walks = [by_range.get(j * G + k, []) for k in range(G)]
        assert all(w == walks[0] for w in walks)


def test_partition_uniform_lengths_never_split(lkv):
    cu = np.arange(65, dtype=np.int32) * 4096
    segs = lkv.plan_segments(0, cu, 1, 1, 64)
    assert len(segs) == 64 and all(s[5] == 1 for s in segs)


def test_partition_tiny_requests_and_short_lengths(lkv):
    cu = np.array([0, 1, 2, 3, 67], dtype=np.int32)
    segs = lkv.plan_segments(0, cu, 1, 1, 74)
    _check_partition(segs, cu.tolist(), 0, 1, 1, 74)
    # L_b < s_q: that request contributes no tiles
    cu = np.array([0, 1, 5], dtype=np.int32)
    segs = lkv.plan_segments(0, cu, 2, 1, 4)
    assert all(s[1] == 1 for s in segs)


def _fake(n):
    return ctypes.c_void_p(n)


def test_validation_errors_need_no_gpu(lkv):
    """Malformed calls are rejected before any CUDA call, so this runs on a CPU-only host."""
    L = lkv
    P16 = _fake(1 << 20)
    cu = _fake(1 << 21)
    args = dict(q=P16, qr=P16, ckv=P16, cs=576, kpe=P16, ks=576, rows=1000, cu=cu, B=2, s_q=1,
                h=128, r=512, dr=64, scale=0.04, dt=0, out=P16, lse=P16, ws=P16, wsb=1 << 30, st=None)

    def call(**kw):
        a = dict(args, **kw)
        return L._mla(a["q"], a["qr"], a["ckv"], a["cs"], a["kpe"], a["ks"], a["rows"], a["cu"],
                      a["B"], a["s_q"], a["h"], a["r"], a["dr"], a["scale"], a["dt"], a["out"],
                      a["lse"], a["ws"], a["wsb"], a["st"])
    assert call(q=None) == L.ERR_INVALID_ARG
    assert call(s_q=3) == L.ERR_UNSUPPORTED
    assert call(B=0) == L.ERR_INVALID_ARG
    assert call(dt=7) == L.ERR_INVALID_ARG
    assert call(r=256) == L.ERR_UNSUPPORTED          # bf16 tensor-core path is r_kv = 512 only
    assert call(h=64) == L.ERR_UNSUPPORTED
    assert call(q=_fake((1 << 20) + 2)) == L.ERR_INVALID_ARG   # not 16-byte aligned
    assert call(cs=500) == L.ERR_INVALID_ARG          # row stride shorter than r_kv
    assert call(cs=580) == L.ERR_INVALID_ARG          # 1160-byte rows are not 16-byte aligned
    assert call(scale=float("nan")) == L.ERR_INVALID_ARG
    assert call(scale=0.0) == L.ERR_INVALID_ARG
    assert call(scale=-0.04) == L.ERR_INVALID_ARG
    assert call(rows=1 << 31) == L.ERR_UNSUPPORTED
    assert call(dt=1, r=2000, cs=2064) == L.ERR_UNSUPPORTED    # fp32 path limit
    # GQLA: h_q not a multiple of g; unsupported head width
    g = L._gqla(P16, P16, P16, 1024, P16, 1024, P16, 64, 1000, cu, 2, 2, 128, 3, 128, 64, 0.07, 0,
                P16, P16, P16, 1 << 30, None)
    assert g == L.ERR_INVALID_ARG
    g = L._gqla(P16, P16, P16, 1024, P16, 1024, P16, 64, 1000, cu, 2, 2, 128, 8, 96, 64, 0.07, 0,
                P16, P16, P16, 1 << 30, None)
    assert g == L.ERR_UNSUPPORTED
    g = L._gla(P16, P16, P16, 512, P16, 64, 1000, cu, 2, 1, 128, 2, 128, 64, 0.05, 0, P16, P16,
               P16, 1 << 30, None)
    assert g == L.ERR_UNSUPPORTED
    # GTA: tied rows shorter than g*d_h; h_q not a multiple of g; unsupported head width
    assert L._gta(P16, P16, P16, 1000, P16, 1088, 1000, cu, 2, 2, 128, 8, 128, 64, 0.07, 0,
                  P16, P16, P16, 1 << 30, None) == L.ERR_INVALID_ARG
    assert L._gta(P16, P16, P16, 1088, P16, 1088, 1000, cu, 2, 2, 128, 3, 128, 64, 0.07, 0,
                  P16, P16, P16, 1 << 30, None) == L.ERR_INVALID_ARG
    assert L._gta(P16, P16, P16, 1088, P16, 1088, 1000, cu, 2, 2, 128, 8, 96, 64, 0.07, 0,
                  P16, P16, P16, 1 << 30, None) == L.ERR_UNSUPPORTED
    # append: misaligned row size
    assert L._append(P16, 24, P16, 24, 10, 24, cu, 1, 1, None) == L.ERR_INVALID_ARG
    assert L._merge(P16, P16, 0, 4, 8, 0, P16, P16, None) == L.ERR_INVALID_ARG
    assert L._merge(P16, P16, 2, 4, 6, 0, P16, P16, None) == L.ERR_INVALID_ARG
    assert L._selftest(0, None) == L.ERR_INVALID_ARG


def test_projection_argument_errors_need_no_gpu(lkv):
    """The projection entry points reject bad arguments before any CUDA call."""
    P = _fake(1 << 20)
    st = ctypes.c_void_p(0)
    assert lkv._absorb(None, P, P, 4, 8, 4, 8, 16, 0, st) == lkv.ERR_INVALID_ARG
    assert lkv._absorb(P, P, P, 4, 6, 4, 8, 16, 0, st) == lkv.ERR_INVALID_ARG      # 6 heads, 4 groups
    assert lkv._absorb(P, P, P, 0, 8, 4, 8, 16, 0, st) == lkv.ERR_INVALID_ARG
    assert lkv._absorb(P, P, P, 4, 8, 4, 8, 16, 1, st) == lkv.ERR_UNSUPPORTED      # fp32
    assert lkv._unabsorb(P, P, None, 4, 8, 4, 16, 8, 0, st) == lkv.ERR_INVALID_ARG
    assert lkv._unabsorb(P, P, P, 4, 8, 3, 16, 8, 0, st) == lkv.ERR_INVALID_ARG
    assert lkv._unabsorb(P, P, P, 4, 8, 4, 16, 8, 1, st) == lkv.ERR_UNSUPPORTED
    assert lkv._expand(P, 8, P, P, 4, 2, 16, 8, 0, st) == lkv.ERR_INVALID_ARG      # row stride < r
    assert lkv._expand(P, 16, P, P, 0, 2, 16, 8, 0, st) == lkv.ERR_INVALID_ARG
    assert lkv._expand(P, 16, P, P, 4, 2, 16, 8, 1, st) == lkv.ERR_UNSUPPORTED
    # the tensor-core GEMM's TMA operands: 16-byte aligned pointers, rows of a multiple of 8 elements
    M = _fake((1 << 20) + 8)
    assert lkv._absorb(M, P, P, 4, 8, 4, 8, 16, 0, st) == lkv.ERR_INVALID_ARG      # misaligned q
    assert lkv._absorb(P, P, P, 4, 8, 4, 12, 16, 0, st) == lkv.ERR_INVALID_ARG     # d_h = 12
    assert lkv._unabsorb(P, P, P, 4, 8, 4, 20, 8, 0, st) == lkv.ERR_INVALID_ARG    # r = 20
    assert lkv._unabsorb(P, P, P, 4, 8, 4, 16, 12, 0, st) == lkv.ERR_INVALID_ARG   # d_v = 12
    assert lkv._unabsorb(P, M, P, 4, 8, 4, 16, 8, 0, st) == lkv.ERR_INVALID_ARG    # misaligned w_uv
    assert lkv._expand(P, 20, P, P, 4, 2, 16, 8, 0, st) == lkv.ERR_INVALID_ARG     # row stride 20
    assert lkv._expand(P, 16, P, P, 4, 2, 16, 12, 0, st) == lkv.ERR_INVALID_ARG    # d = 12
    assert lkv._expand(M, 16, P, P, 4, 2, 16, 8, 0, st) == lkv.ERR_INVALID_ARG     # misaligned c
    assert lkv._oproj(P, P, P, 4, 12, 8, 0, st) == lkv.ERR_INVALID_ARG             # k = 12
    assert lkv._oproj(P, P, P, 4, 16, 12, 1, st) == lkv.ERR_INVALID_ARG            # d_model = 12
    assert lkv._oproj(P, M, P, 4, 16, 8, 1, st) == lkv.ERR_INVALID_ARG             # misaligned w_o


def test_fp8_cache_rows_host_side(lkv):
    """FP8 row size and argument checks: no CUDA call is made for any of these."""
    assert lkv.fp8_cache_row_bytes(512, 64) == 656
    assert lkv.fp8_cache_row_bytes(16, 0) == 32
    assert lkv.fp8_cache_row_bytes(1024, 8) == 1056
    for r, dr in [(0, 64), (500, 64), (1040, 64), (512, 60), (512, -8)]:
        assert lkv.fp8_cache_row_bytes(r, dr) == 0
    P = _fake(1 << 20)
    st = ctypes.c_void_p(0)
    assert lkv._quant_fp8(None, 576, P, 656, 4, 512, 64, st) == lkv.ERR_INVALID_ARG
    assert lkv._quant_fp8(_fake((1 << 20) + 8), 576, P, 656, 4, 512, 64, st) == lkv.ERR_INVALID_ARG  # misaligned
    assert lkv._quant_fp8(P, 570, P, 656, 4, 512, 64, st) == lkv.ERR_INVALID_ARG    # rows shorter than r + d_rope
    assert lkv._quant_fp8(P, 580, P, 656, 4, 512, 64, st) == lkv.ERR_INVALID_ARG    # 1160-byte source rows
    assert lkv._quant_fp8(P, 576, P, 640, 4, 512, 64, st) == lkv.ERR_INVALID_ARG    # cache rows too short
    assert lkv._quant_fp8(P, 576, P, 656, 0, 512, 64, st) == lkv.ERR_INVALID_ARG
    assert lkv._quant_fp8(P, 576, P, 656, 4, 500, 64, st) == lkv.ERR_INVALID_ARG
    assert lkv._append_fp8(P, 576, P, 656, 10, 512, 64, None, 2, 1, st) == lkv.ERR_INVALID_ARG
    assert lkv._append_fp8(P, 576, P, 656, 10, 512, 64, P, 0, 1, st) == lkv.ERR_INVALID_ARG


def test_output_projection_argument_errors_need_no_gpu(lkv):
    P = _fake(1 << 20)
    st = ctypes.c_void_p(0)
    assert lkv._oproj(None, P, P, 4, 16, 8, 1, st) == lkv.ERR_INVALID_ARG
    assert lkv._oproj(P, P, P, 0, 16, 8, 1, st) == lkv.ERR_INVALID_ARG
    assert lkv._oproj(P, P, P, 4, 16, 8, 7, st) == lkv.ERR_INVALID_ARG
