"""The smoke check's own host logic on the CPU: __graft_entry__.smoke() with every device call of the
library answered by the oracle on the same arguments (so only its input building, argument order
and checks run here; the kernels themselves are covered by the -m gpu tests)."""
import numpy as np
import pytest
import torch

import oracle


def _as_out(res):
    o, l = res
    return torch.from_numpy(np.asarray(o)).bfloat16(), torch.from_numpy(np.asarray(l)).float()


def _cu(cu):
    return cu.cpu().numpy().astype(np.int64)


def test_smoke_runs_on_oracle_answers(monkeypatch, lkv_built):
    import __graft_entry__ as ge
    lkv = lkv_built

    class NoBuild:
        def build(self, *a, **k):
            pass

    real_device = torch.device
    monkeypatch.setattr(ge, "_build_module", lambda: NoBuild())
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    monkeypatch.setattr(torch, "device", lambda *a, **k: real_device("cpu"))
    monkeypatch.setattr(lkv, "check_device", lambda clear=True: 0)
    calls = []

    def mla(q, qr, ckv, kpe, cu, scale):
        calls.append("mla")
        return _as_out(oracle.mla_absorbed_decode(q, qr, ckv, kpe, _cu(cu), scale))

    def gqla(q, qr, k, v, kpe, cu, scale):
        calls.append("gqla")
        return _as_out(oracle.gqla_group_decode(q, qr, k, v, kpe, _cu(cu), scale))

    def gta(q, qr, kv, kpe, g, cu, scale):
        calls.append("gta")
        assert kv.shape[1] == g * q.shape[-1] and kpe.shape[1] == qr.shape[-1]
        return _as_out(oracle.gta_group_decode(q, qr, kv.contiguous(), kpe, g, _cu(cu), scale))

    def gla(q, qr, clat, kpe, n_lat, cu, scale):
        calls.append("gla")
        assert clat.shape[1] == n_lat * q.shape[-1]
        return _as_out(oracle.gla_group_decode(q, qr, clat.contiguous(), kpe, n_lat, _cu(cu), scale))

    def gta8(q, qr, rows, g, cu, scale):
        calls.append("gta8")
        width = g * q.shape[-1]
        c, s, k = lkv.fp8_cache_fields(rows, width, qr.shape[-1])
        return _as_out(oracle.fp8.gta_group_decode_fp8(q, qr, c.numpy(), s.numpy(), k, g, _cu(cu), scale))

    monkeypatch.setattr(lkv, "mla_absorbed_decode", mla)
    monkeypatch.setattr(lkv, "gqla_group_decode", gqla)
    monkeypatch.setattr(lkv, "gta_group_decode", gta)
    monkeypatch.setattr(lkv, "gla_group_decode", gla)
    monkeypatch.setattr(lkv, "gta_group_decode_fp8", gta8)
    ge.smoke()
    assert calls == ["mla", "gqla", "gta", "gla", "gta8"]


def test_smoke_rejects_a_wrong_answer(monkeypatch, lkv_built):
    """The smoke's gate is live: an output off by more than the bf16 gate fails it."""
    import __graft_entry__ as ge
    lkv = lkv_built

    class NoBuild:
        def build(self, *a, **k):
            pass

    real_device = torch.device
    monkeypatch.setattr(ge, "_build_module", lambda: NoBuild())
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    monkeypatch.setattr(torch, "device", lambda *a, **k: real_device("cpu"))
    monkeypatch.setattr(lkv, "check_device", lambda clear=True: 0)

    def mla_off(q, qr, ckv, kpe, cu, scale):
        o, l = oracle.mla_absorbed_decode(q, qr, ckv, kpe, _cu(cu), scale)
        return _as_out((o * 1.05, l))

    monkeypatch.setattr(lkv, "mla_absorbed_decode", mla_off)
    with pytest.raises(RuntimeError, match="MLA smoke mismatch"):
        ge.smoke()
