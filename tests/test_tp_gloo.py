"""Group-axis tensor parallelism on CPU: the shard plan, and two gloo ranks (127.0.0.1) that each
decode their groups and project their heads, summed by an all-reduce, against the full
single-process result.  The ranks' compute is the fp64 oracle passed in as the decode and
projection functions, so only the host logic of the library's runner is under test here."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from latent_kv_cache_split_b200.tp import GroupAxisTP, group_shard


@pytest.mark.parametrize("g,h_q", [(8, 128), (4, 128), (2, 128), (8, 8)])
def test_group_shard_covers_every_group_and_head_once(g, h_q):
    hpg = h_q // g
    for world in [w for w in (1, 2, 4, 8) if g % w == 0]:
        groups, heads = [], []
        for rank in range(world):
            sh = group_shard(g, h_q, world, rank)
            groups += list(range(sh.g0, sh.g1))
            heads += list(range(sh.h0, sh.h1))
            assert all(h // hpg in range(sh.g0, sh.g1) for h in range(sh.h0, sh.h1))
            rows = sh.w_o_rows(16)
            assert (rows.start, rows.stop) == (sh.h0 * 16, sh.h1 * 16)
        assert groups == list(range(g)) and heads == list(range(h_q))


def test_group_shard_rejects_uneven_splits():
    with pytest.raises(ValueError):
        group_shard(8, 128, 3, 0)
    with pytest.raises(ValueError):
        group_shard(8, 100, 2, 0)
    with pytest.raises(ValueError):
        group_shard(8, 128, 2, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _inputs():
    rng = np.random.default_rng(31)
    B, S, H, g, d, dr, dm = 2, 2, 8, 4, 6, 4, 10
    lengths = [5, 9]
    cu = np.concatenate([[0], np.cumsum(lengths)])
    T = int(cu[-1])
    return dict(q=rng.standard_normal((B, S, H, d)), qr=rng.standard_normal((B, S, H, dr)),
                k=rng.standard_normal((T, g, d)), v=rng.standard_normal((T, g, d)),
                kpe=rng.standard_normal((T, dr)), cu=cu, w_o=rng.standard_normal((H * d, dm)), g=g, H=H, d=d)


def _oracle_decode(q, qr, k, v, kpe, cu, scale):
    import oracle
    out, lse = oracle.gqla_group_decode(q.numpy(), qr.numpy(), k.numpy(), v.numpy(), kpe.numpy(),
                                        cu.numpy(), scale)
    return torch.from_numpy(out), torch.from_numpy(lse)


def _worker(rank, world, port, q):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = _inputs()
        sh = group_shard(x["g"], x["H"], world, rank)
        tp = GroupAxisTP(sh, decode_fn=_oracle_decode, proj_fn=lambda o, w: o @ w)
        T = lambda a: torch.from_numpy(np.ascontiguousarray(a))
        y, out, _ = tp.step(tp.local_query(T(x["q"])), tp.local_query(T(x["qr"])), tp.local_cache(T(x["k"])),
                            tp.local_cache(T(x["v"])), T(x["kpe"]), T(x["cu"]), 0.4,
                            T(x["w_o"][sh.w_o_rows(x["d"])]))
        q.put((rank, y.numpy(), out.numpy(), (sh.h0, sh.h1)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_sum_to_the_full_projection():
    import oracle
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x = _inputs()
    out, _ = oracle.gqla_group_decode(x["q"], x["qr"], x["k"], x["v"], x["kpe"], x["cu"], 0.4)
    B, S = out.shape[:2]
    y_full = oracle.output_projection(out.reshape(B * S, x["H"], x["d"]), x["w_o"])
    for rank, y, out_local, (h0, h1) in res:
        np.testing.assert_allclose(y, y_full, atol=1e-10)         # every rank holds the full sum
        np.testing.assert_allclose(out_local, out[:, :, h0:h1], atol=1e-12)
    assert res[0][3] == (0, 4) and res[1][3] == (4, 8)


def test_step_checks_local_shapes_and_single_rank_needs_no_process_group():
    sh = group_shard(4, 8, 2, 1)                      # groups 2..3, heads 4..7
    calls = []

    def dec(q, qr, k, v, kpe, cu, scale):
        calls.append(q.shape)
        return torch.ones((q.shape[0], q.shape[1], q.shape[2], 3), dtype=torch.float64), None

    tp = GroupAxisTP(sh, decode_fn=dec, proj_fn=lambda o, w: o @ w, allreduce_fn=lambda y: y)
    q = torch.zeros((2, 1, 8, 3), dtype=torch.float64)
    k = torch.zeros((5, 4, 3), dtype=torch.float64)
    with pytest.raises(ValueError):
        tp.step(q, q, tp.local_cache(k), tp.local_cache(k), None, None, 1.0, torch.zeros((12, 2)))  # all 8 heads
    with pytest.raises(ValueError):
        tp.step(tp.local_query(q), tp.local_query(q), k, k, None, None, 1.0, torch.zeros((12, 2)))   # all 4 groups
    with pytest.raises(ValueError):
        tp.step(tp.local_query(q), tp.local_query(q), tp.local_cache(k), tp.local_cache(k), None, None, 1.0,
                torch.zeros((11, 2), dtype=torch.float64))                                        # W_O rows
    y, out, _ = tp.step(tp.local_query(q), tp.local_query(q), tp.local_cache(k), tp.local_cache(k), None, None, 1.0,
                        torch.ones((12, 2), dtype=torch.float64))
    assert calls[-1] == (2, 1, 4, 3) and y.shape == (2, 2) and torch.all(y == 12)
    # one rank: the default reduction is the identity and needs no process group
    one = GroupAxisTP(group_shard(4, 8, 1, 0), decode_fn=dec, proj_fn=lambda o, w: o @ w)
    y1, _, _ = one.step(q, q, k, k, None, None, 1.0, torch.ones((24, 2), dtype=torch.float64))
    assert torch.all(y1 == 24)
