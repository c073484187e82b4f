"""Group-axis tensor parallelism for the GQA path of GQLA.

The GQA path keeps g expanded key/value groups, and a group's heads read only that group's K_j,
V_j. The GQLA explainer (section 2, "Methodology", GQA path) notes that this allows tensor
parallelism along the group axis, up to 8 ways, with no redundancy. Here each rank holds the cache
of g / world consecutive groups (only the small shared RoPE key is on every rank) and the query
heads of those groups. It decodes them with the library's grouped kernel and multiplies its heads'
outputs by the matching row block of W_O. The full output projection is the sum of the ranks'
partials, one all-reduce over the group.

Host logic only: every computation runs in the library (or in the functions passed in), and the
sum goes through torch.distributed (NCCL on GPUs). A single kernel that fuses the projection with
the reduction over NVLink peer memory is not built.
"""
from __future__ import annotations

from dataclasses import dataclass

__all__ = ["GroupShard", "group_shard", "GroupAxisTP"]


@dataclass(frozen=True)
class GroupShard:
    """The groups [g0, g1) and query heads [h0, h1) that one rank owns."""
    rank: int
    world: int
    g: int
    h_q: int
    g0: int
    g1: int
    h0: int
    h1: int

    @property
    def groups(self) -> int:
        return self.g1 - self.g0

    @property
    def heads(self) -> int:
        return self.h1 - self.h0

    def w_o_rows(self, d_v: int) -> slice:
        """Rows of W_O [h_q * d_v, d_model] that multiply this rank's heads."""
        return slice(self.h0 * d_v, self.h1 * d_v)


def group_shard(g: int, h_q: int, world: int, rank: int) -> GroupShard:
    """Contiguous blocks of g / world groups per rank; heads follow their groups (head h is in
    group h // (h_q / g)). world must divide g and g must divide h_q."""
    if g <= 0 or h_q <= 0 or world <= 0 or not 0 <= rank < world:
        raise ValueError("bad group-axis shard arguments")
    if g % world or h_q % g:
        raise ValueError(f"group-axis TP needs world | g and g | h_q (g={g}, h_q={h_q}, world={world})")
    per = g // world
    hpg = h_q // g
    g0, g1 = rank * per, (rank + 1) * per
    return GroupShard(rank, world, g, h_q, g0, g1, g0 * hpg, g1 * hpg)


class GroupAxisTP:
    """One decode step of the GQA path with the groups split across the ranks of `group`.

    decode_fn(q, q_rope, k, v, kpe, cu_seqlens, scale) -> (out [B, s_q, heads, d_v], lse)
    proj_fn(o [n_tok, heads * d_v], w_o_rows) -> partial y [n_tok, d_model]
    allreduce_fn(y) sums y over the ranks and returns the sum.
    The defaults are the library's grouped decode, its output projection (fp32 partial) and
    torch.distributed.all_reduce over `group` (a no-op for one rank)."""

    def __init__(self, shard: GroupShard, group=None, decode_fn=None, proj_fn=None, allreduce_fn=None):
        self.shard = shard
        self.group = group
        if decode_fn is None or proj_fn is None:
            from . import gqla_group_decode, output_projection
            decode_fn = decode_fn or gqla_group_decode
            proj_fn = proj_fn or output_projection
        self.decode_fn = decode_fn
        self.proj_fn = proj_fn
        self.allreduce_fn = allreduce_fn or self._all_reduce

    def _all_reduce(self, y):
        if self.shard.world > 1:
            import torch.distributed as dist
            dist.all_reduce(y, op=dist.ReduceOp.SUM, group=self.group)
        return y

    def local_query(self, q):
        """This rank's heads of a full [B, s_q, h_q, d] query."""
        return q[:, :, self.shard.h0:self.shard.h1].contiguous()

    def local_cache(self, x):
        """This rank's groups of a full [rows, g, d] expanded cache (a copy, owned by the rank)."""
        return x[:, self.shard.g0:self.shard.g1].contiguous()

    def step(self, q_local, q_rope_local, k_local, v_local, kpe, cu_seqlens, scale, w_o_local):
        """Decode this rank's heads, project them with their rows of W_O, and sum over the ranks.
        Returns (y [B * s_q, d_model], out_local, lse_local); y is the full projection on every rank."""
        sh = self.shard
        if q_local.shape[2] != sh.heads or k_local.shape[1] != sh.groups or v_local.shape[1] != sh.groups:
            raise ValueError("local query heads / cache groups do not match the shard")
        out, lse = self.decode_fn(q_local, q_rope_local, k_local, v_local, kpe, cu_seqlens, scale)
        B, s_q, heads, d_v = out.shape
        if w_o_local.shape[0] != heads * d_v:
            raise ValueError("w_o_local must hold heads * d_v rows")
        y = self.proj_fn(out.reshape(B * s_q, heads * d_v), w_o_local)
        return self.allreduce_fn(y), out, lse
