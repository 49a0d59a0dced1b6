"""Group-axis tensor parallelism of the GQA path over P GPUs.

GQLA's per-group expansion splits along the group axis with no redundancy: P
GPUs each hold g/P of the groups' expanded cache, 8-way at g = 8 and 4-way at
g = 4 (GQLA, paperlayer.ai summary of arXiv:2605.15250v3, sec. 1
Introduction and sec. 4 Roofline Analysis, "Configuration tradeoffs";
gist.science technical summary, sec. 2 "Architektur").

Rank r of P takes groups [r g/P, (r+1) g/P): their planes of the expanded cache
and of W_UK / W_UV, the shared RoPE keys (replicated), and the query heads of
those groups.  Heads map to groups in contiguous blocks of G = h/g, so a
rank's heads are the contiguous block [r h/P, (r+1) h/P).  Attention needs no
exchange: every rank runs the ordinary GQA-path calls (gqla_decode_gqa and
gqla_combine of libgqla) on its own dims (h/P heads over g/P groups).  The
per-head outputs are then gathered so that every rank holds the layer's whole
output: the combine writes a rank's block straight into its slot of a
[P][batch][s_q][h/P][128] buffer and one in-place all-gather (NCCL on GPUs)
fills the other slots.  Head r h/P + j of the layer is local head j of rank r,
so that buffer read as [batch][s_q][P][h/P][128] is the output in head order
(`heads_view`); nothing is copied to put it there.

The absorb path is not split this way: every head attends over the whole
latent row, so splitting its heads would replicate the latent cache.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


class GroupShard:
    """Which groups and heads rank `rank` of `world` owns (host-side arithmetic)."""

    def __init__(self, num_heads: int, num_groups: int, rank: int, world: int):
        if world < 1 or not 0 <= rank < world:
            raise ValueError(f"rank {rank} of {world}")
        if num_groups % world or num_heads % num_groups:
            raise ValueError(f"{num_groups} groups ({num_heads} heads) do not split over {world} ranks")
        self.num_heads, self.num_groups, self.rank, self.world = num_heads, num_groups, rank, world
        self.groups = num_groups // world          # g / P
        self.heads = num_heads // world            # h / P = G g / P
        self.group0 = rank * self.groups
        self.head0 = rank * self.heads

    def group_of_local_head(self, j: int) -> int:
        """Global group of local head j (the layer's head head0 + j)."""
        return (self.head0 + j) // (self.num_heads // self.num_groups)

    def slice_groups(self, t: torch.Tensor, dim: int = 0) -> torch.Tensor:
        """This rank's groups of a per-group tensor ([g][...] weights, or an expanded
        cache [g][slots][256]), as a contiguous tensor."""
        return t.narrow(dim, self.group0, self.groups).contiguous()

    def slice_heads(self, t: torch.Tensor, dim: int = 2) -> torch.Tensor:
        """This rank's heads of a per-head tensor (q [B][s_q][h][192] by default)."""
        return t.narrow(dim, self.head0, self.heads).contiguous()


def gather_heads_(buf: torch.Tensor, rank: int, world: int, group=None) -> torch.Tensor:
    """In-place all-gather over a flat buffer of `world` equal blocks, block `rank`
    already written by this rank: afterwards every rank holds every block."""
    n = buf.numel() // world
    if buf.numel() != n * world or not buf.is_contiguous():
        raise ValueError("the gather buffer must be contiguous and hold world equal blocks")
    if world > 1:
        dist.all_gather_into_tensor(buf, buf[rank * n:(rank + 1) * n], group=group)
    return buf


def rank_block(buf: torch.Tensor, rank: int, world: int, *shape) -> torch.Tensor:
    """Block `rank` of a flat gather buffer of `world` equal blocks, viewed as `shape`."""
    n = buf.numel() // world
    return buf[rank * n:(rank + 1) * n].view(*shape)


def heads_view(buf: torch.Tensor, world: int, batch: int, s_q: int, heads_local: int, *tail):
    """The gathered [P][batch][s_q][h/P](...) buffer as [batch][s_q][P][h/P](...), i.e.
    the layer's heads in order (head r h/P + j at [:, :, r, j]); a view, no copy."""
    return buf.view(world, batch, s_q, heads_local, *tail).movedim(0, 2)


class GqaTensorParallel:
    """One rank's GQA-path decode step under group-axis tensor parallelism.

    The local calls go through libgqla's C ABI (decode_attention_06_b200.gqla);
    the gather through torch.distributed (NCCL process group on GPUs)."""

    def __init__(self, shard: GroupShard, batch: int, s_q: int, num_splits: int, device,
                 softmax_scale=None, group=None):
        from decode_attention_06_b200 import gqla
        self.gqla, self.shard, self.group = gqla, shard, group
        self.batch, self.s_q = batch, s_q
        self.dims = gqla.make_dims(shard.heads, shard.groups, softmax_scale)
        self.bufs = gqla.DecodeBuffers(self.dims, batch, s_q, num_splits, "gqa", device=device)
        P, r = shard.world, shard.rank
        self.out_all = torch.empty(P * batch * s_q * shard.heads * gqla.D_V, dtype=torch.bfloat16,
                                   device=device)
        self.lse_all = torch.empty(P * batch * s_q * shard.heads, dtype=torch.float32, device=device)
        # the combine writes this rank's heads straight into its slot of the gather buffers
        self.bufs.out = rank_block(self.out_all, r, P, batch, s_q, shard.heads, gqla.D_V)
        self.bufs.lse = rank_block(self.lse_all, r, P, batch, s_q, shard.heads)

    def local_step(self, q_local, kv_expanded_local, k_rope, kv, stream=None):
        """This rank's heads: gqla_decode_gqa + gqla_combine on the local dims."""
        self.gqla.decode_step(self.dims, self.bufs, q_local, None, None, kv,
                              kv_expanded=kv_expanded_local, k_rope=k_rope, stream=stream)

    def gather(self):
        """Every rank's heads to every rank; returns (out [B][s_q][P][h/P][128],
        lse [B][s_q][P][h/P]) views in head order."""
        P, r = self.shard.world, self.shard.rank
        gather_heads_(self.out_all, r, P, self.group)
        gather_heads_(self.lse_all, r, P, self.group)
        return (heads_view(self.out_all, P, self.batch, self.s_q, self.shard.heads, self.gqla.D_V),
                heads_view(self.lse_all, P, self.batch, self.s_q, self.shard.heads))

    def step(self, q_local, kv_expanded_local, k_rope, kv, stream=None):
        self.local_step(q_local, kv_expanded_local, k_rope, kv, stream)
        return self.gather()
