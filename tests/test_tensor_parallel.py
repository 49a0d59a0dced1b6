"""Group-axis tensor parallelism of the GQA path on the CPU: the partition of
groups and heads over P ranks, and the in-place all-gather that assembles the
per-head outputs, in a world-size-2 gloo process group.  Each rank's heads are
computed by the fp64 oracle on that rank's slice of the inputs (the CUDA
kernels need a GPU; tests/test_gpu_tp.py runs them on every rank's slice), and
the assembled output must equal the oracle on the whole layer."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from decode_attention_06_b200 import synth
from decode_attention_06_b200.tp import GroupShard, gather_heads_, heads_view, rank_block


@pytest.mark.parametrize("h,g,P", [(128, 8, 1), (128, 8, 2), (128, 8, 4), (128, 8, 8),
                                   (128, 4, 2), (128, 4, 4), (32, 8, 8)])
def test_shards_partition_groups_and_heads(h, g, P):
    G = h // g
    seen_groups, seen_heads = [], []
    for r in range(P):
        s = GroupShard(h, g, r, P)
        assert s.groups == g // P and s.heads == h // P
        seen_groups += list(range(s.group0, s.group0 + s.groups))
        seen_heads += list(range(s.head0, s.head0 + s.heads))
        for j in range(s.heads):  # every local head belongs to one of the rank's own groups
            assert s.group0 <= s.group_of_local_head(j) < s.group0 + s.groups
            assert s.group_of_local_head(j) == (s.head0 + j) // G
    assert seen_groups == list(range(g)) and seen_heads == list(range(h))


def test_shard_rejects_uneven_splits():
    with pytest.raises(ValueError):
        GroupShard(128, 8, 0, 3)
    with pytest.raises(ValueError):
        GroupShard(128, 8, 2, 2)


def test_heads_view_is_head_order():
    P, B, s_q, hl = 4, 2, 2, 3
    buf = torch.arange(P * B * s_q * hl, dtype=torch.float32)
    for r in range(P):
        blk = rank_block(buf, r, P, B, s_q, hl)
        blk.copy_(torch.tensor([[[1000 * r + 100 * b + 10 * s + j for j in range(hl)]
                                 for s in range(s_q)] for b in range(B)], dtype=torch.float32))
    v = heads_view(buf, P, B, s_q, hl)
    assert v.shape == (B, s_q, P, hl)
    full = v.reshape(B, s_q, P * hl)
    for b in range(B):
        for s in range(s_q):
            for h in range(P * hl):
                assert full[b, s, h] == 1000 * (h // hl) + 100 * b + 10 * s + h % hl


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _rank(rank, world, port, h, g, s_q, result):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        case = synth.make_case(h, g, [300, 64, 129], s_q, paged=True, seed=77)  # the same on every rank
        shard = GroupShard(h, g, rank, world)
        B = case["seqlens"].numel()
        # this rank's heads over its groups only: its slice of q and of the weights
        out_loc, lse_loc = oracle.decode(shard.slice_heads(case["q"]), case["latent"], case["page_table"],
                                         case["seqlens"], shard.slice_groups(case["w_uk"]),
                                         shard.slice_groups(case["w_uv"]), shard.groups)
        out_all = torch.full((world * B * s_q * shard.heads * 128,), float("nan"), dtype=torch.float64)
        lse_all = torch.full((world * B * s_q * shard.heads,), float("nan"), dtype=torch.float64)
        rank_block(out_all, rank, world, B, s_q, shard.heads, 128).copy_(torch.from_numpy(out_loc))
        rank_block(lse_all, rank, world, B, s_q, shard.heads).copy_(torch.from_numpy(lse_loc))
        gather_heads_(out_all, rank, world)
        gather_heads_(lse_all, rank, world)
        out = heads_view(out_all, world, B, s_q, shard.heads, 128).reshape(B, s_q, h, 128)
        lse = heads_view(lse_all, world, B, s_q, shard.heads).reshape(B, s_q, h)
        ref, ref_lse = oracle.decode(case["q"], case["latent"], case["page_table"], case["seqlens"],
                                     case["w_uk"], case["w_uv"], g)
        result[rank, 0] = float(np.abs(out.numpy() - ref).max())
        result[rank, 1] = float(np.abs(lse.numpy() - ref_lse).max())
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("h,g,s_q", [(128, 8, 2), (128, 4, 1), (32, 8, 1)])
def test_two_ranks_assemble_the_whole_layer(h, g, s_q):
    world = 2
    result = torch.full((world, 2), float("nan"), dtype=torch.float64).share_memory_()
    mp.start_processes(_rank, args=(world, _free_port(), h, g, s_q, result), nprocs=world,
                       start_method="spawn")
    # each rank's sliced computation is the same fp64 arithmetic as the whole layer's
    assert (result <= 1e-12).all(), result
