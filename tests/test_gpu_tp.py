"""Group-axis tensor parallelism of the GQA path on one GPU: the ranks are run one
after another (no rank waits for another), each through libgqla's C ABI on its
own slice (h/P heads over g/P groups: 4, 2 and 1 groups per rank), and their
per-head blocks are placed as the all-gather would place them.  The assembled
output must match the fp64 oracle on the whole layer."""
import pytest
import torch

from decode_attention_06_b200 import synth
from decode_attention_06_b200.tp import GqaTensorParallel, GroupShard, heads_view, rank_block
from tests.helpers import compare, compare_lse, oracle_ref, to_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")


TP = [
    # id, h, g, P, seqlens, s_q, paged, splits per rank
    ("g8_p2", 128, 8, 2, [700, 64, 1, 333], 2, True, 7),
    ("g8_p4", 128, 8, 4, [1000, 129], 1, True, 5),
    ("g8_p8", 128, 8, 8, [513, 0, 70], 2, False, 4),
    ("g4_p2", 128, 4, 2, [900, 200], 1, True, 6),
    ("g4_p4", 128, 4, 4, [300, 64], 1, False, 3),
    ("h32_g8_p8", 32, 8, 8, [2000, 3], 2, False, 9),
]


@pytest.mark.parametrize("cid,h,g,P,seqlens,s_q,paged,splits", TP, ids=[c[0] for c in TP])
def test_group_parallel_ranks_assemble_the_layer(cid, h, g, P, seqlens, s_q, paged, splits):
    from decode_attention_06_b200 import gqla
    case = synth.make_case(h, g, seqlens, s_q, paged=paged, seed=500 + len(cid) + P)
    gc = to_gpu(case)
    B = len(seqlens)
    kv = gqla.make_kv_index(gc["page_table"], gc["seqlens"], case["num_pages"])
    n = case["num_pages"] * case["page_size"]
    out_all = torch.full((P * B * s_q * (h // P) * 128,), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse_all = torch.full((P * B * s_q * (h // P),), float("nan"), dtype=torch.float32, device="cuda")
    for r in range(P):
        shard = GroupShard(h, g, r, P)
        tp = GqaTensorParallel(shard, B, s_q, splits, "cuda")
        # the rank's own expanded cache: its groups' planes only, from its slice of the weights
        kvx = torch.empty(shard.groups, n, 256, dtype=torch.bfloat16, device="cuda")
        kr = torch.empty(n, 64, dtype=torch.bfloat16, device="cuda")
        gqla.gqla_expand_cache(tp.dims, gc["latent"], shard.slice_groups(gc["w_uk"]),
                               shard.slice_groups(gc["w_uv"]), kvx, kr)
        tp.local_step(shard.slice_heads(gc["q"]), kvx, kr, kv)
        torch.cuda.synchronize()
        assert gqla.gqla_read_device_error(tp.bufs.workspace)[0] == 0
        # what the all-gather delivers: block r of every rank's buffer is rank r's heads
        rank_block(out_all, r, P, B, s_q, h // P, 128).copy_(rank_block(tp.out_all, r, P, B, s_q, h // P, 128))
        rank_block(lse_all, r, P, B, s_q, h // P).copy_(rank_block(tp.lse_all, r, P, B, s_q, h // P))
    out = heads_view(out_all, P, B, s_q, h // P, 128).reshape(B, s_q, h, 128)
    lse = heads_view(lse_all, P, B, s_q, h // P).reshape(B, s_q, h)
    ref, ref_lse = oracle_ref(case)
    compare(out, ref, what=f"tp/{cid}")
    compare_lse(lse, ref_lse, what=f"tp/{cid}")
