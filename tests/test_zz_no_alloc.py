"""gqla_decode_gqa_noalloc: the GQA decode step for callers that cannot allocate
device memory (no partial buffers, no workspace from the caller; the library
keeps its scratch in a fixed device array).

Its output must match the ordinary entry points (gqla_decode_gqa followed by
gqla_combine, with caller-allocated scratch) within the parity tolerance, on
two calls in a row -- the second call reuses the array the first one left
behind.  This file is collected last so that a failure here does not stop a
`-x` run before the rest of the suite.
"""
import ctypes

import pytest
import torch

from decode_attention_06_b200 import synth
from tests.helpers import compare, run_decode, to_gpu


def _noalloc(gcase, num_splits):
    from decode_attention_06_b200 import gqla
    h, g, s_q = gcase["num_heads"], gcase["num_groups"], gcase["s_q"]
    B = gcase["seqlens"].numel()
    dims = gqla.make_dims(h, g)
    kv = gqla.make_kv_index(gcase["page_table"], gcase["seqlens"], gcase["num_pages"])
    n = gcase["num_pages"] * gcase["page_size"]
    kvx = torch.empty(g, n, 256, dtype=torch.bfloat16, device="cuda")
    kr = torch.empty(n, 64, dtype=torch.bfloat16, device="cuda")
    gqla.gqla_expand_cache(dims, gcase["latent"], gcase["w_uk"], gcase["w_uv"], kvx, kr)
    out = torch.full((B, s_q, h, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, s_q, h), float("nan"), dtype=torch.float32, device="cuda")
    err = torch.full((2,), 7, dtype=torch.int32, device="cuda")
    gqla.gqla_decode_gqa_noalloc(dims, gcase["q"], kvx, kr, kv, num_splits, out, lse, err)
    torch.cuda.synchronize()
    return out, lse, err.cpu().tolist()


@pytest.mark.gpu
def test_noalloc_matches_allocating_entry_points_twice():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    cases = [
        (synth.make_case(128, 8, [700, 64, 1, 333], 2, paged=True, seed=301), 11),
        (synth.make_case(32, 8, [2000, 5, 129], 1, paged=False, seed=302), 6),
    ]
    for case, splits in cases:  # two calls in a row, different shapes and data
        g = to_gpu(case)
        ref_out, ref_lse, _, _ = run_decode(g, "gqa", splits)
        out, lse, err = _noalloc(g, splits)
        assert err == [0, 0]
        compare(out, ref_out.float().cpu().double().numpy(), what="noalloc vs allocating")
        torch.testing.assert_close(lse, ref_lse, rtol=0, atol=1e-5)


@pytest.mark.gpu
def test_noalloc_rejects_partials_beyond_the_static_limit():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from decode_attention_06_b200 import gqla
    case = to_gpu(synth.make_case(128, 8, [64], 2, seed=303))
    dims = gqla.make_dims(128, 8)
    kv = gqla.make_kv_index(case["page_table"], case["seqlens"], case["num_pages"])
    n = case["num_pages"] * 64
    kvx = torch.zeros(8, n, 256, dtype=torch.bfloat16, device="cuda")
    kr = torch.zeros(n, 64, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(1, 2, 128, 128, dtype=torch.bfloat16, device="cuda")
    # (1 + 300) * 2 * 128 rows * 516 B > 32 MiB
    with pytest.raises(gqla.GqlaError) as e:
        gqla.gqla_decode_gqa_noalloc(dims, case["q"], kvx, kr, kv, 300, out)
    assert e.value.status == -3
