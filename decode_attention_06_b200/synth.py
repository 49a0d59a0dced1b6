"""Seeded synthetic GQLA decode inputs.

This module is the one piece shared by the CUDA path's tests/benchmark and the
fp64 oracle: it only draws random numbers and lays them out.  It holds none of
the method's arithmetic (no projection, no softmax, no expansion).

Value recipe (the pages ship no data; these stand in for a converted model's
layer):
  * q, latent rows c_t and RoPE keys k^R_t: bf16 of N(0, 1) samples;
  * W_UK, W_UV per group: bf16 of N(0, 1/512) samples, so that
    c W_UK_g and c W_UV_g are again about N(0, 1) and the scaled scores
    q.k / sqrt(192) are about N(0, 1) (with N(0, 1) weights the softmax would
    collapse to one-hot);
  * RoPE is taken as already applied (k^R and q^R are just numbers here);
  * the cache is paged in 64-token pages; a "paged" workload scatters each
    sequence's pages over the pool with a seeded random permutation, the
    others lay them out in order (identity page table).

Named workloads mirror the five layer/batch/context settings the build is
measured on (shapes from the pages: LLaMA-3-8B converted to 32 q heads over
8 groups; a DeepSeek-V3-shaped layer with 128 q heads over 8 groups; latent
512 + RoPE 64 = 576 per token).
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional, Sequence, Tuple

import torch

PAGE_SIZE = 64
D_LATENT, D_ROPE, D_NOPE, D_V = 512, 64, 128, 128
D_QK = D_NOPE + D_ROPE
D_ROW = D_LATENT + D_ROPE


@dataclass(frozen=True)
class Workload:
    name: str
    num_heads: int
    num_groups: int
    batch: int
    lengths: Tuple  # ("fixed", L) or ("uniform", lo, hi) inclusive
    s_q: Tuple[int, ...]
    paged: bool
    seed: int
    expand: bool = False

    def seqlens(self, gen: Optional[torch.Generator] = None) -> torch.Tensor:
        if self.lengths[0] == "fixed":
            return torch.full((self.batch,), int(self.lengths[1]), dtype=torch.int32)
        lo, hi = int(self.lengths[1]), int(self.lengths[2])
        g = gen if gen is not None else torch.Generator().manual_seed(self.seed)
        return torch.randint(lo, hi + 1, (self.batch,), generator=g, dtype=torch.int64).to(torch.int32)


WORKLOADS = {
    w.name: w for w in [
        # LLaMA-3-8B converted single layer, tiny context (the oracle's quick case)
        Workload("llama3_8b_h32_b1_l256", 32, 8, 1, ("fixed", 256), (1,), False, 0),
        # DeepSeek-V3-shaped GQLA layer, s_q = 1
        Workload("dsv3_h128_b32_l4096", 128, 8, 32, ("fixed", 4096), (1,), False, 1),
        # same layer with two MTP query tokens per step
        Workload("dsv3_h128_b64_l8192_mtp2", 128, 8, 64, ("fixed", 8192), (2,), False, 2),
        # long-context paged decode, random page table
        Workload("dsv3_h128_b8_l32k_64k_paged", 128, 8, 8, ("uniform", 32768, 65536), (1, 2),
                 True, 3),
        # LLaMA-3-8B converted shape, large batch of mixed lengths, plus a full-cache expansion
        Workload("llama3_8b_h32_b128_l2k_8k", 32, 8, 128, ("uniform", 2048, 8192), (1, 2),
                 False, 4, expand=True),
        # the (g, s_q) = (4, 1) conversion point: 128 heads over 4 groups, 2176 bytes per
        # expanded token (beyond the five configurations above)
        Workload("dsv3_h128_g4_b32_l4096", 128, 4, 32, ("fixed", 4096), (1,), False, 5),
    ]
}


def pages_for(seqlens: Sequence[int], page_size: int = PAGE_SIZE):
    return [max(1, math.ceil(int(L) / page_size)) for L in seqlens]


def make_case(num_heads: int, num_groups: int, seqlens, s_q: int, paged: bool = False,
              seed: int = 0, page_size: int = PAGE_SIZE, device: str = "cpu",
              spare_pages: int = 0):
    """Draw one decode batch.

    Returns a dict of tensors on ``device``:
      q           bf16  [B][s_q][h][192]   (0..127 nope part, 128..191 RoPE part)
      latent      bf16  [num_pages][page_size][576]  (c_t then k^R_t)
      w_uk, w_uv  bf16  [g][512][128]
      page_table  int32 [B][max_pages]     (unused entries are 0)
      seqlens     int32 [B]
    plus ``num_pages`` and ``page_size``.  ``spare_pages`` extra pool pages are
    drawn too (they are never referenced; useful to check that nothing reads them).
    """
    seqlens = torch.as_tensor(seqlens, dtype=torch.int32).cpu()
    B = int(seqlens.numel())
    n_pages = pages_for(seqlens.tolist(), page_size)
    num_pages = sum(n_pages) + spare_pages
    max_pages = max(n_pages)
    gen = torch.Generator(device=device).manual_seed(seed)
    bf16 = torch.bfloat16
    q = torch.randn(B, s_q, num_heads, D_QK, generator=gen, device=device).to(bf16)
    latent = torch.randn(num_pages, page_size, D_ROW, generator=gen, device=device).to(bf16)
    w_scale = 1.0 / math.sqrt(D_LATENT)
    w_uk = (torch.randn(num_groups, D_LATENT, D_NOPE, generator=gen, device=device)
            * w_scale).to(bf16)
    w_uv = (torch.randn(num_groups, D_LATENT, D_V, generator=gen, device=device)
            * w_scale).to(bf16)
    cpu_gen = torch.Generator().manual_seed(seed + 7919)
    if paged:
        order = torch.randperm(num_pages, generator=cpu_gen)
    else:
        order = torch.arange(num_pages)
    page_table = torch.zeros(B, max_pages, dtype=torch.int32)
    off = 0
    for b in range(B):
        page_table[b, :n_pages[b]] = order[off:off + n_pages[b]].to(torch.int32)
        off += n_pages[b]
    return {
        "q": q, "latent": latent, "w_uk": w_uk, "w_uv": w_uv,
        "page_table": page_table.to(device), "seqlens": seqlens.to(device),
        "num_pages": num_pages, "page_size": page_size,
        "num_heads": num_heads, "num_groups": num_groups, "s_q": s_q,
    }


def make_workload(name: str, s_q: Optional[int] = None, device: str = "cpu"):
    w = WORKLOADS[name]
    s = w.s_q[0] if s_q is None else s_q
    if s not in w.s_q:
        raise ValueError(f"{name} is defined for s_q in {w.s_q}")
    return make_case(w.num_heads, w.num_groups, w.seqlens(), s, paged=w.paged,
                     seed=w.seed, device=device)


def make_topk(seqlens, s_q: int, topk: int, seed: int = 0, unused: int = 0) -> torch.Tensor:
    """Selected token positions for sparse attention: int32 [B][s_q][topk].

    Query token s of sequence b gets min(topk - unused, visible) distinct
    positions drawn uniformly from its visible tokens [0, L_b - s_q + s], in
    random order; the remaining entries are -1 (unused).  The indexer that
    would choose them from the data is outside this path, so a seeded uniform
    choice stands in for it.
    """
    g = torch.Generator().manual_seed(seed)
    sl = [int(x) for x in torch.as_tensor(seqlens).tolist()]
    out = torch.full((len(sl), s_q, topk), -1, dtype=torch.int32)
    for b, L in enumerate(sl):
        for s in range(s_q):
            vis = L - s_q + s + 1
            n = max(0, min(topk - unused, vis))
            if n:
                out[b, s, :n] = torch.randperm(vis, generator=g)[:n].to(torch.int32)
    return out
