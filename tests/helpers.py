"""Shared helpers for the GPU parity tests: run a decode step through the C ABI
and compare it with the fp64 oracle on the same seeded inputs."""
import math

import numpy as np
import torch

import oracle

MAX_ABS = 2e-2   # tolerances of the parity contract: bf16 inputs, fp32 accumulation
REL_FRO = 1e-2


def to_gpu(case):
    out = dict(case)
    for k in ("q", "latent", "w_uk", "w_uv", "page_table", "seqlens"):
        out[k] = case[k].cuda().contiguous()
    return out


def run_decode(gcase, path, num_splits=None, stream=None):
    """One decode step through the binding.  Returns (out bf16, lse fp32, workspace, extras)."""
    from decode_attention_06_b200 import gqla
    h, g, s_q = gcase["num_heads"], gcase["num_groups"], gcase["s_q"]
    dims = gqla.make_dims(h, g)
    kv = gqla.make_kv_index(gcase["page_table"], gcase["seqlens"], gcase["num_pages"])
    B = gcase["seqlens"].numel()
    if num_splits is None:  # as bench.py plans them: from the host copy of the lengths
        num_splits = gqla.plan_splits(path, h, s_q, gcase["seqlens"].cpu())
    bufs = gqla.DecodeBuffers(dims, B, s_q, num_splits, path)
    extras = {}
    if path == "gqa":
        n = gcase["num_pages"] * gcase["page_size"]
        kvx = torch.empty(g, n, 256, dtype=torch.bfloat16, device="cuda")
        kr = torch.empty(n, 64, dtype=torch.bfloat16, device="cuda")
        gqla.gqla_expand_cache(dims, gcase["latent"], gcase["w_uk"], gcase["w_uv"], kvx, kr, stream)
        extras = {"kv_expanded": kvx, "k_rope": kr}
        gqla.decode_step(dims, bufs, gcase["q"], gcase["w_uk"], gcase["w_uv"], kv,
                         kv_expanded=kvx, k_rope=kr, stream=stream)
    else:
        gqla.decode_step(dims, bufs, gcase["q"], gcase["w_uk"], gcase["w_uv"], kv,
                         latent_cache=gcase["latent"], stream=stream)
    torch.cuda.synchronize()
    extras["bufs"] = bufs
    return bufs.out.clone(), bufs.lse.clone(), bufs.workspace, extras


def oracle_ref(case, units=None):
    return oracle.decode(case["q"], case["latent"], case["page_table"], case["seqlens"],
                         case["w_uk"], case["w_uv"], case["num_groups"],
                         page_size=case["page_size"], units=units)


def compare(got_bf16, ref, mask=None, what=""):
    """max-abs <= 2e-2 and ||got - ref||_F / ||ref||_F <= 1e-2 over the selected entries."""
    got = got_bf16.float().cpu().numpy().astype(np.float64)
    if mask is not None:
        got, ref = got[mask], ref[mask]
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = got - ref
    max_abs = float(np.abs(err).max()) if err.size else 0.0
    den = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(err)) / den if den > 0 else float(np.linalg.norm(err))
    assert max_abs <= MAX_ABS, f"{what}: max-abs {max_abs:.3e} > {MAX_ABS}"
    assert rel <= REL_FRO, f"{what}: rel-Frobenius {rel:.3e} > {REL_FRO}"
    return max_abs, rel


def compare_lse(got, ref, mask=None, what="", tol=2e-2):
    g = got.cpu().numpy().astype(np.float64)
    if mask is not None:
        g, ref = g[mask], ref[mask]
    both_inf = np.isneginf(g) & np.isneginf(ref)
    assert (np.isneginf(g) == np.isneginf(ref)).all(), f"{what}: -inf pattern differs"
    d = np.abs(np.where(both_inf, 0.0, g - ref))
    assert d.max(initial=0.0) <= tol, f"{what}: lse max-abs {d.max():.3e}"


def sub_case(case, batch_ids):
    """Compact CPU copy of the chosen sequences (their pages only), for the oracle."""
    pt = case["page_table"].cpu()
    sl = case["seqlens"].cpu()
    ps = case["page_size"]
    pages, rows = [], []
    for b in batch_ids:
        n = max(1, math.ceil(int(sl[b]) / ps))
        rows.append(list(range(len(pages), len(pages) + n)))
        pages.extend(pt[b, :n].tolist())
    latent = case["latent"][torch.tensor(pages, device=case["latent"].device)].cpu()
    maxp = max(len(r) for r in rows)
    new_pt = torch.zeros(len(batch_ids), maxp, dtype=torch.int32)
    for i, r in enumerate(rows):
        new_pt[i, :len(r)] = torch.tensor(r, dtype=torch.int32)
    return {
        "q": case["q"][torch.tensor(batch_ids, device=case["q"].device)].cpu(),
        "latent": latent, "w_uk": case["w_uk"].cpu(), "w_uv": case["w_uv"].cpu(),
        "page_table": new_pt, "seqlens": sl[batch_ids].clone(), "page_size": ps,
        "num_pages": len(pages), "num_groups": case["num_groups"],
        "num_heads": case["num_heads"], "s_q": case["s_q"],
    }


def rising_scores_case(s_q, factor=5.0, seqlens=(256, 200)):
    """A paged batch whose RoPE keys grow with the logical page (by `factor` per page),
    so that row maxima rise from page to page and the kernels' lazy rescaling of O
    (threshold 2^8) runs on every page.  V is the latent part, so it keeps its scale.
    The sequences are short on purpose: a few rescales per row keep the raw scores
    within the range where the absorb path's fp16 partial scores hold 1e-2 accuracy
    (see the absorb kernel's note on score precision)."""
    case = _synth().make_case(128, 8, list(seqlens), s_q, paged=True, seed=131)
    lat = case["latent"].float()
    for b, L in enumerate(case["seqlens"].tolist()):
        for i in range((L + 63) // 64):
            pg = int(case["page_table"][b, i])
            lat[pg, :, 512:] *= 1.0 + factor * i
    case["latent"] = lat.to(torch.bfloat16)
    return case


def _synth():
    from decode_attention_06_b200 import synth
    return synth
