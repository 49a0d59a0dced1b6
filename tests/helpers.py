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
    assert (np.isneginf(g) == np.isneginf(ref)).all(), f"{what}: -inf pattern differs"
    finite = ~np.isneginf(ref)  # the -inf entries agree (checked above); compare the rest
    d = np.abs(g[finite] - ref[finite])
    assert d.max(initial=0.0) <= tol, f"{what}: lse max-abs {d.max(initial=0.0):.3e}"


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


def rising_scores_case(s_q, factor=5.0, seqlens=(256, 200), mode="scale"):
    """A paged batch whose row maxima rise from page to page, so that the kernels' lazy
    rescaling of O (threshold 2^8) runs on every page.  V is the latent part, so it
    keeps its scale; only the RoPE keys k^R change, on logical page i:
      mode "scale":     k^R *= 1 + factor * i.  The score spread grows with the page, so
                        the softmax ends up nearly one-hot.  With the defaults the raw
                        scores reach about 440 (32 nats after the 1/sqrt(192) scale).
      mode "direction": k^R = (1 + factor * i) u + k^R, with one seeded direction u for
                        the whole batch: every token of a page gets nearly the same large
                        RoPE score, which rises page after page, while the spread within a
                        page stays that of the N(0, 1) inputs.  Over 512 / 400 tokens the
                        per-CTA halves of the absorb path's scores (and the scores) reach
                        about 900 (factor 6, ~90 nats), 2900 (factor 20, ~300 nats) and
                        8600 (factor 60, ~900 nats).
    Near a one-hot softmax the output is one row of V, so the GQA path's bf16 expanded
    cache and the bf16 output alone put about 2^-8 |V| of error on it, close to the 2e-2
    bound; the "direction" cases reach far larger scores with the softmax spread over a
    page, so they test the precision of the scores themselves."""
    case = _synth().make_case(128, 8, list(seqlens), s_q, paged=True, seed=131)
    lat = case["latent"].float()
    u = torch.randn(64, generator=torch.Generator().manual_seed(132))
    for b, L in enumerate(case["seqlens"].tolist()):
        for i in range((L + 63) // 64):
            pg = int(case["page_table"][b, i])
            if mode == "scale":
                lat[pg, :, 512:] *= 1.0 + factor * i
            elif mode == "direction":
                lat[pg, :, 512:] += (1.0 + factor * i) * u
            else:
                raise ValueError(mode)
    case["latent"] = lat.to(torch.bfloat16)
    return case


def _synth():
    from decode_attention_06_b200 import synth
    return synth


def expansion_order_case():
    """Hand-built inputs that pin the rounding order of the fp32 cache expansion.

    One latent row and one group; only output columns 0..2 of K_nope (and the same
    columns of V, whose weights are a copy) have nonzero terms c_r * w_r, each exact
    in fp32 (products of powers of two):
      column 0: r = 0, 1, 2..17   -> 1, 2^-8, then sixteen 2^-26
      column 1: r = 494..509, 510, 511 -> sixteen 2^-26, then 2^-8, then 1
      column 2: r = 0, 1, 18      -> 1, 2^-8, 2^-30
    Accumulated in fp32 from +0 in ascending r, one rounding to bf16 at the end:
      column 0: 1 + 2^-8 is exact; each 2^-26 is below half an fp32 ulp of it and is
                lost, so the sum stays 1 + 2^-8, a bf16 tie that rounds to even: 0x3F80;
      column 1: the small terms add up exactly to 2^-22 first, then 2^-8 and 1 give
                1 + 2^-8 + 2^-22 (exact in fp32), above the tie: 0x3F81;
      column 2: 2^-30 is lost against 1 + 2^-8: 0x3F80.
    Other orders give other bits (worked out the same way):
      descending r                      -> 0x3F81, 0x3F80, 0x3F80
      fp64 sum, rounded to fp32, to bf16 -> 0x3F81, 0x3F81, 0x3F80
      exact sum rounded once to bf16    -> 0x3F81, 0x3F81, 0x3F81
    Returns (latent [1][576] fp32, w_uk [1][512][128], w_uv, expected bits [3])."""
    c = np.zeros(576, dtype=np.float32)
    c[0], c[1], c[2:18], c[18] = 1.0, 2.0 ** -8, 2.0 ** -13, 2.0 ** -15
    c[494:510], c[510], c[511] = 2.0 ** -13, 2.0 ** -8, 1.0
    w = np.zeros((1, 512, 128), dtype=np.float32)
    w[0, 0, 0] = w[0, 1, 0] = 1.0
    w[0, 2:18, 0] = 2.0 ** -13
    w[0, 494:510, 1] = 2.0 ** -13
    w[0, 510, 1] = w[0, 511, 1] = 1.0
    w[0, 0, 2] = w[0, 1, 2] = 1.0
    w[0, 18, 2] = 2.0 ** -15
    return c.reshape(1, 576), w, w.copy(), np.array([0x3F80, 0x3F81, 0x3F80], dtype=np.uint16)
