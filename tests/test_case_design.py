"""The rising-score parity cases have teeth: CPU checks of what the GPU tests rely on.

The absorb path splits every score into two halves computed on the two CTAs of a
pair.  An earlier design exchanged those halves in fp16; the "direction" cases of
tests/helpers.rising_scores_case were built so that such an exchange would fail
the parity bound while fp32 halves pass with a wide margin.  This file checks
that property with a numpy emulation of the absorb path's rounding steps (q~ in
bf16, the two halves in fp16 or fp32, P in bf16, the merged latent row in bf16
before W_UV, the output in bf16) against the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
from tests.helpers import MAX_ABS, oracle_ref, rising_scores_case


def _bf16(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).double().numpy()


def _fp16(x):
    return np.asarray(x, dtype=np.float32).astype(np.float16).astype(np.float64)


def _absorb_emulated(case, round_halves):
    """Absorb-path numerics for sequence 0, s_q = 1: [h][128] output."""
    q = case["q"].double().numpy()[0, 0]                                   # [h][192]
    qa = _bf16(oracle.absorb_query(case["q"][:1], case["w_uk"], 8)[0, 0])  # [h][576]
    lat = case["latent"].double().numpy()
    L = int(case["seqlens"][0])
    rows = np.concatenate([lat[int(case["page_table"][0, i])] for i in range((L + 63) // 64)])[:L]
    wv = case["w_uv"].double().numpy()
    h = q.shape[0]
    G = h // 8
    h0 = qa[:, :256] @ rows[:, :256].T + qa[:, 512:544] @ rows[:, 512:544].T
    h1 = qa[:, 256:512] @ rows[:, 256:512].T + qa[:, 544:] @ rows[:, 544:].T
    x = (round_halves(h0) + round_halves(h1)) / math.sqrt(192.0)
    p = _bf16(np.exp(x - x.max(axis=1, keepdims=True)))
    o = _bf16((p @ rows[:, :512]) / p.sum(axis=1, keepdims=True))         # [h][512]
    return np.stack([_bf16(o[hd] @ wv[hd // G]) for hd in range(h)]), max(np.abs(h0).max(), np.abs(h1).max())


@pytest.mark.parametrize("factor,half_lo,half_hi", [(20.0, 2000, 4000), (60.0, 6000, 12000)])
def test_direction_cases_break_an_fp16_exchange_only(factor, half_lo, half_hi):
    case = rising_scores_case(1, factor, (512, 400), mode="direction")
    ref, _ = oracle_ref(case, units=[(0, gi) for gi in range(8)])
    ref = ref[0, 0]
    out16, half = _absorb_emulated(case, _fp16)
    out32, _ = _absorb_emulated(case, lambda v: v)
    assert half_lo < half < half_hi                      # the halves are as large as stated
    assert np.abs(out16 - ref).max() > 1.5 * MAX_ABS     # fp16 halves fail the bound clearly
    assert np.abs(out32 - ref).max() < 0.5 * MAX_ABS     # fp32 halves pass with margin


def test_direction_case_rescales_and_stays_spread():
    case = rising_scores_case(1, 20.0, (512, 400), mode="direction")
    qa = oracle.absorb_query(case["q"], case["w_uk"], 8)
    lat = case["latent"].float().numpy().astype(np.float64)
    L = int(case["seqlens"][0])
    rows = np.concatenate([lat[int(case["page_table"][0, i])] for i in range((L + 63) // 64)])[:L]
    s = qa[0, 0] @ rows.T / math.sqrt(192.0) * math.log2(math.e)        # [h][L], log2 units
    pm = np.stack([s[:, j:j + 64].max(axis=1) for j in range(0, L, 64)], axis=1)
    rises = np.diff(pm, axis=1)
    assert (rises > 8.0).mean() > 0.25      # the lazy rescale runs page after page for many rows
    # the softmax is not one-hot: at least a few tokens carry weight in most rows
    e = np.exp((s - s.max(axis=1, keepdims=True)) * math.log(2.0))
    eff = e.sum(axis=1) ** 2 / (e ** 2).sum(axis=1)                       # effective tokens per row
    assert np.median(eff) > 2.0
