"""Pins for the fp64 oracle: what the pages print, closed forms, library attention.

Every check here ties the oracle to something other than itself:
  * the numbers the pages print (tests/golden/paper_numbers.json),
  * torch's scaled_dot_product_attention on explicitly expanded K/V (a library
    implementation of standard attention, fp64),
  * numpy matmuls for the projections,
  * closed forms: one token, zero query, identical keys, two-token softmax,
    identical scores, empty visible set,
  * invariants: page permutation, causal prefix, absorbed == un-absorbed.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import roofline
from decode_attention_06_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "paper_numbers.json")
SCALE = 1.0 / math.sqrt(192)


def _golden():
    with open(GOLDEN) as f:
        g = json.load(f)
    g.pop("_about")
    return g


def _check(name, got):
    g = _golden()[name]
    assert abs(got - g["value"]) <= g["tol"], (name, got, g)


# ---------------------------------------------------------------- printed numbers

def test_cache_sizes_match_pages():
    _check("cache_bytes_per_token_absorb", roofline.cache_bytes_per_token("absorb"))
    _check("cache_elems_per_token_absorb", roofline.cache_elems_per_token("absorb"))
    _check("cache_bytes_per_token_gqa_g8", roofline.cache_bytes_per_token("gqa", g=8))
    _check("cache_bytes_per_token_gqa_g4", roofline.cache_bytes_per_token("gqa", g=4))
    _check("llama_gqa_cache_elems_per_token", roofline.cache_elems_per_token("llama_gqa"))
    _check("absorb_cache_fraction_of_gqa_baseline",
           roofline.cache_elems_per_token("absorb") / roofline.cache_elems_per_token("llama_gqa"))
    _check("heads_per_group", 128 // 8)


def test_intensities_and_ridges_match_pages():
    _check("intensity_absorb_sq1", roofline.intensity("absorb", h=128, s_q=1))
    _check("intensity_absorb_sq2", roofline.intensity("absorb", h=128, s_q=2))
    _check("intensity_gqa_g8_sq2", roofline.intensity("gqa", h=128, s_q=2, g=8))
    _check("intensity_gqa_g4_sq1", roofline.intensity("gqa", h=128, s_q=1, g=4))
    _check("ridge_h100", roofline.ridge("H100"))
    _check("ridge_h20", roofline.ridge("H20"))
    # the absorb intensity does not depend on g (pwwt sec. 7)
    assert roofline.intensity("absorb", 128, 1) == pytest.approx(
        roofline.flops_per_token("absorb", 128, 1) / 1152)


def test_roofline_step_times_match_pages():
    us = lambda *a, **k: roofline.step_time_s(*a, **k) * 1e6
    _check("step_us_h100_absorb_sq1", us("absorb", "H100", s_q=1))
    _check("step_us_h100_absorb_sq2", us("absorb", "H100", s_q=2))
    _check("mtp_speedup_h100_absorb",
           roofline.tokens_per_s("absorb", "H100", s_q=2) / roofline.tokens_per_s("absorb", "H100", s_q=1))
    _check("step_us_h20_absorb_sq1", us("absorb", "H20", s_q=1))
    _check("step_us_h20_gqa_g8_sq2", us("gqa", "H20", s_q=2, g=8))
    _check("tok_s_h100_absorb_sq1", roofline.tokens_per_s("absorb", "H100", s_q=1))
    _check("tok_s_h20_absorb_sq1", roofline.tokens_per_s("absorb", "H20", s_q=1))
    _check("tok_s_h20_gqa_g8_sq2", roofline.tokens_per_s("gqa", "H20", s_q=2, g=8))
    _check("tok_s_h20_gqa_g4_sq1", roofline.tokens_per_s("gqa", "H20", s_q=1, g=4))
    _check("speedup_h20_gqa_over_mla",
           roofline.tokens_per_s("gqa", "H20", s_q=2, g=8) / roofline.tokens_per_s("absorb", "H20", s_q=1))
    # MLA on H20 is compute-bound, the H100 absorb step at s_q=1 is memory-bound
    assert roofline.intensity("absorb", 128, 1) > roofline.ridge("H20")
    assert roofline.intensity("absorb", 128, 1) < roofline.ridge("H100")


# ---------------------------------------------------------------- helpers

def _np(t):
    return t.float().numpy().astype(np.float64) if t.dtype == torch.bfloat16 else t.numpy()


def _seq_rows(case, b):
    """Latent rows of sequence b in logical order (fp64)."""
    lat = _np(case["latent"])
    pt = case["page_table"].numpy()
    L = int(case["seqlens"][b])
    ps = case["page_size"]
    return np.stack([lat[pt[b, t // ps], t % ps] for t in range(L)]) if L else np.zeros((0, 576))


def _library_attention(case):
    """Expand K/V with numpy, then run torch SDPA (fp64) per (sequence, head)."""
    q = _np(case["q"])
    wk, wv = _np(case["w_uk"]), _np(case["w_uv"])
    B, s_q, h, _ = q.shape
    g = wk.shape[0]
    G = h // g
    out = np.zeros((B, s_q, h, 128))
    for b in range(B):
        rows = _seq_rows(case, b)
        L = rows.shape[0]
        for gi in range(g):
            K = np.concatenate([rows[:, :512] @ wk[gi], rows[:, 512:]], axis=1)
            V = rows[:, :512] @ wv[gi]
            Q = torch.from_numpy(q[b, :, gi * G:(gi + 1) * G].transpose(1, 0, 2).copy())  # [G, s_q, 192]
            t = torch.arange(L)
            mask = torch.stack([t <= L - s_q + s for s in range(s_q)])  # [s_q, L]
            o = torch.nn.functional.scaled_dot_product_attention(
                Q, torch.from_numpy(K).expand(G, L, 192), torch.from_numpy(V).expand(G, L, 128),
                attn_mask=mask.expand(G, s_q, L), scale=SCALE)
            out[b, :, gi * G:(gi + 1) * G] = o.numpy().transpose(1, 0, 2)
    return out


def _run(case, **kw):
    return oracle.decode(case["q"], case["latent"], case["page_table"], case["seqlens"],
                         case["w_uk"], case["w_uv"], case["num_groups"],
                         page_size=case["page_size"], **kw)


# ---------------------------------------------------------------- library attention

@pytest.mark.parametrize("h,seqlens,s_q,paged,seed", [
    (8, [1, 5, 64, 130], 1, False, 11),
    (8, [2, 65, 200], 2, True, 12),
    (32, [96, 3], 2, True, 13),
    (128, [70], 1, False, 14),
])
def test_oracle_matches_library_attention(h, seqlens, s_q, paged, seed):
    case = synth.make_case(h, 8 if h >= 8 else 2, seqlens, s_q, paged=paged, seed=seed)
    out, _ = _run(case)
    ref = _library_attention(case)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


def test_absorbed_form_equals_unabsorbed():
    case = synth.make_case(32, 8, [1, 77, 300], 2, paged=True, seed=21)
    out, lse = _run(case)
    out2, lse2 = oracle.decode_absorbed(case["q"], case["latent"], case["page_table"],
                                        case["seqlens"], case["w_uk"], case["w_uv"], 8)
    np.testing.assert_allclose(out2, out, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse2, lse, rtol=1e-12, atol=1e-12)


def test_units_subset_matches_full_run():
    case = synth.make_case(32, 8, [40, 90], 1, seed=22)
    full, lse = _run(case)
    part, lse_p = _run(case, units=[(1, 3), (0, 7)])
    G = 4
    for b, gi in [(1, 3), (0, 7)]:
        sl = slice(gi * G, (gi + 1) * G)
        np.testing.assert_array_equal(part[b, :, sl], full[b, :, sl])
        np.testing.assert_array_equal(lse_p[b, :, sl], lse[b, :, sl])
    assert np.isnan(part[0, :, 0]).all()


# ---------------------------------------------------------------- closed forms

def test_single_token_returns_its_value():
    case = synth.make_case(16, 8, [1, 1], 1, seed=31)
    out, lse = _run(case)
    wk, wv = _np(case["w_uk"]), _np(case["w_uv"])
    q = _np(case["q"])
    for b in range(2):
        c = _seq_rows(case, b)[0]
        for h in range(16):
            gi = h // 2
            np.testing.assert_allclose(out[b, 0, h], c[:512] @ wv[gi], rtol=1e-12, atol=1e-12)
            k = np.concatenate([c[:512] @ wk[gi], c[512:]])
            assert lse[b, 0, h] == pytest.approx(SCALE * q[b, 0, h] @ k, rel=1e-12)


def test_zero_query_gives_mean_of_visible_values():
    case = synth.make_case(8, 2, [9, 33], 2, seed=32)
    case["q"] = torch.zeros_like(case["q"])
    out, lse = _run(case)
    wv = _np(case["w_uv"])
    for b in range(2):
        rows = _seq_rows(case, b)
        L = rows.shape[0]
        for s in range(2):
            n = L - 2 + s + 1
            for h in range(8):
                np.testing.assert_allclose(out[b, s, h], (rows[:n, :512] @ wv[h // 4]).mean(0),
                                           rtol=1e-11, atol=1e-12)
                assert lse[b, s, h] == pytest.approx(math.log(n), rel=1e-12)


@pytest.mark.parametrize("g", [1, 2, 3])
def test_identical_keys_give_mean_of_values_nullspace(g):
    """c_t = c_0 + n_t with n_t W_UK_j = 0 for every group j and one shared k^R:
    every key is identical, the values are not, so out = mean of V."""
    rng = np.random.default_rng(40 + g)
    h, L = 2 * g, 37
    case = synth.make_case(h, g, [L], 1, seed=40 + g)
    wk = _np(case["w_uk"])
    W = np.concatenate([wk[j] for j in range(g)], axis=1)  # [512, 128 g]
    _, _, vt = np.linalg.svd(W.T)  # rows of vt beyond rank span the left null space of W
    null = vt[128 * g:]
    c0 = rng.standard_normal(512)
    kr = rng.standard_normal(64)
    rows = np.stack([np.concatenate([c0 + null.T @ rng.standard_normal(null.shape[0]), kr])
                     for _ in range(L)])
    cache = rows.reshape(1, L, 576)
    pt = np.zeros((1, 1), np.int32)
    out, lse = oracle.decode(_np(case["q"]), cache, pt, [L], wk, _np(case["w_uv"]), g, page_size=L)
    wv = _np(case["w_uv"])
    for hh in range(h):
        np.testing.assert_allclose(out[0, 0, hh], (rows[:, :512] @ wv[hh // 2]).mean(0),
                                   rtol=1e-9, atol=1e-10)


def test_identical_keys_give_mean_of_values_g8():
    """g = 8 leaves no common null space; W_UK = 0 and one shared k^R make every key equal."""
    case = synth.make_case(128, 8, [50, 129], 2, paged=True, seed=48)
    case["w_uk"] = torch.zeros_like(case["w_uk"])
    lat = case["latent"].clone()
    lat[:, :, 512:] = lat[0, 0, 512:]
    case["latent"] = lat
    out, _ = _run(case)
    wv = _np(case["w_uv"])
    for b, L in enumerate([50, 129]):
        rows = _seq_rows(case, b)
        for s in range(2):
            n = L - 2 + s + 1
            for h in (0, 17, 127):
                np.testing.assert_allclose(out[b, s, h], (rows[:n, :512] @ wv[h // 16]).mean(0),
                                           rtol=1e-11, atol=1e-12)


def test_two_token_softmax_uses_scale_and_rope():
    """W_UK = 0 leaves only the RoPE part of the score: p0/p1 = exp((a0-a1)/sqrt(192))."""
    case = synth.make_case(8, 2, [2], 1, seed=50)
    case["w_uk"] = torch.zeros_like(case["w_uk"])
    out, lse = _run(case)
    q = _np(case["q"])
    rows = _seq_rows(case, 0)
    wv = _np(case["w_uv"])
    for h in range(8):
        a = rows[:, 512:] @ q[0, 0, h, 128:]
        p = np.exp(SCALE * (a - a.max()))
        p /= p.sum()
        np.testing.assert_allclose(out[0, 0, h], p @ (rows[:, :512] @ wv[h // 4]), rtol=1e-12, atol=1e-13)
        assert lse[0, 0, h] == pytest.approx(np.log(np.exp(SCALE * a).sum()), rel=1e-12)


def test_identical_scores_lse_is_score_plus_log_length():
    case = synth.make_case(8, 2, [123], 1, seed=51)
    case["w_uk"] = torch.zeros_like(case["w_uk"])
    lat = case["latent"].clone()
    lat[:, :, 512:] = 0.5
    case["latent"] = lat
    _, lse = _run(case)
    q = _np(case["q"])
    for h in range(8):
        assert lse[0, 0, h] == pytest.approx(SCALE * 0.5 * q[0, 0, h, 128:].sum() + math.log(123),
                                             rel=1e-12, abs=1e-12)


def test_empty_visible_set():
    """s_q = 2 over a single cached token: query 0 sees nothing (out 0, lse -inf)."""
    case = synth.make_case(8, 2, [1], 2, seed=52)
    out, lse = _run(case)
    assert (out[0, 0] == 0).all() and np.isneginf(lse[0, 0]).all()
    assert np.isfinite(out[0, 1]).all() and np.isfinite(lse[0, 1]).all()


# ---------------------------------------------------------------- invariants

def test_causal_first_query_equals_shorter_context():
    case2 = synth.make_case(16, 8, [10, 67], 2, paged=True, seed=60)
    out2, lse2 = _run(case2)
    case1 = dict(case2)
    case1["q"] = case2["q"][:, :1].contiguous()
    case1["seqlens"] = case2["seqlens"] - 1
    out1, lse1 = _run(case1)
    np.testing.assert_allclose(out2[:, 0], out1[:, 0], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse2[:, 0], lse1[:, 0], rtol=1e-13)


def test_page_permutation_invariance():
    case = synth.make_case(8, 2, [100, 190, 64], 1, paged=False, seed=61, spare_pages=3)
    out, lse = _run(case)
    perm = torch.randperm(case["num_pages"], generator=torch.Generator().manual_seed(5))
    lat2 = torch.empty_like(case["latent"])
    lat2[perm] = case["latent"]
    pt2 = perm[case["page_table"].long()].to(torch.int32)
    for b in range(3):  # unused table entries stay unused
        n = math.ceil(int(case["seqlens"][b]) / 64)
        pt2[b, n:] = 0
    case2 = dict(case, latent=lat2, page_table=pt2)
    out2, lse2 = _run(case2)
    np.testing.assert_array_equal(out2, out)
    np.testing.assert_array_equal(lse2, lse)


def test_group_mapping_contiguous_heads():
    """Zeroing W_UV of group 3 zeroes exactly heads 12..15 when h=32, g=8."""
    case = synth.make_case(32, 8, [45], 1, seed=62)
    wv = case["w_uv"].clone()
    wv[3] = 0
    case["w_uv"] = wv
    out, _ = _run(case)
    assert (out[0, 0, 12:16] == 0).all()
    assert (np.abs(out[0, 0, :12]).sum(-1) > 0).all() and (np.abs(out[0, 0, 16:]).sum(-1) > 0).all()


# ---------------------------------------------------------------- projections

def test_absorb_query_matches_numpy():
    case = synth.make_case(32, 8, [4], 2, seed=70)
    qa = oracle.absorb_query(case["q"], case["w_uk"], 8)
    q, wk = _np(case["q"]), _np(case["w_uk"])
    for h in (0, 5, 31):
        np.testing.assert_allclose(qa[0, 1, h, :512], wk[h // 4] @ q[0, 1, h, :128], rtol=1e-12, atol=1e-12)
        np.testing.assert_array_equal(qa[0, 1, h, 512:], q[0, 1, h, 128:])


def test_expand_f64_matches_numpy():
    case = synth.make_case(32, 8, [70], 1, seed=71)
    kv, kr = oracle.expand_f64(case["latent"], case["w_uk"], case["w_uv"])
    lat = _np(case["latent"]).reshape(-1, 576)
    wk, wv = _np(case["w_uk"]), _np(case["w_uv"])
    for gi in (0, 7):
        np.testing.assert_allclose(kv[gi, :, :128], lat[:, :512] @ wk[gi], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(kv[gi, :, 128:], lat[:, :512] @ wv[gi], rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(kr, lat[:, 512:])


def _bits_to_f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_expand_f32seq_close_to_exact_and_rounded_once():
    case = synth.make_case(32, 8, [64], 1, seed=72)
    bits, kr_bits = oracle.expand_f32seq_bits(case["latent"], case["w_uk"], case["w_uv"])
    exact, kr = oracle.expand_f64(case["latent"], case["w_uk"], case["w_uv"])
    got = _bits_to_f64(bits)
    # fp32 accumulation of 512 exact products: |err| <= 512 * 2^-24 * sum|c w|, then one bf16 rounding
    lat = np.abs(_np(case["latent"]).reshape(-1, 576)[:, :512])
    wk, wv = np.abs(_np(case["w_uk"])), np.abs(_np(case["w_uv"]))
    absum = np.stack([np.concatenate([lat @ wk[j], lat @ wv[j]], axis=1) for j in range(8)])
    bound = 512 * 2.0 ** -24 * absum + np.abs(exact) * 2.0 ** -8 + 1e-30
    assert (np.abs(got - exact) <= bound).all()
    np.testing.assert_array_equal(_bits_to_f64(kr_bits), kr)
    # most outputs are the correctly rounded exact value
    exact_rounded = np.array([oracle.bf16_rne_bits(x) for x in exact.ravel()[:2000]], dtype=np.uint16)
    assert (exact_rounded == bits.ravel()[:2000]).mean() > 0.97


def test_expand_f32seq_pins_the_ascending_fp32_order():
    """The fixed rounding order itself: fp32 fused multiply-adds in ascending latent
    index from +0, one bf16 rounding.  The hand-built case gives different bits for
    a descending order, for fp64 accumulation rounded twice and for the exact sum
    rounded once, so this fails for any of them."""
    from tests.helpers import expansion_order_case
    lat, wk, wv, want = expansion_order_case()
    bits, kr_bits = oracle.expand_f32seq_bits(lat, wk, wv)
    assert bits.shape == (1, 1, 256)
    np.testing.assert_array_equal(bits[0, 0, :3], want)
    np.testing.assert_array_equal(bits[0, 0, 128:131], want)
    assert not bits[0, 0, 3:128].any() and not bits[0, 0, 131:].any()
    assert not kr_bits.any()

    # the alternatives really differ on this case (fp32 and fp64 sums by numpy)
    def bf16(x):
        return oracle.bf16_rne_bits(float(np.float32(x)))

    terms = [lat[0, :512].astype(np.float64) * wk[0, :, d].astype(np.float64) for d in range(3)]
    for t in terms:  # every product is exact in fp32
        assert np.array_equal(t.astype(np.float32).astype(np.float64), t)

    def f32_sum(t):
        acc = np.float32(0.0)
        for x in t:
            acc = np.float32(acc + np.float32(x))
        return acc

    ascending = [bf16(f32_sum(t)) for t in terms]
    descending = [bf16(f32_sum(t[::-1])) for t in terms]
    fp64_twice = [bf16(np.float32(sum(t))) for t in terms]
    assert ascending == want.tolist()
    assert descending == [0x3F81, 0x3F80, 0x3F80]
    assert fp64_twice == [0x3F81, 0x3F81, 0x3F80]
    assert len({tuple(ascending), tuple(descending), tuple(fp64_twice)}) == 3


@pytest.mark.parametrize("x,bits", [
    (1.0, 0x3F80),
    (1.0 + 2.0 ** -8, 0x3F80),          # halfway, ties to even (down)
    (1.0 + 3 * 2.0 ** -8, 0x3F82),      # halfway, ties to even (up)
    (1.0 + 2.0 ** -8 + 2.0 ** -20, 0x3F81),  # just above halfway
    (-2.5, 0xC020),
    (0.0, 0x0000),
    (3.0e38, 0x7F62),
    (float("inf"), 0x7F80),
])
def test_bf16_round_nearest_even(x, bits):
    assert oracle.bf16_rne_bits(x) == bits


def test_rising_scores_case_rescales():
    from tests.helpers import rising_scores_case
    # the construction does what the test below relies on: row maxima of the scaled
    # scores rise by more than 2^8 (8 log2 units) between most consecutive pages
    case = rising_scores_case(1)
    qa = oracle.absorb_query(case["q"], case["w_uk"], 8)            # [B][1][h][576]
    lat = case["latent"].float().numpy().astype(np.float64)
    rises = []
    for b, L in enumerate(case["seqlens"].tolist()):
        rows = np.concatenate([lat[int(case["page_table"][b, i])] for i in range((L + 63) // 64)])[:L]
        s = qa[b, 0] @ rows.T / math.sqrt(192.0) * math.log2(math.e)   # [h][L], log2 units
        pm = np.stack([s[:, j:j + 64].max(axis=1) for j in range(0, L, 64)], axis=1)
        rises.append(np.diff(pm, axis=1).ravel())
    rises = np.concatenate(rises)
    assert (rises > 8.0).mean() > 0.4


# ---------------------------------------------------------------- sparse variant

def _sparse_case(h=32, g=8, seqlens=(70, 130), s_q=2, seed=21):
    return synth.make_case(h, g, list(seqlens), s_q, paged=True, seed=seed)


def test_sparse_all_visible_equals_dense():
    """Selecting every visible token is ordinary decode attention (the C oracle)."""
    case = _sparse_case()
    sl, s_q = case["seqlens"].tolist(), case["s_q"]
    idx = synth.make_topk(sl, s_q, max(sl), seed=3)  # topk >= visible: every token, shuffled
    got, got_lse = oracle.decode_sparse(case["q"], case["latent"], case["page_table"], case["seqlens"],
                                        case["w_uk"], case["w_uv"], 8, idx)
    ref, ref_lse = oracle.decode(case["q"], case["latent"], case["page_table"], case["seqlens"],
                                 case["w_uk"], case["w_uv"], 8)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-11)
    np.testing.assert_allclose(got_lse, ref_lse, rtol=0, atol=1e-11)


def test_sparse_single_token_is_its_value_row():
    """One selected token: the output is that token's V row and the LSE its score."""
    case = _sparse_case(h=32, g=8, seqlens=(90,), s_q=1, seed=22)
    t = 37
    idx = torch.full((1, 1, 5), -1, dtype=torch.int32)
    idx[0, 0, 3] = t
    out, lse = oracle.decode_sparse(case["q"], case["latent"], case["page_table"], case["seqlens"],
                                    case["w_uk"], case["w_uv"], 8, idx)
    row = case["latent"].reshape(-1, 576)[int(case["page_table"][0, t // 64]) * 64 + t % 64].double().numpy()
    wk, wv = case["w_uk"].double().numpy(), case["w_uv"].double().numpy()
    q = case["q"].double().numpy()[0, 0]
    for hh in range(32):
        gg = hh // 4
        np.testing.assert_allclose(out[0, 0, hh], row[:512] @ wv[gg], rtol=0, atol=1e-12)
        k = np.concatenate([row[:512] @ wk[gg], row[512:]])
        assert abs(lse[0, 0, hh] - (q[hh] @ k) * SCALE) < 1e-12


def test_sparse_brute_force_tiny():
    """A four-token subset against explicit loops over tokens and dimensions."""
    case = _sparse_case(h=32, g=8, seqlens=(40,), s_q=1, seed=23)
    sel = [3, 17, 31, 39]
    idx = torch.tensor([[sel + [-1, -1]]], dtype=torch.int32)
    out, lse = oracle.decode_sparse(case["q"], case["latent"], case["page_table"], case["seqlens"],
                                    case["w_uk"], case["w_uv"], 8, idx)
    lat = case["latent"].reshape(-1, 576).double().numpy()
    pt = case["page_table"][0].tolist()
    wk, wv = case["w_uk"].double().numpy(), case["w_uv"].double().numpy()
    q = case["q"].double().numpy()[0, 0]
    for hh in (0, 13, 31):
        gg = hh // 4
        scores, values = [], []
        for t in sel:
            c = lat[pt[t // 64] * 64 + t % 64]
            k = [sum(c[i] * wk[gg, i, j] for i in range(512)) for j in range(128)] + list(c[512:])
            scores.append(sum(q[hh, j] * k[j] for j in range(192)) * SCALE)
            values.append([sum(c[i] * wv[gg, i, j] for i in range(512)) for j in range(128)])
        m = max(scores)
        w = [math.exp(x - m) for x in scores]
        want = [sum(w[n] * values[n][j] for n in range(4)) / sum(w) for j in range(128)]
        np.testing.assert_allclose(out[0, 0, hh], want, rtol=0, atol=1e-11)
        assert abs(lse[0, 0, hh] - (m + math.log(sum(w)))) < 1e-11


def test_sparse_order_and_padding_invariant():
    case = _sparse_case(seed=24)
    sl, s_q = case["seqlens"].tolist(), case["s_q"]
    idx = synth.make_topk(sl, s_q, 40, seed=5, unused=9)
    perm = idx.clone()
    for b in range(idx.shape[0]):
        for s in range(s_q):
            perm[b, s] = idx[b, s][torch.randperm(idx.shape[-1], generator=torch.Generator().manual_seed(b * 7 + s))]
    a, la = oracle.decode_sparse(case["q"], case["latent"], case["page_table"], case["seqlens"],
                                 case["w_uk"], case["w_uv"], 8, idx)
    b_, lb = oracle.decode_sparse(case["q"], case["latent"], case["page_table"], case["seqlens"],
                                  case["w_uk"], case["w_uv"], 8, perm)
    np.testing.assert_allclose(a, b_, rtol=0, atol=1e-12)
    np.testing.assert_allclose(la, lb, rtol=0, atol=1e-12)


def test_make_topk_draws_distinct_visible_positions():
    idx = synth.make_topk([10, 300], 2, 64, seed=1, unused=4)
    for b, L in enumerate([10, 300]):
        for s in range(2):
            t = idx[b, s][idx[b, s] >= 0]
            assert t.numel() == min(60, L - 2 + s + 1)
            assert len(set(t.tolist())) == t.numel()
            assert int(t.max()) <= L - 2 + s
