"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Both paths, every workload shape, ragged tails, empty splits and sequences,
random page tables; full-size workloads on sampled (sequence, group) units.
Tolerance: max-abs <= 2e-2 and rel-Frobenius <= 1e-2 (bf16 inputs, fp32
accumulation); the cache expansion is compared bit for bit.
"""
import zlib

import numpy as np
import pytest
import torch

import oracle
from decode_attention_06_b200 import synth
from tests.helpers import (compare, compare_lse, oracle_ref, rising_scores_case, run_decode,
                           sub_case, to_gpu)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")


# ------------------------------------------------------------------ expansion and absorption

@pytest.mark.parametrize("n_pages,extra", [(3, 0), (5, 17)])
def test_expand_cache_bit_exact(n_pages, extra):
    from decode_attention_06_b200 import gqla
    case = synth.make_case(32, 8, [64 * n_pages], 1, seed=100 + n_pages)
    lat = case["latent"].reshape(-1, 576)
    if extra:  # a slot count that is not a multiple of the 128-slot tile
        lat = torch.cat([lat, lat[:extra] * 0.5]).contiguous()
    n = lat.shape[0]
    dims = gqla.make_dims(32, 8)
    kv = torch.empty(8, n, 256, dtype=torch.bfloat16, device="cuda")
    kr = torch.empty(n, 64, dtype=torch.bfloat16, device="cuda")
    gqla.gqla_expand_cache(dims, lat.cuda(), case["w_uk"].cuda(), case["w_uv"].cuda(), kv, kr)
    torch.cuda.synchronize()
    ref_kv, ref_kr = oracle.expand_f32seq_bits(lat, case["w_uk"], case["w_uv"])
    got_kv = kv.cpu().view(torch.int16).numpy().view(np.uint16)
    got_kr = kr.cpu().view(torch.int16).numpy().view(np.uint16)
    assert (got_kv == ref_kv).all(), f"{(got_kv != ref_kv).sum()} expanded values differ"
    assert (got_kr == ref_kr).all()


def test_expand_cache_rounding_order_case():
    """The hand-built case whose bits differ between summation orders: the kernel's
    ascending-order fp32 accumulation gives the bits worked out by hand, in every group."""
    from decode_attention_06_b200 import gqla
    from tests.helpers import expansion_order_case
    lat, wk, wv, want = expansion_order_case()
    g = 8
    lat_t = torch.from_numpy(lat).to(torch.bfloat16)
    wk_t = torch.from_numpy(wk).to(torch.bfloat16).expand(g, -1, -1).contiguous()
    wv_t = torch.from_numpy(wv).to(torch.bfloat16).expand(g, -1, -1).contiguous()
    assert torch.equal(lat_t.float(), torch.from_numpy(lat))  # every input is exact in bf16
    dims = gqla.make_dims(32, g)
    kv = torch.full((g, 1, 256), -1.0, dtype=torch.bfloat16, device="cuda")
    kr = torch.full((1, 64), -1.0, dtype=torch.bfloat16, device="cuda")
    gqla.gqla_expand_cache(dims, lat_t.cuda(), wk_t.cuda(), wv_t.cuda(), kv, kr)
    torch.cuda.synchronize()
    bits = kv.cpu().view(torch.int16).numpy().view(np.uint16)
    for gi in range(g):
        np.testing.assert_array_equal(bits[gi, 0, :3], want)
        np.testing.assert_array_equal(bits[gi, 0, 128:131], want)
        assert not bits[gi, 0, 3:128].any() and not bits[gi, 0, 131:].any()
    assert not kr.cpu().float().any()


@pytest.mark.parametrize("n_pages,extra,g", [(3, 0, 8), (5, 17, 8), (4, 100, 4)])
def test_expand_cache_tc_within_rounding_bound(n_pages, extra, g):
    """Tensor-core expansion: every value within one bf16 rounding of the exact
    product plus the fp32 accumulation bound for 512 terms (the header's contract);
    k_rope copied exactly."""
    from decode_attention_06_b200 import gqla
    case = synth.make_case(128, g, [64 * n_pages], 1, seed=200 + n_pages)
    lat = case["latent"].reshape(-1, 576)
    if extra:  # a slot count that is not a multiple of the 128-slot tile
        lat = torch.cat([lat, lat[:extra] * 0.5]).contiguous()
    n = lat.shape[0]
    dims = gqla.make_dims(128, g)
    kv = torch.empty(g, n, 256, dtype=torch.bfloat16, device="cuda")
    kr = torch.empty(n, 64, dtype=torch.bfloat16, device="cuda")
    gqla.gqla_expand_cache_tc(dims, lat.cuda(), case["w_uk"].cuda(), case["w_uv"].cuda(), kv, kr)
    torch.cuda.synchronize()
    exact, ref_kr = oracle.expand_f64(lat, case["w_uk"], case["w_uv"])
    c = lat[:, :512].double().numpy()
    w = torch.cat([case["w_uk"], case["w_uv"]], dim=2).double().numpy()  # [g][512][256]
    mag = np.einsum("nk,gkc->gnc", np.abs(c), np.abs(w))
    # bf16 rounding to nearest: at most half a unit in the last place, 2^-8 |x|
    bound = 2.0 ** -8 * np.abs(exact) + 2.0 ** -15 * mag
    got = kv.cpu().double().numpy()
    err = np.abs(got - exact)
    excess = err - bound
    assert excess.max() <= 0, f"{(excess > 0).sum()} values outside the bound, worst by {excess.max():.3g}"
    assert np.array_equal(kr.cpu().double().numpy(), ref_kr)
    # and no more than one bf16 step from the sequential-order expansion wherever the
    # two fp32 sums (each within 2^-15 mag of exact) differ by less than one bf16 step
    # (|exact| >= 2^-6 mag); below that, cancellation makes the bound above the test
    seq = torch.empty_like(kv)
    kr2 = torch.empty_like(kr)
    gqla.gqla_expand_cache(dims, lat.cuda(), case["w_uk"].cuda(), case["w_uv"].cuda(), seq, kr2)
    torch.cuda.synchronize()
    a = kv.cpu().view(torch.int16).numpy().astype(np.int32)
    b = seq.cpu().view(torch.int16).numpy().astype(np.int32)
    same_sign = (a ^ b) >= 0
    checked = same_sign & (np.abs(exact) >= 2.0 ** -6 * mag)
    assert checked.mean() > 0.5
    assert np.all(np.abs(a - b)[checked] <= 1), "values more than one bf16 step apart"


@pytest.mark.parametrize("h,B,s_q", [(32, 3, 1), (128, 5, 2), (128, 9, 1)])
def test_absorb_query_matches_oracle(h, B, s_q):
    from decode_attention_06_b200 import gqla
    case = synth.make_case(h, 8, [1] * B, s_q, seed=110 + h + B)
    dims = gqla.make_dims(h, 8)
    qa = torch.empty(B, s_q, h, 576, dtype=torch.bfloat16, device="cuda")
    gqla.gqla_absorb_query(dims, case["q"].cuda(), case["w_uk"].cuda(), qa)
    torch.cuda.synchronize()
    ref = oracle.absorb_query(case["q"], case["w_uk"], 8)
    got = qa.float().cpu().numpy()
    # fp32 accumulation then one bf16 rounding: |err| <= 2^-8 |x| + tiny
    assert (np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-5).all()
    np.testing.assert_array_equal(got[..., 512:], ref[..., 512:])


# ------------------------------------------------------------------ decode parity, small shapes

SMALL = [
    # id, h, seqlens, s_q, paged, num_splits
    ("llama_l256", 32, [256], 1, False, None),
    ("llama_l256_3splits", 32, [256], 1, False, 3),
    ("h128_ragged_paged", 128, [1000, 64, 1, 777], 1, True, 7),
    ("h128_mtp_paged", 128, [513, 130], 2, True, 5),
    ("h32_mtp_ragged", 32, [2000, 3, 70], 2, False, 16),
    ("more_splits_than_pages", 32, [64, 65], 1, False, 9),
    ("one_split", 128, [300, 200], 2, True, 1),
    ("zero_length_sequence", 32, [0, 65, 0], 1, False, 4),
    ("mtp_single_token", 32, [1, 2], 2, False, 2),
    # a sequence over more than 32 splits: the combines take the weights in blocks of 32
    ("many_partials", 128, [5000, 300], 1, True, 70),
    ("many_partials_mtp", 32, [4000, 9], 2, False, 60),
]


@pytest.mark.parametrize("path", ["gqa", "absorb"])
@pytest.mark.parametrize("cid,h,seqlens,s_q,paged,splits", SMALL, ids=[c[0] for c in SMALL])
def test_decode_parity_small(path, cid, h, seqlens, s_q, paged, splits):
    case = synth.make_case(h, 8, seqlens, s_q, paged=paged, seed=zlib.crc32(cid.encode()) % 1000,
                           spare_pages=2)
    out, lse, ws, _ = run_decode(to_gpu(case), path, splits)
    ref, ref_lse = oracle_ref(case)
    compare(out, ref, what=f"{path}/{cid}")
    compare_lse(lse, ref_lse, what=f"{path}/{cid}")
    from decode_attention_06_b200 import gqla
    assert gqla.gqla_read_device_error(ws)[0] == 0


SMALL_G4 = [
    # the (g, s_q) = (4, 1) conversion and its MTP / small-head neighbours: 4 KV groups
    ("g4_h128_paged", 128, [1000, 70], 1, True, 5),
    ("g4_h32_mtp_ragged", 32, [513, 64, 3], 2, False, 6),
]


@pytest.mark.parametrize("path", ["gqa", "absorb"])
@pytest.mark.parametrize("cid,h,seqlens,s_q,paged,splits", SMALL_G4, ids=[c[0] for c in SMALL_G4])
def test_decode_parity_four_groups(path, cid, h, seqlens, s_q, paged, splits):
    case = synth.make_case(h, 4, seqlens, s_q, paged=paged, seed=zlib.crc32(cid.encode()) % 1000)
    out, lse, ws, _ = run_decode(to_gpu(case), path, splits)
    ref, ref_lse = oracle_ref(case)
    compare(out, ref, what=f"{path}/{cid}")
    compare_lse(lse, ref_lse, what=f"{path}/{cid}")
    from decode_attention_06_b200 import gqla
    assert gqla.gqla_read_device_error(ws)[0] == 0


LEAD = [
    # id, h, seqlens, s_q, paged, num_splits, (lead_splits, lead_weight16)
    ("ragged_paged_lead2x", 128, [1000, 64, 1, 777], 1, True, 7, (2, 32)),
    ("mtp_lead3x", 128, [513, 130], 2, True, 5, (1, 48)),
    ("every_chunk_lead", 32, [2000, 3, 70], 2, False, 6, (6, 40)),
    # the lead chunks take nearly everything, the last chunks come out empty
    ("lead_swallows_batch", 128, [300, 200], 2, True, 6, (2, 512)),
    ("zero_length_lead", 32, [0, 65, 0, 700], 1, False, 4, (1, 24)),
    ("headline_shape_lead", 128, [4096, 4096, 4096], 2, True, 9, (2, 30)),
]


@pytest.mark.parametrize("cid,h,seqlens,s_q,paged,splits,lead", LEAD, ids=[c[0] for c in LEAD])
def test_absorb_lead_split_parity(cid, h, seqlens, s_q, paged, splits, lead):
    """Absorb decode and combine on a split plan with lead chunks (the first lead_splits
    chunks lead_weight16 / 16 times as long): the same outputs as the oracle, and within
    fp32 merge rounding of the equal-chunk plan."""
    from decode_attention_06_b200 import gqla
    case = synth.make_case(h, 8, seqlens, s_q, paged=paged, seed=zlib.crc32(cid.encode()) % 1000)
    g = to_gpu(case)
    dims = gqla.make_dims(h, 8)
    kv = gqla.make_kv_index(g["page_table"], g["seqlens"], g["num_pages"])
    B = g["seqlens"].numel()
    bufs = gqla.DecodeBuffers(dims, B, s_q, splits, "absorb")
    gqla.gqla_absorb_query(dims, g["q"], g["w_uk"], bufs.q_absorbed)
    gqla.gqla_decode_absorb(dims, bufs.q_absorbed, g["latent"], kv, splits, bufs.o_part, bufs.lse_part,
                            bufs.workspace, lead=lead)
    gqla.gqla_combine(dims, kv, s_q, splits, 512, bufs.o_part, bufs.lse_part, g["w_uv"], bufs.out,
                      bufs.lse, lead=lead)
    torch.cuda.synchronize()
    assert gqla.gqla_read_device_error(bufs.workspace)[0] == 0
    ref, ref_lse = oracle_ref(case)
    compare(bufs.out, ref, what=f"absorb-lead/{cid}")
    compare_lse(bufs.lse, ref_lse, what=f"absorb-lead/{cid}")
    eq, eq_lse, _, _ = run_decode(g, "absorb", splits)
    d = (bufs.out.float() - eq.float()).abs().max().item()
    assert d <= 2e-2, f"lead plan vs equal chunks: {d}"


def test_plan_lead_on_device():
    """gqla_plan_lead with this device's SM count at the 64 x 8192 s_q = 2 shape: the absorb
    chunks whose 2 x 2 CTAs fit on the SMs the GQA decode's 128 CTAs leave idle."""
    from decode_attention_06_b200 import gqla
    dims = gqla.make_dims(128, 8)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    e, w16 = gqla.gqla_plan_lead(dims, 2, sms, 37, 128, 414.0, 359.0, 37.0)
    assert e == min(max((sms - 128) // 4, 0), 36)
    assert gqla.gqla_plan_lead(dims, 2, sms, 37, sms, 414.0, 359.0, 37.0) == (0, 16)


def test_paths_agree():
    case = synth.make_case(128, 8, [700, 129], 2, paged=True, seed=120)
    g = to_gpu(case)
    a, la, _, _ = run_decode(g, "absorb", 6)
    b, lb, _, _ = run_decode(g, "gqa", 6)
    compare(a, b.float().cpu().numpy().astype(np.float64), what="absorb vs gqa")


RISING = [
    # id, factor, seqlens, mode: raw scores up to ~440 (32 nats, nearly one-hot at the end),
    # then score halves up to ~900, ~2900 and ~8600 (90, 300 and 900 nats) spread over a page
    ("rising", 5.0, (256, 200), "scale"),
    ("steep", 6.0, (512, 400), "direction"),
    ("steeper", 20.0, (512, 400), "direction"),
    ("steepest", 60.0, (512, 400), "direction"),
]


@pytest.mark.parametrize("path", ["gqa", "absorb"])
@pytest.mark.parametrize("s_q", [1, 2])
@pytest.mark.parametrize("cid,factor,seqlens,mode", RISING, ids=[c[0] for c in RISING])
def test_decode_parity_rising_scores(path, s_q, cid, factor, seqlens, mode):
    """Row maxima that rise page after page (the lazy O rescale runs on every page)
    up to large raw scores: both paths form every score in fp32 (an fp16 exchange of
    the absorb path's score halves fails the last two cases, see
    tests/test_case_design.py)."""
    case = rising_scores_case(s_q, factor, seqlens, mode)
    out, lse, ws, _ = run_decode(to_gpu(case), path, 3)
    ref, ref_lse = oracle_ref(case)
    compare(out, ref, what=f"{path}/{cid}_sq{s_q}")
    compare_lse(lse, ref_lse, what=f"{path}/{cid}_sq{s_q}")
    from decode_attention_06_b200 import gqla
    assert gqla.gqla_read_device_error(ws)[0] == 0


def test_bad_page_index_is_reported_not_faulted():
    from decode_attention_06_b200 import gqla
    case = synth.make_case(32, 8, [200, 100], 1, seed=121)
    case["page_table"] = case["page_table"].clone()
    case["page_table"][1, 0] = case["num_pages"] + 5  # outside the pool
    for path in ("gqa", "absorb"):
        _, _, ws, _ = run_decode(to_gpu(case), path, 4)
        st, info = gqla.gqla_read_device_error(ws)
        assert st == -5 and info == 1
        gqla.gqla_clear_device_error(ws)
        assert gqla.gqla_read_device_error(ws)[0] == 0


def test_wait_that_runs_out_is_reported_and_context_survives():
    """A V load that never comes: the bounded wait runs out (about two seconds),
    the call records GQLA_ERR_TIMEOUT instead of hanging, and the next call on the
    same context is correct."""
    from decode_attention_06_b200 import gqla
    case = synth.make_case(128, 8, [700, 300], 1, paged=True, seed=321)
    g = to_gpu(case)
    gqla.gqla_debug_drop_v_load(3)
    out_bad, _, ws, _ = run_decode(g, "gqa", 2)
    st, _ = gqla.gqla_read_device_error(ws)
    assert st == -6
    out, lse, ws2, _ = run_decode(g, "gqa", 2)
    st2, _ = gqla.gqla_read_device_error(ws2)
    assert st2 == 0
    ref, ref_lse = oracle_ref(case)
    compare(out, ref, what="gqa/after-timeout")


def test_absorb_wait_that_runs_out_is_reported_and_context_survives():
    """The absorb decode's CTA pairs: a latent tile that never comes.  The bounded wait
    runs out (about two seconds), the pair drains without a store reaching an exited
    CTA, the call records GQLA_ERR_TIMEOUT, and the next call on the context is correct."""
    from decode_attention_06_b200 import gqla
    case = synth.make_case(128, 8, [700, 300], 1, paged=True, seed=322)
    g = to_gpu(case)
    gqla.gqla_debug_drop_v_load(3)
    _, _, ws, _ = run_decode(g, "absorb", 2)
    st, _ = gqla.gqla_read_device_error(ws)
    assert st == -6
    out, lse, ws2, _ = run_decode(g, "absorb", 2)
    assert gqla.gqla_read_device_error(ws2)[0] == 0
    ref, ref_lse = oracle_ref(case)
    compare(out, ref, what="absorb/after-timeout")
    compare_lse(lse, ref_lse, what="absorb/after-timeout")


def test_sequence_longer_than_page_row_is_reported():
    from decode_attention_06_b200 import gqla
    case = synth.make_case(32, 8, [128, 64], 1, seed=122)
    case["seqlens"] = torch.tensor([128, 64 * 9], dtype=torch.int32)  # row has 2 pages only
    _, _, ws, _ = run_decode(to_gpu(case), "gqa", 2)
    assert gqla.gqla_read_device_error(ws) == (-5, 1)


# ------------------------------------------------------------------ full-size workloads, sampled

FULL = [(name, s, None) for name, w in synth.WORKLOADS.items() for s in w.s_q]
# the bench workload also at the one-wave split counts (chunks holding two sequences' pieces)
FULL += [("dsv3_h128_b32_l4096", 1, "one_wave")]


@pytest.mark.parametrize("path", ["gqa", "absorb"])
@pytest.mark.parametrize("name,s_q,splits", FULL, ids=[f"{n}-sq{s}" + (f"-{m}" if m else "") for n, s, m in FULL])
def test_decode_parity_full_size_sampled(path, name, s_q, splits):
    """Full-size workloads at the split counts bench.py plans (or one wave), sampled."""
    w = synth.WORKLOADS[name]
    case = synth.make_workload(name, s_q=s_q, device="cuda")
    from decode_attention_06_b200 import gqla
    n = gqla.gqla_num_splits_hint(path, w.num_heads, s_q) if splits == "one_wave" else None
    out, lse, ws, _ = run_decode(case, path, n)
    B = w.batch
    rng = np.random.default_rng(w.seed)
    picks = sorted(set([0, B - 1] + rng.integers(0, B, size=2).tolist()))[:3]
    if w.lengths[0] == "uniform" and w.lengths[2] > 16384:
        picks = picks[:2]
    sub = sub_case(case, picks)
    groups = list(range(w.num_groups))  # every group of the sampled sequences
    units = [(i, gi) for i in range(len(picks)) for gi in groups]
    ref, ref_lse = oracle_ref(sub, units=units)
    G = w.num_heads // w.num_groups
    mask = np.zeros(ref.shape[:3], dtype=bool)
    for i, gi in units:
        mask[i, :, gi * G:(gi + 1) * G] = True
    got = out[torch.tensor(picks, device="cuda")]
    compare(got, ref, mask=mask, what=f"{path}/{name}/sq{s_q}")
    compare_lse(lse[torch.tensor(picks, device="cuda")], ref_lse, mask=mask)
    from decode_attention_06_b200 import gqla
    assert gqla.gqla_read_device_error(ws)[0] == 0


# ------------------------------------------------------------------ sparse GQLA (GQA path)

SPARSE = [
    # id, h, g, seqlens, s_q, topk, unused entries, splits
    ("h128_topk256_pad", 128, 8, [1000, 70, 3000], 1, 256, 20, None),
    ("h128_mtp_topk100", 128, 8, [513, 130], 2, 100, 0, 5),
    ("g4_topk64", 128, 4, [700], 1, 64, 0, 3),
    ("h32_mtp_topk300_short", 32, 8, [2000, 3], 2, 300, 7, None),
]


def _sparse_run(case, idx, splits, fused=True):
    from decode_attention_06_b200 import gqla
    g = to_gpu(case)
    h, ng, s_q = case["num_heads"], case["num_groups"], case["s_q"]
    dims = gqla.make_dims(h, ng)
    kv = gqla.make_kv_index(g["page_table"], g["seqlens"], g["num_pages"])
    n = case["num_pages"] * case["page_size"]
    kvx = torch.empty(ng, n, 256, dtype=torch.bfloat16, device="cuda")
    kr = torch.empty(n, 64, dtype=torch.bfloat16, device="cuda")
    gqla.gqla_expand_cache(dims, g["latent"], g["w_uk"], g["w_uv"], kvx, kr)
    B = case["seqlens"].numel()
    if splits is None:
        splits = gqla.gqla_num_splits_hint("gqa", h, 1)
    bufs = gqla.SparseBuffers(dims, B, s_q, idx.shape[-1], splits, fused=fused)
    out, lse = gqla.sparse_gqa_step(dims, bufs, g["q"], kvx, kr, kv, idx.cuda())
    torch.cuda.synchronize()
    return out.clone(), lse.clone(), bufs


@pytest.mark.parametrize("fused", [True, False], ids=["fused", "selected_cache"])
@pytest.mark.parametrize("cid,h,g,seqlens,s_q,topk,unused,splits", SPARSE, ids=[c[0] for c in SPARSE])
def test_sparse_gqa_parity(cid, h, g, seqlens, s_q, topk, unused, splits, fused):
    from decode_attention_06_b200 import gqla
    case = synth.make_case(h, g, seqlens, s_q, paged=True, seed=300 + len(cid))
    idx = synth.make_topk(seqlens, s_q, topk, seed=400 + len(cid), unused=unused)
    out, lse, bufs = _sparse_run(case, idx, splits, fused)
    st, _ = gqla.gqla_read_device_error(bufs.workspace)
    assert st == 0
    ref, ref_lse = oracle.decode_sparse(case["q"], case["latent"], case["page_table"], case["seqlens"],
                                        case["w_uk"], case["w_uv"], g, idx)
    compare(out, ref, what=f"sparse/{cid}")
    compare_lse(lse, ref_lse, what=f"sparse/{cid}")
    counts = (idx >= 0).sum(-1).flatten()
    assert torch.equal(bufs.sel_seqlens.cpu(), counts.to(torch.int32))


@pytest.mark.parametrize("fused", [True, False], ids=["fused", "selected_cache"])
def test_sparse_invalid_position_is_reported_and_skipped(fused):
    from decode_attention_06_b200 import gqla
    case = synth.make_case(128, 8, [300, 200], 1, paged=True, seed=311)
    idx = synth.make_topk([300, 200], 1, 64, seed=312, unused=2)
    idx[1, 0, 62] = 200   # past the last visible token of sequence 1 (199)
    out, lse, bufs = _sparse_run(case, idx, None, fused)
    st, info = gqla.gqla_read_device_error(bufs.workspace)
    assert st == -5 and info == 1
    idx_ok = idx.clone()
    idx_ok[1, 0, 62] = -1
    ref, ref_lse = oracle.decode_sparse(case["q"], case["latent"], case["page_table"], case["seqlens"],
                                        case["w_uk"], case["w_uv"], 8, idx_ok)
    compare(out, ref, what="sparse/invalid-skipped")


# ------------------------------------------------------------------ fused GQA step

FUSED = [
    # id, h, g, seqlens, s_q, paged, splits: one split (no combine launch at all), sequences
    # inside one chunk next to sequences over several, empty sequences, group-split grids
    ("one_split_llama_l256", 32, 8, [256], 1, False, 1),
    ("one_split_mtp_ragged", 128, 8, [700, 0, 65, 1], 2, True, 1),
    ("mixed_single_and_multi", 128, 8, [64, 3000, 10, 0, 700], 1, True, 9),
    ("g4_mtp", 32, 4, [513, 64, 3], 2, False, 4),
    ("many_partials", 128, 8, [5000, 300], 1, True, 70),
    # (g, s_q) = (4, 1) at 128 heads: 32 columns of one query token per group, the
    # 32-column epilogue's final-output and partial writes
    ("g4_h128_one_split", 128, 4, [300, 65], 1, False, 1),
    ("g4_h128_splits", 128, 4, [1000, 130, 0], 1, True, 5),
]


@pytest.mark.parametrize("cid,h,g,seqlens,s_q,paged,splits", FUSED, ids=[c[0] for c in FUSED])
def test_gqa_step_fused_parity(cid, h, g, seqlens, s_q, paged, splits):
    """gqla_decode_gqa_step: the decode writes the output of every sequence that falls in
    one chunk, the combine the others; against the oracle, and bit for bit against the
    separate calls wherever the combine did the work in both."""
    from decode_attention_06_b200 import gqla
    case = synth.make_case(h, g, seqlens, s_q, paged=paged, seed=zlib.crc32(cid.encode()) % 1000)
    gc = to_gpu(case)
    dims = gqla.make_dims(h, g)
    kv = gqla.make_kv_index(gc["page_table"], gc["seqlens"], case["num_pages"])
    n = case["num_pages"] * case["page_size"]
    kvx = torch.empty(g, n, 256, dtype=torch.bfloat16, device="cuda")
    kr = torch.empty(n, 64, dtype=torch.bfloat16, device="cuda")
    gqla.gqla_expand_cache(dims, gc["latent"], gc["w_uk"], gc["w_uv"], kvx, kr)
    B = len(seqlens)
    bufs = gqla.DecodeBuffers(dims, B, s_q, splits, "gqa")
    bufs.out.fill_(float("nan"))
    bufs.lse.fill_(float("nan"))
    if splits == 1:  # one split: the partial buffers are not needed
        gqla.gqla_decode_gqa_step(dims, gc["q"], kvx, kr, kv, 1, None, None, bufs.out, bufs.lse,
                                  bufs.workspace)
    else:
        gqla.decode_step(dims, bufs, gc["q"], None, None, kv, kv_expanded=kvx, k_rope=kr, fused=True)
    torch.cuda.synchronize()
    assert gqla.gqla_read_device_error(bufs.workspace)[0] == 0
    ref, ref_lse = oracle_ref(case)
    compare(bufs.out, ref, what=f"fused/{cid}")
    compare_lse(bufs.lse, ref_lse, what=f"fused/{cid}")
    # the separate calls give the same result to within the bf16 rounding of the output
    out2, lse2, _, _ = run_decode(gc, "gqa", splits)
    torch.testing.assert_close(bufs.out.float(), out2.float(), rtol=2 ** -7, atol=1e-3)
