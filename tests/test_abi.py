"""Host-side checks of the C ABI: the library loads without a GPU, exports every
entry point include/gqla.h declares, and rejects bad arguments before any
launch (no CUDA call is reached by these cases)."""
import ctypes
import math
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gqla.h")


@pytest.fixture(scope="module")
def lib():
    from decode_attention_06_b200 import build_lib
    build_lib.build()
    return ctypes.CDLL(build_lib.LIB)


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gqla_[a-z_]+)\s*\(", text)))


def test_header_declares_the_five_calls():
    names = _declared()
    for n in ["gqla_expand_cache", "gqla_absorb_query", "gqla_decode_absorb",
              "gqla_decode_gqa", "gqla_combine"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_exposes_every_declared_symbol(lib):
    from decode_attention_06_b200 import gqla
    assert sorted(gqla.EXPORTED) == _declared()
    for n in _declared():
        assert callable(getattr(gqla, n))


def test_pure_host_helpers(lib):
    lib.gqla_workspace_bytes.restype = ctypes.c_size_t
    assert lib.gqla_version() == 1
    assert lib.gqla_workspace_bytes() >= 8
    assert lib.gqla_partial_slots(3, 5) == 8
    assert lib.gqla_partial_slots(0, 5) == -1
    lib.gqla_status_string.restype = ctypes.c_char_p
    assert lib.gqla_status_string(0) == b"ok"
    assert lib.gqla_status_string(-6).startswith(b"device-side wait")


class Dims(ctypes.Structure):
    _fields_ = [("num_heads", ctypes.c_int), ("num_groups", ctypes.c_int),
                ("d_latent", ctypes.c_int), ("d_rope", ctypes.c_int),
                ("d_nope", ctypes.c_int), ("d_v", ctypes.c_int),
                ("softmax_scale", ctypes.c_float)]


class KvIndex(ctypes.Structure):
    _fields_ = [("page_table", ctypes.c_void_p), ("seqlens", ctypes.c_void_p),
                ("batch", ctypes.c_int), ("max_pages_per_seq", ctypes.c_int),
                ("page_size", ctypes.c_int), ("num_pages", ctypes.c_int)]


FAKE = ctypes.c_void_p(1 << 20)  # aligned, never dereferenced: every case fails validation first


def _dims(h=128, g=8, lat=512, scale=0.072):
    return Dims(h, g, lat, 64, 128, 128, scale)


def _kv(batch=2, page_size=64):
    return KvIndex(FAKE, FAKE, batch, 4, page_size, 16)


@pytest.mark.parametrize("case,expected", [
    ("null_dims", -1), ("bad_heads", -1), ("latent_256", -2), ("s_q_3", -2), ("s_q_0", -1),
    ("page_32", -2), ("no_workspace", -3), ("small_workspace", -3), ("zero_splits", -1),
    ("null_q", -1), ("misaligned_q", -1), ("slots_mismatch", -1), ("batch_0", -1),
    ("bad_scale", -1),
])
def test_decode_gqa_rejects_bad_arguments(lib, case, expected):
    d, kv = _dims(), _kv()
    s_q, splits, ws, wsb, q, slots = 1, 4, FAKE, 256, FAKE, 16 * 64
    if case == "null_dims":
        dp = None
    else:
        if case == "bad_heads": d.num_heads = 100
        if case == "latent_256": d.d_latent = 256
        if case == "bad_scale": d.softmax_scale = float("nan")
        dp = ctypes.byref(d)
    if case == "s_q_3": s_q = 3
    if case == "s_q_0": s_q = 0
    if case == "page_32": kv.page_size = 32
    if case == "no_workspace": ws = None
    if case == "small_workspace": wsb = 4
    if case == "zero_splits": splits = 0
    if case == "null_q": q = None
    if case == "misaligned_q": q = ctypes.c_void_p((1 << 20) + 2)
    if case == "slots_mismatch": slots = 17
    if case == "batch_0": kv.batch = 0
    st = lib.gqla_decode_gqa(dp, q, s_q, FAKE, FAKE, ctypes.c_int64(slots), ctypes.byref(kv),
                             splits, FAKE, FAKE, ws, ctypes.c_size_t(wsb), None)
    assert st == expected


def test_other_calls_reject_bad_arguments(lib):
    d, kv = _dims(), _kv()
    assert lib.gqla_expand_cache(ctypes.byref(d), None, ctypes.c_int64(64), FAKE, FAKE, FAKE, FAKE, None) == -1
    assert lib.gqla_expand_cache(ctypes.byref(d), FAKE, ctypes.c_int64(-1), FAKE, FAKE, FAKE, FAKE, None) == -1
    assert lib.gqla_absorb_query(ctypes.byref(d), FAKE, 0, 1, FAKE, FAKE, None) == -1
    assert lib.gqla_absorb_query(ctypes.byref(d), FAKE, 2, 5, FAKE, FAKE, None) == -2
    assert lib.gqla_decode_absorb(ctypes.byref(d), FAKE, 1, FAKE, ctypes.byref(kv), 4, FAKE, FAKE,
                                  None, ctypes.c_size_t(0), None) == -3
    # absorb combine needs W_UV, the GQA combine must not get one; d_in must be 512 or 128
    assert lib.gqla_combine(ctypes.byref(d), ctypes.byref(kv), 1, 4, 512, FAKE, FAKE, None, FAKE, None, None) == -1
    assert lib.gqla_combine(ctypes.byref(d), ctypes.byref(kv), 1, 4, 128, FAKE, FAKE, FAKE, FAKE, None, None) == -1
    assert lib.gqla_combine(ctypes.byref(d), ctypes.byref(kv), 1, 4, 256, FAKE, FAKE, None, FAKE, None, None) == -1
    assert lib.gqla_read_device_error(None, None, None) == -1
    assert lib.gqla_num_splits_hint(7, 128, 1) == -1
    assert lib.gqla_num_splits_hint(0, 0, 1) == -1


def test_expand_tc_and_sparse_calls_reject_bad_arguments(lib):
    """The tensor-core expansion and the sparse entry points validate before any launch."""
    d, kv = _dims(), _kv()
    I64 = ctypes.c_int64
    assert lib.gqla_expand_cache_tc(ctypes.byref(d), None, I64(64), FAKE, FAKE, FAKE, FAKE, None) == -1
    assert lib.gqla_expand_cache_tc(ctypes.byref(d), FAKE, I64(-1), FAKE, FAKE, FAKE, FAKE, None) == -1
    assert lib.gqla_expand_cache_tc(ctypes.byref(d), ctypes.c_void_p((1 << 20) + 8), I64(64), FAKE, FAKE,
                                    FAKE, FAKE, None) == -1
    slots = I64(16 * 64)
    ws, wsb = FAKE, ctypes.c_size_t(256)
    # gather: topk out of range, null output, workspace too small, 2 groups unsupported
    assert lib.gqla_sparse_gather(ctypes.byref(d), FAKE, FAKE, slots, ctypes.byref(kv), 1, FAKE, 0,
                                  FAKE, FAKE, FAKE, FAKE, ws, wsb, None) == -1
    assert lib.gqla_sparse_gather(ctypes.byref(d), FAKE, FAKE, slots, ctypes.byref(kv), 1, FAKE, 64,
                                  None, FAKE, FAKE, FAKE, ws, wsb, None) == -1
    assert lib.gqla_sparse_gather(ctypes.byref(d), FAKE, FAKE, slots, ctypes.byref(kv), 1, FAKE, 64,
                                  FAKE, FAKE, FAKE, FAKE, ws, ctypes.c_size_t(4), None) == -3
    d2 = _dims(h=128, g=2)
    assert lib.gqla_sparse_gather(ctypes.byref(d2), FAKE, FAKE, slots, ctypes.byref(kv), 1, FAKE, 64,
                                  FAKE, FAKE, FAKE, FAKE, ws, wsb, None) == -2
    # select: s_q 3, misaligned slot list
    assert lib.gqla_sparse_select(ctypes.byref(d), ctypes.byref(kv), 3, FAKE, 64, FAKE, FAKE, FAKE,
                                  ws, wsb, None) == -2
    assert lib.gqla_sparse_select(ctypes.byref(d), ctypes.byref(kv), 1, FAKE, 64,
                                  ctypes.c_void_p((1 << 20) + 4), FAKE, FAKE, ws, wsb, None) == -1
    # fused decode: a selection whose batch is not a multiple of s_q, zero splits, no slot list
    assert lib.gqla_decode_gqa_sparse(ctypes.byref(d), FAKE, 2, FAKE, FAKE, slots, ctypes.byref(_kv(batch=3)),
                                      FAKE, 4, FAKE, FAKE, ws, wsb, None) == -1
    assert lib.gqla_decode_gqa_sparse(ctypes.byref(d), FAKE, 1, FAKE, FAKE, slots, ctypes.byref(kv),
                                      FAKE, 0, FAKE, FAKE, ws, wsb, None) == -1
    assert lib.gqla_decode_gqa_sparse(ctypes.byref(d), FAKE, 1, FAKE, FAKE, slots, ctypes.byref(kv),
                                      None, 4, FAKE, FAKE, ws, wsb, None) == -1


# ------------------------------------------------------------------ host-side split planning

def _plan_by_hand(lens, max_splits, piece_cost):
    """Every split count tried in turn: chunk loads = pages + piece_cost per sequence
    that starts inside a chunk after its first page; the lightest heaviest chunk wins,
    the smallest count on a tie."""
    pages = [(x + 63) // 64 for x in lens]
    T = sum(pages)
    if T == 0:
        return 1
    starts, acc = [], 0
    for n in pages:
        if n > 0 and acc > 0:
            starts.append(acc)
        acc += n
    best, best_load = None, None
    for n in range(1, max_splits + 1):
        k = -(-T // n)
        load = [min(k, T - c * k) for c in range(-(-T // k))]
        for st in starts:
            if st % k:
                load[st // k] += piece_cost
        if best_load is None or max(load) < best_load:
            best, best_load = n, max(load)
    return best


def _plan(lib, lens, max_splits, piece_cost):
    arr = (ctypes.c_int32 * len(lens))(*lens)
    return lib.gqla_plan_splits(arr, len(lens), max_splits, piece_cost)


def test_plan_splits_uniform_batch(lib):
    lens = [4096] * 32  # 32 sequences of 64 pages
    # without a piece cost: the most splits that shorten the longest chunk (28 pages)
    assert _plan(lib, lens, 74, 0) == 74
    # with one: 64 splits give 32-page chunks inside single sequences, against 28 pages
    # plus a second piece for 74
    assert _plan(lib, lens, 74, 6) == 64
    assert _plan(lib, lens, 148, 2) == 128
    assert _plan(lib, lens, 1, 6) == 1


def test_plan_splits_matches_exhaustive_search(lib):
    import random
    rng = random.Random(11)
    for _ in range(60):
        B = rng.randint(1, 40)
        lens = [rng.choice([0, rng.randint(1, 200), rng.randint(1, 9000)]) for _ in range(B)]
        m, pc = rng.randint(1, 160), rng.randint(0, 9)
        assert _plan(lib, lens, m, pc) == _plan_by_hand(lens, m, pc), (lens, m, pc)


def test_plan_splits_edges(lib):
    assert _plan(lib, [0, 0, 0], 74, 6) == 1          # no pages: one split
    assert _plan(lib, [0, 640, 0], 8, 6) == 5         # 2-page chunks from 5 splits on; empty sequences start no piece
    assert _plan(lib, [64] * 4, 4, 6) == 4            # one page each: one per split
    assert _plan(lib, [-1, 64], 4, 6) == -1
    assert _plan(lib, [64], 0, 6) == -1
    assert _plan(lib, [64], 4, -1) == -1
    assert lib.gqla_plan_splits(None, 1, 4, 6) == -1
    arr = (ctypes.c_int32 * 1)(64)
    assert lib.gqla_plan_splits(arr, 0, 4, 6) == -1


def test_lead_calls_reject_bad_arguments(lib):
    """The lead split plan: 0 .. num_splits lead chunks, each 1 to 64 times as long as the
    others (weight in 1/16); the planner checks its arguments before it asks the device."""
    d, kv = _dims(), _kv()
    wsb = ctypes.c_size_t(256)
    for lead, w16 in ((5, 32), (-1, 32), (1, 15), (1, 1025)):
        assert lib.gqla_decode_absorb_lead(ctypes.byref(d), FAKE, 1, FAKE, ctypes.byref(kv), 4, lead, w16,
                                           FAKE, FAKE, FAKE, wsb, None) == -1, (lead, w16)
        assert lib.gqla_combine_lead(ctypes.byref(d), ctypes.byref(kv), 1, 4, lead, w16, 512, FAKE, FAKE,
                                     FAKE, FAKE, None, None) == -1, (lead, w16)
    # GQA partials never come from a plan with lead chunks
    assert lib.gqla_combine_lead(ctypes.byref(d), ctypes.byref(kv), 1, 4, 1, 32, 128, FAKE, FAKE,
                                 None, FAKE, None, None) == -1
    F = ctypes.c_float
    e, w = ctypes.c_int(), ctypes.c_int()
    plan = lambda *a: lib.gqla_plan_lead(*a)
    D = ctypes.byref(d)
    assert plan(D, 2, 148, 0, 128, F(400), F(350), F(30), ctypes.byref(e), ctypes.byref(w)) == -1
    assert plan(D, 2, 148, 37, 0, F(400), F(350), F(30), ctypes.byref(e), ctypes.byref(w)) == -1
    assert plan(D, 2, 0, 37, 128, F(400), F(350), F(30), ctypes.byref(e), ctypes.byref(w)) == -1
    assert plan(D, 2, 148, 37, 128, F(0), F(350), F(30), ctypes.byref(e), ctypes.byref(w)) == -1
    assert plan(D, 2, 148, 37, 128, F(400), F(-1), F(30), ctypes.byref(e), ctypes.byref(w)) == -1
    assert plan(D, 2, 148, 37, 128, F(400), F(350), F(30), None, ctypes.byref(w)) == -1
    assert plan(D, 3, 148, 37, 128, F(400), F(350), F(30), ctypes.byref(e), ctypes.byref(w)) == -2


def _lead(lib, h, g, s_q, sms, ca, cg, ta, tg, tc):
    d = _dims(h, g)
    e, w = ctypes.c_int(-7), ctypes.c_int(-7)
    F = ctypes.c_float
    st = lib.gqla_plan_lead(ctypes.byref(d), s_q, sms, ca, cg, F(ta), F(tg), F(tc), ctypes.byref(e), ctypes.byref(w))
    assert st == 0
    return e.value, w.value


def _lead_by_hand(h, g, s_q, sms, ca, cg, ta, tg, tc):
    """The plan written out: lead chunks = the absorb chunks (2 CTAs per 128 query rows)
    that fit on the SMs the GQA decode's CTAs (its splits times the group split it takes
    when splits x 4 x gs <= SMs) leave idle; W from equal total work and the lead chunks
    ending the combine's time before the GQA decode."""
    gs = 1
    while gs < g and cg * gs * 4 <= sms:
        gs *= 2
    free = sms - cg * gs
    rb = -(-(s_q * h) // 128)
    e = min(free // (2 * rb) if free > 0 else 0, ca - 1)
    x = float(F32(tg)) - float(F32(tc))
    if e <= 0 or x <= 0:
        return 0, 16
    ta = float(F32(ta))
    den = max(1.0 - x * e / (ca * ta), 0.05)
    wgt = min(1.0 + (x / ta) / den, 64.0)
    return e, int(math.floor(16 * wgt + 0.5))


def F32(v):
    import numpy as np
    return np.float32(v)


def test_plan_lead_matches_the_formula(lib):
    """gqla_plan_lead against the plan written out by hand (host-only: no device)."""
    cases = [
        # (h, g, s_q, sms, absorb splits, gqa splits, T_a, T_g, T_c) in us
        (128, 8, 2, 148, 37, 128, 414.0, 359.0, 37.0),   # the 64 x 8192 step: 5 chunks, W16 30
        (128, 8, 1, 148, 64, 128, 77.6, 93.6, 14.4),
        (32, 8, 1, 148, 4, 1, 16.8, 16.4, 10.0),          # one GQA split, its groups over 8 CTAs
        (128, 8, 2, 148, 37, 148, 414.0, 359.0, 37.0),    # the GQA decode fills the device
        (128, 8, 2, 148, 37, 128, 414.0, 30.0, 37.0),     # x <= 0
        (128, 4, 1, 148, 64, 128, 78.2, 60.2, 14.4),
        (128, 8, 2, 132, 33, 100, 400.0, 380.0, 20.0),    # another SM count
        (128, 8, 2, 148, 3, 100, 50.0, 400.0, 1.0),       # lead capped at splits - 1, W capped at 64
    ]
    for c in cases:
        assert _lead(lib, *c) == _lead_by_hand(*c), c
    assert _lead(lib, *cases[0]) == (5, 30)
