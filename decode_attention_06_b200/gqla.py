"""Python binding of libgqla (include/gqla.h): argument marshalling only.

Every function here checks tensor placement/dtype/shape, passes raw device
pointers and the current CUDA stream to the C ABI, and raises on a non-zero
status.  All arithmetic happens in the CUDA kernels of libgqla.so; there is no
fallback: if the library is missing, importing this module fails.

PyTorch is used for device memory and streams only.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgqla.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(
        f"libgqla.so not found at {_LIB_PATH}; build it with "
        "`python -m decode_attention_06_b200.build_lib` (needs nvcc)")
_lib = ctypes.CDLL(_LIB_PATH)

D_LATENT, D_ROPE, D_NOPE, D_V = 512, 64, 128, 128
D_QK, D_ROW = D_NOPE + D_ROPE, D_LATENT + D_ROPE
PAGE_SIZE = 64

STATUS = {0: "GQLA_OK", -1: "GQLA_ERR_INVALID_ARG", -2: "GQLA_ERR_UNSUPPORTED",
          -3: "GQLA_ERR_WORKSPACE", -4: "GQLA_ERR_CUDA", -5: "GQLA_ERR_DEVICE",
          -6: "GQLA_ERR_TIMEOUT"}


class GqlaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        extra = ""
        if status == -4:
            extra = ": " + _lib.gqla_last_cuda_error().decode()
        super().__init__(f"{fn} returned {status} ({STATUS.get(status, '?')}){extra}")


class gqla_dims(ctypes.Structure):
    _fields_ = [("num_heads", ctypes.c_int), ("num_groups", ctypes.c_int),
                ("d_latent", ctypes.c_int), ("d_rope", ctypes.c_int),
                ("d_nope", ctypes.c_int), ("d_v", ctypes.c_int),
                ("softmax_scale", ctypes.c_float)]


class gqla_kv_index(ctypes.Structure):
    _fields_ = [("page_table", ctypes.c_void_p), ("seqlens", ctypes.c_void_p),
                ("batch", ctypes.c_int), ("max_pages_per_seq", ctypes.c_int),
                ("page_size", ctypes.c_int), ("num_pages", ctypes.c_int)]


_P, _I, _I64, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
_DP, _KP = ctypes.POINTER(gqla_dims), ctypes.POINTER(gqla_kv_index)
_SIGS = {
    "gqla_expand_cache": [_DP, _P, _I64, _P, _P, _P, _P, _P],
    "gqla_expand_cache_tc": [_DP, _P, _I64, _P, _P, _P, _P, _P],
    "gqla_absorb_query": [_DP, _P, _I, _I, _P, _P, _P],
    "gqla_decode_absorb": [_DP, _P, _I, _P, _KP, _I, _P, _P, _P, _SZ, _P],
    "gqla_decode_absorb_lead": [_DP, _P, _I, _P, _KP, _I, _I, _I, _P, _P, _P, _SZ, _P],
    "gqla_decode_gqa": [_DP, _P, _I, _P, _P, _I64, _KP, _I, _P, _P, _P, _SZ, _P],
    "gqla_decode_gqa_step": [_DP, _P, _I, _P, _P, _I64, _KP, _I, _P, _P, _P, _P, _P, _SZ, _P],
    "gqla_combine": [_DP, _KP, _I, _I, _I, _P, _P, _P, _P, _P, _P],
    "gqla_combine_lead": [_DP, _KP, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P],
    "gqla_sparse_gather": [_DP, _P, _P, _I64, _KP, _I, _P, _I, _P, _P, _P, _P, _P, _SZ, _P],
    "gqla_sparse_select": [_DP, _KP, _I, _P, _I, _P, _P, _P, _P, _SZ, _P],
    "gqla_decode_gqa_sparse": [_DP, _P, _I, _P, _P, _I64, _KP, _P, _I, _P, _P, _P, _SZ, _P],
    "gqla_decode_gqa_noalloc": [_DP, _P, _I, _P, _P, _I64, _KP, _I, _P, _P, _P, _P],
    "gqla_partial_slots": [_I, _I],
    "gqla_workspace_bytes": [],
    "gqla_num_splits_hint": [_I, _I, _I],
    "gqla_plan_splits": [_P, _I, _I, _I],
    "gqla_plan_lead": [_DP, _I, _I, _I, _I, ctypes.c_float, ctypes.c_float, ctypes.c_float,
                       ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)],
    "gqla_read_device_error": [_P, ctypes.POINTER(ctypes.c_int), _P],
    "gqla_clear_device_error": [_P, _P],
    "gqla_status_string": [_I],
    "gqla_last_cuda_error": [],
    "gqla_version": [],
    "gqla_debug_drop_v_load": [_I],
}
for _name, _args in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = _I
_lib.gqla_workspace_bytes.restype = _SZ
_lib.gqla_status_string.restype = ctypes.c_char_p
_lib.gqla_last_cuda_error.restype = ctypes.c_char_p

EXPORTED = tuple(_SIGS)


def _check(fn: str, st: int):
    if st != 0:
        raise GqlaError(fn, st)


def _stream(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _dev(t: torch.Tensor, name: str, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return ctypes.c_void_p(t.data_ptr())


def make_dims(num_heads: int, num_groups: int = 8, softmax_scale: Optional[float] = None):
    return gqla_dims(num_heads, num_groups, D_LATENT, D_ROPE, D_NOPE, D_V,
                     1.0 / math.sqrt(D_NOPE + D_ROPE) if softmax_scale is None else softmax_scale)


def make_kv_index(page_table: torch.Tensor, seqlens: torch.Tensor, num_pages: int,
                  page_size: int = PAGE_SIZE):
    pt = _dev(page_table, "page_table", torch.int32)
    sl = _dev(seqlens, "seqlens", torch.int32)
    if page_table.dim() != 2 or seqlens.shape != (page_table.shape[0],):
        raise ValueError("page_table must be [batch][max_pages] and seqlens [batch]")
    idx = gqla_kv_index(pt, sl, page_table.shape[0], page_table.shape[1], page_size, num_pages)
    idx._keep = (page_table, seqlens)  # keep the tensors alive with the struct
    return idx


# ------------------------------------------------------------------ the five calls

def gqla_expand_cache(dims, latent, w_uk, w_uv, kv_expanded, k_rope, stream=None):
    n = latent.numel() // D_ROW
    g = dims.num_groups
    _check("gqla_expand_cache", _lib.gqla_expand_cache(
        ctypes.byref(dims), _dev(latent, "latent", torch.bfloat16), n,
        _dev(w_uk, "w_uk", torch.bfloat16, (g, D_LATENT, D_NOPE)),
        _dev(w_uv, "w_uv", torch.bfloat16, (g, D_LATENT, D_V)),
        _dev(kv_expanded, "kv_expanded", torch.bfloat16, (g, n, D_NOPE + D_V)),
        _dev(k_rope, "k_rope", torch.bfloat16, (n, D_ROPE)), _stream(stream)))


def gqla_expand_cache_tc(dims, latent, w_uk, w_uv, kv_expanded, k_rope, stream=None):
    n = latent.numel() // D_ROW
    g = dims.num_groups
    _check("gqla_expand_cache_tc", _lib.gqla_expand_cache_tc(
        ctypes.byref(dims), _dev(latent, "latent", torch.bfloat16), n,
        _dev(w_uk, "w_uk", torch.bfloat16, (g, D_LATENT, D_NOPE)),
        _dev(w_uv, "w_uv", torch.bfloat16, (g, D_LATENT, D_V)),
        _dev(kv_expanded, "kv_expanded", torch.bfloat16, (g, n, D_NOPE + D_V)),
        _dev(k_rope, "k_rope", torch.bfloat16, (n, D_ROPE)), _stream(stream)))


def gqla_absorb_query(dims, q, w_uk, q_absorbed, stream=None):
    B, s_q, h, _ = q.shape
    _check("gqla_absorb_query", _lib.gqla_absorb_query(
        ctypes.byref(dims), _dev(q, "q", torch.bfloat16, (B, s_q, dims.num_heads, D_QK)), B, s_q,
        _dev(w_uk, "w_uk", torch.bfloat16, (dims.num_groups, D_LATENT, D_NOPE)),
        _dev(q_absorbed, "q_absorbed", torch.bfloat16, (B, s_q, h, D_ROW)), _stream(stream)))


def gqla_decode_absorb(dims, q_absorbed, latent_cache, kv, num_splits, o_part, lse_part,
                       workspace, stream=None, lead=None):
    """lead = (lead_splits, lead_weight16) calls gqla_decode_absorb_lead."""
    B, s_q, h, _ = q_absorbed.shape
    slots = gqla_partial_slots(kv.batch, num_splits)
    fn, extra = ("gqla_decode_absorb", ()) if lead is None else ("gqla_decode_absorb_lead", tuple(lead))
    _check(fn, getattr(_lib, fn)(
        ctypes.byref(dims), _dev(q_absorbed, "q_absorbed", torch.bfloat16, (kv.batch, s_q, dims.num_heads, D_ROW)),
        s_q, _dev(latent_cache, "latent_cache", torch.bfloat16, (kv.num_pages, kv.page_size, D_ROW)),
        ctypes.byref(kv), num_splits, *extra,
        _dev(o_part, "o_part", torch.float32, (slots, s_q, h, D_LATENT)),
        _dev(lse_part, "lse_part", torch.float32, (slots, s_q, h)),
        _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(), _stream(stream)))


def gqla_decode_absorb_lead(dims, q_absorbed, latent_cache, kv, num_splits, lead_splits, lead_weight16,
                            o_part, lse_part, workspace, stream=None):
    gqla_decode_absorb(dims, q_absorbed, latent_cache, kv, num_splits, o_part, lse_part, workspace,
                       stream, lead=(lead_splits, lead_weight16))


def gqla_decode_gqa(dims, q, kv_expanded, k_rope, kv, num_splits, o_part, lse_part, workspace,
                    stream=None):
    B, s_q, h, _ = q.shape
    n = kv.num_pages * kv.page_size
    slots = gqla_partial_slots(kv.batch, num_splits)
    _check("gqla_decode_gqa", _lib.gqla_decode_gqa(
        ctypes.byref(dims), _dev(q, "q", torch.bfloat16, (kv.batch, s_q, dims.num_heads, D_QK)), s_q,
        _dev(kv_expanded, "kv_expanded", torch.bfloat16, (dims.num_groups, n, D_NOPE + D_V)),
        _dev(k_rope, "k_rope", torch.bfloat16, (n, D_ROPE)), n, ctypes.byref(kv), num_splits,
        _dev(o_part, "o_part", torch.float32, (slots, s_q, h, D_V)),
        _dev(lse_part, "lse_part", torch.float32, (slots, s_q, h)),
        _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(), _stream(stream)))


def gqla_decode_gqa_step(dims, q, kv_expanded, k_rope, kv, num_splits, o_part, lse_part, out, lse_out,
                         workspace, stream=None):
    """gqla_decode_gqa + gqla_combine in one call; sequences that fall in one chunk get
    their output from the decode itself (o_part / lse_part may be None for one split)."""
    B, s_q, h, _ = q.shape
    n = kv.num_pages * kv.page_size
    slots = gqla_partial_slots(kv.batch, num_splits)
    _check("gqla_decode_gqa_step", _lib.gqla_decode_gqa_step(
        ctypes.byref(dims), _dev(q, "q", torch.bfloat16, (kv.batch, s_q, dims.num_heads, D_QK)), s_q,
        _dev(kv_expanded, "kv_expanded", torch.bfloat16, (dims.num_groups, n, D_NOPE + D_V)),
        _dev(k_rope, "k_rope", torch.bfloat16, (n, D_ROPE)), n, ctypes.byref(kv), num_splits,
        None if o_part is None else _dev(o_part, "o_part", torch.float32, (slots, s_q, h, D_V)),
        None if lse_part is None else _dev(lse_part, "lse_part", torch.float32, (slots, s_q, h)),
        _dev(out, "out", torch.bfloat16, (kv.batch, s_q, h, D_V)),
        None if lse_out is None else _dev(lse_out, "lse_out", torch.float32, (kv.batch, s_q, h)),
        _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(), _stream(stream)))


def gqla_combine(dims, kv, s_q, num_splits, d_in, o_part, lse_part, w_uv, out, lse_out=None,
                 stream=None, lead=None):
    """lead = (lead_splits, lead_weight16), as given to the decode, calls gqla_combine_lead."""
    slots = gqla_partial_slots(kv.batch, num_splits)
    h = dims.num_heads
    fn, extra = ("gqla_combine", ()) if lead is None else ("gqla_combine_lead", tuple(lead))
    _check(fn, getattr(_lib, fn)(
        ctypes.byref(dims), ctypes.byref(kv), s_q, num_splits, *extra, d_in,
        _dev(o_part, "o_part", torch.float32, (slots, s_q, h, d_in)),
        _dev(lse_part, "lse_part", torch.float32, (slots, s_q, h)),
        None if w_uv is None else _dev(w_uv, "w_uv", torch.bfloat16, (dims.num_groups, D_LATENT, D_V)),
        _dev(out, "out", torch.bfloat16, (kv.batch, s_q, h, D_V)),
        None if lse_out is None else _dev(lse_out, "lse_out", torch.float32, (kv.batch, s_q, h)),
        _stream(stream)))


def gqla_sparse_gather(dims, kv_expanded, k_rope, kv, s_q, topk_idx, kv_sel, k_rope_sel,
                       sel_page_table, sel_seqlens, workspace, stream=None):
    B = kv.batch
    n = kv.num_pages * kv.page_size
    topk = topk_idx.shape[-1]
    cap = (topk + PAGE_SIZE - 1) // PAGE_SIZE * PAGE_SIZE
    ns = B * s_q * cap
    _check("gqla_sparse_gather", _lib.gqla_sparse_gather(
        ctypes.byref(dims), _dev(kv_expanded, "kv_expanded", torch.bfloat16, (dims.num_groups, n, D_NOPE + D_V)),
        _dev(k_rope, "k_rope", torch.bfloat16, (n, D_ROPE)), n, ctypes.byref(kv), s_q,
        _dev(topk_idx, "topk_idx", torch.int32, (B, s_q, topk)), topk,
        _dev(kv_sel, "kv_sel", torch.bfloat16, (dims.num_groups, ns, D_NOPE + D_V)),
        _dev(k_rope_sel, "k_rope_sel", torch.bfloat16, (ns, D_ROPE)),
        _dev(sel_page_table, "sel_page_table", torch.int32, (B * s_q, cap // PAGE_SIZE)),
        _dev(sel_seqlens, "sel_seqlens", torch.int32, (B * s_q,)),
        _dev(workspace, "workspace", torch.uint8), workspace.numel(), _stream(stream)))


def gqla_sparse_select(dims, kv, s_q, topk_idx, sel_slot, sel_page_table, sel_seqlens, workspace,
                       stream=None):
    B = kv.batch
    topk = topk_idx.shape[-1]
    cap = (topk + PAGE_SIZE - 1) // PAGE_SIZE * PAGE_SIZE
    _check("gqla_sparse_select", _lib.gqla_sparse_select(
        ctypes.byref(dims), ctypes.byref(kv), s_q, _dev(topk_idx, "topk_idx", torch.int32, (B, s_q, topk)), topk,
        _dev(sel_slot, "sel_slot", torch.int32, (B * s_q * cap,)),
        _dev(sel_page_table, "sel_page_table", torch.int32, (B * s_q, cap // PAGE_SIZE)),
        _dev(sel_seqlens, "sel_seqlens", torch.int32, (B * s_q,)),
        _dev(workspace, "workspace", torch.uint8), workspace.numel(), _stream(stream)))


def gqla_decode_gqa_sparse(dims, q, kv_expanded, k_rope, num_slots, sel, sel_slot, num_splits, o_part,
                           lse_part, workspace, stream=None):
    B, s_q, h, _ = q.shape
    slots = gqla_partial_slots(sel.batch, num_splits)
    _check("gqla_decode_gqa_sparse", _lib.gqla_decode_gqa_sparse(
        ctypes.byref(dims), _dev(q, "q", torch.bfloat16, (sel.batch // s_q, s_q, dims.num_heads, D_QK)), s_q,
        _dev(kv_expanded, "kv_expanded", torch.bfloat16, (dims.num_groups, num_slots, D_NOPE + D_V)),
        _dev(k_rope, "k_rope", torch.bfloat16, (num_slots, D_ROPE)), num_slots, ctypes.byref(sel),
        _dev(sel_slot, "sel_slot", torch.int32), num_splits,
        _dev(o_part, "o_part", torch.float32, (slots, 1, h, D_V)),
        _dev(lse_part, "lse_part", torch.float32, (slots, 1, h)),
        _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(), _stream(stream)))


def gqla_decode_gqa_noalloc(dims, q, kv_expanded, k_rope, kv, num_splits, out, lse_out=None,
                            device_error=None, stream=None):
    """GQA decode step with library-owned static scratch (no o_part/lse_part/workspace)."""
    B, s_q, h, _ = q.shape
    n = kv.num_pages * kv.page_size
    _check("gqla_decode_gqa_noalloc", _lib.gqla_decode_gqa_noalloc(
        ctypes.byref(dims), _dev(q, "q", torch.bfloat16, (kv.batch, s_q, dims.num_heads, D_QK)), s_q,
        _dev(kv_expanded, "kv_expanded", torch.bfloat16, (dims.num_groups, n, D_NOPE + D_V)),
        _dev(k_rope, "k_rope", torch.bfloat16, (n, D_ROPE)), n, ctypes.byref(kv), num_splits,
        _dev(out, "out", torch.bfloat16, (kv.batch, s_q, h, D_V)),
        None if lse_out is None else _dev(lse_out, "lse_out", torch.float32, (kv.batch, s_q, h)),
        None if device_error is None else _dev(device_error, "device_error", torch.int32, (2,)),
        _stream(stream)))


# ------------------------------------------------------------------ helpers

def gqla_partial_slots(batch: int, num_splits: int) -> int:
    n = _lib.gqla_partial_slots(batch, num_splits)
    if n < 0:
        raise GqlaError("gqla_partial_slots", n)
    return n


def gqla_workspace_bytes() -> int:
    return int(_lib.gqla_workspace_bytes())


def gqla_num_splits_hint(path: str, num_heads: int, s_q: int) -> int:
    n = _lib.gqla_num_splits_hint({"absorb": 0, "gqa": 1}[path], num_heads, s_q)
    if n < 0:
        raise GqlaError("gqla_num_splits_hint", n)
    return n


def gqla_combine_lead(dims, kv, s_q, num_splits, lead_splits, lead_weight16, d_in, o_part, lse_part, w_uv,
                      out, lse_out=None, stream=None):
    gqla_combine(dims, kv, s_q, num_splits, d_in, o_part, lse_part, w_uv, out, lse_out, stream,
                 lead=(lead_splits, lead_weight16))


def gqla_plan_lead(dims, s_q: int, num_sms: int, absorb_splits: int, gqa_splits: int,
                   absorb_decode_us: float, gqa_decode_us: float, absorb_combine_us: float):
    """(lead_splits, lead_weight16) for the absorb decode beside the GQA path on a device
    with num_sms SMs."""
    e, w = ctypes.c_int(0), ctypes.c_int(16)
    _check("gqla_plan_lead", _lib.gqla_plan_lead(
        ctypes.byref(dims), s_q, num_sms, absorb_splits, gqa_splits, absorb_decode_us, gqa_decode_us,
        absorb_combine_us, ctypes.byref(e), ctypes.byref(w)))
    return e.value, w.value


def gqla_plan_splits(seqlens, max_splits: int, piece_cost_pages: int) -> int:
    """Split count for known lengths (host int32 values: a CPU tensor or a list)."""
    lens = torch.as_tensor(seqlens, dtype=torch.int32, device="cpu").contiguous()
    n = _lib.gqla_plan_splits(ctypes.c_void_p(lens.data_ptr()), lens.numel(), max_splits, piece_cost_pages)
    if n < 0:
        raise GqlaError("gqla_plan_splits", n)
    return n


# What a chunk's second piece costs, in pages of the chunk, for the two decode
# kernels on B200 (sweeps of split counts: over 32 sequences of 4096 tokens the
# absorb decode's time grows by ~0.9 us per page of its longest chunk and by
# ~6 us when that chunk holds two pieces; the GQA decode, bound by the HBM
# stream, gains little from more CTAs and loses 8-10 pages' worth per extra
# piece: 389 us at 128 splits of 64 pages, each inside one sequence, against
# 401 us at 147 splits of 56 pages over 64 sequences of 8192 tokens, s_q = 2).
PIECE_COST_PAGES = {"absorb": 6, "gqa": 8}


# Below this many pages in the batch, one split is fastest for gqla_decode_gqa_step: the
# decode then writes every output itself (its groups spread over up to 8 CTAs) and no
# combine runs.  Measured on B200 at one sequence of 256 tokens (4 pages): 14.4 us with
# one split against 18.5 us with 2 to 8 splits and the combine.
SINGLE_SPLIT_MAX_PAGES = 8


def plan_splits(path: str, num_heads: int, s_q: int, seqlens, fused: bool = False) -> int:
    """gqla_plan_splits up to one wave of the device, with the path's piece cost; for the
    fused GQA step (gqla_decode_gqa_step), one split when the batch is tiny."""
    if fused and path == "gqa":
        lens = torch.as_tensor(seqlens, dtype=torch.int64, device="cpu")
        if int(((lens + PAGE_SIZE - 1) // PAGE_SIZE).sum()) <= SINGLE_SPLIT_MAX_PAGES:
            return 1
    return gqla_plan_splits(seqlens, gqla_num_splits_hint(path, num_heads, s_q), PIECE_COST_PAGES[path])


def gqla_read_device_error(workspace: torch.Tensor, stream=None):
    info = ctypes.c_int(0)
    st = _lib.gqla_read_device_error(_dev(workspace, "workspace"), ctypes.byref(info), _stream(stream))
    return st, info.value


def gqla_clear_device_error(workspace: torch.Tensor, stream=None):
    _check("gqla_clear_device_error", _lib.gqla_clear_device_error(_dev(workspace, "workspace"), _stream(stream)))


def gqla_status_string(status: int) -> str:
    return _lib.gqla_status_string(status).decode()


def gqla_last_cuda_error() -> str:
    return _lib.gqla_last_cuda_error().decode()


def gqla_version() -> int:
    return _lib.gqla_version()


def gqla_debug_drop_v_load(unit: int):
    """Diagnostic: the next decode call of this thread leaves out one load (GQA decode:
    a V load; absorb decode: a latent tile), so its bounded wait runs out and the call
    records GQLA_ERR_TIMEOUT (-1 cancels)."""
    _check("gqla_debug_drop_v_load", _lib.gqla_debug_drop_v_load(unit))


def new_workspace(device=None) -> torch.Tensor:
    """A zeroed workspace of gqla_workspace_bytes() bytes."""
    return torch.zeros(gqla_workspace_bytes(), dtype=torch.uint8, device=device or "cuda")


class DecodeBuffers:
    """Device buffers for one decode step (allocated once, reused every step)."""

    def __init__(self, dims, batch: int, s_q: int, num_splits: int, path: str, device="cuda"):
        h = dims.num_heads
        slots = gqla_partial_slots(batch, num_splits)
        d_in = D_LATENT if path == "absorb" else D_V
        self.path, self.s_q, self.num_splits, self.d_in = path, s_q, num_splits, d_in
        self.q_absorbed = (torch.empty(batch, s_q, h, D_ROW, dtype=torch.bfloat16, device=device)
                           if path == "absorb" else None)
        self.o_part = torch.empty(slots, s_q, h, d_in, dtype=torch.float32, device=device)
        self.lse_part = torch.empty(slots, s_q, h, dtype=torch.float32, device=device)
        self.out = torch.empty(batch, s_q, h, D_V, dtype=torch.bfloat16, device=device)
        self.lse = torch.empty(batch, s_q, h, dtype=torch.float32, device=device)
        self.workspace = new_workspace(device)


class SparseBuffers:
    """Device buffers of one sparse GQA step: the selection (its slot list for the
    fused path, or a selected cache), its index, and the decode buffers of the
    batch * s_q selected sequences."""

    def __init__(self, dims, batch: int, s_q: int, topk: int, num_splits: int, device="cuda",
                 fused: bool = False):
        self.s_q, self.topk, self.fused = s_q, topk, fused
        self.cap = (topk + PAGE_SIZE - 1) // PAGE_SIZE * PAGE_SIZE
        v = batch * s_q
        if fused:
            self.sel_slot = torch.empty(v * self.cap, dtype=torch.int32, device=device)
            self.kv_sel = self.k_rope_sel = None
        else:
            self.sel_slot = None
            self.kv_sel = torch.empty(dims.num_groups, v * self.cap, D_NOPE + D_V, dtype=torch.bfloat16,
                                      device=device)
            self.k_rope_sel = torch.empty(v * self.cap, D_ROPE, dtype=torch.bfloat16, device=device)
        self.sel_page_table = torch.empty(v, self.cap // PAGE_SIZE, dtype=torch.int32, device=device)
        self.sel_seqlens = torch.empty(v, dtype=torch.int32, device=device)
        self.sel_index = make_kv_index(self.sel_page_table, self.sel_seqlens, v * self.cap // PAGE_SIZE)
        self.dec = DecodeBuffers(dims, v, 1, num_splits, "gqa", device=device)
        self.workspace = self.dec.workspace


def sparse_gqa_step(dims, bufs: SparseBuffers, q, kv_expanded, k_rope, kv, topk_idx, stream=None):
    """Sparse GQA step through the C ABI: the selection, then the GQA decode (the
    fused one gathering the selected rows itself, or the plain one over a selected
    cache) and the combine over batch * s_q one-token queries.  Returns
    (out [batch][s_q][h][128] bf16, lse [batch][s_q][h])."""
    B, s_q, h, _ = q.shape
    if bufs.fused:
        gqla_sparse_select(dims, kv, s_q, topk_idx, bufs.sel_slot, bufs.sel_page_table, bufs.sel_seqlens,
                           bufs.workspace, stream)
        gqla_decode_gqa_sparse(dims, q, kv_expanded, k_rope, kv.num_pages * kv.page_size, bufs.sel_index,
                               bufs.sel_slot, bufs.dec.num_splits, bufs.dec.o_part, bufs.dec.lse_part,
                               bufs.workspace, stream)
    else:
        gqla_sparse_gather(dims, kv_expanded, k_rope, kv, s_q, topk_idx, bufs.kv_sel, bufs.k_rope_sel,
                           bufs.sel_page_table, bufs.sel_seqlens, bufs.workspace, stream)
        q1 = q.view(B * s_q, 1, h, D_QK)
        gqla_decode_gqa(dims, q1, bufs.kv_sel, bufs.k_rope_sel, bufs.sel_index, bufs.dec.num_splits,
                        bufs.dec.o_part, bufs.dec.lse_part, bufs.workspace, stream)
    gqla_combine(dims, bufs.sel_index, 1, bufs.dec.num_splits, D_V, bufs.dec.o_part, bufs.dec.lse_part,
                 None, bufs.dec.out, bufs.dec.lse, stream)
    return bufs.dec.out.view(B, s_q, h, D_V), bufs.dec.lse.view(B, s_q, h)


def decode_step(dims, bufs: DecodeBuffers, q, w_uk, w_uv, kv, latent_cache=None,
                kv_expanded=None, k_rope=None, stream=None, fused=False):
    """One decode step through the C ABI: absorb path = absorb_query ->
    decode_absorb -> combine(W_UV); GQA path = decode_gqa -> combine, or with
    `fused` the one call gqla_decode_gqa_step."""
    if bufs.path == "gqa" and fused:
        gqla_decode_gqa_step(dims, q, kv_expanded, k_rope, kv, bufs.num_splits, bufs.o_part,
                             bufs.lse_part, bufs.out, bufs.lse, bufs.workspace, stream)
        return bufs.out, bufs.lse
    if bufs.path == "absorb":
        gqla_absorb_query(dims, q, w_uk, bufs.q_absorbed, stream)
        gqla_decode_absorb(dims, bufs.q_absorbed, latent_cache, kv, bufs.num_splits, bufs.o_part,
                           bufs.lse_part, bufs.workspace, stream)
        gqla_combine(dims, kv, bufs.s_q, bufs.num_splits, D_LATENT, bufs.o_part, bufs.lse_part,
                     w_uv, bufs.out, bufs.lse, stream)
    else:
        gqla_decode_gqa(dims, q, kv_expanded, k_rope, kv, bufs.num_splits, bufs.o_part,
                        bufs.lse_part, bufs.workspace, stream)
        gqla_combine(dims, kv, bufs.s_q, bufs.num_splits, D_V, bufs.o_part, bufs.lse_part,
                     None, bufs.out, bufs.lse, stream)
    return bufs.out, bufs.lse
