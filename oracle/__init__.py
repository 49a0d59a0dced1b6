"""fp64 CPU oracle for GQLA decode attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never calls it and
shares no code with it; the only thing both sides share is the seeded input
generator, which holds none of the method's arithmetic.

The arithmetic lives in ``gqla_oracle.c`` (plain C, fp64, OpenMP over
independent (sequence, group) units); this module compiles it with gcc on first
use and marshals numpy arrays into it.  ``roofline.py`` holds the closed-form
cache-size / arithmetic-intensity / roofline-time model the pages print.

Sources, by page and section:
  * GQLA, paperlayer.ai summary (arXiv:2605.15250v3): sec. 3 Methods
    (architecture, the two equivalent decoding paths), sec. 4 Roofline
    Analysis (intensities, step times), sec. 5 Experiments (576 elements per
    token, 2*g*d_h + d_R for the per-group path).
  * GQLA, gist.science technical summary: sec. 2 Methodik (group-indexed
    W_UK / W_UV, the two paths).
  * GQLA, pwwt.cn article: sec. 3 (4224 B / 1152 B per token, 16 heads per
    group), sec. 4 (LLaMA-3-8B 2048-element GQA cache, 28.125 %), sec. 5
    (sparse attention: each new token attends to a selected subset).

``decode_sparse`` is numpy (fp64, library matmuls), not C: the sparse variant
is small and its per-query selection makes the C unit loop a poor fit.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gqla_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libgqla_oracle.so")
_lock = threading.Lock()
_lib = None

D_LATENT, D_ROPE, D_NOPE, D_V = 512, 64, 128, 128
D_QK = D_NOPE + D_ROPE
D_ROW = D_LATENT + D_ROPE


def build(force: bool = False) -> str:
    """Compile gqla_oracle.c into a shared library next to it (gcc, -O2, OpenMP).

    No -ffast-math: the fp32 expansion reference relies on IEEE fmaf.
    """
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
               "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            P = ctypes.c_void_p
            I = ctypes.c_int
            lib.gqla_oracle_decode.argtypes = [I, I, I, I, I, I, P, P, P, P, P, P,
                                               ctypes.c_double, P, I, P, P]
            lib.gqla_oracle_decode.restype = I
            lib.gqla_oracle_decode_absorbed.argtypes = [I, I, I, I, I, I, P, P, P, P, P, P,
                                                        ctypes.c_double, P, P]
            lib.gqla_oracle_decode_absorbed.restype = I
            lib.gqla_oracle_absorb_query.argtypes = [I, I, I, P, P, P]
            lib.gqla_oracle_absorb_query.restype = I
            lib.gqla_oracle_expand_f64.argtypes = [ctypes.c_int64, I, P, P, P, P, P]
            lib.gqla_oracle_expand_f64.restype = None
            lib.gqla_oracle_expand_f32seq.argtypes = [ctypes.c_int64, I, P, P, P, P, P]
            lib.gqla_oracle_expand_f32seq.restype = None
            lib.gqla_oracle_bf16_rne.argtypes = [ctypes.c_float]
            lib.gqla_oracle_bf16_rne.restype = ctypes.c_uint16
            lib.gqla_oracle_num_threads.argtypes = []
            lib.gqla_oracle_num_threads.restype = I
            _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    a = _to_numpy(a)
    return np.ascontiguousarray(a, dtype=np.float64)


def _f32(a) -> np.ndarray:
    a = _to_numpy(a)
    return np.ascontiguousarray(a, dtype=np.float32)


def _i32(a) -> np.ndarray:
    a = _to_numpy(a)
    return np.ascontiguousarray(a, dtype=np.int32)


def _to_numpy(a):
    if hasattr(a, "detach"):  # torch tensor (bf16 is widened exactly to fp32 first)
        import torch
        t = a.detach().cpu()
        if t.dtype in (torch.bfloat16, torch.float16):
            t = t.float()
        return t.numpy()
    return np.asarray(a)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return _load().gqla_oracle_num_threads()


def default_scale() -> float:
    """1/sqrt(d_nope + d_R) = 1/sqrt(192): the MLA convention (a reading; the pages are silent)."""
    return 1.0 / np.sqrt(D_QK)


def decode(q, cache, page_table, seqlens, w_uk, w_uv, num_groups, page_size=64,
           scale=None, units=None):
    """Un-absorbed (GQA-path) definition of GQLA decode attention.

    q [B][s_q][h][192], cache [pages][page_size][576], page_table [B][max_pages],
    seqlens [B], w_uk / w_uv [g][512][128].  Returns (out [B][s_q][h][128],
    lse [B][s_q][h]) in fp64.  ``units``: optional list of (b, group) pairs to
    compute; other entries are NaN.
    """
    lib = _load()
    q = _f64(q); cache = _f64(cache); pt = _i32(page_table); sl = _i32(seqlens)
    wk = _f64(w_uk); wv = _f64(w_uv)
    B, s_q, h, dqk = q.shape
    assert dqk == D_QK and cache.shape[-1] == D_ROW and cache.shape[1] == page_size
    assert wk.shape == (num_groups, D_LATENT, D_NOPE) and wv.shape == (num_groups, D_LATENT, D_V)
    out = np.full((B, s_q, h, D_V), np.nan)
    lse = np.full((B, s_q, h), np.nan)
    if units is None:
        u_ptr, n_units = None, 0
    else:
        u = np.ascontiguousarray(np.asarray(units, dtype=np.int32).reshape(-1, 2))
        u_ptr, n_units = _ptr(u), u.shape[0]
    rc = lib.gqla_oracle_decode(B, s_q, h, num_groups, page_size, pt.shape[1], _ptr(q),
                                _ptr(cache), _ptr(pt), _ptr(sl), _ptr(wk), _ptr(wv),
                                float(default_scale() if scale is None else scale),
                                u_ptr, n_units, _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("gqla_oracle_decode: bad arguments")
    return out, lse


def decode_sparse(q, cache, page_table, seqlens, w_uk, w_uv, num_groups, topk_idx, page_size=64,
                  scale=None):
    """Sparse GQLA (paperlayer.ai summary, sec. 2 "Sparse GQLA"; pwwt.cn article,
    sec. 5): query token s of sequence b attends only to the token positions in
    topk_idx[b][s] (the same set for every head; -1 = unused entry), with the
    un-absorbed definition of ``decode`` otherwise: K = [c W_UK_g | k^R],
    V = c W_UV_g, softmax of q.K * scale over the set, out = sum p V.
    Positions must be visible (0 <= t <= L_b - s_q + s).  Returns
    (out [B][s_q][h][128], lse [B][s_q][h]) in fp64; an empty set gives out = 0
    and lse = -inf.
    """
    q = _f64(q); pages = _f64(cache); pt = _i32(page_table); sl = _i32(seqlens)
    wk = _f64(w_uk); wv = _f64(w_uv); idx = np.asarray(_to_numpy(topk_idx), dtype=np.int64)
    B, s_q, h, dqk = q.shape
    assert dqk == D_QK and pages.shape[1] == page_size and pages.shape[-1] == D_ROW
    G = h // num_groups
    sc = default_scale() if scale is None else scale
    out = np.zeros((B, s_q, h, D_V))
    lse = np.full((B, s_q, h), -np.inf)
    for b in range(B):
        for s in range(s_q):
            t = idx[b, s][idx[b, s] >= 0]
            if t.size == 0:
                continue
            assert t.max() <= sl[b] - s_q + s, "a selected token is not visible"
            rows = pages[pt[b, t // page_size], t % page_size]     # [n][576]
            c, kr = rows[:, :D_LATENT], rows[:, D_LATENT:]
            for g in range(num_groups):
                K = np.concatenate([c @ wk[g], kr], axis=1)       # [n][192]
                V = c @ wv[g]                                      # [n][128]
                x = (q[b, s, g * G:(g + 1) * G] @ K.T) * sc        # [G][n]
                m = x.max(axis=1, keepdims=True)
                e = np.exp(x - m)
                l = e.sum(axis=1, keepdims=True)
                out[b, s, g * G:(g + 1) * G] = (e / l) @ V
                lse[b, s, g * G:(g + 1) * G] = (m + np.log(l))[:, 0]
    return out, lse


def decode_absorbed(q, cache, page_table, seqlens, w_uk, w_uv, num_groups, page_size=64,
                    scale=None):
    """MQA-absorb form of the same attention (independent code path, fp64)."""
    lib = _load()
    q = _f64(q); cache = _f64(cache); pt = _i32(page_table); sl = _i32(seqlens)
    wk = _f64(w_uk); wv = _f64(w_uv)
    B, s_q, h, _ = q.shape
    out = np.zeros((B, s_q, h, D_V))
    lse = np.zeros((B, s_q, h))
    rc = lib.gqla_oracle_decode_absorbed(B, s_q, h, num_groups, page_size, pt.shape[1],
                                         _ptr(q), _ptr(cache), _ptr(pt), _ptr(sl), _ptr(wk),
                                         _ptr(wv),
                                         float(default_scale() if scale is None else scale),
                                         _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("gqla_oracle_decode_absorbed: bad arguments")
    return out, lse


def absorb_query(q, w_uk, num_groups):
    """q~ = [W_UK_{g(h)} q^C ; q^R] for every row of q [..., h, 192] -> [..., h, 576]."""
    lib = _load()
    q = _f64(q); wk = _f64(w_uk)
    h = q.shape[-2]
    rows = int(np.prod(q.shape[:-1]))
    qa = np.zeros(q.shape[:-1] + (D_ROW,))
    rc = lib.gqla_oracle_absorb_query(rows, h, num_groups, _ptr(q), _ptr(wk), _ptr(qa))
    if rc != 0:
        raise ValueError("gqla_oracle_absorb_query: bad arguments")
    return qa


def expand_f64(latent, w_uk, w_uv):
    """Exact expansion: returns (kv [g][n][256] = [c W_UK_g | c W_UV_g], k_rope [n][64])."""
    lib = _load()
    lat = _f64(latent).reshape(-1, D_ROW); wk = _f64(w_uk); wv = _f64(w_uv)
    n, g = lat.shape[0], wk.shape[0]
    kv = np.zeros((g, n, D_NOPE + D_V))
    kr = np.zeros((n, D_ROPE))
    lib.gqla_oracle_expand_f64(n, g, _ptr(lat), _ptr(wk), _ptr(wv), _ptr(kv), _ptr(kr))
    return kv, kr


def expand_f32seq_bits(latent, w_uk, w_uv):
    """Expansion with the fixed fp32 rounding order; returns bf16 bit patterns (uint16)."""
    lib = _load()
    lat = _f32(latent).reshape(-1, D_ROW); wk = _f32(w_uk); wv = _f32(w_uv)
    n, g = lat.shape[0], wk.shape[0]
    kv = np.zeros((g, n, D_NOPE + D_V), dtype=np.uint16)
    kr = np.zeros((n, D_ROPE), dtype=np.uint16)
    lib.gqla_oracle_expand_f32seq(n, g, _ptr(lat), _ptr(wk), _ptr(wv), _ptr(kv), _ptr(kr))
    return kv, kr


def bf16_rne_bits(x: float) -> int:
    """bf16 bit pattern of float32(x) rounded to nearest, ties to even."""
    return int(_load().gqla_oracle_bf16_rne(float(x)))
