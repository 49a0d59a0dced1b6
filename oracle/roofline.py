"""Closed-form cache-size, arithmetic-intensity and roofline model of GQLA decode.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

This restates the analytical model the pages use (GQLA, paperlayer.ai summary,
sec. 4 Roofline Analysis; pwwt.cn article, sec. 2, 3 and 7):

  * attainable throughput = min(I * BW, FLOPs_max), ridge I* = FLOPs_max / BW;
  * cache bytes per token per layer: absorb path (r_kv + d_R) * 2 B,
    GQA path (2 * g * d_h + d_R) * 2 B (paperlayer.ai sec. 5, "Conversion setup");
  * decode FLOPs per cached token: every query row (h_q * s_q of them) takes a
    dot product over the key width and an accumulate over the value width,
    2 * h_q * s_q * (d_key + d_value); the cache is read once per step whatever
    s_q is (paperlayer.ai sec. 4, "MQA-absorb path").

The pages never state the context length or the peak figures behind their step
times.  The reading that reproduces every printed number is: one sequence, one
layer, L = 8192 cached tokens, H100 = 3.35 TB/s and 989 TFLOP/s dense bf16,
H20 = 4.0 TB/s and 148 TFLOP/s (the H20 pair is printed in the pwwt.cn article,
sec. 2).  Those assumptions live in ``PAPER_HW`` and ``PAPER_CONTEXT``.
"""
from __future__ import annotations

BF16_BYTES = 2
D_LATENT, D_ROPE, D_HEAD = 512, 64, 128

PAPER_HW = {
    "H100": {"bw": 3.35e12, "flops": 989e12},
    "H20": {"bw": 4.0e12, "flops": 148e12},
}
PAPER_CONTEXT = 8192


def cache_elems_per_token(path: str, g: int = 8) -> int:
    if path == "absorb":
        return D_LATENT + D_ROPE
    if path == "gqa":
        return 2 * g * D_HEAD + D_ROPE
    if path == "llama_gqa":  # original LLaMA-3-8B cache: 8 KV groups x 128 x (K, V)
        return 2 * 8 * D_HEAD
    raise ValueError(path)


def cache_bytes_per_token(path: str, g: int = 8) -> int:
    return BF16_BYTES * cache_elems_per_token(path, g)


def flops_per_token(path: str, h: int, s_q: int) -> float:
    if path == "absorb":  # scores over 576, accumulate over the 512-d latent
        return 2.0 * h * s_q * ((D_LATENT + D_ROPE) + D_LATENT)
    if path == "gqa":  # scores over 192, accumulate over the 128-d value
        return 2.0 * h * s_q * ((D_HEAD + D_ROPE) + D_HEAD)
    raise ValueError(path)


def intensity(path: str, h: int = 128, s_q: int = 1, g: int = 8) -> float:
    """FLOPs per byte of cache read."""
    return flops_per_token(path, h, s_q) / cache_bytes_per_token(path, g)


def ridge(hw: str) -> float:
    return PAPER_HW[hw]["flops"] / PAPER_HW[hw]["bw"]


def step_time_s(path: str, hw: str, h: int = 128, s_q: int = 1, g: int = 8,
                context: int = PAPER_CONTEXT) -> float:
    """Roofline step time: the slower of moving the cache and doing the FLOPs."""
    p = PAPER_HW[hw]
    t_mem = context * cache_bytes_per_token(path, g) / p["bw"]
    t_cmp = context * flops_per_token(path, h, s_q) / p["flops"]
    return max(t_mem, t_cmp)


def tokens_per_s(path: str, hw: str, h: int = 128, s_q: int = 1, g: int = 8,
                 context: int = PAPER_CONTEXT) -> float:
    """Generated tokens per second: s_q tokens per decode step."""
    return s_q / step_time_s(path, hw, h, s_q, g, context)
