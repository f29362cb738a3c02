"""Algorithmic bytes and FLOPs of one decode step (the roofline model of the hot path).

TEST INFRASTRUCTURE (part of the oracle package; see its header). The bench computes its own
counts; a CPU test checks them against these closed forms.

Source: « Résumé technique : GQLA … », « 1. Énoncé du problème » and « Chemin MQA-Absorbé »
(≈242 FLOPs per byte for the absorbed path at s_q = 1, ridge ≈295 on H100 and ≈37 on H20), and
« Chemin GQA » / « Sélection du chemin » (g and s_q move the grouped path's intensity).

Counting rules:
  * absorbed path, per cached position and query token: the score contraction over d_c + d_r and
    the P·c contraction over d_c, i.e. 2·H·(2·d_c + d_r) FLOPs; the cache row (d_c + d_r values)
    is read once per step whatever s_q is.
  * GQA path, per position and query token: 2·H·(D + d_r) + 2·H·d_v FLOPs; the row holds
    2·g·D + d_r values (K and V of g groups plus the RoPE key).
"""
from __future__ import annotations


def absorbed_flops_per_position(H: int, d_c: int, d_r: int, s_q: int = 1) -> int:
    return 2 * H * (2 * d_c + d_r) * s_q


def absorbed_bytes_per_position(d_c: int, d_r: int, bytes_per_value: int = 2) -> int:
    return (d_c + d_r) * bytes_per_value


def absorbed_intensity(H: int, d_c: int, d_r: int, s_q: int = 1, bytes_per_value: int = 2) -> float:
    return absorbed_flops_per_position(H, d_c, d_r, s_q) / absorbed_bytes_per_position(d_c, d_r, bytes_per_value)


def gqa_flops_per_position(H: int, D: int, d_r: int, d_v: int, s_q: int = 1) -> int:
    return (2 * H * (D + d_r) + 2 * H * d_v) * s_q


def gqa_bytes_per_position(g: int, D: int, d_r: int, bytes_per_value: int = 2) -> int:
    return (2 * g * D + d_r) * bytes_per_value


def gqa_intensity(H: int, g: int, D: int, d_r: int, d_v: int, s_q: int = 1, bytes_per_value: int = 2) -> float:
    return gqa_flops_per_position(H, D, d_r, d_v, s_q) / gqa_bytes_per_position(g, D, d_r, bytes_per_value)


def ridge(flops_per_s: float, bytes_per_s: float) -> float:
    return flops_per_s / bytes_per_s


def decode_step_counts(H, d_c, d_r, d_v, seqlens, s_q=1, bytes_per_value=2):
    """(bytes, flops) of the absorbed decode kernel for one step.

    bytes: every cached row once, plus q_abs in and o_lat (storage type) and lse (fp32) out.
    flops: 2·H·(2·d_c + d_r) per visible (position, query token) pair; the causal triangle among
    the s_q new tokens is not counted.
    """
    total_pos = int(sum(int(L) for L in seqlens))
    B = len(seqlens)
    row = (d_c + d_r) * bytes_per_value
    bytes_ = total_pos * row + B * s_q * H * ((d_c + d_r) + d_c) * bytes_per_value + B * s_q * H * 4
    visible = sum(int(L) * s_q - s_q * (s_q - 1) // 2 for L in seqlens)
    flops = 2 * H * (2 * d_c + d_r) * visible
    return bytes_, flops
