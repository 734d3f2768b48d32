"""Closed-form cost counts of an MoE FFN layer -- part of the oracle (test infrastructure).

From "MoE 到底省了什么" (clxhxhhr.top):
  section 2:   N_e = 3 d f                        parameters of one SwiGLU expert
  section 3:   F_expert = 2 N_e sum_e t_e = 2 N_e B k      (dropless)
               R_expert = b_W N_e U                U = distinct experts read
  section 4:   F_layer  = 2 m N_s + 2 sum_e t_e N_e        (with a shared expert, m tokens)
  section 4.1: routed params per layer 3 E d f; per-token expert FLOPs 6 k d f
"""
from __future__ import annotations

from typing import Iterable


def expert_params(d: int, f: int) -> int:
    """N_e = 3 d f (gate, up and down matrices of one expert)."""
    return 3 * d * f


def expert_flops(rows_per_expert: Iterable[int], d: int, f: int) -> int:
    """F_expert = 2 N_e sum_e t_e, counted from the rows each expert actually received."""
    return 2 * expert_params(d, f) * sum(int(t) for t in rows_per_expert)


def expert_weight_bytes(distinct_experts: int, d: int, f: int, bytes_per_weight: int = 2) -> int:
    """R_expert = b_W N_e U."""
    return bytes_per_weight * expert_params(d, f) * distinct_experts


def layer_flops(rows_per_expert: Iterable[int], m: int, d: int, f: int, f_s: int) -> int:
    """F = 2 m N_s + 2 sum_e t_e N_e (shared expert of width f_s on all m tokens)."""
    return 2 * m * expert_params(d, f_s) + expert_flops(rows_per_expert, d, f)


def routed_params(E: int, d: int, f: int) -> int:
    """3 E d f: every routed expert's parameters in one layer."""
    return E * expert_params(d, f)


def flops_per_token(k: int, d: int, f: int) -> int:
    """6 k d f: expert FLOPs of one token."""
    return 2 * k * expert_params(d, f)


def distinct_experts(counts: Iterable[int]) -> int:
    """U: experts that received at least one row."""
    return sum(1 for c in counts if int(c) > 0)
