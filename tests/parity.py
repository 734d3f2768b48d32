"""Comparison of the CUDA path with the CPU oracle (test helper).

Acceptance rules for one layer call:
  * selected experts: equal as sets on every token whose oracle probability gap
    p_(K) - p_(K+1) exceeds NEAR_TIE; on near-tie tokens the CUDA selection must still
    be a valid top-K up to that gap (every chosen expert has p >= p_(K) - NEAR_TIE);
  * routing weights: |alpha_gpu - alpha_oracle| <= W_TOL for every matched expert (on
    tokens whose set differs, the oracle renormalises over the CUDA path's set);
  * output: |y_gpu - y_oracle| <= Y_TOL * RMS(y_oracle) + half_ulp_bf16(y) elementwise,
    where tokens whose CUDA selection differs are compared with the oracle output for that
    selection.  The half-ulp term is the rounding of the exact value to the bf16 output
    format itself: no bf16 number is closer than that to a value midway between two bf16
    neighbours, so without it the bound could not be met by elements beyond ~5 x RMS.
    Intermediate fp32 results (out_acc, y_sorted) are checked against the plain bound.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

NEAR_TIE = 1e-4
W_TOL = 1e-3
Y_TOL = 2e-2


@dataclasses.dataclass
class RouteReport:
    near_tie: int
    differing_sets: np.ndarray  # token ids whose CUDA set differs (all near ties)
    max_w_err: float


def half_ulp_bf16(v: np.ndarray) -> np.ndarray:
    """Half the spacing of bf16 numbers (8 significant bits) at |v|."""
    a = np.abs(np.asarray(v, np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.exp2(e - 8), 0.0)


def output_error(y_gpu_bf16: np.ndarray, y_ref: np.ndarray):
    """(max |dy|, RMS(y_ref), worst fraction of the allowed bound) for a bf16 output."""
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    d = np.abs(y_gpu_bf16 - y_ref)
    allow = Y_TOL * rms + half_ulp_bf16(np.maximum(np.abs(y_ref), np.abs(y_gpu_bf16)))
    return float(d.max()) if d.size else 0.0, rms, float((d / allow).max()) if d.size else 0.0


def check_route(orc, gpu_idx, gpu_w, gpu_counts=None, select_bias=None,
                bf16_weights=False) -> RouteReport:
    """orc: oracle.route(...) dict; gpu_*: numpy arrays.  The selection keys are the scores
    plus the selection-only bias; with bf16 weights both sides round independently, so one
    bf16 ulp of the weight is allowed on top of W_TOL."""
    o_idx, o_alpha, probs, gap = orc["idx"], orc["alpha"], orc["probs"], orc["gap"]
    T, K = o_idx.shape
    sb = None if select_bias is None else np.asarray(
        select_bias.cpu() if hasattr(select_bias, "cpu") else select_bias, np.float64)
    keys = probs if sb is None else probs + sb
    assert gpu_idx.shape == (T, K)
    assert np.all((gpu_idx >= 0) & (gpu_idx < probs.shape[1])), "index out of range"
    for t in range(T):
        assert len(set(gpu_idx[t].tolist())) == K, f"token {t}: repeated expert"
    near = gap <= NEAR_TIE
    same = np.array([set(gpu_idx[t]) == set(o_idx[t]) for t in range(T)], dtype=bool)
    bad = ~same & ~near
    assert not bad.any(), f"selection differs on non-near-tie tokens {np.nonzero(bad)[0][:10]}"
    # near-tie tokens: the CUDA choice must be a valid top-K within the tie gap
    for t in np.nonzero(~same)[0]:
        kth = keys[t, o_idx[t, K - 1]]
        chosen = keys[t, gpu_idx[t]]
        assert np.all(chosen >= kth - NEAR_TIE), f"token {t}: invalid near-tie selection"
    # weights: compare per expert; renormalise the oracle scores over the CUDA set
    sel = np.take_along_axis(probs, gpu_idx.astype(np.int64), axis=1)
    ref_w = sel / sel.sum(1, keepdims=True)
    allow = W_TOL + (2 * half_ulp_bf16(ref_w) if bf16_weights else 0.0)
    w_err = float(np.abs(gpu_w - ref_w).max()) if T else 0.0
    assert np.all(np.abs(gpu_w - ref_w) <= allow), f"routing weight error {w_err}"
    # the CUDA list is ordered by descending key
    gk = np.take_along_axis(keys, gpu_idx.astype(np.int64), axis=1)
    assert np.all(np.diff(gk, axis=1) <= 1e-6), "selection not in descending key order"
    if gpu_counts is not None:
        bc = np.bincount(gpu_idx.reshape(-1), minlength=len(gpu_counts))
        np.testing.assert_array_equal(gpu_counts, bc)
    return RouteReport(int(near.sum()), np.nonzero(~same)[0], w_err)


def compact_weights(inp, experts: np.ndarray):
    """Copy only the listed experts' weights to the host (for multi-GB layers)."""
    ex = torch.as_tensor(np.asarray(experts, np.int64), device=inp.w_gate_up.device)
    return inp.w_gate_up.index_select(0, ex).cpu(), inp.w_down.index_select(0, ex).cpu()


def oracle_outputs(orc_mod, inp, idx, alpha, tokens, shared_gate=None):
    """Oracle y for `tokens` with the given routing (idx/alpha [T,K], oracle-side)."""
    sub_idx = idx[tokens]
    uniq, inv = np.unique(sub_idx, return_inverse=True)
    gu, wd = compact_weights(inp, uniq)
    local_idx = inv.reshape(sub_idx.shape).astype(np.int32)
    x_sub = inp.x[torch.as_tensor(tokens, device=inp.x.device)].cpu()
    sg = None if shared_gate is None else np.asarray(shared_gate)[tokens]
    return orc_mod.experts(x_sub, local_idx, alpha[tokens], gu, wd, None,
                           None if inp.w_shared_gate_up is None else inp.w_shared_gate_up.cpu(),
                           None if inp.w_shared_down is None else inp.w_shared_down.cpu(), sg)


def check_layer(orc_mod, inp, y_gpu, gpu_idx, gpu_w, tokens=None, orc=None, score="softmax",
                select_bias=None, bf16_weights=False, residual=None, capacity=None):
    """Route on the oracle (all tokens), compare routing, then compare y (+ residual) on
    `tokens` (all when None); with an expert capacity C the oracle drops every assignment
    past the first C of its expert (token order) of that routing.  Returns a dict of
    measured errors."""
    cfg = inp.cfg
    if orc is None:
        orc = orc_mod.route(inp.x, inp.w_router, cfg.K, inp.logit_bias, inp.w_shared_gate,
                            score, select_bias, bf16_weights)
    rep = check_route(orc, gpu_idx, gpu_w, select_bias=select_bias, bf16_weights=bf16_weights)
    T = cfg.T
    toks = np.arange(T) if tokens is None else np.asarray(tokens)
    # forced routing: the oracle's own weights over the CUDA set for differing tokens
    idx = orc["idx"].copy()
    alpha = orc["alpha"].copy()
    for t in rep.differing_sets:
        idx[t] = gpu_idx[t]
        p = orc["probs"][t, gpu_idx[t]]
        alpha[t] = p / p.sum()
        if bf16_weights:
            alpha[t] = torch.tensor(alpha[t]).float().bfloat16().double().numpy()
    dropped = 0
    if capacity is not None:
        keep = orc_mod.capacity_keep(idx, cfg.E, capacity)
        alpha = np.where(keep, alpha, 0.0)
        dropped = int((~keep).sum())
    y_ref = oracle_outputs(orc_mod, inp, idx, alpha, toks, orc["shared_gate"])
    if residual is not None:
        y_ref = y_ref + residual[torch.as_tensor(toks, device=residual.device)].cpu().double().numpy()
    y = y_gpu[torch.as_tensor(toks, device=y_gpu.device)].float().cpu().numpy().astype(np.float64)
    err, rms, used = output_error(y, y_ref)
    assert rms > 0
    assert used <= 1.0, (f"output error {err:.3e} exceeds {Y_TOL} x RMS {rms:.3e} + half a bf16 "
                         f"ulp ({used:.2f} of the bound)")
    return dict(near_tie=rep.near_tie, differing=len(rep.differing_sets), w_err=rep.max_w_err,
                y_err=err, y_rms=rms, y_rel=err / rms, bound_used=used, dropped=dropped)
