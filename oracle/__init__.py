"""CPU oracle for the top-k MoE SwiGLU layer forward -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may
import this package.  The product library never links or calls it, and it imports
nothing from the product package.

``moe_oracle.c`` holds the arithmetic (fp64, plain loops, one function per step of the
method, each citing its passage); this module compiles it with gcc, loads it with
ctypes and marshals numpy arrays.  ``accounting`` holds the closed-form FLOP and byte
counts of "MoE 到底省了什么" (clxhxhhr.top), sections 2-4.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

from . import accounting  # noqa: F401  (re-export)

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fopenmp", "-shared", "-fPIC",
                               "-std=c11", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        # ORACLE_LIB lets the mutation test point the pins at a deliberately broken build.
        alt = os.environ.get("ORACLE_LIB")
        lib = ctypes.CDLL(alt if alt else build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.oracle_route.argtypes = [P, P, P, P, I, I, I, I, P, P, P, P, P]
        lib.oracle_route_ex.argtypes = [P, P, P, P, I, I, I, I, I, P, I, P, P, P, P, P]
        lib.oracle_route_ex.restype = ctypes.c_int
        lib.oracle_experts.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, P, I, P]
        lib.oracle_dense_masked.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, P]
        lib.oracle_permute.argtypes = [P, I, I, I, P, P, P, P, P]
        lib.oracle_expert_capacity.argtypes = [I, I, I, ctypes.c_double, I]
        lib.oracle_expert_capacity.restype = ctypes.c_longlong
        lib.oracle_capacity_keep.argtypes = [P, I, I, I, ctypes.c_longlong, P]
        lib.oracle_capacity_keep.restype = ctypes.c_int
        for fn in (lib.oracle_route, lib.oracle_experts, lib.oracle_dense_masked,
                   lib.oracle_permute):
            fn.restype = ctypes.c_int
        _lib = lib
    return _lib


def bits(t) -> np.ndarray:
    """bf16 tensor (torch) or uint16 array -> contiguous uint16 numpy array of its bits."""
    if isinstance(t, np.ndarray):
        assert t.dtype == np.uint16
        return np.ascontiguousarray(t)
    import torch
    assert t.dtype == torch.bfloat16
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_to_f64(t) -> np.ndarray:
    """Exact widening of bf16 bits to float64 (for tests that need the values)."""
    b = bits(t).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f64_vec(v):
    if v is None:
        return None
    return np.ascontiguousarray(np.asarray(v.cpu() if hasattr(v, "cpu") else v, dtype=np.float64))


def route(x, w_router, K: int, logit_bias=None, w_shared_gate=None, score: str = "softmax",
          select_bias=None, bf16_weights: bool = False):
    """Router: returns dict(idx [T,K] int32, alpha [T,K] f64, probs [T,E] f64 (the scores:
    softmax probabilities or sigmoid affinities), gap [T] f64 (of the selection keys),
    shared_gate [T] f64 or None)."""
    xb, wb = bits(x), bits(w_router)
    T, D = xb.shape
    E = wb.shape[0]
    bias = _f64_vec(logit_bias)
    sbias = _f64_vec(select_bias)
    mode = {"softmax": 0, "sigmoid": 1}[score]
    sg = None if w_shared_gate is None else bits(w_shared_gate)
    idx = np.zeros((T, K), np.int32)
    alpha = np.zeros((T, K), np.float64)
    probs = np.zeros((T, E), np.float64)
    gap = np.zeros((T,), np.float64)
    sgate = np.zeros((T,), np.float64) if sg is not None else None
    rc = _load().oracle_route_ex(_ptr(xb), _ptr(wb), _ptr(bias), _ptr(sg), T, D, E, K, mode,
                                 _ptr(sbias), int(bool(bf16_weights)), _ptr(idx), _ptr(alpha),
                                 _ptr(probs), _ptr(gap), _ptr(sgate))
    if rc != 0:
        raise ValueError(f"oracle_route failed ({rc})")
    return dict(idx=idx, alpha=alpha, probs=probs, gap=gap, shared_gate=sgate)


def experts(x, idx, alpha, w_gate_up, w_down, tokens=None, w_shared_gate_up=None,
            w_shared_down=None, shared_gate=None):
    """Sparse layer output y [ntok, D] (f64) for the listed tokens (all when None)."""
    xb = bits(x)
    T, D = xb.shape
    gu, wd = bits(w_gate_up), bits(w_down)
    E, twof, _ = gu.shape
    f = twof // 2
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    alpha = np.ascontiguousarray(alpha, dtype=np.float64)
    K = idx.shape[1]
    tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int32)
    ntok = T if tok is None else len(tok)
    sgu = None if w_shared_gate_up is None else bits(w_shared_gate_up)
    sd = None if w_shared_down is None else bits(w_shared_down)
    sgt = None if shared_gate is None else np.ascontiguousarray(shared_gate, dtype=np.float64)
    f_s = 0 if sgu is None else sgu.shape[0] // 2
    y = np.zeros((ntok, D), np.float64)
    rc = _load().oracle_experts(_ptr(xb), _ptr(idx), _ptr(alpha), _ptr(gu), _ptr(wd),
                                _ptr(sgu), _ptr(sd), _ptr(sgt), D, E, K, f, f_s,
                                _ptr(tok), ntok, _ptr(y))
    if rc != 0:
        raise ValueError(f"oracle_experts failed ({rc})")
    return y


def dense_masked(x, dense_alpha, w_gate_up, w_down, w_shared_gate_up=None,
                 w_shared_down=None, shared_gate=None):
    """Brute force: all E experts on all tokens, weighted by dense_alpha [T,E]."""
    xb = bits(x)
    T, D = xb.shape
    gu, wd = bits(w_gate_up), bits(w_down)
    E, twof, _ = gu.shape
    f = twof // 2
    da = np.ascontiguousarray(dense_alpha, dtype=np.float64)
    sgu = None if w_shared_gate_up is None else bits(w_shared_gate_up)
    sd = None if w_shared_down is None else bits(w_shared_down)
    sgt = None if shared_gate is None else np.ascontiguousarray(shared_gate, dtype=np.float64)
    f_s = 0 if sgu is None else sgu.shape[0] // 2
    y = np.zeros((T, D), np.float64)
    rc = _load().oracle_dense_masked(_ptr(xb), _ptr(da), _ptr(gu), _ptr(wd), _ptr(sgu),
                                     _ptr(sd), _ptr(sgt), T, D, E, f, f_s, _ptr(y))
    if rc != 0:
        raise ValueError(f"oracle_dense_masked failed ({rc})")
    return y


def permute(idx, E: int):
    """Group (token, slot) pairs by expert, tokens ascending within a group."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, K = idx.shape
    counts = np.zeros((E,), np.int32)
    offsets = np.zeros((E + 1,), np.int32)
    sorted_token = np.zeros((T * K,), np.int32)
    sorted_slot = np.zeros((T * K,), np.int32)
    slot_to_row = np.zeros((T * K,), np.int32)
    rc = _load().oracle_permute(_ptr(idx), T, E, K, _ptr(counts), _ptr(offsets),
                                _ptr(sorted_token), _ptr(sorted_slot), _ptr(slot_to_row))
    if rc != 0:
        raise ValueError(f"oracle_permute failed ({rc})")
    return dict(counts=counts, offsets=offsets, sorted_token=sorted_token,
                sorted_slot=sorted_slot, slot_to_row=slot_to_row)


def expert_capacity(T: int, K: int, E: int, capacity_factor: float, min_capacity: int = 0) -> int:
    """Assignments an expert may take: max(min_capacity, ceil(capacity_factor*T*K/E))
    ("1.6 混合专家（MoE）", expert capacity and token dropping)."""
    c = _load().oracle_expert_capacity(T, K, E, float(capacity_factor), int(min_capacity))
    if c < 0:
        raise ValueError("oracle_expert_capacity: bad arguments")
    return int(c)


def capacity_keep(idx, E: int, C: int) -> np.ndarray:
    """bool [T, K]: the assignment is among the first C of its expert in token order."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, K = idx.shape
    keep = np.zeros((T * K,), np.uint8)
    rc = _load().oracle_capacity_keep(_ptr(idx), T, K, E, int(C), _ptr(keep))
    if rc != 0:
        raise ValueError(f"oracle_capacity_keep failed ({rc})")
    return keep.reshape(T, K).astype(bool)


def layer(inp, tokens=None, score: str = "softmax", select_bias=None, bf16_weights=False,
          residual=None, capacity=None):
    """Whole layer for a ``workloads.LayerInputs``: route every token, then the sparse
    expert sum for ``tokens`` (all when None), plus the residual h (bf16 [T, D]) when given
    ("MoE", section 4: h_out = h + y).  With ``capacity`` = C, each expert keeps only its
    first C assignments in token order and the dropped ones contribute nothing.
    Returns (route dict, y [ntok, D])."""
    r = route(inp.x, inp.w_router, inp.cfg.K, inp.logit_bias, inp.w_shared_gate, score,
              select_bias, bf16_weights)
    alpha = r["alpha"]
    if capacity is not None:
        r["keep"] = capacity_keep(r["idx"], inp.cfg.E, capacity)
        alpha = np.where(r["keep"], alpha, 0.0)
    y = experts(inp.x, r["idx"], alpha, inp.w_gate_up, inp.w_down, tokens,
                inp.w_shared_gate_up, inp.w_shared_down, r["shared_gate"])
    if residual is not None:
        h = bf16_to_f64(residual)
        y = y + (h if tokens is None else h[np.asarray(tokens)])
    return r, y
