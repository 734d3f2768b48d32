"""The C ABI without a GPU: the library builds, loads, exports every entry point that
include/moe_api.h declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

import top_routing_grouped_03_b200 as moe
from top_routing_grouped_03_b200 import build as moe_build

MOE_OK, ARG, UNSUP, ALIGN, WS = 0, -1, -2, -3, -6


@pytest.fixture(scope="module")
def lib():
    moe_build.build()
    return moe.lib()


def declared_symbols():
    text = open(moe.HEADER_PATH, encoding="utf-8").read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)))


def test_header_declares_the_layer_api():
    names = declared_symbols()
    for n in ("moe_route", "moe_permute", "moe_grouped_swiglu", "moe_combine",
              "moe_layer_forward", "moe_workspace_size", "moe_read_device_status"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    raw = ctypes.CDLL(moe.LIB_PATH)
    for n in declared_symbols():
        assert hasattr(raw, n), f"{n} not exported"


def test_version_and_status_strings(lib):
    assert moe.version() >= 100
    assert moe.status_string(0) == "ok"
    assert "unsupported" in moe.status_string(UNSUP)
    assert moe.status_string(12345) == "unknown status"


def test_workspace_size(lib):
    a = moe.workspace_size(64, 2048, 256, 8, 512)
    b = moe.workspace_size(128, 2048, 256, 8, 512)
    assert 0 < a < b
    assert moe.workspace_size(64, 2048, 256, 8, 512, 512) > a
    assert a % 256 == 0
    # T*K*D bf16 gathered rows alone must fit
    assert a >= 64 * 8 * 2048 * 2
    assert moe.workspace_size(0, 2048, 256, 8, 512) > 0
    for bad in [(64, 100, 256, 8, 512), (64, 2048, 513, 8, 512), (64, 2048, 8, 9, 512),
                (64, 2048, 256, 17, 512), (64, 2048, 256, 8, 500), (-1, 2048, 256, 8, 512)]:
        assert moe.workspace_size(*bad) == 0, bad


def _fake(addr):
    return ctypes.c_void_p(addr)


def test_host_validation_returns_before_launch(lib):
    L = lib
    A = 0x10000  # aligned fake device addresses: never dereferenced by the host checks
    ws = _fake(A)
    # moe_route
    assert L.moe_route(_fake(A), _fake(A), None, None, 4, 256, 16, 17, _fake(A), _fake(A),
                       _fake(A), None, ws, 1 << 30, None) == UNSUP
    assert L.moe_route(_fake(A + 2), _fake(A), None, None, 4, 256, 16, 4, _fake(A), _fake(A),
                       _fake(A), None, ws, 1 << 30, None) == ALIGN
    assert L.moe_route(None, _fake(A), None, None, 4, 256, 16, 4, _fake(A), _fake(A),
                       _fake(A), None, ws, 1 << 30, None) == ARG
    assert L.moe_route(_fake(A), _fake(A), None, _fake(A), 4, 256, 16, 4, _fake(A), _fake(A),
                       _fake(A), None, ws, 1 << 30, None) == ARG  # gate vector without output
    assert L.moe_route(_fake(A), _fake(A), None, None, 4, 256, 16, 4, _fake(A), _fake(A),
                       _fake(A), None, ws, 16, None) == WS
    # moe_permute
    assert L.moe_permute(_fake(A), None, None, 4, 16, 4, _fake(A), _fake(A), None, _fake(A),
                         None, None) == ARG
    assert L.moe_permute(_fake(A), None, _fake(A), 4, 600, 4, _fake(A), _fake(A), None,
                         _fake(A), None, None) == UNSUP
    # moe_grouped_swiglu
    assert L.moe_grouped_swiglu(_fake(A), _fake(A), _fake(A), None, _fake(A), _fake(A), 4, 16,
                                256, 16, 128, None, None, ws, 1 << 30, None) == ARG
    assert L.moe_grouped_swiglu(_fake(A), None, _fake(A), None, _fake(A), _fake(A), 4, 16,
                                256, 16, 128, None, _fake(A), ws, 1 << 30, None) == ARG
    assert L.moe_grouped_swiglu(_fake(A), _fake(A), _fake(A), None, _fake(A + 8), _fake(A), 4,
                                16, 256, 16, 128, None, _fake(A), ws, 1 << 30, None) == ALIGN
    assert L.moe_grouped_swiglu(_fake(A), _fake(A), _fake(A), None, _fake(A), _fake(A), 4, 16,
                                256, 16, 128, None, _fake(A), ws, 100, None) == WS
    # moe_combine
    assert L.moe_combine(None, None, None, None, None, None, 4, 256, 4, None, None) == ARG
    assert L.moe_combine(None, _fake(A), None, None, None, None, 4, 256, 4, _fake(A), None) == ARG
    assert L.moe_combine(None, None, None, None, _fake(A), None, 4, 256, 4, _fake(A), None) == ARG
    # moe_layer_forward
    assert L.moe_layer_forward(None, _fake(A), ws, 1 << 30, None) == ARG
    p = moe.LayerParams(_fake(A), _fake(A), None, _fake(A), _fake(A), None, None, None,
                        64, 2048, 256, 8, 512, 0, 0, None, None, None)
    assert L.moe_layer_forward(ctypes.byref(p), _fake(A), ws, 100, None) == WS
    assert L.moe_layer_forward(ctypes.byref(p), _fake(A), _fake(A + 16), 1 << 40, None) == ALIGN
    p.f_s = 512  # shared width without shared weights
    assert L.moe_layer_forward(ctypes.byref(p), _fake(A), ws, 1 << 40, None) == ARG
    p.f_s, p.D = 0, 2000
    assert L.moe_layer_forward(ctypes.byref(p), _fake(A), ws, 1 << 40, None) == UNSUP
    p.D = 2048
    for bad in (-1.0, float("nan"), float("inf")):  # capacity factor
        p.capacity_factor = bad
        assert L.moe_layer_forward(ctypes.byref(p), _fake(A), ws, 1 << 40, None) == ARG
    p.capacity_factor, p.min_capacity = 1.25, -1
    assert L.moe_layer_forward(ctypes.byref(p), _fake(A), ws, 1 << 40, None) == ARG
    # moe_permute_ex: same checks as moe_permute
    assert L.moe_permute_ex(_fake(A), None, None, 4, 16, 4, 3, _fake(A), _fake(A), None,
                            _fake(A), None, None) == ARG
    assert L.moe_read_device_status(None, None) == WS


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(moe, "_lib", None)
    monkeypatch.setattr(moe, "LIB_PATH", str(tmp_path / "nope.so"))
    with pytest.raises(ImportError):
        moe.lib()


def test_python_binding_needs_cuda_tensors(lib):
    import torch
    with pytest.raises(ValueError):
        moe._p(torch.zeros(4))


def test_python_binding_checks_element_types(lib):
    """A tensor of another element type than the C ABI reads at that pointer is refused
    (checked before anything touches the device)."""
    import torch
    with pytest.raises(TypeError):
        moe._p(torch.zeros(4), moe.BF16)
    with pytest.raises(TypeError):
        moe._p(torch.zeros(4, dtype=torch.int64), moe.I32)
    with pytest.raises(TypeError):
        moe.combine(2, 128, 1, out=torch.empty((2, 128), dtype=torch.bfloat16),
                    out_acc=torch.zeros((2, 128), dtype=torch.float64))


def test_expert_capacity_matches_oracle(lib, oracle_mod):
    """The layer's capacity C (host arithmetic of the library) equals the oracle's for the
    same float capacity factor, over sizes, factors and minimums."""
    import numpy as np
    for T, K, E in [(64, 8, 256), (8192, 8, 128), (4096, 10, 512), (1, 8, 128), (1000, 2, 3),
                    (7, 1, 7), (300, 6, 128), (0, 4, 16)]:
        for cf in (0.5, 0.75, 1.0, 1.1, 1.25, 2.0, 3.3):
            cf32 = float(np.float32(cf))
            for mn in (0, 4, 1000):
                assert moe.expert_capacity(T, K, E, cf, mn) == \
                    oracle_mod.expert_capacity(T, K, E, cf32, mn), (T, K, E, cf, mn)
    assert moe.expert_capacity(64, 8, 256, 0.0) == -1
    assert moe.expert_capacity(64, 8, 256, -1.0) == -1
    assert moe.expert_capacity(64, 8, 0, 1.25) == -1


def _plan(L, T, D, E, K, f, f_s=0, flags=0):
    A = 0x10000
    p = moe.LayerParams()
    p.x, p.w_router, p.w_gate_up, p.w_down = A, A, A, A
    if f_s:
        p.w_shared_gate, p.w_shared_gate_up, p.w_shared_down = A, A, A
    p.T, p.D, p.E, p.K, p.f, p.f_s, p.flags = T, D, E, K, f, f_s, flags
    mask, n = ctypes.c_uint(0), ctypes.c_int(0)
    assert L.moe_layer_plan(ctypes.byref(p), ctypes.byref(mask), ctypes.byref(n)) == MOE_OK
    steps = {name for i, name in enumerate(moe.STEP_EVENT_NAMES) if mask.value >> i & 1}
    return steps, n.value


def test_layer_plan_names_the_launched_steps(lib):
    """moe_layer_plan (host only): which steps launch kernels and how many, per regime."""
    # decode: router, one-CTA permutation, gate_up, down (which also writes the output)
    assert _plan(lib, 64, 2048, 256, 8, 512) == ({"router", "permute", "gate_up", "down"}, 4)
    # fixed-order combine: one more kernel
    assert _plan(lib, 64, 2048, 256, 8, 512, flags=1) == (
        {"router", "permute", "gate_up", "down", "combine"}, 5)
    # fine-grained + shared: tensor-core router (logits GEMM + selection), chunked
    # permutation (histograms + scatter), the shared expert's two launches (the last one
    # writes the output)
    assert _plan(lib, 4096, 4096, 512, 10, 1024, 1024) == (
        {"router", "permute", "gate_up", "down", "shared"}, 8)
    assert _plan(lib, 4096, 4096, 512, 10, 1024, 512) == (
        {"router", "permute", "gate_up", "down", "shared"}, 8)
    # prefill: CTA pairs, whose gate_up first copies the token rows into expert order and
    # whose down writes weighted bf16 rows that a fixed-order combine sums
    assert _plan(lib, 8192, 4096, 128, 8, 1536) == (
        {"router", "permute", "gate_up", "down", "combine"}, 8)
    # E > 256 with few tokens: the permutation is a launch of its own
    assert _plan(lib, 70, 256, 512, 16, 128) == ({"router", "permute", "gate_up", "down"}, 4)
    assert _plan(lib, 0, 256, 16, 4, 128) == (set(), 0)
