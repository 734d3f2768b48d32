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
