"""top_routing_grouped_03_b200 -- one top-k MoE SwiGLU FFN layer forward on a B200.

A thin ctypes binding over ``libmoe_b200.so`` (C ABI in ``include/moe_api.h``).  Every
step of the layer runs in the library's sm_100a kernels; this module only allocates
tensors with PyTorch, passes their device pointers and the current CUDA stream, and turns
status codes into exceptions.  There is no fallback: without the built library (or on a
machine without a CUDA device) the calls raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "moe_api.h")

MOE_FLAG_DETERMINISTIC = 1
MOE_FLAG_BF16_WEIGHTS = 2
SCORES = {"softmax": 0, "sigmoid": 1}

_lib = None


class MoEError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {status_string(code)} ({code})")


class LayerParams(ctypes.Structure):
    _fields_ = [
        ("x", ctypes.c_void_p), ("w_router", ctypes.c_void_p), ("logit_bias", ctypes.c_void_p),
        ("w_gate_up", ctypes.c_void_p), ("w_down", ctypes.c_void_p),
        ("w_shared_gate", ctypes.c_void_p), ("w_shared_gate_up", ctypes.c_void_p),
        ("w_shared_down", ctypes.c_void_p),
        ("T", ctypes.c_int), ("D", ctypes.c_int), ("E", ctypes.c_int), ("K", ctypes.c_int),
        ("f", ctypes.c_int), ("f_s", ctypes.c_int), ("flags", ctypes.c_uint),
        ("topk_idx_out", ctypes.c_void_p), ("topk_w_out", ctypes.c_void_p),
        ("expert_counts_out", ctypes.c_void_p), ("step_events", ctypes.c_void_p),
        ("score_mode", ctypes.c_int), ("select_bias", ctypes.c_void_p),
        ("residual", ctypes.c_void_p),
        ("capacity_factor", ctypes.c_float), ("min_capacity", ctypes.c_int),
    ]


# Step boundaries recorded by moe_layer_forward when step_events is given.
STEP_EVENT_NAMES = ("start", "router", "permute", "gate_up", "down", "shared", "combine",
                    "end")
NUM_STEP_EVENTS = len(STEP_EVENT_NAMES)


def lib() -> ctypes.CDLL:
    """Load the C library (built in-tree by ``build.build()`` / ``__graft_entry__.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m top_routing_grouped_03_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        L.moe_status_string.argtypes = [I]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_version.argtypes = []
        L.moe_version.restype = I
        L.moe_workspace_size.argtypes = [I, I, I, I, I, I]
        L.moe_workspace_size.restype = Z
        L.moe_route.argtypes = [P, P, P, P, I, I, I, I, P, P, P, P, P, Z, P]
        L.moe_route.restype = I
        L.moe_route_ex.argtypes = [P, P, P, P, I, I, I, I, I, P, ctypes.c_uint, P, P, P, P, P,
                                   Z, P]
        L.moe_route_ex.restype = I
        L.moe_permute.argtypes = [P, P, P, I, I, I, P, P, P, P, P, P]
        L.moe_permute.restype = I
        L.moe_permute_ex.argtypes = [P, P, P, I, I, I, ctypes.c_longlong, P, P, P, P, P, P]
        L.moe_permute_ex.restype = I
        L.moe_expert_capacity.argtypes = [I, I, I, ctypes.c_float, I]
        L.moe_expert_capacity.restype = ctypes.c_longlong
        L.moe_grouped_swiglu.argtypes = [P, P, P, P, P, P, I, I, I, I, I, P, P, P, Z, P]
        L.moe_grouped_swiglu.restype = I
        L.moe_combine.argtypes = [P, P, P, P, P, P, I, I, I, P, P]
        L.moe_combine.restype = I
        L.moe_layer_forward.argtypes = [ctypes.POINTER(LayerParams), P, P, Z, P]
        L.moe_layer_forward.restype = I
        L.moe_read_device_status.argtypes = [P, P]
        L.moe_read_device_status.restype = I
        L.moe_route_noalloc.argtypes = [P, P, P, P, I, I, I, I, P, P, P, P, P]
        L.moe_route_noalloc.restype = I
        L.moe_launch_count.argtypes = []
        L.moe_launch_count.restype = ctypes.c_ulonglong
        L.moe_ep_dispatch_rows.argtypes = [P, P, I, I, P, P]
        L.moe_ep_dispatch_rows.restype = I
        L.moe_ep_recv_layout.argtypes = [P, I, I, I, P, P, P, P]
        L.moe_ep_recv_layout.restype = I
        L.moe_ep_return_rows.argtypes = [P, P, I, I, P, P]
        L.moe_ep_return_rows.restype = I
        L.moe_layer_plan.argtypes = [ctypes.POINTER(LayerParams), P, P]
        L.moe_layer_plan.restype = I
        L.moe_set_grid_wait_budget_ns.argtypes = [ctypes.c_ulonglong]
        L.moe_set_grid_wait_budget_ns.restype = ctypes.c_ulonglong
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().moe_status_string(int(code)).decode()


def version() -> int:
    return lib().moe_version()


def _check(rc: int, what: str):
    if rc != 0:
        raise MoEError(rc, what)


BF16, F32, I32, U8 = torch.bfloat16, torch.float32, torch.int32, torch.uint8


def _p(t: Optional[torch.Tensor], dtype: Optional[torch.dtype] = None):
    """Device pointer of a contiguous CUDA tensor (None -> NULL), of the element type the
    C ABI reads there when ``dtype`` is given."""
    if t is None:
        return None
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"expected a {dtype} tensor, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def workspace_size(T: int, D: int, E: int, K: int, f: int, f_s: int = 0) -> int:
    return int(lib().moe_workspace_size(T, D, E, K, f, f_s))


def alloc_workspace(T, D, E, K, f, f_s=0, device=None) -> torch.Tensor:
    n = workspace_size(T, D, E, K, f, f_s)
    if n == 0:
        raise MoEError(-2, "moe_workspace_size")
    ws = torch.empty(n, dtype=torch.uint8, device=device or "cuda")
    ws[:256].zero_()  # the device status word starts clear
    return ws


def route(x, w_router, K, logit_bias=None, w_shared_gate=None, workspace=None, stream=None,
          score="softmax", select_bias=None, bf16_weights=False):
    """Router step.  Returns (topk_idx [T,K] int32, topk_w [T,K] f32, expert_counts [E]
    int32, shared_gate [T] f32 or None).  score / select_bias / bf16_weights select the
    router variants of moe_route_ex."""
    T, D = x.shape
    E = w_router.shape[0]
    dev = x.device
    ws = workspace if workspace is not None else alloc_workspace(T, D, E, K, 128, 0, dev)
    idx = torch.empty((T, K), dtype=torch.int32, device=dev)
    w = torch.empty((T, K), dtype=torch.float32, device=dev)
    counts = torch.empty((E,), dtype=torch.int32, device=dev)
    sg = torch.empty((T,), dtype=torch.float32, device=dev) if w_shared_gate is not None else None
    if score == "softmax" and select_bias is None and not bf16_weights:
        rc = lib().moe_route(_p(x, BF16), _p(w_router, BF16), _p(logit_bias, F32),
                             _p(w_shared_gate, BF16), T, D, E, K, _p(idx), _p(w), _p(counts),
                             _p(sg), _p(ws, U8), ws.numel(), _stream(stream))
    else:
        rc = lib().moe_route_ex(_p(x, BF16), _p(w_router, BF16), _p(logit_bias, F32),
                                _p(w_shared_gate, BF16), T, D, E, K, SCORES[score],
                                _p(select_bias, F32),
                                MOE_FLAG_BF16_WEIGHTS if bf16_weights else 0, _p(idx), _p(w),
                                _p(counts), _p(sg), _p(ws, U8), ws.numel(), _stream(stream))
    _check(rc, "moe_route")
    return idx, w, counts, sg


def route_noalloc(x, w_router, K, logit_bias=None, w_shared_gate=None, stream=None):
    """Router step with no workspace: the library's own 1 MiB device scratch is used (see
    moe_route_noalloc in moe_api.h for the size limit and the sharing rules).  Only the
    outputs are allocated here, by the caller's side of the binding."""
    T, D = x.shape
    E = w_router.shape[0]
    dev = x.device
    idx = torch.empty((T, K), dtype=torch.int32, device=dev)
    w = torch.empty((T, K), dtype=torch.float32, device=dev)
    counts = torch.empty((E,), dtype=torch.int32, device=dev)
    sg = torch.empty((T,), dtype=torch.float32, device=dev) if w_shared_gate is not None else None
    rc = lib().moe_route_noalloc(_p(x, BF16), _p(w_router, BF16), _p(logit_bias, F32),
                                 _p(w_shared_gate, BF16), T, D, E, K, _p(idx), _p(w),
                                 _p(counts), _p(sg), _stream(stream))
    _check(rc, "moe_route_noalloc")
    return idx, w, counts, sg


def expert_capacity(T, K, E, capacity_factor, min_capacity=0) -> int:
    """Assignments per expert the layer keeps (moe_expert_capacity); -1: no capacity."""
    return int(lib().moe_expert_capacity(T, K, E, float(capacity_factor), int(min_capacity)))


def permute(topk_idx, topk_w, expert_counts, E, workspace=None, stream=None, capacity=None):
    """Permutation step.  Returns dict(offsets [E+1], sorted_token, sorted_w, slot_to_row).
    ``capacity``: keep each expert's first ``capacity`` entries (moe_permute_ex)."""
    T, K = topk_idx.shape
    dev = topk_idx.device
    off = torch.empty((E + 1,), dtype=torch.int32, device=dev)
    st = torch.empty((T * K,), dtype=torch.int32, device=dev)
    sw = torch.empty((T * K,), dtype=torch.float32, device=dev) if topk_w is not None else None
    s2r = torch.empty((T * K,), dtype=torch.int32, device=dev)
    if workspace is None and T > 0:
        workspace = alloc_workspace(T, 128, E, K, 128, 0, dev)
    cap = -1 if capacity is None else int(capacity)
    rc = lib().moe_permute_ex(_p(topk_idx, I32), _p(topk_w, F32), _p(expert_counts, I32), T, E,
                              K, cap, _p(off), _p(st), _p(sw), _p(s2r), _p(workspace, U8),
                              _stream(stream))
    _check(rc, "moe_permute_ex")
    return dict(offsets=off, sorted_token=st, sorted_w=sw, slot_to_row=s2r)


def grouped_swiglu(x, sorted_token, offsets, sorted_w, w_gate_up, w_down, rows,
                   out_acc=None, y_sorted=None, workspace=None, stream=None):
    """Grouped SwiGLU experts over the sorted rows; writes out_acc (+=) and/or y_sorted."""
    T, D = x.shape
    E, twof, _ = w_gate_up.shape
    f = twof // 2
    if workspace is None:
        Kr = max(1, -(-rows // max(T, 1)))
        workspace = alloc_workspace(max(T, 1), D, E, min(Kr, E, 16), f, 0, x.device)
    rc = lib().moe_grouped_swiglu(_p(x, BF16), _p(sorted_token, I32), _p(offsets, I32),
                                  _p(sorted_w, F32), _p(w_gate_up, BF16), _p(w_down, BF16), T,
                                  rows, D, E, f, _p(y_sorted, F32), _p(out_acc, F32),
                                  _p(workspace, U8), workspace.numel(), _stream(stream))
    _check(rc, "moe_grouped_swiglu")


def combine(T, D, K, out=None, out_acc=None, y_sorted=None, slot_to_row=None, topk_w=None,
            shared_out=None, shared_gate=None, device=None, stream=None):
    dev = device or "cuda"
    out = out if out is not None else torch.empty((T, D), dtype=torch.bfloat16, device=dev)
    rc = lib().moe_combine(_p(out_acc, F32), _p(y_sorted, F32), _p(slot_to_row, I32),
                           _p(topk_w, F32), _p(shared_out, BF16), _p(shared_gate, F32), T, D, K,
                           _p(out, BF16), _stream(stream))
    _check(rc, "moe_combine")
    return out


def ep_dispatch_rows(x, sorted_token, rows, stream=None):
    """x_sorted [rows, D] bf16 = x[sorted_token[:rows]] (moe_ep_dispatch_rows)."""
    out = torch.empty((rows, x.shape[1]), dtype=BF16, device=x.device)
    _check(lib().moe_ep_dispatch_rows(_p(x, BF16), _p(sorted_token, I32), rows, x.shape[1],
                                      _p(out, BF16), _stream(stream)), "moe_ep_dispatch_rows")
    return out


def ep_recv_layout(recv_counts, n, workspace=None, stream=None):
    """(recv_offsets [El+1], recv_row [n]) from the received counts [G, El] (device int32)."""
    G, El = recv_counts.shape
    off = torch.empty((El + 1,), dtype=I32, device=recv_counts.device)
    row = torch.empty((n,), dtype=I32, device=recv_counts.device)
    _check(lib().moe_ep_recv_layout(_p(recv_counts, I32), G, El, n, _p(off), _p(row),
                                    _p(workspace, U8), _stream(stream)), "moe_ep_recv_layout")
    return off, row


def ep_return_rows(y, recv_row, stream=None):
    """y_ret [n, D] fp32 with y_ret[recv_row[j]] = y[j] (moe_ep_return_rows)."""
    n, D = y.shape
    out = torch.empty_like(y)
    _check(lib().moe_ep_return_rows(_p(y, F32), _p(recv_row, I32), n, D, _p(out, F32),
                                    _stream(stream)), "moe_ep_return_rows")
    return out


def launch_count() -> int:
    """Kernels launched by the library in this process so far."""
    return int(lib().moe_launch_count())


def set_grid_wait_budget_ns(ns: int) -> int:
    """Bound of the layer's grid-wide wait for later calls (moe_set_grid_wait_budget_ns);
    returns the previous bound."""
    return int(lib().moe_set_grid_wait_budget_ns(int(ns)))


def event_array(events):
    """ctypes array of raw cudaEvent_t handles of recorded ``torch.cuda.Event`` objects
    (None entries are not recorded by the layer)."""
    assert len(events) == NUM_STEP_EVENTS
    arr = (ctypes.c_void_p * NUM_STEP_EVENTS)()
    for i, e in enumerate(events):
        if e is None:
            arr[i] = None
            continue
        if not e.cuda_event:
            raise ValueError("record each event once before passing it (creates the handle)")
        arr[i] = e.cuda_event
    return arr


def read_device_status(workspace, stream=None) -> int:
    return int(lib().moe_read_device_status(_p(workspace), _stream(stream)))


class MoELayer:
    """One MoE layer with resident weights and a reusable workspace.

    ``layer(x)`` runs moe_layer_forward on the current stream and returns y [T, D] bf16.
    """

    def __init__(self, w_router, w_gate_up, w_down, K, logit_bias=None, w_shared_gate=None,
                 w_shared_gate_up=None, w_shared_down=None, deterministic=False,
                 score="softmax", select_bias=None, bf16_weights=False, capacity_factor=0.0,
                 min_capacity=0):
        self.w_router, self.w_gate_up, self.w_down = w_router, w_gate_up, w_down
        self.logit_bias = logit_bias
        self.w_shared_gate, self.w_shared_gate_up = w_shared_gate, w_shared_gate_up
        self.w_shared_down = w_shared_down
        self.E, self.D = w_router.shape
        self.f = w_gate_up.shape[1] // 2
        self.f_s = 0 if w_shared_gate_up is None else w_shared_gate_up.shape[0] // 2
        self.K = K
        self.flags = (MOE_FLAG_DETERMINISTIC if deterministic else 0) | \
            (MOE_FLAG_BF16_WEIGHTS if bf16_weights else 0)
        self.score_mode = SCORES[score]
        self.select_bias = select_bias
        self.capacity_factor = float(capacity_factor)
        self.min_capacity = int(min_capacity)
        self._ws = None
        self._ws_T = -1
        self._copy_streams = None

    @classmethod
    def from_inputs(cls, inp, deterministic=False, **router):
        return cls(inp.w_router, inp.w_gate_up, inp.w_down, inp.cfg.K, inp.logit_bias,
                   inp.w_shared_gate, inp.w_shared_gate_up, inp.w_shared_down, deterministic,
                   **router)

    def workspace(self, T: int) -> torch.Tensor:
        if self._ws is None or self._ws_T < T:
            self._ws = alloc_workspace(T, self.D, self.E, self.K, self.f, self.f_s,
                                       self.w_router.device)
            self._ws_T = T
        return self._ws

    def params(self, x, topk_idx=None, topk_w=None, counts=None, events=None,
               residual=None) -> LayerParams:
        T = x.shape[0]
        ev = None if events is None else ctypes.cast(events, ctypes.c_void_p)
        return LayerParams(_p(x, BF16), _p(self.w_router, BF16), _p(self.logit_bias, F32),
                           _p(self.w_gate_up, BF16), _p(self.w_down, BF16),
                           _p(self.w_shared_gate, BF16), _p(self.w_shared_gate_up, BF16),
                           _p(self.w_shared_down, BF16), T, self.D, self.E, self.K, self.f,
                           self.f_s, self.flags, _p(topk_idx, I32), _p(topk_w, F32),
                           _p(counts, I32), ev, self.score_mode, _p(self.select_bias, F32),
                           _p(residual, BF16), self.capacity_factor, self.min_capacity)

    def __call__(self, x, out=None, topk_idx=None, topk_w=None, counts=None, stream=None,
                 step_events=None, residual=None):
        """y = layer(x) (+ residual h) on the device.  ``step_events``: an
        ``event_array(...)`` to time each kernel of the call."""
        T = x.shape[0]
        if x.shape[1] != self.D:
            raise MoEError(-1, "moe_layer_forward (x has the wrong width)")
        out = out if out is not None else torch.empty((T, self.D), dtype=torch.bfloat16,
                                                      device=x.device)
        ws = self.workspace(T)
        prm = self.params(x, topk_idx, topk_w, counts, step_events, residual)
        rc = lib().moe_layer_forward(ctypes.byref(prm), _p(out, BF16), _p(ws, U8), ws.numel(),
                                     _stream(stream))
        _check(rc, "moe_layer_forward")
        return out

    def plan(self, T: int):
        """(steps that launch kernels, kernels per call) for T tokens, from moe_layer_plan:
        the step names of STEP_EVENT_NAMES whose interval holds work of their own."""
        x = torch.empty((0, self.D), dtype=BF16, device=self.w_router.device)
        prm = self.params(x)
        prm.T = T
        mask, n = ctypes.c_uint(0), ctypes.c_int(0)
        _check(lib().moe_layer_plan(ctypes.byref(prm), ctypes.byref(mask), ctypes.byref(n)),
               "moe_layer_plan")
        steps = [name for i, name in enumerate(STEP_EVENT_NAMES) if mask.value >> i & 1]
        return steps, n.value

    def forward_host(self, x_host, y_host, x_dev, y_dev, stream=None):
        """End to end from host memory: copy x (pinned host) in, run the layer, copy y
        out to pinned host memory; everything enqueued on one stream."""
        x_dev.copy_(x_host, non_blocking=True)
        self(x_dev, out=y_dev, stream=stream)
        y_host.copy_(y_dev, non_blocking=True)
        return y_host

    def forward_host_stream(self, x_hosts, y_hosts, x_devs, y_devs, stream=None):
        """End to end for a sequence of batches from host memory, each batch's copies
        overlapping the layer on its neighbours: batch i's x (pinned host) goes in on a copy
        stream while batch i-1 runs, its y comes back to pinned host memory on another copy
        stream while batch i+1 runs.  x_devs and y_devs hold two device buffers each (used
        in turn).  The layer runs on `stream` (default: the current stream), which at the end
        waits for the last copy out; returns y_hosts."""
        cur = torch.cuda.current_stream() if stream is None else stream
        if self._copy_streams is None:
            self._copy_streams = (torch.cuda.Stream(device=cur.device),
                                  torch.cuda.Stream(device=cur.device))
        h2d, d2h = self._copy_streams
        start = torch.cuda.Event()
        start.record(cur)
        h2d.wait_event(start)
        d2h.wait_event(start)
        ran, out = [], []
        for i, (xh, yh) in enumerate(zip(x_hosts, y_hosts)):
            b = i % 2
            with torch.cuda.stream(h2d):
                if i >= 2:
                    h2d.wait_event(ran[i - 2])  # the layer is done with x buffer b
                x_devs[b].copy_(xh, non_blocking=True)
                arrived = torch.cuda.Event()
                arrived.record(h2d)
            cur.wait_event(arrived)
            if i >= 2:
                cur.wait_event(out[i - 2])  # y buffer b has been copied out
            self(x_devs[b], out=y_devs[b], stream=cur)
            done = torch.cuda.Event()
            done.record(cur)
            ran.append(done)
            with torch.cuda.stream(d2h):
                d2h.wait_event(done)
                yh.copy_(y_devs[b], non_blocking=True)
                copied = torch.cuda.Event()
                copied.record(d2h)
            out.append(copied)
        if out:
            cur.wait_event(out[-1])
        return y_hosts

    def device_status(self, stream=None) -> int:
        return read_device_status(self._ws, stream) if self._ws is not None else 0
