"""moe_route_noalloc, the router entry point for callers that cannot allocate device
memory (a plugin whose host framework owns every allocation, or latency-critical code that
cannot pay for cudaMalloc's synchronisation): its scratch is the library's fixed 1 MiB
device array, so the caller passes only inputs and outputs.

Its outputs must match moe_route's (which uses a caller-provided workspace) on two calls
in a row, the second with a different, smaller problem so that stale scratch contents
from the first call would show.  Where moe_route takes its logits from the tensor cores
(T >= 256, E a multiple of 128) the two agree within the router's parity rules, checked
against the oracle.  The device's free memory does not move across a call.  This file is
collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from parity import W_TOL, check_route
from workloads import CONFIGS, LayerConfig, make_inputs

pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().cpu().numpy()


def test_route_noalloc_matches_route_on_two_calls():
    import top_routing_grouped_03_b200 as moe
    cases = [CONFIGS["decode_concentrated"],
             LayerConfig("noalloc_shared", T=37, D=256, E=16, K=4, f=128, f_s=128, seed=9)]
    for cfg in cases:
        inp = make_inputs(cfg).to("cuda")
        ref = moe.route(inp.x, inp.w_router, cfg.K, inp.logit_bias, inp.w_shared_gate)
        got = moe.route_noalloc(inp.x, inp.w_router, cfg.K, inp.logit_bias, inp.w_shared_gate)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(_np(got[0]), _np(ref[0]))
        assert np.abs(_np(got[1]) - _np(ref[1])).max() <= W_TOL
        np.testing.assert_array_equal(_np(got[2]), _np(ref[2]))
        if ref[3] is not None:
            assert np.abs(_np(got[3]) - _np(ref[3])).max() <= 1e-5


def test_route_noalloc_where_route_uses_tensor_cores(oracle_mod):
    """T = 512, E = 128: moe_route sums the logits on the tensor cores, the no-allocation
    entry point on the CUDA cores; both must pass the router's parity rules against the
    oracle (exact experts off near ties, weights within 1e-3)."""
    import top_routing_grouped_03_b200 as moe
    cfg = LayerConfig("noalloc_tc", T=512, D=256, E=128, K=8, f=128, seed=17)
    inp = make_inputs(cfg).to("cuda")
    orc = oracle_mod.route(inp.x, inp.w_router, cfg.K)
    for call in (moe.route, moe.route_noalloc):
        idx, w, counts, _ = call(inp.x, inp.w_router, cfg.K)
        torch.cuda.synchronize()
        rep = check_route(orc, _np(idx), _np(w), _np(counts))
        print(call.__name__, "near ties", rep.near_tie, "differing", len(rep.differing_sets))


def test_route_noalloc_leaves_free_memory_unchanged():
    """Outputs allocated first, then the C entry point called directly: the device's free
    memory (cudaMemGetInfo) is the same before and after the call."""
    import top_routing_grouped_03_b200 as moe
    cfg = LayerConfig("noalloc_mem", T=200, D=512, E=64, K=6, f=128, seed=23)
    inp = make_inputs(cfg).to("cuda")
    T, D, E, K = cfg.T, cfg.D, cfg.E, cfg.K
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, K), dtype=torch.float32, device="cuda")
    counts = torch.empty((E,), dtype=torch.int32, device="cuda")
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    args = (ctypes.c_void_p(inp.x.data_ptr()), ctypes.c_void_p(inp.w_router.data_ptr()), None,
            None, T, D, E, K, ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(w.data_ptr()),
            ctypes.c_void_p(counts.data_ptr()), None, s)
    assert moe.lib().moe_route_noalloc(*args) == 0  # first call: module and scratch set up
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    assert moe.lib().moe_route_noalloc(*args) == 0
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert int(counts.sum()) == T * K


def test_route_noalloc_rejects_sizes_beyond_its_scratch():
    import top_routing_grouped_03_b200 as moe
    x = torch.zeros((1100, 128), dtype=torch.bfloat16, device="cuda")  # 1100 x 257 floats > 1 MiB
    w_r = torch.zeros((256, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoEError) as err:
        moe.route_noalloc(x, w_r, 8)
    assert err.value.code == -2  # MOE_ERR_UNSUPPORTED
