"""moe_route_noalloc, the router entry point for callers that cannot allocate device
memory (a plugin whose host framework owns every allocation, or latency-critical code that
cannot pay for cudaMalloc's synchronisation): its scratch is the library's fixed 1 MiB
device array, so the caller passes only inputs and outputs.

Its outputs must match moe_route's (which uses a caller-provided workspace) on two calls
in a row, the second with a different, smaller problem so that stale scratch contents
from the first call would show.  This file is collected last on purpose."""
import numpy as np
import pytest
import torch

from parity import W_TOL
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


def test_route_noalloc_rejects_sizes_beyond_its_scratch():
    import top_routing_grouped_03_b200 as moe
    x = torch.zeros((1100, 128), dtype=torch.bfloat16, device="cuda")  # 1100 x 257 floats > 1 MiB
    w_r = torch.zeros((256, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoEError) as err:
        moe.route_noalloc(x, w_r, 8)
    assert err.value.code == -2  # MOE_ERR_UNSUPPORTED
