"""Failure detection on the GPU without a hang or a fault: the layer's grid-wide wait (the
last down kernel converts the output only after every CTA of its grid has added its
tiles) gives up after a run-time budget.  With a budget of 0 every CTA but the last to
arrive gives up at its first look, records MOE_ERR_TIMEOUT in the workspace's status word
and returns; the host reads that status, and the next call with the default budget is
parity-green again."""
import numpy as np
import pytest
import torch

from parity import check_layer
from workloads import CONFIGS, LayerConfig, make_inputs

pytestmark = pytest.mark.gpu

MOE_ERR_TIMEOUT = -5
DEFAULT_NS = 2_000_000_000


@pytest.mark.parametrize("name", ["decode", "shared"])
def test_grid_wait_timeout_is_reported_then_recovers(moe, oracle_mod, name):
    cfg = CONFIGS["decode"] if name == "decode" else \
        LayerConfig("timeout_shared", T=96, D=512, E=32, K=4, f=256, f_s=256, seed=19)
    inp = make_inputs(cfg).to("cuda")
    layer = moe.MoELayer.from_inputs(inp)
    T, K = cfg.T, cfg.K
    statuses = []
    prev = moe.set_grid_wait_budget_ns(0)
    try:
        # the first CTA to finish finds the grid incomplete (CTAs finish microseconds
        # apart); a few calls make a run where every CTA arrives at once irrelevant
        for _ in range(5):
            layer(inp.x)
            torch.cuda.synchronize()
            statuses.append(layer.device_status())
            if statuses[-1] == MOE_ERR_TIMEOUT:
                break
    finally:
        assert moe.set_grid_wait_budget_ns(prev) == 0
    assert prev == DEFAULT_NS
    assert statuses[-1] == MOE_ERR_TIMEOUT and set(statuses) <= {0, MOE_ERR_TIMEOUT}, statuses
    # the context is usable and the default budget gives a correct layer again
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, K), dtype=torch.float32, device="cuda")
    y = layer(inp.x, topk_idx=idx, topk_w=w)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    rep = check_layer(oracle_mod, inp, y, idx.cpu().numpy(), w.cpu().numpy())
    assert np.isfinite(rep["y_err"])
