"""The seeded synthetic inputs (CPU): reproducible bits, the stated distributions, and the
routing regimes they are built to produce."""
import math

import numpy as np
import pytest
import torch

from workloads import (CONFIGS, LayerConfig, crafted_routing, make_inputs, random_routing,
                       routing_bias)


def test_same_seed_same_bits_other_seed_other_bits():
    cfg = LayerConfig("w", T=16, D=128, E=8, K=2, f=128, f_s=128)
    a, b, c = make_inputs(cfg), make_inputs(cfg), make_inputs(cfg, seed=1)
    for name in ("x", "w_router", "w_gate_up", "w_down", "w_shared_gate", "w_shared_gate_up",
                 "w_shared_down"):
        ta, tb, tc = getattr(a, name), getattr(b, name), getattr(c, name)
        assert ta.dtype == torch.bfloat16
        assert torch.equal(ta.view(torch.int16), tb.view(torch.int16)), name
        assert not torch.equal(ta.view(torch.int16), tc.view(torch.int16)), name


def test_shapes_and_scales():
    cfg = CONFIGS["decode"]
    inp = make_inputs(cfg)
    T, D, E, f = cfg.T, cfg.D, cfg.E, cfg.f
    assert inp.x.shape == (T, D) and inp.w_router.shape == (E, D)
    assert inp.w_gate_up.shape == (E, 2 * f, D) and inp.w_down.shape == (E, D, f)
    assert inp.logit_bias is None and inp.w_shared_gate is None

    def std(t):
        return float(t.float().std())
    assert std(inp.x) == pytest.approx(1.0, rel=0.02)
    assert std(inp.w_router) == pytest.approx(1 / math.sqrt(D), rel=0.02)
    assert std(inp.w_gate_up[:, :f]) == pytest.approx(1 / math.sqrt(D), rel=0.02)
    assert std(inp.w_gate_up[:, f:]) == pytest.approx(1 / math.sqrt(D), rel=0.02)
    assert std(inp.w_down) == pytest.approx(1 / math.sqrt(f), rel=0.02)


def test_concentrated_bias_and_regime(oracle_mod):
    """+20 on the same 8 experts (randperm(E, seed 1)[:8]) sends every token to that set."""
    cfg = CONFIGS["decode_concentrated"]
    b = routing_bias(cfg).numpy()
    hot = np.flatnonzero(b)
    assert len(hot) == 8 and np.all(b[hot] == 20.0)
    perm = torch.randperm(cfg.E, generator=torch.Generator().manual_seed(1)).numpy()
    assert sorted(hot.tolist()) == sorted(perm[:8].tolist())
    inp = make_inputs(cfg)
    r = oracle_mod.route(inp.x, inp.w_router, cfg.K, inp.logit_bias)
    assert all(sorted(row) == sorted(hot.tolist()) for row in r["idx"].tolist())


def test_zipf_bias():
    """b_e = 2 ln(rank_e^-1.2) = -2.4 ln(rank_e), ranks 1..E from randperm(E, seed 2)."""
    cfg = CONFIGS["zipf@T16"]
    b = routing_bias(cfg).numpy().astype(np.float64)
    rank = np.exp(-b / 2.4)
    np.testing.assert_allclose(np.sort(rank), np.arange(1, cfg.E + 1), rtol=1e-5)
    perm = torch.randperm(cfg.E, generator=torch.Generator().manual_seed(2)).numpy()
    assert b[perm[0]] == 0.0  # rank 1
    np.testing.assert_allclose(b[perm], -2.4 * np.log(np.arange(1, cfg.E + 1)), rtol=1e-6,
                               atol=1e-6)


def test_natural_routing_has_no_bias():
    for name in ("tiny", "decode", "prefill", "finegrained"):
        assert routing_bias(CONFIGS[name]) is None


@pytest.mark.parametrize("T,E,K", [(64, 256, 8), (37, 16, 4), (1, 8, 8)])
def test_random_routing_distinct_experts(T, E, K):
    idx = random_routing(T, E, K, seed=3)
    assert idx.shape == (T, K) and idx.dtype == torch.int32
    assert all(len(set(row)) == K for row in idx.tolist())
    assert int(idx.min()) >= 0 and int(idx.max()) < E


def test_crafted_routings():
    u = crafted_routing(64, 256, 8, "uniform").numpy()
    assert np.all(np.bincount(u.reshape(-1), minlength=256) == 2)   # 2 rows per expert
    c = crafted_routing(64, 256, 8, "concentrated").numpy()
    assert set(np.unique(c)) == set(range(8))                       # U = K
    h = crafted_routing(300, 16, 4, "one_hot_expert").numpy()
    assert np.all(h[:, 0] == 0)
    assert all(len(set(row)) == 4 for row in h.tolist())
