"""Expert capacity and token dropping on the GPU ("1.6 混合专家（MoE）", section 三, expert
capacity and token dropping): the capacity-limited permutation bit-exactly against the
oracle's keep mask, and whole layers against the oracle layer with the same capacity."""
import numpy as np
import pytest
import torch

from parity import check_layer
from workloads import CONFIGS, LayerConfig, crafted_routing, make_inputs, random_routing

pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().cpu().numpy()


def _expected_permutation(oracle_mod, idx, E, C):
    """The oracle's permutation restricted to the oracle's kept assignments."""
    ref = oracle_mod.permute(idx, E)
    keep = oracle_mod.capacity_keep(idx, E, C).reshape(-1)
    T, K = idx.shape
    kept_rows = [r for r in range(T * K) if keep[ref["sorted_slot"][r]]]
    sorted_token = ref["sorted_token"][kept_rows]
    sorted_slot = ref["sorted_slot"][kept_rows]
    slot_to_row = np.full(T * K, -1, np.int32)
    slot_to_row[sorted_slot] = np.arange(len(kept_rows), dtype=np.int32)
    kept_counts = np.minimum(ref["counts"], C)
    offsets = np.concatenate([[0], np.cumsum(kept_counts)]).astype(np.int32)
    return offsets, sorted_token, sorted_slot, slot_to_row


@pytest.mark.parametrize("kind,T,E,K,C", [
    ("random", 64, 256, 8, 2),           # decode sizes, one CTA
    ("concentrated", 64, 256, 8, 5),     # 8 experts of 64 entries, 5 kept each
    ("one_hot_expert", 300, 16, 4, 40),
    ("random", 4096, 128, 8, 200),       # several chunks
    ("concentrated", 2048, 128, 8, 300),
    ("random", 700, 32, 4, 0),           # capacity 0: everything dropped
    ("random", 900, 64, 6, 10 ** 6),     # capacity above every group: dropless
])
def test_permute_with_capacity_bitexact(moe, oracle_mod, kind, T, E, K, C):
    idx = (random_routing(T, E, K, seed=T + C) if kind == "random"
           else crafted_routing(T, E, K, kind)).numpy()
    w = torch.rand((T, K), generator=torch.Generator().manual_seed(3))
    counts = np.bincount(idx.reshape(-1), minlength=E).astype(np.int32)
    offsets, sorted_token, sorted_slot, slot_to_row = _expected_permutation(oracle_mod, idx, E, C)
    ws = moe.alloc_workspace(T, 128, E, K, 128)
    ws.zero_()
    out = moe.permute(torch.as_tensor(idx).cuda(), w.cuda(), torch.as_tensor(counts).cuda(), E,
                      workspace=ws, capacity=C)
    torch.cuda.synchronize()
    assert moe.read_device_status(ws) == 0
    n = int(offsets[-1])
    np.testing.assert_array_equal(_np(out["offsets"]), offsets)
    np.testing.assert_array_equal(_np(out["slot_to_row"]), slot_to_row)
    np.testing.assert_array_equal(_np(out["sorted_token"])[:n], sorted_token)
    np.testing.assert_array_equal(_np(out["sorted_w"])[:n], w.numpy().reshape(-1)[sorted_slot])
    # the rows past the kept total belong to no group: token 0, weight 0
    assert np.all(_np(out["sorted_token"])[n:] == 0)
    assert np.all(_np(out["sorted_w"])[n:] == 0.0)


CAP_LAYERS = {
    # every token picks the same 8 experts; C = max(0, ceil(1.0 * 64 * 8 / 256)) = 2 of 64
    "decode_concentrated": (CONFIGS["decode_concentrated"], 1.0, 0),
    "decode": (CONFIGS["decode"], 1.25, 4),
    "tiny": (CONFIGS["tiny"], 1.0, 0),
    "shared_small": (LayerConfig("shared_small", T=40, D=256, E=16, K=4, f=128, f_s=256),
                     0.75, 0),
    # tensor-core router, shared expert
    "tc_router_shared": (LayerConfig("tc_router_shared", T=300, D=384, E=128, K=6, f=128,
                                     f_s=256, seed=8), 1.25, 4),
    "few_tokens": (LayerConfig("few_tokens", T=12, D=256, E=8, K=4, f=256, seed=9), 1.0, 0),
    # shared expert as wide as the routed ones, with tokens dropped from the routed groups
    "shared_fused": (LayerConfig("shared_fused", T=100, D=256, E=16, K=4, f=256, f_s=256,
                                 seed=16), 0.8, 2),
}


def _run(moe, inp, cf, mn, det, residual=None):
    cfg = inp.cfg
    layer = moe.MoELayer.from_inputs(inp, deterministic=det, capacity_factor=cf,
                                     min_capacity=mn)
    idx = torch.empty((cfg.T, cfg.K), dtype=torch.int32, device="cuda")
    w = torch.empty((cfg.T, cfg.K), dtype=torch.float32, device="cuda")
    y = layer(inp.x, topk_idx=idx, topk_w=w, residual=residual)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    return y, idx, w


@pytest.mark.parametrize("det", [False, True])
@pytest.mark.parametrize("name", sorted(CAP_LAYERS))
def test_layer_with_capacity(moe, oracle_mod, name, det):
    cfg, cf, mn = CAP_LAYERS[name]
    inp = make_inputs(cfg).to("cuda")
    C = moe.expert_capacity(cfg.T, cfg.K, cfg.E, cf, mn)
    assert C == oracle_mod.expert_capacity(cfg.T, cfg.K, cfg.E, float(np.float32(cf)), mn)
    h = torch.randn((cfg.T, cfg.D), generator=torch.Generator().manual_seed(5))
    h = h.to(torch.bfloat16).cuda()
    y, idx, w = _run(moe, inp, cf, mn, det, residual=h)
    rep = check_layer(oracle_mod, inp, y, _np(idx), _np(w), residual=h, capacity=C)
    print(name, det, "C =", C, rep)
    if name == "decode_concentrated":
        assert rep["dropped"] == cfg.T * cfg.K - 8 * C  # only 2 of each expert's 64 stay


def test_fully_dropped_tokens_pass_the_residual_through(moe):
    """Every token routes to experts 0..K-1; with C = 3 the tokens from the fourth on lose
    every assignment: their output is the residual, bit for bit."""
    cfg = LayerConfig("cap", T=20, D=256, E=16, K=2, f=128)
    inp = make_inputs(cfg).to("cuda")
    bias = torch.zeros(16)
    bias[:2] = 30.0
    inp.logit_bias = bias.cuda()
    h = torch.randn((cfg.T, cfg.D), generator=torch.Generator().manual_seed(6))
    h = h.to(torch.bfloat16).cuda()
    y, idx, _ = _run(moe, inp, 1.0, 3, False, residual=h)
    assert moe.expert_capacity(20, 2, 16, 1.0, 3) == 3
    assert np.all(np.sort(_np(idx), axis=1) == [0, 1])
    assert torch.equal(y[3:], h[3:])
    assert not torch.equal(y[:3], h[:3])


def test_capacity_above_every_group_equals_dropless(moe):
    inp = make_inputs(CONFIGS["tiny"]).to("cuda")
    y0, _, _ = _run(moe, inp, 0.0, 0, True)
    y1, _, _ = _run(moe, inp, 100.0, 0, True)
    assert torch.equal(y0, y1)


@pytest.mark.parametrize("name,cf", [("zipf@T1024", 1.25), ("prefill", 1.0)])
def test_full_size_layer_with_capacity(moe, oracle_mod, name, cf):
    """Hot experts far over capacity (Zipf), and ~half the experts over it (prefill); the
    outputs of a sample of tokens against the oracle."""
    cfg = CONFIGS[name]
    inp = make_inputs(cfg, device="cuda")
    C = moe.expert_capacity(cfg.T, cfg.K, cfg.E, cf, 4)
    y, idx, w = _run(moe, inp, cf, 4, False)
    gi = _np(idx)
    rng = np.random.default_rng(0)
    toks = np.unique(np.concatenate([np.arange(8), cfg.T - 1 - np.arange(8),
                                     rng.choice(cfg.T, 24, replace=False)]))
    rep = check_layer(oracle_mod, inp, y, gi, _np(w), tokens=toks, capacity=C)
    assert rep["dropped"] > 0
    print(name, "C =", C, rep)
