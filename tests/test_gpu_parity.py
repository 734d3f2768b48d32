"""Parity of the CUDA path (through the C ABI) with the CPU oracle, on a B200.

Small layers are compared element by element on every token; the multi-GB layers on the
full routing plus a sample of tokens (first, last, ragged tail, hot expert, random).
"""
import numpy as np
import pytest
import torch

from parity import Y_TOL, check_layer, check_route, oracle_outputs, output_error
from workloads import CONFIGS, LayerConfig, crafted_routing, make_inputs, random_routing

pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().cpu().numpy()


def _run_layer(moe, inp, deterministic=False):
    layer = moe.MoELayer.from_inputs(inp, deterministic=deterministic)
    T, K, E = inp.cfg.T, inp.cfg.K, inp.cfg.E
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, K), dtype=torch.float32, device="cuda")
    counts = torch.empty((E,), dtype=torch.int32, device="cuda")
    y = layer(inp.x, topk_idx=idx, topk_w=w, counts=counts)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    return layer, y, idx, w, counts


SMALL_LAYERS = {
    "tiny": CONFIGS["tiny"],
    "decode": CONFIGS["decode"],
    "decode_concentrated": CONFIGS["decode_concentrated"],
    "shared_small": LayerConfig("shared_small", T=40, D=256, E=16, K=4, f=128, f_s=256),
    "ragged_T": LayerConfig("ragged_T", T=203, D=384, E=24, K=6, f=256, seed=3),
    "single_token": LayerConfig("single_token", T=1, D=512, E=64, K=8, f=128, seed=4),
    "dense_E1": LayerConfig("dense_E1", T=33, D=256, E=1, K=1, f=384, seed=5),
    "all_experts": LayerConfig("all_experts", T=50, D=256, E=8, K=8, f=128, seed=6),
    "hot_rows": LayerConfig("hot_rows", T=300, D=256, E=4, K=2, f=128, seed=7),
    # few tiles with deep reductions (D = 1024 for gate_up, f = 1024 for down), routed and
    # shared
    "deep_gate_up": LayerConfig("deep_gate_up", T=40, D=1024, E=8, K=2, f=256, seed=10),
    "deep_down": LayerConfig("deep_down", T=48, D=512, E=4, K=2, f=1024, seed=11),
    "deep_shared": LayerConfig("deep_shared", T=40, D=1024, E=8, K=2, f=256, f_s=512,
                               seed=12),
    # the largest sizes the library takes: K = 16 of E = 512 experts (16 logits per lane
    # in the selection, 512 groups), D = 8192 (128 KiB of staged tokens in the router,
    # 128 K steps), f = 8192 (64 feature blocks, 128 K steps in down)
    "max_k_e": LayerConfig("max_k_e", T=70, D=256, E=512, K=16, f=128, seed=13),
    "max_d": LayerConfig("max_d", T=24, D=8192, E=8, K=2, f=128, seed=14),
    "max_f": LayerConfig("max_f", T=24, D=256, E=4, K=2, f=8192, seed=15),
    # at most 16 tokens: weights-on-M grouped GEMMs, routed and shared
    "few_tokens_shared": LayerConfig("few_tokens_shared", T=12, D=256, E=32, K=4, f=256,
                                     f_s=128, seed=9),
    # shared expert as wide as the routed ones, on the tokens-on-M kernel (routed groups of
    # a few to ~50 rows; then many small groups with the tensor-core router and several
    # shared row blocks)
    "shared_fused": LayerConfig("shared_fused", T=100, D=256, E=16, K=4, f=256, f_s=256,
                                seed=16),
    "shared_fused_tc": LayerConfig("shared_fused_tc", T=520, D=512, E=128, K=8, f=256,
                                   f_s=256, seed=18),
    # T >= 256 and E % 128 == 0: router logits on the tensor cores, shared gate in the
    # selection kernel
    "tc_router_shared": LayerConfig("tc_router_shared", T=300, D=384, E=128, K=6, f=128,
                                    f_s=256, seed=8),
}


# ------------------------------------------------------------------ router


@pytest.mark.parametrize("name", sorted(SMALL_LAYERS))
def test_route_matches_oracle(moe, oracle_mod, name):
    cfg = SMALL_LAYERS[name]
    inp = make_inputs(cfg).to("cuda")
    idx, w, counts, sg = moe.route(inp.x, inp.w_router, cfg.K, inp.logit_bias, inp.w_shared_gate)
    torch.cuda.synchronize()
    orc = oracle_mod.route(inp.x, inp.w_router, cfg.K, inp.logit_bias, inp.w_shared_gate)
    check_route(orc, _np(idx), _np(w), _np(counts))
    if sg is not None:
        np.testing.assert_allclose(_np(sg), orc["shared_gate"], rtol=0, atol=1e-5)


def test_route_worked_example(moe):
    """x = 0, bias = ln(score): p is proportional to the scores, so the top-2 of
    (.1, .9, .2, .3, .6, .05, .05, .05) renormalise to 0.9/1.5 = 0.6 and 0.6/1.5 = 0.4."""
    scores = np.array([0.1, 0.9, 0.2, 0.3, 0.6, 0.05, 0.05, 0.05])
    x = torch.zeros((3, 128), dtype=torch.bfloat16, device="cuda")
    w_r = torch.zeros((8, 128), dtype=torch.bfloat16, device="cuda")
    bias = torch.tensor(np.log(scores), dtype=torch.float32, device="cuda")
    idx, w, counts, _ = moe.route(x, w_r, 2, bias)
    torch.cuda.synchronize()
    assert _np(idx).tolist() == [[1, 4]] * 3
    np.testing.assert_allclose(_np(w), [[0.6, 0.4]] * 3, atol=1e-6)
    assert _np(counts).tolist() == [0, 3, 0, 0, 3, 0, 0, 0]


def test_route_ties_go_to_lower_index(moe):
    x = torch.zeros((2, 128), dtype=torch.bfloat16, device="cuda")
    w_r = torch.zeros((40, 128), dtype=torch.bfloat16, device="cuda")
    bias = torch.zeros(40, dtype=torch.float32, device="cuda")
    bias[[3, 7, 35, 36]] = 1.0
    idx, w, _, _ = moe.route(x, w_r, 6, bias)
    torch.cuda.synchronize()
    assert _np(idx).tolist() == [[3, 7, 35, 36, 0, 1]] * 2


@pytest.mark.parametrize("T,D,E,K", [(1, 128, 16, 4), (9, 256, 16, 16), (37, 1024, 64, 8),
                                     (130, 512, 512, 10), (64, 2048, 256, 8), (5, 8192, 32, 3),
                                     # tensor-core logits (T >= 256, E % 128 == 0)
                                     (256, 128, 128, 8), (1000, 2048, 256, 8),
                                     (777, 512, 512, 10), (4099, 4096, 128, 8)])
def test_route_shapes(moe, oracle_mod, T, D, E, K):
    cfg = LayerConfig("r", T=T, D=D, E=E, K=K, f=128, seed=T + E)
    inp = make_inputs(cfg).to("cuda")
    idx, w, counts, _ = moe.route(inp.x, inp.w_router, K)
    torch.cuda.synchronize()
    orc = oracle_mod.route(inp.x, inp.w_router, K)
    check_route(orc, _np(idx), _np(w), _np(counts))


@pytest.mark.parametrize("T,D,E,K", [(1000, 2048, 256, 8), (4099, 4096, 128, 8)])
def test_route_repeatable(moe, T, D, E, K):
    """The tensor-core router's split reduction adds its partial planes in a fixed order:
    two calls give the same bits."""
    cfg = LayerConfig("r", T=T, D=D, E=E, K=K, f=128, seed=1)
    inp = make_inputs(cfg).to("cuda")
    a = moe.route(inp.x, inp.w_router, K)
    b = moe.route(inp.x, inp.w_router, K)
    torch.cuda.synchronize()
    for u, v in zip(a[:3], b[:3]):
        assert torch.equal(u, v)


# ------------------------------------------------------------------ permutation


@pytest.mark.parametrize("kind,T,E,K", [("uniform", 64, 256, 8), ("concentrated", 64, 256, 8),
                                        ("one_hot_expert", 300, 16, 4), ("random", 1, 8, 3),
                                        ("random", 517, 128, 8), ("random", 4096, 512, 10),
                                        ("random", 3000, 4, 4),
                                        # several chunks: hot experts, 256 chunks of a length
                                        # that is not a multiple of 1024
                                        ("concentrated", 2048, 256, 8),
                                        ("one_hot_expert", 9000, 64, 6),
                                        ("random", 70001, 64, 4)])
def test_permute_bitexact(moe, oracle_mod, kind, T, E, K):
    idx = (random_routing(T, E, K, seed=T) if kind == "random"
           else crafted_routing(T, E, K, kind)).numpy()
    w = torch.rand((T, K), generator=torch.Generator().manual_seed(1))
    counts = np.bincount(idx.reshape(-1), minlength=E).astype(np.int32)
    ref = oracle_mod.permute(idx, E)
    ws = moe.alloc_workspace(max(T, 1), 128, E, K, 128)
    ws.zero_()
    out = moe.permute(torch.as_tensor(idx).cuda(), w.cuda(), torch.as_tensor(counts).cuda(), E,
                      workspace=ws)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(_np(out["offsets"]), ref["offsets"])
    np.testing.assert_array_equal(_np(out["sorted_token"]), ref["sorted_token"])
    np.testing.assert_array_equal(_np(out["slot_to_row"]), ref["slot_to_row"])
    np.testing.assert_array_equal(_np(out["sorted_w"]), w.numpy().reshape(-1)[ref["sorted_slot"]])
    assert moe.read_device_status(ws) == 0


def test_permute_flags_inconsistent_counts(moe):
    idx = torch.tensor([[0, 1], [1, 2]], dtype=torch.int32, device="cuda")
    bad_counts = torch.tensor([1, 1, 1, 0], dtype=torch.int32, device="cuda")  # sums to 3 != 4
    ws = moe.alloc_workspace(2, 128, 4, 2, 128)
    ws.zero_()
    moe.permute(idx, None, bad_counts, 4, workspace=ws)
    assert moe.read_device_status(ws) == -7  # MOE_ERR_DEVICE


@pytest.mark.parametrize("delta", [-1, 1])
def test_permute_flags_inconsistent_counts_chunked(moe, delta):
    T, E, K = 3000, 8, 4   # 12000 entries: several chunks
    idx = random_routing(T, E, K, seed=5)
    counts = np.bincount(idx.numpy().reshape(-1), minlength=E).astype(np.int32)
    counts[3] += delta
    counts[5] -= delta        # the total stays right, two groups do not
    ws = moe.alloc_workspace(T, 128, E, K, 128)
    ws.zero_()
    moe.permute(idx.cuda(), None, torch.as_tensor(counts).cuda(), E, workspace=ws)
    assert moe.read_device_status(ws) == -7  # MOE_ERR_DEVICE


# ------------------------------------------------------------------ grouped SwiGLU


@pytest.mark.parametrize("kind,T,D,E,K,f", [
    ("uniform", 64, 2048, 256, 8, 512),        # 2 rows per expert (the pages' uniform case)
    ("concentrated", 64, 2048, 256, 8, 512),   # 64 rows on 8 experts
    ("one_hot_expert", 300, 256, 16, 4, 128),  # one expert with every token
    ("one_hot_expert", 200, 256, 8, 2, 128),   # one 200-row group, the rest ~29 rows
    # at most 16 tokens: the weights-on-M orientation (narrow token tiles)
    ("concentrated", 16, 2048, 256, 8, 512),   # 16 rows on each of 8 experts
    ("random", 13, 512, 4, 2, 384),            # ragged groups of a few rows
    ("random", 1, 256, 8, 3, 256),
    ("random", 777, 512, 12, 3, 384),          # ragged groups, several row blocks
])
def test_grouped_swiglu_crafted_routing(moe, oracle_mod, kind, T, D, E, K, f):
    cfg = LayerConfig("g", T=T, D=D, E=E, K=K, f=f, seed=11)
    inp = make_inputs(cfg).to("cuda")
    idx = (random_routing(T, E, K, seed=3) if kind == "random"
           else crafted_routing(T, E, K, kind)).numpy()
    alpha = torch.rand((T, K), generator=torch.Generator().manual_seed(2), dtype=torch.float64)
    alpha = (alpha / alpha.sum(1, keepdim=True)).numpy()
    counts = np.bincount(idx.reshape(-1), minlength=E).astype(np.int32)
    pm = moe.permute(torch.as_tensor(idx).cuda(), torch.as_tensor(alpha, dtype=torch.float32).cuda(),
                     torch.as_tensor(counts).cuda(), E)
    out_acc = torch.zeros((T, D), dtype=torch.float32, device="cuda")
    y_sorted = torch.empty((T * K, D), dtype=torch.float32, device="cuda")
    moe.grouped_swiglu(inp.x, pm["sorted_token"], pm["offsets"], pm["sorted_w"], inp.w_gate_up,
                       inp.w_down, T * K, out_acc=out_acc, y_sorted=y_sorted)
    torch.cuda.synchronize()
    alpha32 = alpha.astype(np.float32).astype(np.float64)  # the weights the GPU was given
    y_ref = oracle_outputs(oracle_mod, inp, idx, alpha32, np.arange(T))
    rms = np.sqrt(np.mean(y_ref ** 2))
    err = np.abs(_np(out_acc).astype(np.float64) - y_ref).max()
    assert err <= Y_TOL * rms, (err, rms)
    # the fp32 per-row outputs, combined in slot order into bf16, give the same result
    y2 = moe.combine(T, D, K, y_sorted=y_sorted, slot_to_row=pm["slot_to_row"])
    err2, _, used = output_error(_np(y2.float()).astype(np.float64), y_ref)
    assert used <= 1.0, (err2, rms, used)


def test_grouped_swiglu_dense_identity(moe, oracle_mod):
    """E = 1, identity rows, weight 1: a dense SwiGLU FFN over all tokens."""
    cfg = LayerConfig("d", T=130, D=256, E=1, K=1, f=256, seed=12)
    inp = make_inputs(cfg).to("cuda")
    off = torch.tensor([0, cfg.T], dtype=torch.int32, device="cuda")
    out_acc = torch.zeros((cfg.T, cfg.D), dtype=torch.float32, device="cuda")
    moe.grouped_swiglu(inp.x, None, off, None, inp.w_gate_up, inp.w_down, cfg.T, out_acc=out_acc)
    torch.cuda.synchronize()
    y_ref = oracle_outputs(oracle_mod, inp, np.zeros((cfg.T, 1), np.int32),
                           np.ones((cfg.T, 1)), np.arange(cfg.T))
    rms = np.sqrt(np.mean(y_ref ** 2))
    assert np.abs(_np(out_acc) - y_ref).max() <= Y_TOL * rms


# ------------------------------------------------------------------ whole layer


@pytest.mark.parametrize("name", sorted(SMALL_LAYERS))
def test_layer_matches_oracle(moe, oracle_mod, name):
    inp = make_inputs(SMALL_LAYERS[name]).to("cuda")
    _, y, idx, w, _ = _run_layer(moe, inp)
    rep = check_layer(oracle_mod, inp, y, _np(idx), _np(w))
    print(name, rep)


# decode (its last wave's gate_up tiles), deep_gate_up, decode_concentrated (every tile) and
# single_token (weights on M) cut gate_up tiles into K slices: the slices' partial sums are
# added in slice order, so the fixed-order mode stays bit-for-bit repeatable
@pytest.mark.parametrize("name", ["tiny", "decode", "shared_small", "ragged_T", "deep_gate_up",
                                  "deep_down", "deep_shared", "shared_fused",
                                  "decode_concentrated", "single_token"])
def test_layer_deterministic_mode(moe, oracle_mod, name):
    inp = make_inputs(SMALL_LAYERS[name]).to("cuda")
    layer, y1, idx, w, _ = _run_layer(moe, inp, deterministic=True)
    y2 = layer(inp.x)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    check_layer(oracle_mod, inp, y1, _np(idx), _np(w))


def test_layer_zero_input(moe):
    cfg = LayerConfig("z", T=16, D=256, E=16, K=4, f=128, f_s=128)
    inp = make_inputs(cfg).to("cuda")
    inp.x = torch.zeros_like(inp.x)
    _, y, idx, w, _ = _run_layer(moe, inp)
    assert torch.count_nonzero(y) == 0
    assert _np(idx).tolist() == [[0, 1, 2, 3]] * 16
    np.testing.assert_allclose(_np(w), 0.25)


def test_layer_empty_batch(moe):
    cfg = LayerConfig("e", T=0, D=256, E=16, K=4, f=128)
    inp = make_inputs(cfg).to("cuda")
    layer = moe.MoELayer.from_inputs(inp)
    y = layer(inp.x)
    torch.cuda.synchronize()
    assert y.shape == (0, 256)


def test_layer_cuda_graph_replay(moe):
    inp = make_inputs(CONFIGS["decode"]).to("cuda")
    layer = moe.MoELayer.from_inputs(inp)
    ref = layer(inp.x).clone()
    out = torch.empty_like(ref)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        layer(inp.x, out=out)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        layer(inp.x, out=out)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    diff = (out.float() - ref.float()).abs().max().item()
    assert diff <= 1e-2 * ref.float().pow(2).mean().sqrt().item()


def test_rejects_bad_arguments(moe):
    inp = make_inputs(CONFIGS["tiny"]).to("cuda")
    with pytest.raises(moe.MoEError):
        moe.route(inp.x, inp.w_router, 17)            # K > E
    odd = torch.empty(inp.x.numel() + 1, dtype=torch.bfloat16, device="cuda")[1:].view_as(inp.x)
    with pytest.raises(moe.MoEError):
        moe.route(odd, inp.w_router, 4)                # misaligned
    layer = moe.MoELayer.from_inputs(inp)
    with pytest.raises(moe.MoEError):
        layer(torch.empty((4, 200), dtype=torch.bfloat16, device="cuda"))  # D mismatch


# ------------------------------------------------------------------ full-size layers


def _sample_tokens(T, idx, n_random=24, seed=0, tile_rows=128):
    """Tokens to check element by element on a multi-GB layer: for every expert hit, the
    tokens of its first and last row (rows are in ascending token order within a group);
    in the hottest group, the tokens on both sides of every tile_rows boundary (the
    tokens-on-M tile height; the CTA pairs' 256-row tiles fall on every other one); the
    first and last 6 tokens; 24 random ones."""
    rng = np.random.default_rng(seed)
    K = idx.shape[1]
    flat = idx.reshape(-1)
    tok = np.repeat(np.arange(T), K)
    order = np.argsort(flat, kind="stable")
    se, st = flat[order], tok[order]
    starts = np.r_[0, np.nonzero(np.diff(se))[0] + 1]
    ends = np.r_[starts[1:], len(se)] - 1
    pick = set(st[starts].tolist()) | set(st[ends].tolist())
    hot = int(np.bincount(flat).argmax())
    hot_rows = st[se == hot]
    for b in range(tile_rows, len(hot_rows), tile_rows):
        pick |= {int(hot_rows[b - 1]), int(hot_rows[b])}
    pick |= set(range(min(T, 6))) | set(range(max(0, T - 6), T))
    pick |= set(rng.choice(T, size=min(T, n_random), replace=False).tolist())
    return np.array(sorted(pick), dtype=np.int64)


@pytest.mark.slow
@pytest.mark.parametrize("name", ["prefill", "finegrained", "zipf@T1", "zipf@T16", "zipf@T128",
                                  "zipf@T1024", "zipf@T16384"])
def test_full_size_layer(moe, oracle_mod, name):
    cfg = CONFIGS[name]
    inp = make_inputs(cfg, device="cuda")
    _, y, idx, w, counts = _run_layer(moe, inp)
    gi = _np(idx)
    toks = _sample_tokens(cfg.T, gi)
    rep = check_layer(oracle_mod, inp, y, gi, _np(w), tokens=toks)
    np.testing.assert_array_equal(_np(counts), np.bincount(gi.reshape(-1), minlength=cfg.E))
    hit = np.unique(gi)
    covered = np.unique(gi[toks])
    # every expert hit has at least its first and last row checked element by element
    assert np.array_equal(covered, hit)
    print(f"{name}: {len(toks)} tokens checked, {len(hit)} groups, bound used "
          f"{rep['bound_used']:.3f}, near ties {rep['near_tie']}, differing sets "
          f"{rep['differing']}, max|dy| {rep['y_err']:.3e} ({rep['y_rel']:.2e} x RMS)")


# ------------------------------------------------------------------ router variants, residual


VARIANTS = [
    dict(score="sigmoid"),
    dict(score="sigmoid", select_bias=True),
    dict(score="softmax", select_bias=True),
    dict(score="softmax", bf16_weights=True),
    dict(score="sigmoid", select_bias=True, bf16_weights=True),
]


def _variant(cfg, v):
    sb = None
    if v.get("select_bias"):
        g = torch.Generator().manual_seed(21)
        sb = (0.05 * torch.randn(cfg.E, generator=g)).float().cuda()
    return dict(score=v.get("score", "softmax"), select_bias=sb,
                bf16_weights=bool(v.get("bf16_weights", False)))


@pytest.mark.parametrize("vi", range(len(VARIANTS)))
@pytest.mark.parametrize("name", ["decode", "tc_router_shared", "single_token"])
def test_route_variants(moe, oracle_mod, name, vi):
    cfg = SMALL_LAYERS[name]
    inp = make_inputs(cfg).to("cuda")
    v = _variant(cfg, VARIANTS[vi])
    idx, w, counts, sg = moe.route(inp.x, inp.w_router, cfg.K, inp.logit_bias, inp.w_shared_gate,
                                   **v)
    torch.cuda.synchronize()
    orc = oracle_mod.route(inp.x, inp.w_router, cfg.K, inp.logit_bias, inp.w_shared_gate,
                           v["score"], v["select_bias"], v["bf16_weights"])
    check_route(orc, _np(idx), _np(w), _np(counts), select_bias=v["select_bias"],
                bf16_weights=v["bf16_weights"])


def test_route_sigmoid_worked_example(moe):
    """The worked example in its own form: sigmoid affinities 0.9 and 0.6 win and are
    renormalised to 0.6 and 0.4; a selection bias of 0.35 on the 0.3 expert makes it win
    the second slot while the weights still use the raw scores (0.9/1.2, 0.3/1.2)."""
    s = np.array([0.2, 0.9, 0.3, 0.1, 0.6, 0.05, 0.05, 0.05])
    x = torch.zeros((2, 128), dtype=torch.bfloat16, device="cuda")
    w_r = torch.zeros((8, 128), dtype=torch.bfloat16, device="cuda")
    bias = torch.tensor(np.log(s / (1 - s)), dtype=torch.float32, device="cuda")
    idx, w, _, _ = moe.route(x, w_r, 2, bias, score="sigmoid")
    torch.cuda.synchronize()
    assert _np(idx).tolist() == [[1, 4]] * 2
    np.testing.assert_allclose(_np(w), [[0.6, 0.4]] * 2, atol=1e-6)
    sb = torch.zeros(8, dtype=torch.float32, device="cuda")
    sb[2] = 0.35
    idx, w, _, _ = moe.route(x, w_r, 2, bias, score="sigmoid", select_bias=sb)
    torch.cuda.synchronize()
    assert _np(idx).tolist() == [[1, 2]] * 2
    np.testing.assert_allclose(_np(w), [[0.75, 0.25]] * 2, atol=1e-6)


@pytest.mark.parametrize("det", [False, True])
@pytest.mark.parametrize("vi", [0, 2, 4])
@pytest.mark.parametrize("name", ["tiny", "tc_router_shared", "shared_fused"])
def test_layer_variants_with_residual(moe, oracle_mod, name, vi, det):
    cfg = SMALL_LAYERS[name]
    inp = make_inputs(cfg).to("cuda")
    v = _variant(cfg, VARIANTS[vi])
    g = torch.Generator().manual_seed(31)
    h = torch.randn((cfg.T, cfg.D), generator=g).to(torch.bfloat16).cuda()
    layer = moe.MoELayer.from_inputs(inp, deterministic=det, **v)
    idx = torch.empty((cfg.T, cfg.K), dtype=torch.int32, device="cuda")
    w = torch.empty((cfg.T, cfg.K), dtype=torch.float32, device="cuda")
    y = layer(inp.x, topk_idx=idx, topk_w=w, residual=h)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    rep = check_layer(oracle_mod, inp, y, _np(idx), _np(w), residual=h, **v)
    print(name, VARIANTS[vi], det, rep)
