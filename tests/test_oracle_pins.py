"""Pins of the CPU oracle to facts fixed outside it: values the pages print, closed forms,
special cases that reduce to library routines, and brute force on tiny inputs.

Each test would fail on a plausible slip in the oracle: a dropped term (the up projection,
the routing weight, the shared expert), a wrong sign (SiLU, sigmoid), a wrong index or a
swapped operand (gate vs up rows, a transposed down matrix), a wrong renormalisation set,
or ties broken the wrong way.
"""
import math

import numpy as np
import pytest
import scipy.special
import torch

from conftest import golden, size_bytes

from workloads import LayerConfig, crafted_routing, make_inputs, random_routing


def _bf16(a) -> torch.Tensor:
    return torch.as_tensor(np.asarray(a), dtype=torch.float32).to(torch.bfloat16)


def _f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).numpy()


# ---------------------------------------------------------------- router


def test_renorm_worked_example(oracle_mod):
    """The pages' E=5, k=2 example: scores (.., 0.90, .., .., 0.60) -> weights 0.60 / 0.40.
    With x = 0 the logits equal the bias, so a bias of ln(score) makes p proportional to the
    scores and the renormalised top-2 weights are score / (0.90 + 0.60)."""
    g = golden("renorm_worked_example.txt")
    E, K = int(g["E"]), int(g["K"])
    scores = np.array([float(g[f"score {i}"]) for i in range(1, E + 1)])
    x = torch.zeros((1, 8), dtype=torch.bfloat16)
    w_r = torch.zeros((E, 8), dtype=torch.bfloat16)
    r = oracle_mod.route(x, w_r, K, logit_bias=np.log(scores))
    assert list(r["idx"][0]) == [1, 4]          # experts 2 and 5, 1-based, by descending p
    np.testing.assert_allclose(r["alpha"][0], [float(g["weight 2"]), float(g["weight 5"])],
                               rtol=0, atol=1e-12)
    assert r["alpha"][0].sum() == pytest.approx(float(g["weight_sum"]), abs=1e-15)


def test_sigmoid_worked_example(oracle_mod):
    """The worked example exactly as the page states it: sigmoid affinities (x = 0 and a
    logit bias of logit(score) make s_i equal the printed scores), top-2, weights
    0.90/1.50 = 0.60 and 0.40."""
    g = golden("renorm_worked_example.txt")
    E, K = int(g["E"]), int(g["K"])
    scores = np.array([float(g[f"score {i}"]) for i in range(1, E + 1)])
    x = torch.zeros((1, 8), dtype=torch.bfloat16)
    w_r = torch.zeros((E, 8), dtype=torch.bfloat16)
    r = oracle_mod.route(x, w_r, K, logit_bias=np.log(scores / (1 - scores)), score="sigmoid")
    assert list(r["idx"][0]) == [1, 4]
    np.testing.assert_allclose(r["probs"][0], scores, rtol=0, atol=1e-15)
    np.testing.assert_allclose(r["alpha"][0], [float(g["weight 2"]), float(g["weight 5"])],
                               rtol=0, atol=1e-12)


def test_selection_only_bias(oracle_mod):
    """"1.6 混合专家（MoE）", section 三 (DeepSeek-V3 bias method): the bias b_i is added to the
    affinity for selection only; the weights normalise the raw s_i.  With s = (0.2, 0.9,
    0.3, 0.1, 0.6) and b = 0.55 on expert 3 (1-based) the keys are (0.2, 0.9, 0.85, 0.1,
    0.6): experts 2 and 3 win, weighted 0.9/1.2 = 0.75 and 0.3/1.2 = 0.25 -- not by the
    biased keys (0.9/1.75) and not the unbiased winners (2 and 5)."""
    s = np.array([0.2, 0.9, 0.3, 0.1, 0.6])
    b = np.array([0.0, 0.0, 0.55, 0.0, 0.0])
    x = torch.zeros((1, 8), dtype=torch.bfloat16)
    w_r = torch.zeros((5, 8), dtype=torch.bfloat16)
    r = oracle_mod.route(x, w_r, 2, logit_bias=np.log(s / (1 - s)), score="sigmoid",
                         select_bias=b)
    assert list(r["idx"][0]) == [1, 2]
    np.testing.assert_allclose(r["alpha"][0], [0.75, 0.25], rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["gap"][0], 0.85 - 0.6, atol=1e-12)


@pytest.mark.parametrize("with_bias", [False, True])
def test_sigmoid_router_matches_library(oracle_mod, with_bias):
    """Sigmoid scores = scipy expit of the logits; selection = stable sort of the keys
    (scores + selection bias); weights = selected raw scores over their sum."""
    x, w = _random_router(23, 128, 32, seed=9)
    b = np.linspace(-0.3, 0.3, 32) if with_bias else None
    r = oracle_mod.route(x, w, 6, score="sigmoid", select_bias=b)
    s = scipy.special.expit(_f64(x) @ _f64(w).T)
    np.testing.assert_allclose(r["probs"], s, rtol=1e-13)
    key = s + (b if with_bias else 0.0)
    order = np.argsort(-key, axis=1, kind="stable")[:, :6]
    np.testing.assert_array_equal(r["idx"], order)
    sel = np.take_along_axis(s, order, axis=1)
    np.testing.assert_allclose(r["alpha"], sel / sel.sum(1, keepdims=True), rtol=1e-12)


def test_softmax_with_selection_bias(oracle_mod):
    """Softmax scores with a selection-only bias: keys = p + b, weights from p alone."""
    x, w = _random_router(15, 64, 16, seed=10)
    b = np.linspace(0.0, 0.2, 16)
    r = oracle_mod.route(x, w, 4, select_bias=b)
    p = scipy.special.softmax(_f64(x) @ _f64(w).T, axis=1)
    order = np.argsort(-(p + b), axis=1, kind="stable")[:, :4]
    np.testing.assert_array_equal(r["idx"], order)
    sel = np.take_along_axis(p, order, axis=1)
    np.testing.assert_allclose(r["alpha"], sel / sel.sum(1, keepdims=True), rtol=1e-12)


def test_bf16_routing_weights(oracle_mod):
    """"MoE", section 2: the renormalised fp32 weights are cast back to the model dtype --
    the fp64 weights rounded to fp32 and then to bf16 by torch (round to nearest even)."""
    x, w = _random_router(31, 128, 24, seed=11)
    ref = oracle_mod.route(x, w, 5)
    r = oracle_mod.route(x, w, 5, bf16_weights=True)
    np.testing.assert_array_equal(r["idx"], ref["idx"])
    want = torch.tensor(ref["alpha"]).to(torch.float32).to(torch.bfloat16).to(torch.float64)
    np.testing.assert_array_equal(r["alpha"], want.numpy())


def test_residual_is_added(oracle_mod):
    """"MoE", section 4: h_out = h + y_MoE."""
    cfg = LayerConfig("res", T=6, D=64, E=4, K=2, f=32)
    inp = make_inputs(cfg)
    h = (torch.randn((6, 64), generator=torch.Generator().manual_seed(3))).to(torch.bfloat16)
    _, y = oracle_mod.layer(inp)
    _, yh = oracle_mod.layer(inp, residual=h)
    np.testing.assert_allclose(yh, y + _f64(h), rtol=0, atol=0)


def _random_router(T, D, E, seed):
    gen = torch.Generator().manual_seed(seed)
    x = torch.randn((T, D), generator=gen).to(torch.bfloat16)
    w = (torch.randn((E, D), generator=gen) / math.sqrt(D)).to(torch.bfloat16)
    return x, w


def test_full_k_is_softmax(oracle_mod):
    """K = E: the renormalisation is the identity, so the weights are the plain softmax of
    the logits (scipy), listed in descending order."""
    x, w = _random_router(9, 64, 6, seed=1)
    r = oracle_mod.route(x, w, 6)
    logits = _f64(x) @ _f64(w).T
    sm = scipy.special.softmax(logits, axis=1)
    np.testing.assert_allclose(r["probs"], sm, rtol=1e-12, atol=0)
    got = np.zeros_like(sm)
    np.put_along_axis(got, r["idx"].astype(np.int64), r["alpha"], axis=1)
    np.testing.assert_allclose(got, sm, rtol=1e-12, atol=0)
    assert np.all(np.isinf(r["gap"]))


@pytest.mark.parametrize("T,D,E,K", [(40, 128, 16, 4), (17, 64, 64, 8), (5, 256, 256, 10)])
def test_topk_matches_stable_sort(oracle_mod, T, D, E, K):
    """TopK against a library stable sort of the softmax (descending, equal -> lower index);
    alpha against the selected probabilities over their sum; gap against the sorted probs."""
    x, w = _random_router(T, D, E, seed=T)
    r = oracle_mod.route(x, w, K)
    probs = scipy.special.softmax(_f64(x) @ _f64(w).T, axis=1)
    order = np.argsort(-probs, axis=1, kind="stable")
    np.testing.assert_array_equal(r["idx"], order[:, :K])
    sel = np.take_along_axis(probs, order[:, :K], axis=1)
    np.testing.assert_allclose(r["alpha"], sel / sel.sum(1, keepdims=True), rtol=1e-12)
    srt = -np.sort(-probs, axis=1)
    np.testing.assert_allclose(r["gap"], srt[:, K - 1] - srt[:, K], rtol=1e-9, atol=1e-15)


def test_topk_ties_go_to_lower_index(oracle_mod):
    x = torch.zeros((1, 8), dtype=torch.bfloat16)
    w_r = torch.zeros((6, 8), dtype=torch.bfloat16)
    bias = np.array([0.0, 1.0, 0.5, 1.0, 1.0, 0.5])
    r = oracle_mod.route(x, w_r, 4, logit_bias=bias)
    assert list(r["idx"][0]) == [1, 3, 4, 2]
    assert r["gap"][0] == 0.0


def test_bias_enters_before_softmax(oracle_mod):
    """A logit bias shifts the probabilities like an extra logit term (scipy softmax)."""
    x, w = _random_router(7, 64, 12, seed=3)
    bias = np.linspace(-2.0, 3.0, 12)
    r = oracle_mod.route(x, w, 3, logit_bias=bias)
    probs = scipy.special.softmax(_f64(x) @ _f64(w).T + bias, axis=1)
    np.testing.assert_allclose(r["probs"], probs, rtol=1e-12)


def test_shared_gate_is_sigmoid(oracle_mod):
    x, w = _random_router(11, 64, 4, seed=4)
    ws = (torch.randn(64, generator=torch.Generator().manual_seed(5)) / 8).to(torch.bfloat16)
    r = oracle_mod.route(x, w, 2, w_shared_gate=ws)
    np.testing.assert_allclose(r["shared_gate"], scipy.special.expit(_f64(x) @ _f64(ws)),
                               rtol=1e-13)


# ---------------------------------------------------------------- experts


def _torch_swiglu(x, w_gu, w_d):
    """Library SwiGLU in float64: W_d (silu(W_g x) * W_u x), gate = first half of rows."""
    x64, gu, d = x.to(torch.float64), w_gu.to(torch.float64), w_d.to(torch.float64)
    f = gu.shape[0] // 2
    return (torch.nn.functional.silu(x64 @ gu[:f].T) * (x64 @ gu[f:].T)) @ d.T


def test_single_expert_is_dense_swiglu(oracle_mod):
    """E = 1, K = 1: alpha = 1 and the layer is one dense SwiGLU FFN (torch silu, float64).
    Non-square shapes (D=64, f=48) catch a transposed operand."""
    cfg = LayerConfig("e1", T=10, D=64, E=1, K=1, f=48)
    inp = make_inputs(cfg)
    r, y = oracle_mod.layer(inp)
    assert np.all(r["alpha"] == 1.0) and np.all(r["idx"] == 0)
    ref = _torch_swiglu(inp.x, inp.w_gate_up[0], inp.w_down[0]).numpy()
    np.testing.assert_allclose(y, ref, rtol=1e-10, atol=1e-12)


def test_shared_expert_matches_library(oracle_mod):
    """One routed expert plus a shared expert of another width (f_s = 32 != f = 48):
    y = SwiGLU_0(x) + sigmoid(w_s . x) SwiGLU_s(x)  (torch silu/sigmoid, float64)."""
    cfg = LayerConfig("e1s", T=6, D=64, E=1, K=1, f=48, f_s=32)
    inp = make_inputs(cfg)
    r, y = oracle_mod.layer(inp)
    x64 = inp.x.to(torch.float64)
    gate = torch.sigmoid(x64 @ inp.w_shared_gate.to(torch.float64))
    ref = _torch_swiglu(inp.x, inp.w_gate_up[0], inp.w_down[0]) + \
        gate[:, None] * _torch_swiglu(inp.x, inp.w_shared_gate_up, inp.w_shared_down)
    np.testing.assert_allclose(y, ref.numpy(), rtol=1e-10, atol=1e-12)


def test_routed_sum_matches_library(oracle_mod):
    """Several experts: y_t = sum_k alpha_k SwiGLU_{e_k}(x_t), each term by torch."""
    cfg = LayerConfig("small", T=5, D=64, E=6, K=3, f=32)
    inp = make_inputs(cfg)
    r, y = oracle_mod.layer(inp)
    ref = np.zeros_like(y)
    for t in range(cfg.T):
        for k in range(cfg.K):
            e = int(r["idx"][t, k])
            ref[t] += r["alpha"][t, k] * _torch_swiglu(inp.x[t:t + 1], inp.w_gate_up[e],
                                                       inp.w_down[e]).numpy()[0]
    np.testing.assert_allclose(y, ref, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("shared", [False, True])
def test_dense_masked_equals_sparse(oracle_mod, shared):
    """Brute force: every expert evaluated on every token and weighted by alpha (0 off the
    selection) equals the sparse sum over the K selected experts."""
    cfg = LayerConfig("bf", T=12, D=64, E=8, K=3, f=32, f_s=16 if shared else 0)
    inp = make_inputs(cfg)
    r, y = oracle_mod.layer(inp)
    dense = np.zeros((cfg.T, cfg.E))
    np.put_along_axis(dense, r["idx"].astype(np.int64), r["alpha"], axis=1)
    yd = oracle_mod.dense_masked(inp.x, dense, inp.w_gate_up, inp.w_down,
                                 inp.w_shared_gate_up, inp.w_shared_down, r["shared_gate"])
    np.testing.assert_allclose(y, yd, rtol=1e-12, atol=1e-13)
    assert np.abs(y).max() > 0.1


def test_zero_input_gives_zero(oracle_mod):
    cfg = LayerConfig("z", T=4, D=64, E=8, K=2, f=32, f_s=16)
    inp = make_inputs(cfg)
    inp.x = torch.zeros_like(inp.x)
    r, y = oracle_mod.layer(inp)
    assert np.all(y == 0.0)
    np.testing.assert_allclose(r["shared_gate"], 0.5)


def test_token_subset_matches_full(oracle_mod):
    cfg = LayerConfig("sub", T=9, D=64, E=8, K=2, f=32)
    inp = make_inputs(cfg)
    r, y = oracle_mod.layer(inp)
    toks = np.array([8, 0, 5], np.int32)
    _, ys = oracle_mod.layer(inp, tokens=toks)
    np.testing.assert_array_equal(ys, y[toks])


# ---------------------------------------------------------------- permutation


@pytest.mark.parametrize("T,E,K", [(0, 8, 2), (1, 4, 4), (37, 16, 4), (300, 64, 8)])
def test_permute_matches_stable_sort(oracle_mod, T, E, K):
    """Rows grouped by expert, tokens ascending inside a group: a library stable argsort of
    the flattened expert ids; counts = bincount; slot_to_row inverts the order."""
    idx = random_routing(T, E, K, seed=T).numpy()
    p = oracle_mod.permute(idx, E)
    flat = idx.reshape(-1)
    order = np.argsort(flat, kind="stable")
    np.testing.assert_array_equal(p["sorted_slot"], order)
    np.testing.assert_array_equal(p["sorted_token"], order // K)
    np.testing.assert_array_equal(p["counts"], np.bincount(flat, minlength=E))
    np.testing.assert_array_equal(p["offsets"], np.concatenate([[0], np.cumsum(p["counts"])]))
    inv = np.empty_like(order)
    inv[order] = np.arange(T * K)
    np.testing.assert_array_equal(p["slot_to_row"], inv)


def test_permute_rejects_out_of_range(oracle_mod):
    with pytest.raises(ValueError):
        oracle_mod.permute(np.array([[0, 9]], np.int32), 4)


# ---------------------------------------------------------------- closed forms


def test_closed_forms_of_the_pages(oracle_mod):
    """Section 2.1 / 3 / 7 / 10 numbers of the 35B-A3B layer, with F counted from the rows
    the oracle's permutation assigns and U from its counts, under crafted uniform (2 rows
    per expert) and concentrated (64 rows on 8 experts) routings."""
    acc = oracle_mod.accounting
    g = golden("closed_forms.txt")
    d, f, E, k, B = (int(g[n]) for n in ("d", "f", "E", "k", "B"))
    Ne = acc.expert_params(d, f)
    assert Ne == int(g["N_e"])
    assert 2 * Ne == size_bytes(g["N_e_bytes_bf16"])
    assert acc.expert_weight_bytes(E, d, f) == size_bytes(g["all_routed_bytes"])
    assert acc.expert_weight_bytes(k, d, f) == size_bytes(g["one_token_bytes"])

    res = {}
    for kind in ("uniform", "concentrated"):
        p = oracle_mod.permute(crafted_routing(B, E, k, kind).numpy(), E)
        U = acc.distinct_experts(p["counts"])
        res[kind] = (acc.expert_flops(p["counts"], d, f), acc.expert_weight_bytes(U, d, f),
                     p["counts"][p["counts"] > 0])
    (Fu, Ru, cu), (Fc, Rc, cc) = res["uniform"], res["concentrated"]
    assert Fu == Fc == 2 * Ne * B * k == 3_221_225_472
    assert float(g["F_expert"].split()[0]) == round(Fu / 1e9, 2)
    assert Ru == size_bytes(g["R_uniform"]) and Rc == size_bytes(g["R_concentrated"])
    assert Ru / Rc == float(g["ratio"])
    assert set(cu) == {int(g["rows_uniform"])} and set(cc) == {int(g["rows_concentrated"])}
    L = int(g["layers"])
    assert L * Ru == size_bytes(g["layers_uniform"])
    assert L * Rc == size_bytes(g["layers_concentrated"])
    # section 10: the read volume depends on U, not on the batch
    p32 = oracle_mod.permute(crafted_routing(int(g["selftest_B"]), E, k, "uniform").numpy(), E)
    U32 = acc.distinct_experts(p32["counts"])
    assert U32 == E and acc.expert_weight_bytes(U32, d, f) == size_bytes(g["selftest_bytes"])


def test_granularity_invariant(oracle_mod):
    acc = oracle_mod.accounting
    g = golden("granularity.txt")

    def parse(s):
        v = s.split()
        return dict(zip(v[0::2], map(int, v[1::2])))

    for pair in ("pair1", "pair2"):
        a, b, d = parse(g[f"{pair}_a"]), parse(g[f"{pair}_b"]), int(g[f"{pair}_d"])
        assert a["E"] == 2 * b["E"] or b["E"] == 4 * a["E"]
        assert acc.routed_params(a["E"], d, a["f"]) == acc.routed_params(b["E"], d, b["f"])
        assert acc.flops_per_token(a["k"], d, a["f"]) == acc.flops_per_token(b["k"], d, b["f"])
    # and on real routings: the oracle's counts give the same layer FLOPs for both shapes
    a, b = parse(g["pair2_a"]), parse(g["pair2_b"])
    T = 16
    for s in (a, b):
        p = oracle_mod.permute(random_routing(T, s["E"], s["k"], seed=7).numpy(), s["E"])
        s["F"] = acc.expert_flops(p["counts"], int(g["pair2_d"]), s["f"])
    assert a["F"] == b["F"] == T * acc.flops_per_token(a["k"], int(g["pair2_d"]), a["f"])


def test_shared_expert_flops_formula(oracle_mod):
    """Section 4: F = 2 m N_s + 2 sum t_e N_e.  Pinned through expert_flops (itself pinned
    to the printed 3.22 GFLOPs): a shared expert is one more group that receives all m
    tokens, and -- an expert's FLOPs being linear in its width -- a shared expert of width
    2f is two such groups of width f.  Counts come from the oracle's permutation of a real
    routing; without a shared expert the layer is its routed experts alone."""
    acc = oracle_mod.accounting
    m, E, K, d, f = 24, 16, 4, 64, 32
    counts = oracle_mod.permute(random_routing(m, E, K, seed=5).numpy(), E)["counts"]
    routed = [int(c) for c in counts]
    assert acc.layer_flops(routed, m=m, d=d, f=f, f_s=0) == acc.expert_flops(routed, d, f)
    assert acc.layer_flops(routed, m=m, d=d, f=f, f_s=f) == acc.expert_flops(routed + [m], d, f)
    assert acc.layer_flops(routed, m=m, d=d, f=f, f_s=2 * f) == \
        acc.expert_flops(routed + [m, m], d, f)
    # the shared term grows with every token, the routed one with the routed rows only
    assert acc.layer_flops(routed, m=2 * m, d=d, f=f, f_s=f) - \
        acc.layer_flops(routed, m=m, d=d, f=f, f_s=f) == acc.expert_flops([m], d, f)


# ---------------------------------------------------------------- expert capacity


def _pairs(text):
    return np.array([[int(v) for v in p.split()] for p in text.split(",")], dtype=np.int32)


def test_capacity_values(oracle_mod):
    """C = max(min_capacity, ceil(cf * T * K / E)) against hand-worked values for the
    configuration the pages print (capacity_factor 1.25, min_capacity 4)."""
    g = golden("capacity.txt")
    cf, mn = float(g["capacity_factor"]), int(g["min_capacity"])
    n = 0
    for key, val in g.items():
        if key.startswith("cap "):
            T, K, E = map(int, key.split()[1:])
            assert oracle_mod.expert_capacity(T, K, E, cf, mn) == int(val), key
            n += 1
        elif key.startswith("cap0 "):
            T, K, E = map(int, key.split()[1:])
            assert oracle_mod.expert_capacity(T, K, E, 1.0, 0) == int(val), key
    assert n == 5


def test_capacity_keep_worked_example(oracle_mod):
    g = golden("capacity.txt")
    idx, keep = _pairs(g["route"]), _pairs(g["keep"]).astype(bool)
    np.testing.assert_array_equal(oracle_mod.capacity_keep(idx, 3, 2), keep)


@pytest.mark.parametrize("T,E,K,C", [(50, 8, 3, 4), (200, 16, 4, 30), (64, 256, 8, 2), (7, 4, 4, 0)])
def test_capacity_keep_is_first_c_in_token_order(oracle_mod, T, E, K, C):
    """Brute force: for every expert, the kept assignments are exactly the first C tokens
    (ascending) that chose it."""
    idx = random_routing(T, E, K, seed=T + C).numpy()
    keep = oracle_mod.capacity_keep(idx, E, C)
    for e in range(E):
        toks = [t for t in range(T) if e in idx[t]]
        kept = [t for t in range(T) for k in range(K) if idx[t, k] == e and keep[t, k]]
        assert kept == toks[:C], e


def test_capacity_drops_whole_tokens_to_zero(oracle_mod):
    """Every token picks experts 0..K-1: with C = 3 only tokens 0, 1, 2 keep anything.  The
    later tokens get y = 0 exactly (they pass through the residual alone); the first three
    are unchanged from the dropless layer."""
    cfg = LayerConfig("cap", T=9, D=64, E=8, K=2, f=32)
    inp = make_inputs(cfg)
    big = torch.zeros(8)
    big[:2] = 30.0   # every token routes to experts 0 and 1
    inp.logit_bias = big
    r0, y0 = oracle_mod.layer(inp)
    r, y = oracle_mod.layer(inp, capacity=3)
    assert np.all(np.sort(r["idx"], axis=1) == [0, 1])
    assert np.all(y[3:] == 0.0)
    np.testing.assert_array_equal(y[:3], y0[:3])


def test_capacity_keeps_weights_unrenormalised(oracle_mod):
    """A token that loses one of its two experts keeps alpha_kept * E_kept(x) -- the surviving
    weight is not renormalised (torch float64 SwiGLU)."""
    cfg = LayerConfig("cap", T=5, D=64, E=16, K=2, f=48)
    inp = make_inputs(cfg)
    bias = torch.zeros(16)
    bias[0] = 30.0   # expert 0 is every token's first choice; C = 1 leaves it to token 0
    inp.logit_bias = bias
    r, y = oracle_mod.layer(inp, capacity=1)
    checked = 0
    for t in range(1, cfg.T):
        k0 = int(np.where(r["idx"][t] == 0)[0][0])
        assert not r["keep"][t, k0]
        if not r["keep"][t, 1 - k0]:
            continue  # its second expert was already taken by an earlier token
        e2 = int(r["idx"][t, 1 - k0])
        ref = r["alpha"][t, 1 - k0] * _torch_swiglu(inp.x[t:t + 1], inp.w_gate_up[e2],
                                                    inp.w_down[e2]).numpy()[0]
        np.testing.assert_allclose(y[t], ref, rtol=1e-10, atol=1e-12)
        checked += 1
    assert checked >= 2


def test_capacity_at_or_above_every_group_is_dropless(oracle_mod):
    cfg = LayerConfig("cap", T=40, D=64, E=8, K=3, f=32, f_s=32, seed=4)
    inp = make_inputs(cfg)
    _, y0 = oracle_mod.layer(inp)
    _, y = oracle_mod.layer(inp, capacity=cfg.T)
    np.testing.assert_array_equal(y, y0)
