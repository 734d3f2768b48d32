"""Expert parallelism on one GPU: G ranks emulated in one process, each with its own tokens
and 1/G of the experts, the two all-to-all exchanges done by slicing and concatenating on
the device (the layer's phases run exactly as they would between G processes).  Every
rank's output must pass the layer's parity rules against the oracle on that rank's tokens,
with the full set of experts."""
import numpy as np
import pytest
import torch

from parity import check_layer
from workloads import LayerConfig, LayerInputs, make_inputs

pytestmark = pytest.mark.gpu


def _run_virtual(layers, xs):
    G = len(layers)
    sts = [l.dispatch(x) for l, x in zip(layers, xs)]
    # rank r receives row r of every source's count table, and the source's rows for r
    recv_counts = [torch.stack([sts[s].send_counts[r] for s in range(G)]) for r in range(G)]

    def seg(rows, splits, i):
        a = sum(splits[:i])
        return rows[a:a + splits[i]]

    recv_x = [torch.cat([seg(sts[s].x_sorted, sts[s].send_splits, r) for s in range(G)])
              for r in range(G)]
    y_ret = [layers[r].experts(recv_x[r], recv_counts[r]) for r in range(G)]
    recv_splits = [[sts[s].send_splits[r] for s in range(G)] for r in range(G)]
    # source s gets back, rank by rank, the rows it sent there
    y_back = [torch.cat([seg(y_ret[r], recv_splits[r], s) for r in range(G)]) for s in range(G)]
    outs = [layers[s].combine(sts[s], y_back[s]) for s in range(G)]
    torch.cuda.synchronize()
    return sts, outs


CASES = {
    "g2": (LayerConfig("ep_g2", T=96, D=256, E=16, K=4, f=128, seed=30), 2, [48, 48], None),
    "g4_shared_uneven": (LayerConfig("ep_g4", T=200, D=512, E=64, K=8, f=256, f_s=256, seed=31),
                         4, [40, 60, 50, 50], None),
    # every token prefers rank 0's experts: the other ranks receive nothing
    "g4_all_to_rank0": (LayerConfig("ep_hot", T=64, D=256, E=32, K=4, f=128, seed=32), 4,
                        [16, 16, 16, 16], "rank0"),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_expert_parallel_layer_matches_oracle(moe, oracle_mod, name):
    from top_routing_grouped_03_b200.ep import ExpertParallelLayer
    cfg, G, tokens, bias = CASES[name]
    inp = make_inputs(cfg).to("cuda")
    if bias == "rank0":
        b = torch.zeros(cfg.E, dtype=torch.float32)
        b[: cfg.E // G] = 30.0
        inp.logit_bias = b.cuda()
    El = cfg.E // G
    layers = [ExpertParallelLayer(r, G, inp.w_router, inp.w_gate_up[r * El:(r + 1) * El],
                                  inp.w_down[r * El:(r + 1) * El], cfg.K, inp.logit_bias,
                                  inp.w_shared_gate, inp.w_shared_gate_up, inp.w_shared_down)
              for r in range(G)]
    starts = np.cumsum([0] + tokens)
    xs = [inp.x[starts[r]:starts[r + 1]].contiguous() for r in range(G)]
    sts, outs = _run_virtual(layers, xs)
    if bias == "rank0":
        assert all(int(st.send_counts[1:].sum()) == 0 for st in sts)
    for r in range(G):
        sub = LayerInputs(LayerConfig(f"{cfg.name}_r{r}", T=tokens[r], D=cfg.D, E=cfg.E,
                                      K=cfg.K, f=cfg.f, f_s=cfg.f_s),
                          xs[r], inp.w_router, inp.w_gate_up, inp.w_down, inp.logit_bias,
                          inp.w_shared_gate, inp.w_shared_gate_up, inp.w_shared_down)
        rep = check_layer(oracle_mod, sub, outs[r], sts[r].topk_idx.cpu().numpy(),
                          sts[r].topk_w.cpu().numpy())
        print(name, "rank", r, rep)
