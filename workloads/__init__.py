"""Seeded synthetic workloads for the top-k MoE SwiGLU layer.

This module only draws inputs: it holds none of the layer's arithmetic, so both
the CPU oracle (``oracle/``) and the CUDA path (``top_routing_grouped_03_b200``)
can be fed the very same bf16 bits from here without sharing any computation.

Shapes follow the layers the source pages discuss:
  * "tiny":        T=64,   D=256,  E=16,  K=4,  f=128
  * "decode":      T=64,   D=2048, E=256, K=8,  f=512   (the Qwen3.6-35B-A3B-like layer of
                   "MoE 到底省了什么" §2.1/§3: N_e = 3*2048*512, B=64, k=8)
  * "prefill":     T=8192, D=4096, E=128, K=8,  f=1536  (the 128 x 1536 x top-8 shape of §4)
  * "finegrained": T=4096, D=4096, E=512, K=10, f=1024, plus one shared expert f_s=1024
                   (the 512-routed / top-10 / 1-shared layer of the "MoE" page §1.1)
  * "zipf":        the prefill shape with a Zipf(s=1.2) logit bias over a random expert
                   permutation, T in {1, 16, 128, 1024, 16384}

Recipe (fixed order, one generator): x ~ N(0,1); W_r ~ N(0,1/D); W_gate ~ N(0,1/D);
W_up ~ N(0,1/D); W_down ~ N(0,1/f); then, with a shared expert, w_s ~ N(0,1/D),
W_s_gate, W_s_up ~ N(0,1/D), W_s_down ~ N(0,1/f_s).  Every draw is fp32 from
``torch.randn`` scaled by the standard deviation and rounded to bf16 (round to nearest
even).  Weights are drawn expert by expert so memory stays bounded.

Routing regimes that need a logit bias (added to the router logits before the softmax):
  * "concentrated": +20 on the 8 experts ``randperm(E, seed 1)[:8]``, so every token
    picks that same set (U = 8 distinct experts).
  * "zipf": b_e = 2*ln(rank_e ** -1.2) = -2.4*ln(rank_e), ranks 1..E assigned by
    ``randperm(E, seed 2)``.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int
    D: int
    E: int
    K: int
    f: int
    f_s: int = 0            # 0: no shared expert
    routing: str = "natural"  # natural | concentrated | zipf
    seed: int = 0

    @property
    def has_shared(self) -> bool:
        return self.f_s > 0

    def with_tokens(self, T: int) -> "LayerConfig":
        return dataclasses.replace(self, T=T, name=f"{self.name.split('@')[0]}@T{T}")


CONFIGS = {
    "tiny": LayerConfig("tiny", T=64, D=256, E=16, K=4, f=128),
    "decode": LayerConfig("decode", T=64, D=2048, E=256, K=8, f=512),
    "decode_concentrated": LayerConfig("decode_concentrated", T=64, D=2048, E=256, K=8, f=512,
                                       routing="concentrated"),
    "prefill": LayerConfig("prefill", T=8192, D=4096, E=128, K=8, f=1536),
    "finegrained": LayerConfig("finegrained", T=4096, D=4096, E=512, K=10, f=1024, f_s=1024),
}
# the prefill layer's per-expert shape (512 rows per expert, D=4096, f=1536) with 32 experts:
# the same kernels and tiles on ~1.2 GB of weights, small enough for profiler captures
CONFIGS["prefill_e32"] = LayerConfig("prefill_e32", T=2048, D=4096, E=32, K=8, f=1536)
# the fine-grained layer's per-expert shape (~80 rows per expert, D=4096, f=f_s=1024, top-10,
# shared expert) with 64 experts and 512 tokens: 1.6 GB of weights, for profiler captures
CONFIGS["finegrained_e64"] = LayerConfig("finegrained_e64", T=512, D=4096, E=64, K=10, f=1024,
                                         f_s=1024)
# the fine-grained layer's router (T=4096, D=4096, E=512, K=10, shared gate) with narrow
# experts (f=f_s=128): the same router kernels on 1.6 GB of weights, for profiler captures
CONFIGS["finegrained_router"] = LayerConfig("finegrained_router", T=4096, D=4096, E=512, K=10,
                                            f=128, f_s=128)
# one token on the prefill/Zipf expert shape (D=4096, f=1536, top-8) with 16 experts: the
# few-token kernels on 0.6 GB of weights, for profiler captures
CONFIGS["zipf_e16@T1"] = LayerConfig("zipf_e16@T1", T=1, D=4096, E=16, K=8, f=1536)
ZIPF_TOKENS = (1, 16, 128, 1024, 16384)
for _t in ZIPF_TOKENS:
    CONFIGS[f"zipf@T{_t}"] = LayerConfig(f"zipf@T{_t}", T=_t, D=4096, E=128, K=8, f=1536,
                                         routing="zipf")


@dataclasses.dataclass
class LayerInputs:
    """bf16 tensors (uint16 bit patterns are ``t.view(torch.int16)``) and an fp32 bias."""
    cfg: LayerConfig
    x: torch.Tensor            # [T, D]
    w_router: torch.Tensor     # [E, D]
    w_gate_up: torch.Tensor    # [E, 2f, D]  rows [0,f) gate, [f,2f) up
    w_down: torch.Tensor       # [E, D, f]
    logit_bias: Optional[torch.Tensor] = None      # [E] fp32
    w_shared_gate: Optional[torch.Tensor] = None   # [D]
    w_shared_gate_up: Optional[torch.Tensor] = None  # [2f_s, D]
    w_shared_down: Optional[torch.Tensor] = None     # [D, f_s]

    def to(self, device) -> "LayerInputs":
        def mv(t):
            return None if t is None else t.to(device)
        return LayerInputs(self.cfg, mv(self.x), mv(self.w_router), mv(self.w_gate_up),
                           mv(self.w_down), mv(self.logit_bias), mv(self.w_shared_gate),
                           mv(self.w_shared_gate_up), mv(self.w_shared_down))


def _normal_bf16(gen: torch.Generator, shape, std: float, device) -> torch.Tensor:
    t = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch.bfloat16)


def routing_bias(cfg: LayerConfig) -> Optional[torch.Tensor]:
    """The fp32 logit bias of the routing regime (None for natural routing)."""
    E = cfg.E
    if cfg.routing == "natural":
        return None
    if cfg.routing == "concentrated":
        perm = torch.randperm(E, generator=torch.Generator().manual_seed(1))
        b = torch.zeros(E, dtype=torch.float32)
        b[perm[:8]] = 20.0
        return b
    if cfg.routing == "zipf":
        perm = torch.randperm(E, generator=torch.Generator().manual_seed(2))
        rank = torch.empty(E, dtype=torch.float64)
        rank[perm] = torch.arange(1, E + 1, dtype=torch.float64)
        return (2.0 * torch.log(rank ** -1.2)).to(torch.float32)
    raise ValueError(cfg.routing)


def make_inputs(cfg: LayerConfig, device="cpu", seed: Optional[int] = None) -> LayerInputs:
    """Draw one layer's inputs.  ``device='cpu'`` gives bits identical on every machine;
    ``device='cuda'`` draws with a seeded CUDA generator (same recipe, different stream of
    numbers) for the multi-GB layers."""
    seed = cfg.seed if seed is None else seed
    dev = torch.device(device)
    gen = torch.Generator(device=dev).manual_seed(seed)
    T, D, E, f = cfg.T, cfg.D, cfg.E, cfg.f
    x = _normal_bf16(gen, (T, D), 1.0, dev)
    w_r = _normal_bf16(gen, (E, D), 1.0 / math.sqrt(D), dev)
    w_gu = torch.empty((E, 2 * f, D), dtype=torch.bfloat16, device=dev)
    for e in range(E):                       # gate rows of every expert first ...
        w_gu[e, :f] = _normal_bf16(gen, (f, D), 1.0 / math.sqrt(D), dev)
    for e in range(E):                       # ... then the up rows
        w_gu[e, f:] = _normal_bf16(gen, (f, D), 1.0 / math.sqrt(D), dev)
    w_d = torch.empty((E, D, f), dtype=torch.bfloat16, device=dev)
    for e in range(E):
        w_d[e] = _normal_bf16(gen, (D, f), 1.0 / math.sqrt(f), dev)
    inp = LayerInputs(cfg, x, w_r, w_gu, w_d)
    b = routing_bias(cfg)
    inp.logit_bias = None if b is None else b.to(dev)
    if cfg.has_shared:
        fs = cfg.f_s
        inp.w_shared_gate = _normal_bf16(gen, (D,), 1.0 / math.sqrt(D), dev)
        gu = torch.empty((2 * fs, D), dtype=torch.bfloat16, device=dev)
        gu[:fs] = _normal_bf16(gen, (fs, D), 1.0 / math.sqrt(D), dev)
        gu[fs:] = _normal_bf16(gen, (fs, D), 1.0 / math.sqrt(D), dev)
        inp.w_shared_gate_up = gu
        inp.w_shared_down = _normal_bf16(gen, (D, fs), 1.0 / math.sqrt(fs), dev)
    return inp


def random_routing(T: int, E: int, K: int, seed: int = 0) -> torch.Tensor:
    """Hand-built routing for exercising the permutation alone: K distinct experts per
    token drawn uniformly (int32 [T, K])."""
    g = torch.Generator().manual_seed(seed)
    return torch.stack([torch.randperm(E, generator=g)[:K] for _ in range(T)]).to(torch.int32) \
        if T > 0 else torch.empty((0, K), dtype=torch.int32)


def crafted_routing(T: int, E: int, K: int, kind: str) -> torch.Tensor:
    """Routings with a known structure (int32 [T, K]).

    * "uniform": token t -> experts {K*(t mod (E/K)) + j}: every expert gets exactly
      T*K/E rows when T is a multiple of E/K (the 2-rows-per-expert case of the pages'
      B=64, k=8, E=256 example).
    * "concentrated": every token -> experts {0..K-1} (U = K).
    * "one_hot_expert": every token's first slot is expert 0 (a hot expert), the other
      slots spread uniformly.
    """
    t = torch.arange(T, dtype=torch.int64)[:, None]
    j = torch.arange(K, dtype=torch.int64)[None, :]
    if kind == "uniform":
        groups = E // K
        return (K * (t % groups) + j).to(torch.int32)
    if kind == "concentrated":
        return j.expand(T, K).to(torch.int32).contiguous()
    if kind == "one_hot_expert":
        rest = 1 + ((t * (K - 1) + (j - 1)) % (E - 1))
        return torch.where(j == 0, torch.zeros_like(rest), rest).to(torch.int32)
    raise ValueError(kind)
