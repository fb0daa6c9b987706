"""Seeded synthetic inputs for one MoE layer.

This module draws random numbers and nothing else: it holds none of the
layer's arithmetic (no routing, no softmax, no re-indexing, no FFN).  Both
the CUDA path and the CPU oracle are fed from it, so the two see the same
bits.  The shapes and value distributions follow the workloads the layer is
measured on: the configurations in CONFIGS below, with the distributions
their fields name.

All draws come from one ``torch.Generator`` seeded per call, in a fixed
order: logits (+ per-expert bias, + planted-group boosts), activations,
routed expert weights (gate, up, down), shared expert weights.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int            # tokens
    d: int            # d_model
    f: int            # d_ff of a routed expert
    E: int            # routed experts
    k: int            # top-k
    R: int            # simulated expert-parallel ranks
    renorm: int = 0   # 1: softmax over the k selected logits
    S: int = 0        # always-on shared experts
    fs: int = 0       # d_ff of a shared expert
    dtype: str = "bf16"
    x_std: float = 1.0
    w_std: float = 0.02
    bias_std: float = 0.0      # per-expert logit bias (load skew)
    groups: int = 0            # planted co-activation groups (0 = none)
    group_p: float = 0.8       # probability a token routes inside one group
    group_boost: float = 8.0   # logit boost given to the chosen group
    seed: int = 0

    @property
    def L(self) -> int:
        return self.E // self.R

    @property
    def cap(self) -> int:
        """Row capacity of the SFD state: T * min(k, R)."""
        return self.T * min(self.k, self.R)

    def with_(self, **kw) -> "LayerConfig":
        return replace(self, **kw)


CONFIGS: dict[str, LayerConfig] = {
    # tiny MoE layer (fp32 and bf16 variants are both exercised by the tests)
    "tiny": LayerConfig("tiny", T=256, d=128, f=256, E=8, k=2, R=4),
    # OLMoE-shaped layer: activations and weights N(0, 0.02), biased logits
    "olmoe": LayerConfig("olmoe", T=4096, d=2048, f=1024, E=64, k=8, R=8,
                         x_std=0.02, bias_std=0.5),
    # Mixtral-shaped layer: 8 experts, top-2 with renormalised softmax
    "mixtral": LayerConfig("mixtral", T=8192, d=4096, f=14336, E=8, k=2, R=8, renorm=1),
    # DeepSeek-V2-Lite-shaped layer: 64 routed top-6 plus 2 shared experts
    "dsv2lite": LayerConfig("dsv2lite", T=16384, d=2048, f=1408, E=64, k=6, R=8,
                            S=2, fs=1408),
    # correlated-routing stress, decode and prefill sizes, 8 planted groups
    "corr_decode": LayerConfig("corr_decode", T=64, d=4096, f=2048, E=64, k=6, R=8, groups=8),
    "corr_prefill": LayerConfig("corr_prefill", T=32768, d=4096, f=2048, E=64, k=6, R=8,
                                groups=8),
}


def torch_dtype(cfg: LayerConfig) -> torch.dtype:
    return {"bf16": torch.bfloat16, "f32": torch.float32}[cfg.dtype]


def group_members(E: int, groups: int, seed: int = 0) -> torch.Tensor:
    """Planted group of every expert: group(e) = perm(e) mod groups, where perm
    is a seeded random permutation (so groups are not contiguous id ranges)."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    perm = torch.randperm(E, generator=g)
    return perm % groups


def make_logits(cfg: LayerConfig, device="cpu", seed: int | None = None) -> torch.Tensor:
    """Router logits, float32 [T, E]."""
    seed = cfg.seed if seed is None else seed
    g = torch.Generator(device=device).manual_seed(seed)
    logits = torch.randn(cfg.T, cfg.E, generator=g, device=device, dtype=torch.float32)
    if cfg.bias_std > 0:
        bias = torch.randn(cfg.E, generator=g, device=device, dtype=torch.float32) * cfg.bias_std
        logits = logits + bias
    if cfg.groups > 0:
        member = group_members(cfg.E, cfg.groups).to(device)
        grouped = torch.rand(cfg.T, generator=g, device=device) < cfg.group_p
        pick = torch.randint(0, cfg.groups, (cfg.T,), generator=g, device=device)
        boost = (member[None, :] == pick[:, None]) & grouped[:, None]
        logits = logits + boost.to(torch.float32) * cfg.group_boost
    return logits.contiguous()


def make_layer_pair_logits(cfg: LayerConfig, follow_p: float = 0.8, device="cpu",
                           seed: int | None = None) -> tuple[torch.Tensor, torch.Tensor]:
    """Router logits of two consecutive layers, float32 [T, E] each, with
    planted inter-layer affinity.  A token routes inside a planted group with
    probability cfg.group_p at both layers (the same tokens); its layer-(l+1)
    group is next(g) for its layer-l group g with probability follow_p, else a
    uniform draw, where next is a seeded permutation of the groups.  The
    layer-(l+1) groups come from their own seeded expert permutation."""
    assert cfg.groups > 0, "planted groups are needed"
    seed = cfg.seed if seed is None else seed
    g = torch.Generator(device=device).manual_seed(seed)
    G = cfg.groups
    member1 = group_members(cfg.E, G, seed=0).to(device)
    member2 = group_members(cfg.E, G, seed=1).to(device)
    nxt = torch.randperm(G, generator=torch.Generator().manual_seed(2)).to(device)
    l1 = torch.randn(cfg.T, cfg.E, generator=g, device=device, dtype=torch.float32)
    l2 = torch.randn(cfg.T, cfg.E, generator=g, device=device, dtype=torch.float32)
    grouped = torch.rand(cfg.T, generator=g, device=device) < cfg.group_p
    g1 = torch.randint(0, G, (cfg.T,), generator=g, device=device)
    follow = torch.rand(cfg.T, generator=g, device=device) < follow_p
    g2 = torch.where(follow, nxt[g1], torch.randint(0, G, (cfg.T,), generator=g, device=device))
    l1 = l1 + ((member1[None, :] == g1[:, None]) & grouped[:, None]).float() * cfg.group_boost
    l2 = l2 + ((member2[None, :] == g2[:, None]) & grouped[:, None]).float() * cfg.group_boost
    return l1.contiguous(), l2.contiguous()


def make_inputs(cfg: LayerConfig, device="cpu", seed: int | None = None,
                weights: bool = True) -> dict[str, torch.Tensor]:
    """All tensors of one layer invocation.

    logits f32 [T,E]; x [T,d]; wg, wu [E,f,d]; wd [E,d,f];
    sg, su [S,fs,d]; sd [S,d,fs] (only when S > 0).  Weights are in
    expert-id order and K-contiguous (the last axis is the reduction axis).
    """
    seed = cfg.seed if seed is None else seed
    dt = torch_dtype(cfg)
    out = {"logits": make_logits(cfg, device, seed)}
    g = torch.Generator(device=device).manual_seed(seed + 1000003)
    out["x"] = (torch.randn(cfg.T, cfg.d, generator=g, device=device) * cfg.x_std).to(dt)
    if weights:
        def w(*shape):
            return (torch.randn(*shape, generator=g, device=device) * cfg.w_std).to(dt)
        out["wg"] = w(cfg.E, cfg.f, cfg.d)
        out["wu"] = w(cfg.E, cfg.f, cfg.d)
        out["wd"] = w(cfg.E, cfg.d, cfg.f)
        if cfg.S > 0:
            out["sg"] = w(cfg.S, cfg.fs, cfg.d)
            out["su"] = w(cfg.S, cfg.fs, cfg.d)
            out["sd"] = w(cfg.S, cfg.d, cfg.fs)
    return out


def contiguous_placement(E: int) -> torch.Tensor:
    """slot_of[e] = e: rank r holds experts [r*L, (r+1)*L)."""
    return torch.arange(E, dtype=torch.int32)


def random_topk(T: int, E: int, k: int, seed: int = 0, device="cpu") -> torch.Tensor:
    """k distinct uniformly random expert ids per token, int32 [T, k]."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    idx = torch.argsort(torch.rand(T, E, generator=g), dim=1)[:, :k]
    return idx.to(torch.int32).contiguous().to(device)
