"""Seeded synthetic inputs for routed-MoE expert projections.

This module only draws random numbers.  It holds none of the method's
arithmetic (no pruning, no quantization, no routing sort, no GEMM), so that
both the CUDA path and the CPU oracle can be fed the very same tensors.

Workloads are shaped like the expert FFNs of the models the paper measures
("Hardware-Native Joint Sparse-Quantization for Trillion-Scale
Mixture-of-Experts", §4.1 setup and §D.2 kernel benchmark): a 30B-A3B-shaped
model (hidden 2048, expert FFN 768, 128 experts, top-8) and a 1T-shaped model
(hidden 7168, expert FFN 2048, 384 experts, top-8).  No model weights or
datasets are used: weights are N(0, sigma) in fp32, activations N(0, 1) in
bf16 with a few scaled outlier channels, routing is uniform or Zipf.

Seed streams (base seed 0): expert e's weight -> 1000 + e (a layer's down-projection:
3000 + e), activations -> 1, routing -> 2, gate logits -> 3, outlier channels -> 4.
"""
from __future__ import annotations

import dataclasses

import torch

SEED_X = 1
SEED_ROUTE = 2
SEED_GATES = 3
SEED_OUTLIERS = 4
SEED_W_BASE = 1000


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    """One grouped expert projection: E experts, Y_e = X_e . W_e^T with W_e [N, K]."""
    name: str
    E: int
    K: int
    N: int
    T: int                 # tokens
    top_k: int
    routing: str           # "uniform" or "zipf"
    zipf_s: float = 0.0
    w_sigma: float = 0.02
    outlier_frac: float = 0.0
    outlier_scale: float = 1.0

    @property
    def R(self) -> int:
        """Routed rows: every token appears once per selected expert."""
        return self.T * self.top_k


CONFIGS = {
    "tiny": MoEConfig("tiny", E=4, K=256, N=128, T=32, top_k=2, routing="uniform",
                      w_sigma=0.02),
    "30b_up_prefill": MoEConfig("30b_up_prefill", E=128, K=2048, N=1536, T=512, top_k=8,
                                routing="zipf", zipf_s=1.0, w_sigma=0.02,
                                outlier_frac=0.01, outlier_scale=20.0),
    "30b_down_decode": MoEConfig("30b_down_decode", E=128, K=768, N=2048, T=64, top_k=8,
                                 routing="uniform", w_sigma=0.02),
    "1t_up_prefill": MoEConfig("1t_up_prefill", E=384, K=7168, N=4096, T=8192, top_k=8,
                               routing="zipf", zipf_s=1.1, w_sigma=0.015,
                               outlier_frac=0.005, outlier_scale=30.0),
}
for _b in (1, 32, 128, 256):
    CONFIGS[f"1t_down_decode_b{_b}"] = MoEConfig(
        f"1t_down_decode_b{_b}", E=384, K=2048, N=7168, T=_b, top_k=8,
        routing="uniform", w_sigma=0.015)
# The 1T prefill up-projection on 64 of its experts with the same average rows per expert
# (1368 tokens top-8 = 171 per expert): the same kernel instantiation (128-token tiles) on
# 0.65 GB of weights, small enough for profiler captures of all counters.
CONFIGS["1t_up_prefill_e64"] = MoEConfig("1t_up_prefill_e64", E=64, K=7168, N=4096, T=1368, top_k=8,
                                         routing="zipf", zipf_s=1.1, w_sigma=0.015,
                                         outlier_frac=0.005, outlier_scale=30.0)
# The 1T prefill up-projection at 65,536 tokens top-8 (R = 524,288): eight times the rows on the
# same weights, 30.8 dense-equivalent TFLOP against 10.2 GB of algorithmic traffic (packed weights,
# activation codes and scales, bf16 output), past the ridge point of the sparse NVFP4 tensor roof.
# A measurement of the kernel where the tensor pipe, not HBM, is the binding roof; not one of the
# expert-projection workloads.  The _e64 variant keeps its rows per expert on 64 experts (10,920
# tokens) for profiler captures.
CONFIGS["1t_up_prefill_65k"] = MoEConfig("1t_up_prefill_65k", E=384, K=7168, N=4096, T=65536, top_k=8,
                                         routing="zipf", zipf_s=1.1, w_sigma=0.015,
                                         outlier_frac=0.005, outlier_scale=30.0)
CONFIGS["1t_up_prefill_65k_e64"] = MoEConfig("1t_up_prefill_65k_e64", E=64, K=7168, N=4096, T=10920, top_k=8,
                                             routing="zipf", zipf_s=1.1, w_sigma=0.015,
                                             outlier_frac=0.005, outlier_scale=30.0)


@dataclasses.dataclass(frozen=True)
class MoELayer:
    """A routed MoE FFN layer: up-projection with fused gate|up weights [2I, H], SwiGLU, then the
    down-projection [H, I], over the same routed tokens.  Shapes of the expert FFNs of the
    30B-A3B-shaped and 1T-shaped models (see the module docstring)."""
    name: str
    E: int
    H: int                 # hidden size: K of the up-projection, N of the down-projection
    I: int                 # expert FFN size: N/2 of the up-projection, K of the down-projection
    T: int
    top_k: int
    routing: str
    zipf_s: float = 0.0
    w_sigma: float = 0.02
    outlier_frac: float = 0.0
    outlier_scale: float = 1.0

    @property
    def R(self) -> int:
        return self.T * self.top_k

    def up(self) -> MoEConfig:
        """The up-projection (its activations, routing and gates are the layer's)."""
        return MoEConfig(self.name + "_up", E=self.E, K=self.H, N=2 * self.I, T=self.T, top_k=self.top_k,
                         routing=self.routing, zipf_s=self.zipf_s, w_sigma=self.w_sigma,
                         outlier_frac=self.outlier_frac, outlier_scale=self.outlier_scale)

    def down(self) -> MoEConfig:
        return MoEConfig(self.name + "_down", E=self.E, K=self.I, N=self.H, T=self.T, top_k=self.top_k,
                         routing=self.routing, zipf_s=self.zipf_s, w_sigma=self.w_sigma)


LAYERS = {
    "tiny_layer": MoELayer("tiny_layer", E=4, H=256, I=256, T=32, top_k=2, routing="uniform"),
    "30b_layer": MoELayer("30b_layer", E=128, H=2048, I=768, T=512, top_k=8, routing="zipf", zipf_s=1.0,
                          w_sigma=0.02, outlier_frac=0.01, outlier_scale=20.0),
    "1t_layer": MoELayer("1t_layer", E=384, H=7168, I=2048, T=1024, top_k=8, routing="zipf", zipf_s=1.1,
                         w_sigma=0.015, outlier_frac=0.005, outlier_scale=30.0),
}
SEED_W_DOWN_BASE = 3000


def down_weight(layer: MoELayer, e: int, device: str = "cpu") -> torch.Tensor:
    """Expert e's down-projection weight fp32 [H, I] ~ N(0, w_sigma) (its own seed stream)."""
    g = _gen(SEED_W_DOWN_BASE + e, device)
    w = torch.randn(layer.H, layer.I, generator=g, device=device, dtype=torch.float32)
    return w.mul_(layer.w_sigma)


def _gen(seed: int, device: str) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def expert_weight(cfg: MoEConfig, e: int, device: str = "cpu") -> torch.Tensor:
    """W_e fp32 [N, K] ~ N(0, w_sigma), K contiguous."""
    g = _gen(SEED_W_BASE + e, device)
    w = torch.randn(cfg.N, cfg.K, generator=g, device=device, dtype=torch.float32)
    return w.mul_(cfg.w_sigma)


def all_weights(cfg: MoEConfig, device: str = "cpu") -> torch.Tensor:
    """W fp32 [E, N, K]; only sensible for the small configs."""
    return torch.stack([expert_weight(cfg, e, device) for e in range(cfg.E)])


def activations(cfg: MoEConfig, device: str = "cpu") -> torch.Tensor:
    """X bf16 [T, K] ~ N(0, 1); a seeded set of round(frac*K) channels is scaled."""
    g = _gen(SEED_X, device)
    x = torch.randn(cfg.T, cfg.K, generator=g, device=device, dtype=torch.float32)
    n_out = int(round(cfg.outlier_frac * cfg.K))
    if n_out > 0:
        go = _gen(SEED_OUTLIERS, "cpu")
        ch = torch.randperm(cfg.K, generator=go)[:n_out].to(device)
        x[:, ch] *= cfg.outlier_scale
    return x.to(torch.bfloat16)


def expert_probs(cfg: MoEConfig) -> torch.Tensor:
    """Per-expert selection weights: uniform, or Zipf(s) over a seeded permutation."""
    if cfg.routing == "uniform":
        return torch.full((cfg.E,), 1.0 / cfg.E, dtype=torch.float64)
    g = _gen(SEED_ROUTE, "cpu")
    perm = torch.randperm(cfg.E, generator=g)
    rank_w = torch.arange(1, cfg.E + 1, dtype=torch.float64).pow(-cfg.zipf_s)
    p = torch.empty(cfg.E, dtype=torch.float64)
    p[perm] = rank_w           # expert perm[i] gets weight (i+1)^-s
    return p / p.sum()


def routing(cfg: MoEConfig) -> torch.Tensor:
    """topk ids int32 [T, top_k]: each token draws top_k distinct experts."""
    p = expert_probs(cfg)
    g = _gen(SEED_ROUTE + 100, "cpu")
    ids = torch.multinomial(p.expand(cfg.T, cfg.E), cfg.top_k, replacement=False, generator=g)
    return ids.to(torch.int32).contiguous()


def gates(cfg: MoEConfig) -> torch.Tensor:
    """gates fp32 [T, top_k]: softmax of N(0,1) logits over the selected experts."""
    g = _gen(SEED_GATES, "cpu")
    logits = torch.randn(cfg.T, cfg.top_k, generator=g, dtype=torch.float32)
    return torch.softmax(logits, dim=-1).contiguous()


def random_bf16(shape, seed: int, device: str = "cpu", scale: float = 1.0) -> torch.Tensor:
    """A seeded bf16 tensor (used to feed the scatter step in isolation)."""
    g = _gen(seed, device)
    return (torch.randn(*shape, generator=g, device=device) * scale).to(torch.bfloat16)


def custom_config(name: str, E: int, K: int, N: int, T: int, top_k: int,
                  routing: str = "uniform", zipf_s: float = 0.0, w_sigma: float = 0.02,
                  outlier_frac: float = 0.0, outlier_scale: float = 1.0) -> MoEConfig:
    return MoEConfig(name, E=E, K=K, N=N, T=T, top_k=top_k, routing=routing, zipf_s=zipf_s,
                     w_sigma=w_sigma, outlier_frac=outlier_frac, outlier_scale=outlier_scale)


def routed_counts(ids: torch.Tensor, E: int) -> torch.Tensor:
    """Rows per expert (a plain histogram of the ids; used only for sizing launches)."""
    return torch.bincount(ids.reshape(-1).long(), minlength=E)


def expert_flops(cfg: MoEConfig) -> float:
    """Dense-equivalent flops 2*R*N*K, the unit the sparse tensor peak is quoted in."""
    return 2.0 * cfg.R * cfg.N * cfg.K


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


__all__ = ["MoEConfig", "CONFIGS", "expert_weight", "all_weights", "activations", "routing",
           "gates", "random_bf16", "custom_config", "routed_counts", "expert_flops",
           "expert_probs", "ceil_div"]
