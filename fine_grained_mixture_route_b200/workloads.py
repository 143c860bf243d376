"""Seeded synthetic inputs for the DeepSeekMoE layer forward.

This module only draws random tensors of the right shapes and distributions; it holds none
of the layer's arithmetic.  It is the one module that both the CUDA path (bench, GPU tests)
and the fp64 oracle's tests take their inputs from.

Shapes follow the layer as described in "《DeepSeekMoE》深度解读报告" §2.2-§2.3 and §3.1
(N_m fine-grained routed experts, top-N_r routing, K_s shared experts) with the per-expert
SwiGLU FFN of the `Expert` module in "DeepSeek MoE模型优化与未来演进及字节超稀疏内存技术"
(w1, w3: [inter, dim]; w2: [dim, inter]; every Linear with a bias).  The initial standard
deviation 0.006 for every learnable tensor is the one stated in §3.3 of the DeepSeekMoE
report.

Every tensor, and every expert slice of a stacked tensor, has its own torch.Generator seeded
from (seed, tensor id, expert), so a slice can be regenerated on its own and the values
never depend on the order of generation.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import torch

INIT_STD = 0.006          # "all learnable parameters", DeepSeekMoE report §3.3
ZIPF_S = 1.1              # centroid-norm exponent of the skewed prefill workload


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int                 # tokens
    d: int                 # hidden size
    n_experts: int         # N_m
    inter: int             # routed intermediate size
    top_k: int             # N_r
    n_shared: int          # K_s
    inter_shared: int      # shared intermediate size
    has_bias: bool
    dtype: torch.dtype
    centroid_init: str     # "normal_std", "normal_inv_sqrt_d", "uniform_inv_sqrt_d", "zipf_norm"

    @property
    def slots(self) -> int:
        return self.T * self.top_k

    def flops(self) -> float:
        """Algorithmic FLOPs of one layer call (2 per multiply-add): router scores plus
        three d x inter contractions per routed pick and per shared expert."""
        return (2.0 * self.T * 3 * self.d * (self.top_k * self.inter + self.n_shared * self.inter_shared)
                + 2.0 * self.T * self.d * self.n_experts)

    def elem_bytes(self) -> int:
        return torch.tensor([], dtype=self.dtype).element_size()


CONFIGS: Dict[str, LayerConfig] = {
    # tiny fp32 layer: 16 routed experts of inter 64, top-4, one shared expert, biases on
    "tiny": LayerConfig("tiny", 128, 256, 16, 64, 4, 1, 64, True, torch.float32, "normal_std"),
    # small fine-grained layer: 64 experts of inter 320, top-7 + 1 shared
    "small": LayerConfig("small", 2048, 1280, 64, 320, 7, 1, 320, True, torch.bfloat16, "normal_inv_sqrt_d"),
    # mid-size layer: 64 experts of inter 1408, top-6 + 2 shared, no bias, balanced routing
    "mid": LayerConfig("mid", 4096, 2048, 64, 1408, 6, 2, 1408, False, torch.bfloat16, "uniform_inv_sqrt_d"),
    # decode-shaped V3 expert layer: T=256, d=7168, 256 experts of inter 2048, top-8 + 1 shared
    "decode": LayerConfig("decode", 256, 7168, 256, 2048, 8, 1, 2048, True, torch.bfloat16, "normal_std"),
    # prefill-shaped layer, same experts, T=16384, Zipf(1.1)-skewed centroid norms
    "prefill": LayerConfig("prefill", 16384, 7168, 256, 2048, 8, 1, 2048, True, torch.bfloat16, "zipf_norm"),
    # profiling slice of the prefill layer, a few GB on the device: the same expert shape and
    # Zipf routing over 32 experts, T chosen so that the mean tokens per expert (512) match
    "prefill_slice": LayerConfig("prefill_slice", 2048, 7168, 32, 2048, 8, 1, 2048, True, torch.bfloat16, "zipf_norm"),
}

# tensor ids used to derive per-tensor seeds
_TID = {"x": 1, "centroids": 2, "zipf_rank": 3,
        "w1": 10, "b1": 11, "w3": 12, "b3": 13, "w2": 14, "b2": 15,
        "sw1": 20, "sb1": 21, "sw3": 22, "sb3": 23, "sw2": 24, "sb2": 25}


def seed_for(seed: int, tensor: str, expert: int = 0) -> int:
    """Deterministic 63-bit seed for one tensor slice (splitmix64 finaliser of a packed key)."""
    z = (seed * 0x9E3779B97F4A7C15 + _TID[tensor] * 0xBF58476D1CE4E5B9 + (expert + 1) * 0x94D049BB133111EB) & (2**64 - 1)
    z ^= z >> 30
    z = (z * 0xBF58476D1CE4E5B9) & (2**64 - 1)
    z ^= z >> 27
    z = (z * 0x94D049BB133111EB) & (2**64 - 1)
    z ^= z >> 31
    return z & (2**63 - 1)


def _gen(device, seed: int, tensor: str, expert: int = 0) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed_for(seed, tensor, expert))
    return g


def _normal(shape, std, device, seed, tensor, expert=0):
    t = torch.empty(shape, dtype=torch.float32, device=device)
    t.normal_(0.0, std, generator=_gen(device, seed, tensor, expert))
    return t


def make_x(cfg: LayerConfig, device="cpu", seed: int = 0, T: Optional[int] = None) -> torch.Tensor:
    T = cfg.T if T is None else T
    return _normal((T, cfg.d), 1.0, device, seed, "x").to(cfg.dtype)


def make_centroids(cfg: LayerConfig, device="cpu", seed: int = 0) -> torch.Tensor:
    N, d = cfg.n_experts, cfg.d
    kind = cfg.centroid_init
    if kind == "normal_std":
        c = _normal((N, d), INIT_STD, device, seed, "centroids")
    elif kind == "normal_inv_sqrt_d":
        c = _normal((N, d), 1.0 / math.sqrt(d), device, seed, "centroids")
    elif kind == "uniform_inv_sqrt_d":
        a = math.sqrt(3.0) / math.sqrt(d)           # std 1/sqrt(d)
        c = torch.empty((N, d), dtype=torch.float32, device=device)
        c.uniform_(-a, a, generator=_gen(device, seed, "centroids"))
    elif kind == "zipf_norm":
        # e_i = R * rank_i^-s * v_i / |v_i|, R = INIT_STD * sqrt(d) (the norm of a std-0.006
        # centroid), v_i ~ N(0, I), ranks a seeded permutation of 1..N
        v = _normal((N, d), 1.0, device, seed, "centroids")
        rank = torch.randperm(N, generator=_gen("cpu", seed, "zipf_rank")).to(torch.float32) + 1.0
        R = INIT_STD * math.sqrt(d)
        scale = (R * rank.pow(-ZIPF_S)).to(device)
        c = v / v.norm(dim=1, keepdim=True) * scale[:, None]
    else:
        raise ValueError(kind)
    return c.to(cfg.dtype)


def make_expert_stack(cfg: LayerConfig, shared: bool, device="cpu", seed: int = 0,
                      experts: Optional[range] = None) -> Dict[str, Optional[torch.Tensor]]:
    """Stacked expert weights in nn.Linear layout: w1,w3 [E, inter, d], w2 [E, d, inter],
    b1,b3 [E, inter], b2 [E, d] (biases None when the config has none).  `experts` selects a
    sub-range of expert indices (for streaming the large configs one slice at a time)."""
    E = cfg.n_shared if shared else cfg.n_experts
    I = cfg.inter_shared if shared else cfg.inter
    d = cfg.d
    p = "s" if shared else ""
    ids = range(E) if experts is None else experts
    n = len(ids)
    out: Dict[str, Optional[torch.Tensor]] = {}
    shapes = {"w1": (I, d), "w3": (I, d), "w2": (d, I), "b1": (I,), "b3": (I,), "b2": (d,)}
    # W1 and W3 are the two halves of one buffer, so the up-projection can fetch a tile of both
    # with one request
    w13 = torch.empty((2, n, I, d), dtype=cfg.dtype, device=device)
    for name, shp in shapes.items():
        if name.startswith("b") and not cfg.has_bias:
            out[name] = None
            continue
        t = w13[0] if name == "w1" else w13[1] if name == "w3" else torch.empty((n,) + shp, dtype=cfg.dtype,
                                                                                  device=device)
        for j, e in enumerate(ids):
            t[j] = _normal(shp, INIT_STD, device, seed, p + name, e).to(cfg.dtype)
        out[name] = t
    return out


def make_layer(cfg: LayerConfig, device="cpu", seed: int = 0) -> Dict[str, object]:
    """All inputs of one layer call: x, centroids, routed and shared expert stacks."""
    return {
        "x": make_x(cfg, device, seed),
        "centroids": make_centroids(cfg, device, seed),
        "routed": make_expert_stack(cfg, False, device, seed),
        "shared": make_expert_stack(cfg, True, device, seed) if cfg.n_shared > 0 else None,
    }


def scaled(cfg: LayerConfig, **kw) -> LayerConfig:
    """A copy of a config with some fields replaced (smaller test cases of the same family)."""
    return dataclasses.replace(cfg, **kw)
