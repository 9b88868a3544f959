"""Seeded synthetic inputs for the fine-grained MoE expert layer.

The pages benchmark real MoE model shapes (OLMoE, Qwen3, DeepSeek-V3, ...) with
trained weights; here random tensors of those shapes and of the stated value
distributions stand in for them. Every tensor comes from its own seeded torch
generator (Philox on CUDA, MT19937 on CPU), so the same (config, device) always
gives the same bytes.

Recipe per config (sizes from the workload descriptions):
  X   [T, d]      bf16  N(0, x_std)
  W1  [E, d, 2n]  bf16  N(0, 0.02)   columns [0, n) gate, [n, 2n) up
  W2  [E, n, d]   bf16  N(0, 0.02)
  Wr  [d, E]      fp32  N(0, 0.02)
  b   [E]         fp32  router logit bias giving skewed expert loads:
                        "normal": N(0, 0.5); "zipf": -1.1 * ln(rank_e) with rank
                        a seeded permutation of 1..E; "none": absent
  dO  [T, d]      bf16  N(0, 1)

This module holds no arithmetic of the layer itself.
"""
from __future__ import annotations

import dataclasses
import numpy as np


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int
    d: int
    E: int
    n: int
    K: int
    x_std: float = 1.0
    w_std: float = 0.02
    wr_std: float = 0.02
    bias: str = "none"          # "none" | "normal" | "zipf"
    bias_std: float = 0.5
    zipf_s: float = 1.1
    seed: int = 0
    round_mode: int = 0         # 0 off, 1 nearest, 2 stochastic

    def with_(self, **kw) -> "MoEConfig":
        return dataclasses.replace(self, **kw)

    @property
    def flops_fwd(self) -> int:
        """Expert-GEMM FLOPs of the forward: up 4*T*K*d*n + down 2*T*K*d*n."""
        return 6 * self.T * self.K * self.d * self.n

    @property
    def flops_bwd(self) -> int:
        """dH 2 + dW2 2 + dX~ 4 + dW1 4, all times T*K*d*n."""
        return 12 * self.T * self.K * self.d * self.n

    def describe(self) -> dict:
        return {"T": self.T, "d": self.d, "E": self.E, "n": self.n, "K": self.K,
                "bias": self.bias, "seed": self.seed, "round_mode": self.round_mode}


def _sweep(E: int, n: int, tr: bool, idx: int) -> MoEConfig:
    return MoEConfig(name=f"sweep_E{E}_n{n}" + ("_tr" if tr else ""), T=16384, d=1536,
                     E=E, n=n, K=8, bias="normal", seed=30 + idx,
                     round_mode=2 if tr else 0)


CONFIGS: dict[str, MoEConfig] = {
    # tiny layer: every tensor N(0, 0.02), no router bias
    "tiny": MoEConfig("tiny", T=512, d=128, E=16, n=64, K=2, x_std=0.02, seed=0),
    # fine-grained 7B-class layer with skewed router
    "7b": MoEConfig("7b", T=16384, d=1536, E=128, n=256, K=8, bias="normal", seed=1),
    # Qwen3-MoE-shaped layer, balanced router
    "qwen3": MoEConfig("qwen3", T=32768, d=2048, E=128, n=768, K=8, seed=2),
    # DeepSeek-V3-shaped layer, Zipf(1.1) expert popularity
    "dsv3": MoEConfig("dsv3", T=8192, d=7168, E=256, n=2048, K=8, bias="zipf", seed=4),
    # OLMoE-shaped layer (the pages' runtime-breakdown workload), balanced router
    "olmoe": MoEConfig("olmoe", T=32768, d=2048, E=64, n=1024, K=8, seed=5),
    # a small layer with the DeepSeek-V3-shaped layer's load pattern (many
    # experts of a few dozen rows, a Zipf head), about 4 GB resident: for
    # profiler captures of the weight-gradient kernels' short tiles
    "smallexp": MoEConfig("smallexp", T=4096, d=2048, E=256, n=512, K=8, bias="zipf", seed=6),
}
for _i, (_E, _n) in enumerate([(64, 512), (128, 256), (256, 128), (512, 64)]):
    for _tr in (False, True):
        _c = _sweep(_E, _n, _tr, _i)
        CONFIGS[_c.name] = _c


def get_config(name: str) -> MoEConfig:
    return CONFIGS[name]


def _gen(torch, device, seed: int):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def make_inputs(cfg: MoEConfig, device="cpu", need_grad_inputs: bool = True, rank: int = 0,
                experts=None) -> dict:
    """Return the seeded input tensors of `cfg` on `device` (torch tensors).

    Large weight tensors are produced one expert at a time, each expert from
    its own seed, so that the fp32 temporaries stay small and a subset of the
    experts can be produced alone: with `experts` (a list of expert ids) W1
    and W2 hold only those experts, in that order, with the same values the
    full tensors hold for them.  `rank` selects a different batch of tokens
    (X and dO) for data-parallel replica `rank`; the weights do not depend on
    it.
    """
    import torch

    dev = torch.device(device)
    base = 1000 * (cfg.seed + 1)
    data = base + 100 * int(rank)
    out = {}
    g = _gen(torch, dev, data + 1)
    out["X"] = (torch.randn(cfg.T, cfg.d, generator=g, device=dev) * cfg.x_std).to(torch.bfloat16)

    ids = list(range(cfg.E)) if experts is None else [int(e) for e in experts]

    def expert_weights(shape_e, seed):
        w = torch.empty((len(ids),) + shape_e, dtype=torch.bfloat16, device=dev)
        for i, e in enumerate(ids):
            g_ = _gen(torch, dev, seed * 1_000_003 + e)
            w[i] = (torch.randn(shape_e, generator=g_, device=dev) * cfg.w_std).to(torch.bfloat16)
        return w

    out["W1"] = expert_weights((cfg.d, 2 * cfg.n), base + 2)
    out["W2"] = expert_weights((cfg.n, cfg.d), base + 3)
    g = _gen(torch, dev, base + 4)
    out["Wr"] = torch.randn(cfg.d, cfg.E, generator=g, device=dev) * cfg.wr_std
    if cfg.bias == "normal":
        g = _gen(torch, dev, base + 5)
        out["bias"] = torch.randn(cfg.E, generator=g, device=dev) * cfg.bias_std
    elif cfg.bias == "zipf":
        g = _gen(torch, "cpu", base + 5)
        rank = torch.randperm(cfg.E, generator=g).to(torch.float64) + 1.0
        out["bias"] = (-cfg.zipf_s * torch.log(rank)).to(torch.float32).to(dev)
    else:
        out["bias"] = None
    if need_grad_inputs:
        g = _gen(torch, dev, data + 6)
        out["dO"] = torch.randn(cfg.T, cfg.d, generator=g, device=dev).to(torch.bfloat16)
    return out


def bf16_round_np(x) -> np.ndarray:
    """Round an array to the nearest bfloat16 value (ties to even); float32 out."""
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = a.view(np.uint32).astype(np.uint64)
    rounded = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    nan = np.isnan(a)
    r = rounded.astype(np.uint32).view(np.float32).copy()
    r[nan] = np.nan
    return r


def realised_loads(counts) -> dict:
    c = np.asarray(counts, dtype=np.int64)
    return {"min": int(c.min()), "mean": float(c.mean()), "max": int(c.max()),
            "max_over_mean": float(c.max() / max(c.mean(), 1e-9)),
            "pad_rows_128": int(sum((-int(x)) % 128 for x in c))}
