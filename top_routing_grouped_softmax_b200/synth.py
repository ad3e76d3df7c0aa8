"""Seeded synthetic inputs for the sparse-MoE block forward.

This module only draws random numbers and lays them out; it holds none of the
block's arithmetic.  Both the CUDA path and the CPU oracle are fed from it, so
the two sides see identical bf16 bytes.

Recipe (the pages publish no dataset or weights; these stand in for the
workloads they describe):

* ``torch.Generator`` on the CPU, ``manual_seed(seed)``.
* fp32 ``randn`` draws, in this order: ``x [T, d]``; ``W_router [d, E]``;
  ``W_gate[e] [d, f]`` for e = 0..E-1; ``W_up[e] [d, f]`` for e = 0..E-1;
  ``W_down[e] [f, d]`` for e = 0..E-1.  Weights are scaled by ``sigma``; every
  tensor is then rounded to bf16 (round-to-nearest-even, torch's cast).
* Load-skewed configurations then draw ``randperm(E)`` from the same
  generator.  Expert ``perm[i]`` gets rank ``i + 1`` and the bias
  ``b_e = 2.0 * log(1 / rank_e ** 1.2)`` (natural log, computed in fp64,
  stored as fp32), a Zipf(s = 1.2) preference over a seeded expert ranking.
  The bias is added to the router logits before the softmax, as in the
  gated-router formula ``G(x) = Softmax(W_g x + b_g)`` of the Hunyuan-Large
  overview page (section 2.1, "gating network").

Per-expert draws keep peak host memory near one expert's weights even for
the coarse configuration (E = 8, d = 4096, f = 14336).
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np
import torch


@dataclass(frozen=True)
class MoEConfig:
    """Shape and generation parameters of one synthetic MoE-block workload."""

    name: str
    T: int          # tokens (batch x sequence, flattened)
    d: int          # hidden size
    E: int          # experts
    k: int          # experts per token (top-k)
    f: int          # expert SwiGLU intermediate size
    sigma: float    # std of every weight tensor (x is N(0, 1))
    seed: int
    skew: bool = False  # add the Zipf expert bias to the router logits

    def with_(self, **kw) -> "MoEConfig":
        return replace(self, **kw)

    @property
    def flops(self) -> int:
        """Algorithmic FLOPs of one forward: 2*T*(d*E + 3*k*d*f)."""
        return 2 * self.T * (self.d * self.E + 3 * self.k * self.d * self.f)


# The five workloads.  "qwen" is the Qwen3-MoE-shaped layer; "coarse" mirrors
# the 8-expert top-2 block the Qwen3MoeSparseMoeBlock article benchmarks;
# "fine" is the fine-grained regime of the SonicMoE comparison page.
CONFIGS = {
    "tiny": MoEConfig("tiny", T=256, d=256, E=8, k=2, f=512, sigma=0.02, seed=0),
    "qwen": MoEConfig("qwen", T=8192, d=2048, E=128, k=8, f=768, sigma=0.02, seed=1),
    "fine": MoEConfig("fine", T=16384, d=1536, E=256, k=8, f=256, sigma=0.02, seed=2),
    "coarse": MoEConfig("coarse", T=4096, d=4096, E=8, k=2, f=14336, sigma=0.01, seed=3),
    "skew": MoEConfig("skew", T=32768, d=2048, E=128, k=8, f=768, sigma=0.02, seed=4, skew=True),
}


@dataclass
class MoEInputs:
    """bf16 tensors on the CPU (torch.bfloat16) plus an optional fp32 bias."""

    cfg: MoEConfig
    x: torch.Tensor          # [T, d]
    W_router: torch.Tensor   # [d, E]
    W_gate: torch.Tensor     # [E, d, f]
    W_up: torch.Tensor       # [E, d, f]
    W_down: torch.Tensor     # [E, f, d]
    bias: torch.Tensor | None  # [E] fp32 or None

    def bits(self, name: str) -> np.ndarray:
        """The raw bf16 bit patterns of one tensor as a uint16 numpy array."""
        return bf16_bits(getattr(self, name))

    def bias_np(self) -> np.ndarray | None:
        return None if self.bias is None else self.bias.numpy()


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """View a bf16 tensor's storage as uint16 (no copy, no rounding)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def bits_to_bf16(a: np.ndarray) -> torch.Tensor:
    """Inverse of bf16_bits."""
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def _randn_bf16(gen: torch.Generator, shape, scale: float) -> torch.Tensor:
    t = torch.randn(*shape, generator=gen, dtype=torch.float32)
    if scale != 1.0:
        t.mul_(scale)
    return t.to(torch.bfloat16)


def zipf_bias(E: int, gen: torch.Generator, s: float = 1.2, scale: float = 2.0) -> torch.Tensor:
    """Per-expert bias b_e = scale * log(1 / rank_e**s) over a seeded ranking."""
    order = torch.randperm(E, generator=gen)
    rank = np.empty(E, dtype=np.float64)
    rank[order.numpy()] = np.arange(1, E + 1, dtype=np.float64)
    b = scale * np.log(1.0 / rank ** s)
    return torch.from_numpy(b.astype(np.float32))


def make_inputs(cfg: MoEConfig | str, **overrides) -> MoEInputs:
    """Draw one workload's inputs following the recipe in the module docstring."""
    if isinstance(cfg, str):
        cfg = CONFIGS[cfg]
    if overrides:
        cfg = cfg.with_(**overrides)
    T, d, E, f = cfg.T, cfg.d, cfg.E, cfg.f
    gen = torch.Generator(device="cpu")
    gen.manual_seed(cfg.seed)
    x = _randn_bf16(gen, (T, d), 1.0)
    W_router = _randn_bf16(gen, (d, E), cfg.sigma)
    W_gate = torch.empty(E, d, f, dtype=torch.bfloat16)
    W_up = torch.empty(E, d, f, dtype=torch.bfloat16)
    W_down = torch.empty(E, f, d, dtype=torch.bfloat16)
    for e in range(E):
        W_gate[e] = _randn_bf16(gen, (d, f), cfg.sigma)
    for e in range(E):
        W_up[e] = _randn_bf16(gen, (d, f), cfg.sigma)
    for e in range(E):
        W_down[e] = _randn_bf16(gen, (f, d), cfg.sigma)
    bias = zipf_bias(E, gen) if cfg.skew else None
    return MoEInputs(cfg, x, W_router, W_gate, W_up, W_down, bias)


def make_shared_weights(cfg: MoEConfig, n_shared: int, f_shared: int | None = None) -> dict:
    """Weights of ``n_shared`` shared experts (every token passes through
    them with weight one): bf16 W_gate_s, W_up_s [n_shared, d, f_s] and
    W_down_s [n_shared, f_s, d], f_s = f_shared or cfg.f.  Drawn like the
    routed experts (fp32 randn * sigma, rounded to bf16; gate of every
    shared expert, then up, then down) from their own generator seeded with
    seed + 100000, so adding shared experts leaves the other inputs of the
    workload unchanged."""
    fs = cfg.f if f_shared is None else f_shared
    gen = torch.Generator(device="cpu")
    gen.manual_seed(cfg.seed + 100000)
    W_gate_s = torch.empty(n_shared, cfg.d, fs, dtype=torch.bfloat16)
    W_up_s = torch.empty(n_shared, cfg.d, fs, dtype=torch.bfloat16)
    W_down_s = torch.empty(n_shared, fs, cfg.d, dtype=torch.bfloat16)
    for s in range(n_shared):
        W_gate_s[s] = _randn_bf16(gen, (cfg.d, fs), cfg.sigma)
    for s in range(n_shared):
        W_up_s[s] = _randn_bf16(gen, (cfg.d, fs), cfg.sigma)
    for s in range(n_shared):
        W_down_s[s] = _randn_bf16(gen, (fs, cfg.d), cfg.sigma)
    return {"W_gate_s": W_gate_s, "W_up_s": W_up_s, "W_down_s": W_down_s}


def make_dout(T: int, d: int, seed: int) -> torch.Tensor:
    """The output gradient for a backward check: fp32 [T, d], N(0, 1), drawn
    from its own generator (seed + 200000) so the forward inputs of the
    same seed are unchanged."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed + 200000)
    return torch.randn(T, d, generator=gen, dtype=torch.float32)


def sample_tokens(T: int, n: int, seed: int, must_include=()) -> np.ndarray:
    """A seeded, sorted, duplicate-free sample of n token indices in [0, T).

    ``must_include`` tokens (for example ones routed to the smallest and the
    largest expert group) are always part of the sample.
    """
    if n >= T:
        return np.arange(T, dtype=np.int64)
    rng = np.random.default_rng(seed + 7919)
    pick = set(int(t) for t in must_include)
    rest = rng.choice(T, size=n, replace=False)
    for t in rest:
        if len(pick) >= max(n, len(must_include)):
            break
        pick.add(int(t))
    return np.array(sorted(pick), dtype=np.int64)


__all__ = [
    "MoEConfig", "MoEInputs", "CONFIGS", "make_inputs", "bf16_bits", "bits_to_bf16",
    "zipf_bias", "sample_tokens", "make_shared_weights", "make_dout",
]
