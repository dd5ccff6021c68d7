"""Seeded synthetic inputs for the routed sigmoid top-k MoE FFN.

This module is the one piece shared by the CUDA path's tests/benchmark and by
the CPU oracle's tests.  It only draws random numbers and builds id patterns;
it holds none of the method's arithmetic (no routing, no matmul, no SwiGLU).

Workloads (shapes and value distributions follow the routed-matmul and MoE
FFN pages; sizes are the ones this library is measured on):

* ``tiny``:   matmul by expert id, m=4, k=64, n=32, E=8, top_k=2; x ~N(0,1),
  W ~N(0,0.05), ids uniform and distinct per token.
* ``decode``: matmul by expert id, m=8, k=4096, n=1536, E=256, top_k=8;
  x ~N(0,1), W ~N(0,0.02), ids uniform and distinct per token.
* ``prefill``: full MoE FFN layer, m=4096, hidden 4096, inter 1536, E=256,
  top-8 sigmoid + selection-bias routing (logits ~N(0,1), bias ~U(-0.1,0.1)),
  weights ~N(0,0.02), x ~N(0,1).
* ``skewed``: the ``prefill`` layer with every token forced onto experts 0..7
  (the maximally skewed distinct routing profile of mlx-native's
  ``DenseMatmulIdRoutingProfile``).
* ``long``:   m=16384, hidden 2048, inter 768, E=128, top-8, slotted input
  rows ``[m, top_k, hidden]``, routing as in ``prefill``.
* ``prefill_e32``: the ``prefill`` layer cut to 32 experts and m=512 (profiling).
* ``skewed_e8``: the ``skewed`` layer with only its 8 experts allocated (profiling).
* ``long_e16``: the ``long`` layer cut to 16 experts and m=2048 (profiling).

Draw order for one seed (``torch.Generator(device).manual_seed(seed)``):
logits, bias, x, W_gate, W_up, W_down (or W), then ids.  bf16 values are
normal draws in f32 scaled by the std, rounded to bf16 (round to nearest
even, torch's conversion).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

SHARED_PER_TOKEN = 0
SLOTTED = 1


@dataclass(frozen=True)
class MatmulIdConfig:
    name: str
    m: int
    n: int
    k: int
    n_experts: int
    top_k: int
    w_std: float
    layout: int = SHARED_PER_TOKEN


@dataclass(frozen=True)
class FfnConfig:
    name: str
    m: int
    hidden: int
    inter: int
    n_experts: int
    top_k: int
    w_std: float = 0.02
    layout: int = SHARED_PER_TOKEN
    routing: str = "router"          # "router" | "skewed" | "balanced" | "may_repeat"
    extra: dict = field(default_factory=dict)


TINY = MatmulIdConfig("tiny", m=4, n=32, k=64, n_experts=8, top_k=2, w_std=0.05)
DECODE = MatmulIdConfig("decode", m=8, n=1536, k=4096, n_experts=256, top_k=8, w_std=0.02)
PREFILL = FfnConfig("prefill", m=4096, hidden=4096, inter=1536, n_experts=256, top_k=8)
SKEWED = FfnConfig("skewed", m=4096, hidden=4096, inter=1536, n_experts=256, top_k=8,
                   routing="skewed")
LONG = FfnConfig("long", m=16384, hidden=2048, inter=768, n_experts=128, top_k=8,
                 layout=SLOTTED)

# The prefill layer with 32 experts and m=512 (same 128 routed rows per expert,
# 1.2 GB of weights): small enough for multi-pass profiler captures.
PREFILL_E32 = FfnConfig("prefill_e32", m=512, hidden=4096, inter=1536, n_experts=32, top_k=8)

# The skewed layer with only the 8 experts it uses allocated (0.3 GB of
# weights): the tensor-bound case for multi-pass profiler captures.
SKEWED_E8 = FfnConfig("skewed_e8", m=4096, hidden=4096, inter=1536, n_experts=8, top_k=8,
                      routing="skewed")

# The long layer cut to 16 experts and m=2048 (the same 1024 routed rows per
# expert, 150 MB of weights, slotted input): for multi-pass profiler captures.
LONG_E16 = FfnConfig("long_e16", m=2048, hidden=2048, inter=768, n_experts=16, top_k=8,
                     layout=SLOTTED)

CONFIGS = {c.name: c for c in (TINY, DECODE, PREFILL, SKEWED, LONG, PREFILL_E32, SKEWED_E8,
                               LONG_E16)}


def generator(seed: int = 0, device: str | torch.device = "cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def bf16_normal(shape, std: float, gen: torch.Generator, device="cpu") -> torch.Tensor:
    """Normal(0, std) draws rounded to bf16."""
    return (torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * std).to(
        torch.bfloat16)


def uniform_bias(n: int, half_width: float, gen: torch.Generator, device="cpu") -> torch.Tensor:
    """U(-half_width, half_width) in f32."""
    return (torch.rand(n, generator=gen, device=device, dtype=torch.float32) * 2.0 - 1.0) * half_width


def uniform_distinct_ids(m: int, n_experts: int, top_k: int, gen: torch.Generator,
                         device="cpu") -> torch.Tensor:
    """Per token, top_k distinct experts drawn uniformly (a random permutation prefix)."""
    keys = torch.rand((m, n_experts), generator=gen, device=device)
    return keys.argsort(dim=1)[:, :top_k].to(torch.int32).contiguous()


def balanced_ids(m: int, n_experts: int, top_k: int, device="cpu") -> torch.Tensor:
    """ids[t, j] = (t + j) mod E (mlx-native's Balanced routing profile)."""
    t = torch.arange(m, device=device, dtype=torch.int64)[:, None]
    j = torch.arange(top_k, device=device, dtype=torch.int64)[None, :]
    return ((t + j) % n_experts).to(torch.int32).contiguous()


def skewed_ids(m: int, top_k: int, device="cpu") -> torch.Tensor:
    """ids[t, j] = j (mlx-native's MaximallySkewedDistinct routing profile)."""
    j = torch.arange(top_k, device=device, dtype=torch.int32)[None, :]
    return j.expand(m, top_k).contiguous()


def may_repeat_ids(m: int, n_experts: int, top_k: int, device="cpu") -> torch.Tensor:
    """ids[t, j] = t mod E for every slot j (mlx-native's MayRepeat routing
    profile: every slot of a token picks the same expert)."""
    t = torch.arange(m, device=device, dtype=torch.int64)[:, None]
    return (t % n_experts).expand(m, top_k).to(torch.int32).contiguous()


def matmul_id_inputs(cfg: MatmulIdConfig, seed: int = 0, device="cpu", m: int | None = None):
    """x, W, ids for a matmul-by-expert-id workload (optionally with another m)."""
    m = cfg.m if m is None else m
    g = generator(seed, device)
    x_rows = m if cfg.layout == SHARED_PER_TOKEN else m * cfg.top_k
    x = bf16_normal((x_rows, cfg.k), 1.0, g, device)
    if cfg.layout == SLOTTED:
        x = x.view(m, cfg.top_k, cfg.k)
    W = bf16_normal((cfg.n_experts, cfg.n, cfg.k), cfg.w_std, g, device)
    ids = uniform_distinct_ids(m, cfg.n_experts, cfg.top_k, g, device)
    return {"x": x, "W": W, "ids": ids}


def ffn_inputs(cfg: FfnConfig, seed: int = 0, device="cpu", m: int | None = None,
               n_experts: int | None = None):
    """logits, bias, x, W_gate, W_up, W_down (+ forced ids for skewed/balanced)."""
    m = cfg.m if m is None else m
    E = cfg.n_experts if n_experts is None else n_experts
    g = generator(seed, device)
    logits = torch.randn((m, E), generator=g, device=device, dtype=torch.float32)
    bias = uniform_bias(E, 0.1, g, device)
    x_rows = m if cfg.layout == SHARED_PER_TOKEN else m * cfg.top_k
    x = bf16_normal((x_rows, cfg.hidden), 1.0, g, device)
    if cfg.layout == SLOTTED:
        x = x.view(m, cfg.top_k, cfg.hidden)
    W_gate = bf16_normal((E, cfg.inter, cfg.hidden), cfg.w_std, g, device)
    W_up = bf16_normal((E, cfg.inter, cfg.hidden), cfg.w_std, g, device)
    W_down = bf16_normal((E, cfg.hidden, cfg.inter), cfg.w_std, g, device)
    out = {"logits": logits, "bias": bias, "x": x, "W_gate": W_gate, "W_up": W_up,
           "W_down": W_down}
    if cfg.routing == "skewed":
        out["ids"] = skewed_ids(m, cfg.top_k, device)
    elif cfg.routing == "balanced":
        out["ids"] = balanced_ids(m, E, cfg.top_k, device)
    elif cfg.routing == "may_repeat":
        out["ids"] = may_repeat_ids(m, E, cfg.top_k, device)
    return out


def shared_expert_inputs(hidden: int, inter_sh: int, seed: int = 0, device="cpu",
                         w_std: float = 0.02, gate_std: float = 0.02):
    """Shared expert weights: gate row w_sh [hidden], W_sh_gate / W_sh_up
    [inter_sh, hidden], W_sh_down [hidden, inter_sh] (bf16 normals)."""
    g = generator(seed + 7919, device)
    return {"w_sh": bf16_normal((hidden,), gate_std, g, device),
            "W_sh_gate": bf16_normal((inter_sh, hidden), w_std, g, device),
            "W_sh_up": bf16_normal((inter_sh, hidden), w_std, g, device),
            "W_sh_down": bf16_normal((hidden, inter_sh), w_std, g, device)}


def bf16_bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (host copy)."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view("uint16")
