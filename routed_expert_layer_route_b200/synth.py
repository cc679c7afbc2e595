"""Seeded synthetic inputs for the routed-expert MoE layer.

This module only draws random numbers and prepares inputs; it holds none of
the layer's arithmetic.  The tests feed what it returns to both the GPU
library and the CPU oracle, and the benchmark uses it for its workloads.

Recipe (shared by every workload):
  * x      : N(0, 1) draws, RMS-normalised per token (eps 1e-6, unit scale,
             float32), then rounded to bfloat16 (float32 kept for the tiny
             all-float32 case);
  * W_r    : router weights [E x d], N(0, 0.02);
  * b      : router bias [E]: none, N(0, 0.5) ("overlap"), or a Zipf(s)
             popularity bias b_e = -s * ln(rank_e) with rank a seeded
             permutation of 1..E;
  * W_gate, W_up [E x I x d], W_down [E x d x I]: N(0, 0.02).
Draw order per layer: x, W_r, b, W_gate, W_up, W_down, from one generator
seeded with ``layer_seed(seed, layer)``.  Weights are drawn directly in the
target dtype.
"""
from dataclasses import dataclass
from typing import Optional

import torch

RMS_EPS = 1e-6
W_STD = 0.02


def layer_seed(seed: int, layer: int) -> int:
    return int(seed) * 1_000_003 + int(layer) + 1


def make_generator(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def rms_normalised_tokens(T: int, d: int, g: torch.Generator, device, dtype=torch.bfloat16):
    x = torch.randn((T, d), generator=g, device=device, dtype=torch.float32)
    x = x * torch.rsqrt(x.pow(2).mean(dim=-1, keepdim=True) + RMS_EPS)
    return x.to(dtype)


def normal(shape, std: float, g: torch.Generator, device, dtype):
    t = torch.empty(shape, device=device, dtype=dtype)
    t.normal_(0.0, std, generator=g)
    return t


def router_bias(kind: Optional[str], E: int, g: torch.Generator, device, zipf_s: float = 1.1):
    if kind is None or kind == "none":
        return None
    if kind == "normal":
        return normal((E,), 0.5, g, device, torch.float32)
    if kind == "zipf":
        rank = torch.randperm(E, generator=g, device=device).to(torch.float64) + 1.0
        return (-zipf_s * torch.log(rank)).to(torch.float32)
    raise ValueError("unknown bias kind %r" % (kind,))


@dataclass
class Layer:
    x: torch.Tensor            # [T x d]
    w_router: torch.Tensor     # [E x d]
    bias: Optional[torch.Tensor]  # [E] float32 or None
    w_gate: torch.Tensor       # [E x I x d]
    w_up: torch.Tensor         # [E x I x d]
    w_down: torch.Tensor       # [E x d x I]


def make_layer(T, d, E, I, *, seed=0, layer=0, device="cpu", dtype=torch.bfloat16,
               bias: Optional[str] = None, zipf_s: float = 1.1, with_x: bool = True) -> Layer:
    g = make_generator(device, layer_seed(seed, layer))
    x = rms_normalised_tokens(T, d, g, device, dtype) if with_x else None
    w_router = normal((E, d), W_STD, g, device, dtype)
    b = router_bias(bias, E, g, device, zipf_s)
    w_gate = normal((E, I, d), W_STD, g, device, dtype)
    w_up = normal((E, I, d), W_STD, g, device, dtype)
    w_down = normal((E, d, I), W_STD, g, device, dtype)
    return Layer(x, w_router, b, w_gate, w_up, w_down)


def make_tokens(T, d, *, seed=0, stream=0, device="cpu", dtype=torch.bfloat16):
    """Extra token batches drawn from their own generator (stream >= 0)."""
    g = make_generator(device, layer_seed(seed + 7919, stream))
    return rms_normalised_tokens(T, d, g, device, dtype)


def make_logits(T, E, *, seed=0, scale=1.0, device="cpu"):
    """Float32 router logits for routing-only tests."""
    g = make_generator(device, layer_seed(seed + 104729, 0))
    return torch.randn((T, E), generator=g, device=device, dtype=torch.float32) * scale


# The five workloads of the method's evaluation (shapes, value recipe, sweep).
WORKLOADS = {
    "tiny": dict(T=4, d=64, E=16, I=32, layers=1, dtype="float32", bias=None,
                 sweep=[(2, 2), (2, 4), (2, 16)]),
    "decode_b1": dict(T=1, d=2048, E=128, I=768, layers=48, dtype="bfloat16", bias=None,
                      sweep=[(8, 8), (8, 16), (8, 128), (4, 4), (4, 16), (4, 128)]),
    "decode_small_batch": dict(T=(8, 32), d=2048, E=128, I=768, layers=48, dtype="bfloat16",
                               bias="normal", sweep=[(8, 8), (4, 16)]),
    "prefill": dict(T=4096, d=2048, E=128, I=768, layers=4, dtype="bfloat16", bias="zipf",
                    sweep=[(8, 16), (4, 16)]),
    "large": dict(T=(1, 64), d=4096, E=512, I=1024, layers=8, dtype="bfloat16", bias=None,
                  sweep=[(10, 10), (5, 20)]),
}


def torch_dtype(name: str):
    return {"float32": torch.float32, "bfloat16": torch.bfloat16}[name]


def bf16_bits(t: torch.Tensor):
    """numpy uint16 view of a bfloat16 tensor (the oracle reads these as bf16)."""
    assert t.dtype == torch.bfloat16
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")


def to_numpy(t: Optional[torch.Tensor]):
    """Oracle-ready numpy array: bf16 tensors become uint16 bit arrays."""
    if t is None:
        return None
    if t.dtype == torch.bfloat16:
        return bf16_bits(t)
    return t.detach().cpu().contiguous().numpy()
