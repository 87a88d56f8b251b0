"""Seeded synthetic inputs for the streaming-experts MoE layer.

This module is shared by the CPU oracle side (tests) and the CUDA side (tests,
benchmark).  It only draws random numbers and shapes them; it holds none of the
layer's arithmetic.  Every tensor is drawn from its own stream, seeded by
(config seed, replica, tensor name, expert), so any subset of experts can be
generated on its own and always comes out the same.

Recipe (the pages print no dataset; shapes follow the Qwen3.5-397B-shaped
layer they run: hidden 4096, 512 experts, K=4, [hakusoku] "モデルアーキテクチャ"):
  * expert weights  fp32 N(0, 0.02), then packed to 4 or 2 bits
  * shared expert   bf16 of N(0, 0.02)
  * router matrix   bf16 of N(0, 0.02)
  * router bias     -1.1 * ln(rank_e), rank a seeded permutation of 1..E
                    (Zipf(1.1)-skewed expert popularity); zero for "uniform"
  * gamma           bf16 of 1 + N(0, 0.02)
  * x, residual     bf16 of N(0, 1), fresh per token
"""
from dataclasses import dataclass, replace
import hashlib

import numpy as np


@dataclass(frozen=True)
class LayerShape:
    name: str
    hidden: int
    inter: int
    n_experts: int
    top_k: int
    bits: int = 4
    group: int = 64
    eps: float = 1e-6
    has_shared: int = 1
    tokens: int = 1
    routing: str = "zipf"  # "zipf" or "uniform" (zero bias)
    seed: int = 0


TINY = LayerShape("tiny", 256, 128, 16, 2, tokens=4, routing="uniform")
QWEN_4BIT = LayerShape("h4096_e512_k4_i1024_4bit", 4096, 1024, 512, 4, tokens=1)
QWEN_2BIT = replace(QWEN_4BIT, name="h4096_e512_k4_i1024_2bit", bits=2)


def _seed(*parts) -> int:
    h = hashlib.sha256("/".join(str(p) for p in parts).encode()).digest()
    return int.from_bytes(h[:8], "little")


def rng(*parts) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(_seed(*parts)))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest even) and return the 16-bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lower = u & 0xFFFF
    upper = u >> 16
    up = (lower > 0x8000) | ((lower == 0x8000) & ((upper & 1) == 1))
    out = (upper + up.astype(np.uint64)) & 0xFFFF
    nan = np.isnan(np.ascontiguousarray(a, dtype=np.float32))
    out = np.where(nan, (upper | 0x40) & 0xFFFF, out)
    return out.astype(np.uint16)


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    return (np.asarray(a, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def expert_weights(s: LayerShape, e: int, replica: int = 0):
    """fp32 (w_gate [I][H], w_up [I][H], w_down [H][I]) of expert e."""
    g = rng(s.seed, replica, "expert", e, s.hidden, s.inter)
    wg = g.standard_normal((s.inter, s.hidden), dtype=np.float32) * np.float32(0.02)
    wu = g.standard_normal((s.inter, s.hidden), dtype=np.float32) * np.float32(0.02)
    wd = g.standard_normal((s.hidden, s.inter), dtype=np.float32) * np.float32(0.02)
    return wg, wu, wd


def router_bias(s: LayerShape, replica: int = 0) -> np.ndarray:
    if s.routing == "uniform":
        return np.zeros(s.n_experts, dtype=np.float32)
    rank = rng(s.seed, replica, "zipf_rank", s.n_experts).permutation(s.n_experts) + 1
    return (-1.1 * np.log(rank.astype(np.float64))).astype(np.float32)


def dense_weights(s: LayerShape, replica: int = 0):
    """bf16 bit patterns of router, shared expert and gamma, plus the bias."""
    g = rng(s.seed, replica, "dense", s.hidden, s.inter, s.n_experts)
    wr = f32_to_bf16_bits(g.standard_normal((s.n_experts, s.hidden), dtype=np.float32) * np.float32(0.02))
    sg = f32_to_bf16_bits(g.standard_normal((s.inter, s.hidden), dtype=np.float32) * np.float32(0.02))
    su = f32_to_bf16_bits(g.standard_normal((s.inter, s.hidden), dtype=np.float32) * np.float32(0.02))
    sd = f32_to_bf16_bits(g.standard_normal((s.hidden, s.inter), dtype=np.float32) * np.float32(0.02))
    gamma = f32_to_bf16_bits(1.0 + g.standard_normal(s.hidden, dtype=np.float32) * np.float32(0.02))
    return dict(wr=wr, bias=router_bias(s, replica), shared_gate=sg, shared_up=su,
                shared_down=sd, gamma=gamma)


def activations(s: LayerShape, step: int = 0, tokens: int = None, replica: int = 0):
    """bf16 bit patterns of x [T][H] and residual [T][H] for one step."""
    T = s.tokens if tokens is None else tokens
    g = rng(s.seed, replica, "act", step, T, s.hidden)
    x = f32_to_bf16_bits(g.standard_normal((T, s.hidden), dtype=np.float32))
    res = f32_to_bf16_bits(g.standard_normal((T, s.hidden), dtype=np.float32))
    return x, res


def prenorm_inputs(s: LayerShape, step: int = 0, tokens: int = None, replica: int = 0):
    """bf16 bit patterns of a residual stream h [T][H] (normal values, a
    per-token scale e^U(-1, 2), every 64th channel 8x larger) and of the
    pre-norm weight gamma_pre [H] (1 + 0.02 N(0, 1))."""
    T = s.tokens if tokens is None else tokens
    g = rng(s.seed, replica, "prenorm", step, T, s.hidden)
    h = g.standard_normal((T, s.hidden), dtype=np.float32)
    h *= np.exp(g.uniform(-1.0, 2.0, (T, 1))).astype(np.float32)
    h[:, ::64] *= np.float32(8.0)
    gp = 1.0 + g.standard_normal(s.hidden, dtype=np.float32) * np.float32(0.02)
    return f32_to_bf16_bits(h), f32_to_bf16_bits(gp)


def torch_expert_weights(s: LayerShape, e0: int, n: int, replica: int, device):
    """Device-side fp32 expert weights for experts e0..e0+n-1 (benchmark scale).

    Drawn with torch's seeded device generator: same distribution as
    expert_weights, not the same numbers.  Shapes: [n][I][H], [n][I][H],
    [n][H][I]."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(_seed(s.seed, replica, "texpert", e0, n) & 0x7FFFFFFFFFFFFFFF)
    wg = torch.randn((n, s.inter, s.hidden), generator=gen, device=device) * 0.02
    wu = torch.randn((n, s.inter, s.hidden), generator=gen, device=device) * 0.02
    wd = torch.randn((n, s.hidden, s.inter), generator=gen, device=device) * 0.02
    return wg, wu, wd
