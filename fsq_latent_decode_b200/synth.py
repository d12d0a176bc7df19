"""Seeded synthetic inputs shaped like the Qwen3 decode workloads.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic (no encoder, quantiser, packing or attention).  The test
suite and the benchmark use it to feed the same inputs to the CUDA library and
to the CPU oracle.

Distributions (per token, per layer):
  x     ~ N(0, 1)        residual states [N, C]          (bf16)
  E     ~ N(0, 4/C)      encoder [G, C]                   (bf16)
  W_kv  ~ N(0, 1/G)      shared decoder [2*n_kv*d_h, G]   (bf16); at L levels
                         other than 16 the standard deviation is scaled by
                         16/L (exact in bf16: a power of two), so that keys
                         and values keep the magnitude they have at 16 levels
  q     ~ N(0, 1)        queries [B, n_q, d_h]            (bf16)
  u     ~ N(0, 4)        pre-activations [N, G] (fp32): the law of E x under
                         the two lines above, used to make large caches
                         without materialising x
Draw order within one workload: x, E, W_kv, q.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    n_q: int
    n_kv: int
    d_h: int
    G: int
    C: int
    batches: tuple
    lengths: tuple
    n_new: int = 0          # tokens encoded and appended (prefill / append leg)
    note: str = ""
    levels: int = 16        # L: 4, 16 or 256 levels per coordinate (2, 4, 8 bits)


# The five seeded workloads (Qwen3-shaped single layer, L=16 levels), then the
# level-grid comparison: the same 8B-shaped layer at fixed code budgets of 80
# and 144 B/token with 4 or 256 levels (2- or 8-bit codes), the budget setting
# the latent width G = 8 * budget / b.
WORKLOADS = {
    "tiny_0p6b": Workload("tiny_0p6b", 16, 8, 128, 256, 1024, (1,), (1024,), 1024,
                          "0.6B-shaped, codes from encoding x end to end"),
    "qwen3_1p7b_32x": Workload("qwen3_1p7b_32x", 16, 8, 128, 256, 2048, (1, 4, 8), (32768,), 4096,
                               "1.7B-shaped layer, 128 B/token"),
    "qwen3_8b_32x": Workload("qwen3_8b_32x", 32, 8, 128, 256, 4096, (1, 4, 16), (8192, 32768, 131072), 4096,
                             "8B-shaped layer, 128 B/token vs 4096 B bf16"),
    "qwen3_8b_97x": Workload("qwen3_8b_97x", 32, 8, 128, 84, 4096, (1, 4, 16), (8192, 32768, 131072), 4096,
                             "8B-shaped layer, 42 B/token"),
    "long_8b_97x": Workload("long_8b_97x", 32, 8, 128, 84, 4096, (1,), (1 << 20,), 4096,
                            "8B-shaped layer, 1,048,576 cached tokens, chunked prefill of 4096"),
    "qwen3_8b_l4_80B": Workload("qwen3_8b_l4_80B", 32, 8, 128, 320, 4096, (16,), (32768,), 4096,
                                "8B-shaped layer, 4 levels (2-bit codes), 80 B/token", 4),
    "qwen3_8b_l256_80B": Workload("qwen3_8b_l256_80B", 32, 8, 128, 80, 4096, (16,), (32768,), 4096,
                                  "8B-shaped layer, 256 levels (8-bit codes), 80 B/token", 256),
    "qwen3_8b_l4_144B": Workload("qwen3_8b_l4_144B", 32, 8, 128, 576, 4096, (16,), (32768,), 4096,
                                 "8B-shaped layer, 4 levels (2-bit codes), 144 B/token", 4),
    "qwen3_8b_l256_144B": Workload("qwen3_8b_l256_144B", 32, 8, 128, 144, 4096, (16,), (32768,), 4096,
                                   "8B-shaped layer, 256 levels (8-bit codes), 144 B/token", 256),
}


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal(shape, std, gen, dtype=torch.bfloat16, device="cpu"):
    """N(0, std^2) drawn in fp32 from `gen`, then cast to `dtype`."""
    t = torch.randn(*shape, generator=gen, dtype=torch.float32, device=device)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def encoder_inputs(n_tok, C, G, gen, device="cpu"):
    """x [n_tok, C] ~ N(0,1) and E [G, C] ~ N(0, 4/C), both bf16 (x first)."""
    x = normal((n_tok, C), 1.0, gen, device=device)
    E = normal((G, C), (4.0 / C) ** 0.5, gen, device=device)
    return x, E


def decoder_inputs(B, n_q, n_kv, d_h, G, gen, device="cpu", levels=16):
    """W_kv [2*n_kv*d_h, G] ~ N(0, 1/G) (std x 16/L) then q [B, n_q, d_h] ~ N(0,1), bf16."""
    W_kv = normal((2 * n_kv * d_h, G), (1.0 / G) ** 0.5, gen, device=device)
    if levels != 16:
        W_kv = W_kv * (16.0 / levels)  # a power of two: exact in bf16
    q = normal((B, n_q, d_h), 1.0, gen, device=device)
    return W_kv, q


def preactivations(n_tok, G, gen, std=2.0, device="cpu"):
    """u [n_tok, G] fp32 ~ N(0, std^2); std=2 is the law of E x above."""
    return normal((n_tok, G), std, gen, dtype=torch.float32, device=device)


def random_bytes(shape, gen, device="cpu"):
    """Uniform bytes (any byte is a valid group of 2-, 4- or 8-bit codes)."""
    return torch.randint(0, 256, shape, generator=gen, dtype=torch.uint8, device=device)


def workload_seed(seed: int, *parts: int) -> int:
    """A derived seed for a sub-stream (batch row, chunk, ...) of one workload."""
    s = int(seed) & 0xFFFFFFFF
    for p in parts:
        s = (s * 1000003 + int(p) + 1) & 0x7FFFFFFFFFFF
    return s
