"""Seeded synthetic inputs for the layer-streamed NF4 LoRA linear.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic (no quantisation, no matmul).  Both the CUDA path and the
CPU oracle take their inputs from here, so a parity test compares the two on
identical bits.

Generators (all counter-based, so any tensor can be regenerated alone):

* host side: numpy's Philox-4x32-10 bit generator (Salmon et al., "Parallel
  random numbers: as easy as 1, 2, 3", SC'11), keyed by a ``SeedSequence`` of
  (seed, *stream ids);
* device side (large benchmark tensors only): torch's CUDA Philox generator
  seeded from the same (seed, *stream ids) hash.

Distributions follow the workloads' stated recipes: base weights
W ~ N(0, 0.02) in fp32, LoRA A ~ U(-1/sqrt(K), 1/sqrt(K)), B ~ N(0, 0.01),
activations and output gradients ~ N(0, 1); the second parameter of N(.,.) is
read as the standard deviation.  bf16 tensors are the round-to-nearest-even
bf16 of the fp32 draw and travel to the oracle as uint16 bit patterns.
"""
from __future__ import annotations

import hashlib
from dataclasses import dataclass, field

import numpy as np

SEED = 1234

# Tensor ids used in stream keys.
T_W, T_X, T_DY, T_A, T_B, T_EMB, T_TOK = range(7)
PROJ_NAMES = ("q", "k", "v", "o", "gate", "up", "down")


def _key(seed: int, ids) -> list[int]:
    return [int(seed)] + [int(i) for i in ids]


def host_rng(seed: int, *ids) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(np.random.SeedSequence(_key(seed, ids))))


def stream_seed(seed: int, *ids) -> int:
    """A 63-bit integer seed derived from (seed, *ids) for torch generators."""
    h = hashlib.sha256(repr(_key(seed, ids)).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even) and return the bits."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_f32(shape, std: float, seed: int, *ids) -> np.ndarray:
    return (host_rng(seed, *ids).standard_normal(size=shape, dtype=np.float32) * np.float32(std)).astype(np.float32)


def uniform_f32(shape, bound: float, seed: int, *ids) -> np.ndarray:
    u = host_rng(seed, *ids).random(size=shape, dtype=np.float32)
    return ((u * np.float32(2.0) - np.float32(1.0)) * np.float32(bound)).astype(np.float32)


@dataclass
class LinearCase:
    """One LoRA linear's inputs: W fp32 [N,K]; x [T,K], dY [T,N], A [r,K], B [N,r] as bf16 bits."""
    T: int
    K: int
    N: int
    r: int
    alpha: float
    W: np.ndarray
    x: np.ndarray
    dY: np.ndarray
    A: np.ndarray
    B: np.ndarray
    meta: dict = field(default_factory=dict)

    @property
    def scale(self) -> float:
        return self.alpha / self.r


def linear_case(T: int, K: int, N: int, r: int, alpha: float, seed: int = SEED, layer: int = 0, proj: int = 0,
                w_std: float = 0.02, b_std: float = 0.01, with_w: bool = True) -> LinearCase:
    ids = (layer, proj)
    W = normal_f32((N, K), w_std, seed, *ids, T_W) if with_w else None
    x = to_bf16_bits(normal_f32((T, K), 1.0, seed, *ids, T_X))
    dY = to_bf16_bits(normal_f32((T, N), 1.0, seed, *ids, T_DY))
    A = to_bf16_bits(uniform_f32((r, K), 1.0 / np.sqrt(K), seed, *ids, T_A))
    B = to_bf16_bits(normal_f32((N, r), b_std, seed, *ids, T_B))
    return LinearCase(T, K, N, r, alpha, W, x, dY, A, B)


# ------------------------------------------------------------ workloads ---

@dataclass(frozen=True)
class StackConfig:
    """A synthetic decoder stack: per layer the seven projections (K -> N)."""
    name: str
    layers: int
    hidden: int
    kv: int
    mlp: int
    tokens: int
    rank: int
    alpha: float
    base: str            # "nf4" or "bf16"
    vocab: int = 0

    @property
    def projections(self):
        h, kv, m = self.hidden, self.kv, self.mlp
        return (("q", h, h), ("k", h, kv), ("v", h, kv), ("o", h, h),
                ("gate", h, m), ("up", h, m), ("down", m, h))

    def params_per_layer(self) -> int:
        return sum(k * n for _, k, n in self.projections)

    def flop_per_token_per_layer(self) -> int:
        """fwd + bwd (dX, dA, dB) of the seven LoRA linears, no recompute, no dW."""
        base = sum(4 * k * n for _, k, n in self.projections)
        lora = sum(6 * self.rank * (k + n) for _, k, n in self.projections)
        return base + lora


STACKS = {
    # Qwen2.5-0.5B shape, bf16 base, 2-layer pool, batch 1 x seq 512.
    "0.5b": StackConfig("qwen2.5-0.5b-shape", 24, 896, 128, 4864, 512, 16, 32.0, "bf16", vocab=151936),
    # Qwen2.5-3B shape, un-quantised bf16 base, batch 1 x seq 1024.
    "3b": StackConfig("qwen2.5-3b-shape", 36, 2048, 256, 11008, 1024, 16, 32.0, "bf16"),
    # Llama-3.1-8B shape, NF4 base, batch 1 x seq 2048.
    "8b": StackConfig("llama-3.1-8b-shape", 32, 4096, 1024, 14336, 2048, 16, 32.0, "nf4"),
    # Qwen2.5-72B shape, NF4 base, 2-layer pool, batch 1 x seq 1024.
    "72b": StackConfig("qwen2.5-72b-shape", 80, 8192, 1024, 29568, 1024, 16, 32.0, "nf4"),
}

# The single-linear case: 256 tokens, 512 -> 512, r = 8, alpha = 16.
SINGLE = dict(T=256, K=512, N=512, r=8, alpha=16.0)


def device_normal(shape, std: float, seed: int, *ids, device="cuda", dtype=None):
    """N(0, std) drawn on the device by torch's Philox generator (benchmark-size tensors)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(stream_seed(seed, *ids))
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    t.mul_(std)
    return t if dtype is None else t.to(dtype)


def device_uniform(shape, bound: float, seed: int, *ids, device="cuda", dtype=None):
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(stream_seed(seed, *ids))
    t = torch.rand(shape, generator=g, device=device, dtype=torch.float32)
    t.mul_(2.0).sub_(1.0).mul_(bound)
    return t if dtype is None else t.to(dtype)


def device_token_ids(T: int, vocab: int, seed: int, device="cuda"):
    """T token ids uniform over [0, vocab) (torch's Philox generator on the device)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(stream_seed(seed, T_TOK))
    return torch.randint(0, vocab, (T,), generator=g, device=device, dtype=torch.int64)
