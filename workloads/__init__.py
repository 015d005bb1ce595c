"""Seeded synthetic inputs for the NVFP4 W4A16 linear layer.

This module only draws random numbers and shapes them into the workloads
below; it holds none of the format's arithmetic (no rounding onto E2M1 or
E4M3, no scales, no dot products).  Both the CPU oracle and the CUDA path
are fed from here.

Shapes follow a 27B-class decoder layer (hidden 5120, MLP 17408) as used on
the model card "Qwen3.8-27B-NVFP4 (compressed-tensors)", section
"Measurements": batch-1 decode, 32-user decode and a 512-token prefill.
The MLP down projection of the same layer (N=5120, K=17408) is the skinny
decode shape.  There is no dataset: every tensor is drawn from a fixed seed.

Recipe (all draws from ``numpy.random.default_rng(seed).spawn(4)``; stream 0
for W, 1 for the per-row jitter, 2 for the outlier mask, 3 for x):
  * plain W:   fp32 N(0, 0.02), cast to BF16 with round-to-nearest-even.
  * layer W:   fp32 N(0, 0.02) * per-row U(0.5, 2) * (20 where a Bernoulli(1e-3)
               mask is set, else 1), then cast to BF16.
  * x / X:     fp32 N(0, 1), cast to BF16.
  * merged W:  five members q, k, v [5120, 5120] and gate, up [17408, 5120],
               each a layer W drawn from seed 16 * seed + member index, rescaled in fp32
               so that the member amaxes are A * (1, 1/3.7, 1/3.7, 1/2, 1/1.5),
               then cast to BF16 and stacked along rows.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

HIDDEN = 5120
MLP = 17408


@dataclass(frozen=True)
class LayerConfig:
    """One workload: activations X [M, K] times NVFP4 weights W [N, K]."""

    name: str
    M: int
    N: int
    K: int
    seed: int
    weights: str  # "plain", "layer" or "merged"


CONFIGS = {
    "tiny": LayerConfig("tiny N=K=1024 decode GEMV", 1, 1024, 1024, 0, "plain"),
    "decode": LayerConfig("decode GEMV N=17408 K=5120", 1, MLP, HIDDEN, 1, "layer"),
    "merged": LayerConfig("merged qkv+gate/up decode GEMV N=50176 K=5120", 1,
                          3 * HIDDEN + 2 * MLP, HIDDEN, 2, "merged"),
    "batch32": LayerConfig("32-user decode GEMM M=32 N=17408 K=5120", 32, MLP, HIDDEN, 3, "layer"),
    "prefill": LayerConfig("prefill GEMM M=512 N=17408 K=5120", 512, MLP, HIDDEN, 4, "layer"),
    # the MLP down projection of the same layer: few rows, long K (split-K decode GEMV)
    "down": LayerConfig("down-projection decode GEMV N=5120 K=17408", 1, HIDDEN, MLP, 5, "layer"),
}

# Relative amax of the five merged members (q, k, v, gate, up): a 3.7x spread,
# the largest the model card reports inside one merged group.
MERGED_MEMBER_ROWS = (HIDDEN, HIDDEN, HIDDEN, MLP, MLP)
MERGED_MEMBER_AMAX = (1.0, 1.0 / 3.7, 1.0 / 3.7, 1.0 / 2.0, 1.0 / 1.5)


def _streams(seed: int):
    return np.random.default_rng(seed).spawn(4)


def to_bf16(a: np.ndarray) -> torch.Tensor:
    """fp32 numpy array -> BF16 torch tensor (round to nearest even)."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def plain_weight_f32(N: int, K: int, seed: int) -> np.ndarray:
    rw = _streams(seed)[0]
    return rw.normal(0.0, 0.02, size=(N, K)).astype(np.float32)


def layer_weight_f32(N: int, K: int, seed: int) -> np.ndarray:
    rw, rj, ro, _ = _streams(seed)
    w = rw.normal(0.0, 0.02, size=(N, K)).astype(np.float32)
    w *= rj.uniform(0.5, 2.0, size=(N, 1)).astype(np.float32)
    mask = ro.random(size=(N, K)) < 1e-3
    w[mask] *= np.float32(20.0)
    return w


def activations(M: int, K: int, seed: int) -> torch.Tensor:
    rx = _streams(seed)[3]
    return to_bf16(rx.normal(0.0, 1.0, size=(M, K)).astype(np.float32))


def merged_members(seed: int, K: int = HIDDEN, rows=MERGED_MEMBER_ROWS,
                   rel_amax=MERGED_MEMBER_AMAX) -> list[torch.Tensor]:
    """The five members of a merged q/k/v + gate/up weight, BF16 each."""
    members = []
    target = None
    for i, (n, rel) in enumerate(zip(rows, rel_amax)):
        w = layer_weight_f32(n, K, seed * 16 + i)
        a = float(np.max(np.abs(w)))
        if target is None:
            target = a
        w *= np.float32(target * rel / a)
        members.append(to_bf16(w))
    return members


def weight_bf16(cfg: LayerConfig) -> torch.Tensor:
    """The BF16 weight W [N, K] of a workload (merged members stacked)."""
    if cfg.weights == "plain":
        return to_bf16(plain_weight_f32(cfg.N, cfg.K, cfg.seed))
    if cfg.weights == "layer":
        return to_bf16(layer_weight_f32(cfg.N, cfg.K, cfg.seed))
    if cfg.weights == "merged":
        return torch.cat(merged_members(cfg.seed, cfg.K), dim=0)
    raise ValueError(cfg.weights)


def random_bf16(shape, seed: int, std: float = 1.0) -> torch.Tensor:
    """Small seeded BF16 tensors for tests of arbitrary shape."""
    r = np.random.default_rng(seed)
    return to_bf16(r.normal(0.0, std, size=shape).astype(np.float32))


def random_codes(N: int, K: int, seed: int):
    """Random packed nibbles [N, K/2] and E4M3 scale bytes [N, K/16] (finite,
    non-negative scales in [2^-6, 15]) for tests that feed the GEMV/GEMM
    directly without quantizing."""
    r = np.random.default_rng(seed)
    q = r.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    # exponent field 1..10, any mantissa: normal E4M3 values in [2^-6, 15]
    e = r.integers(1, 11, size=(N, K // 16), dtype=np.uint8)
    m = r.integers(0, 8, size=(N, K // 16), dtype=np.uint8)
    s = ((e << 3) | m).astype(np.uint8)
    return torch.from_numpy(q), torch.from_numpy(s)
