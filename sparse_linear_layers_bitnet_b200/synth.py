"""Seeded synthetic inputs shared by the tests, the benchmark and the smoke check.

This module holds no arithmetic of the method: it only draws random numbers
with fixed seeds in the shapes and distributions of the workloads (Gaussian
master weights, Gaussian activations with sparse outliers, random-walk weight
updates).  Both the CUDA path and the CPU oracle receive copies of the same
arrays, so neither depends on the other's random number generator.
"""
from __future__ import annotations

import numpy as np

# Shapes of the workloads (output features x input features).
LLAMA_2B = dict(hidden=2560, ffn=6912)
LLAMA_3B = dict(hidden=3200, ffn=8640, layers=26, heads=32)

DECODE_2B_MATRICES = [  # (name, K, N_out)
    ("qkv", 2560, 3840),
    ("o", 2560, 2560),
    ("gate_up", 2560, 13824),
    ("down", 6912, 2560),
]

PREFILL_7B_GEMMS = [  # (name, T, K, N_out)
    ("up", 4096, 4096, 11008),
    ("down", 4096, 11008, 4096),
]

LAYER_3B_MATRICES = [  # (name, N_out, K) for the per-step pack over a 3B model
    ("q", 3200, 3200), ("k", 3200, 3200), ("v", 3200, 3200), ("o", 3200, 3200),
    ("gate", 8640, 3200), ("up", 8640, 3200), ("down", 3200, 8640),
]


def rng(seed: int) -> np.random.Generator:
    return np.random.default_rng(seed)


def master_weights(n_out: int, k: int, sigma: float = 0.02, seed: int = 0) -> np.ndarray:
    """fp32 master weights ~ N(0, sigma), shape [n_out, k]."""
    return rng(seed).normal(0.0, sigma, size=(n_out, k)).astype(np.float32)


def activations(t: int, k: int, seed: int = 1, outlier_p: float = 0.0,
                outlier_scale: float = 20.0) -> np.ndarray:
    """fp32 activations ~ N(0, 1) [t, k]; each element independently, with
    probability outlier_p, multiplied by outlier_scale."""
    g = rng(seed)
    x = g.normal(0.0, 1.0, size=(t, k)).astype(np.float32)
    if outlier_p > 0:
        hit = g.random(size=(t, k)) < outlier_p
        x = np.where(hit, x * np.float32(outlier_scale), x).astype(np.float32)
    return x


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even) and return the uint16 bits.
    Inputs are drawn in fp32 and then stored as bf16; this is data preparation,
    not part of the method."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(u16: np.ndarray) -> np.ndarray:
    return (u16.astype(np.uint32) << np.uint32(16)).view(np.float32)


def random_walk_step(w: np.ndarray, sigma: float = 1e-4, seed: int = 0) -> np.ndarray:
    """W_{s+1} = W_s + N(0, sigma) (one step of the per-step pack workload)."""
    return (w + rng(seed).normal(0.0, sigma, size=w.shape).astype(np.float32)).astype(np.float32)


def torch_master_weights(n_out: int, k: int, sigma: float = 0.02, seed: int = 0, device="cuda"):
    """Same distribution as master_weights(), drawn on the device by torch
    (for the large benchmark workloads; the oracle gets a host copy)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return torch.randn((n_out, k), generator=g, device=device, dtype=torch.float32) * sigma


def torch_activations(t: int, k: int, seed: int = 1, outlier_p: float = 0.0,
                      outlier_scale: float = 20.0, dtype=None, device="cuda"):
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    x = torch.randn((t, k), generator=g, device=device, dtype=torch.float32)
    if outlier_p > 0:
        hit = torch.rand((t, k), generator=g, device=device) < outlier_p
        x = torch.where(hit, x * outlier_scale, x)
    if dtype is not None:
        x = x.to(dtype)
    return x


def torch_random_walk_(w, sigma: float = 1e-4, seed: int = 0):
    import torch
    g = torch.Generator(device=w.device)
    g.manual_seed(seed)
    w.add_(torch.randn(w.shape, generator=g, device=w.device, dtype=w.dtype) * sigma)
    return w
