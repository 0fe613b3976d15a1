"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds no attention arithmetic: it only draws seeded normal numbers and rounds
them to bfloat16 (round to nearest even), so that the CPU oracle and the CUDA path see the
very same bf16 values.  Seeds follow one recipe: ``seed = 1000 * workload + 16 * layer +
tensor_id`` with the tensor ids below.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

TENSOR_ID = {"q": 0, "k": 1, "v": 2, "k_enc": 3, "v_enc": 4, "k_dec": 5, "v_dec": 6,
             "k_new": 7, "v_new": 8, "k_cache": 9, "v_cache": 10, "dout": 11}


def seed_for(workload: int, layer: int, tensor: str) -> int:
    return 1000 * workload + 16 * layer + TENSOR_ID[tensor]


def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest, ties to even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    return r


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


@dataclass
class Bf16Array:
    """A bf16 tensor held as its bit pattern plus the exact float32 value of each element."""

    bits: np.ndarray  # uint16
    f32: np.ndarray   # float32, exactly representable in bf16

    @property
    def shape(self):
        return self.bits.shape


def normal_bf16(shape, seed: int, sigma: float = 1.0) -> Bf16Array:
    """N(0, sigma^2) samples rounded to bf16."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(size=shape, dtype=np.float32) * np.float32(sigma)
    bits = round_to_bf16_bits(x)
    return Bf16Array(bits=bits, f32=bf16_bits_to_f32(bits))


def constant_bf16(shape, value: float) -> Bf16Array:
    bits = round_to_bf16_bits(np.full(shape, value, dtype=np.float32))
    return Bf16Array(bits=bits, f32=bf16_bits_to_f32(bits))


def to_torch(a: Bf16Array, device="cpu"):
    """Upload the bit pattern as a torch.bfloat16 tensor (no rounding happens here)."""
    import torch

    t = torch.from_numpy(a.bits.view(np.int16).copy()).view(torch.bfloat16)
    return t.to(device)
