"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module only makes random numbers: it holds none of the attention
arithmetic.  Two generators:

* ``normal_bf16_bits``: numpy PCG64 standard normals, rounded to bf16 with
  round-to-nearest-even on the bit pattern, returned as uint16.  Used for every
  input the CPU oracle must see in full.
* ``cuda_normal_bf16``: torch's CUDA generator, for the multi-GB tensors of the
  long-context and decode workloads.  Tests that check those read the sampled
  slices they need back to the host before handing them to the oracle.

Seeds are ``BASE_SEED + tensor id`` with the ids below, so a given tensor of a
given workload is always the same bits.
"""

from __future__ import annotations

import numpy as np

BASE_SEED = 1234
TENSOR_ID = {"q": 0, "k": 1, "v": 2, "do": 3, "k_cache": 4, "v_cache": 5, "q_t": 6}


def seed_of(name: str, extra: int = 0) -> int:
    return BASE_SEED + TENSOR_ID[name] + 1000 * extra


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest-even) and return the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def normal_bf16_bits(shape, seed: int) -> np.ndarray:
    """Standard normal draws (PCG64, float32) rounded to bf16; uint16 bit patterns."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return f32_to_bf16_bits(rng.standard_normal(size=shape, dtype=np.float32))


def bits_to_torch(bits: np.ndarray, device="cpu"):
    """uint16 bf16 bit patterns -> torch.bfloat16 tensor on `device` (same bits)."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(device)


def torch_to_bits(t) -> np.ndarray:
    """torch.bfloat16 tensor (any device) -> numpy uint16 bit patterns."""
    import torch

    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def cuda_normal_bf16(shape, seed: int, device="cuda"):
    """Standard normal bf16 tensor drawn on the device with torch's generator."""
    import torch

    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)
