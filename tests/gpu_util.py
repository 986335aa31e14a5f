"""Helpers of the GPU parity tests: bf16 bit conversion between numpy and torch."""
import numpy as np
import torch

import oracle


def to_dev(bits: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bits -> bf16 CUDA tensor (bit-exact)."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def from_dev(t: torch.Tensor) -> np.ndarray:
    """bf16 CUDA tensor -> float64 numpy (exact)."""
    bits = t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return oracle.bf16_bits_to_f64(bits)


def rand_bf16(rng: np.random.Generator, shape, std=1.0) -> np.ndarray:
    """Random bf16-valued fp64 array (the oracle's input form)."""
    return oracle.bf16_round(rng.standard_normal(shape) * std)


def f64_to_dev(x: np.ndarray) -> torch.Tensor:
    return to_dev(oracle.f64_to_bf16_bits(x))


def i64(a) -> torch.Tensor:
    return torch.as_tensor(np.asarray(a, dtype=np.int64)).cuda()


def i32(a) -> torch.Tensor:
    return torch.as_tensor(np.asarray(a, dtype=np.int32)).cuda()
