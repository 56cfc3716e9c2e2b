"""Seeded synthetic inputs shaped like the workloads on the bitsandbytes / QLoRA
pages (7B/8B-class linear layers).  This module holds no quantization
arithmetic: it only draws random numbers, so both the CPU oracle (in the tests)
and the CUDA library can be fed the same arrays.

Recipe (numpy PCG64, float64 draws cast once to the stated dtype):
  weights      standard_normal * 0.02          -> fp32 (RN) or bf16 (RNE via torch)
  outliers     0.1% of entries, chosen without replacement with their own seed, x20
  activations  standard_normal                 -> bf16
bf16 arrays are returned as uint16 bit patterns (numpy has no bf16 dtype).
"""
from __future__ import annotations

import numpy as np

WEIGHT_STD = 0.02
OUTLIER_FRACTION = 0.001
OUTLIER_FACTOR = 20.0

# an 8B llama-shaped decoder layer: (name, rows N = out features, cols K = in features)
LLAMA8B_LAYER = (
    ("q", 4096, 4096),
    ("k", 1024, 4096),
    ("v", 1024, 4096),
    ("o", 4096, 4096),
    ("gate", 14336, 4096),
    ("up", 14336, 4096),
    ("down", 4096, 14336),
)
LLAMA8B_LAYERS = 32


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest even) with torch's CPU cast; return uint16 bits."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_weights(shape, seed: int, std: float = WEIGHT_STD, dtype: str = "f32") -> np.ndarray:
    w = (rng(seed).standard_normal(shape) * std).astype(np.float32)
    return w if dtype == "f32" else f32_to_bf16_bits(w)


def add_outliers(w_f32: np.ndarray, seed: int, fraction: float = OUTLIER_FRACTION,
                 factor: float = OUTLIER_FACTOR) -> np.ndarray:
    """Multiply `fraction` of the entries (chosen without replacement) by `factor`."""
    flat = np.array(w_f32, dtype=np.float32, copy=True).reshape(-1)
    count = int(round(flat.size * fraction))
    idx = rng(seed).choice(flat.size, size=count, replace=False)
    flat[idx] = flat[idx] * np.float32(factor)
    return flat.reshape(np.shape(w_f32))


def activations(shape, seed: int) -> np.ndarray:
    """bf16 bit patterns of standard-normal activations."""
    return f32_to_bf16_bits(rng(seed).standard_normal(shape).astype(np.float32))


def fp32_1024x1024_weight() -> np.ndarray:
    """fp32 1024x1024 ~N(0, 0.02), seed 1001 (round-trip case)."""
    return normal_weights((1024, 1024), 1001)


def bf16_4096x4096_outlier_weight() -> np.ndarray:
    """bf16 4096x4096 ~N(0, 0.02) with 0.1% x20 outliers (seeds 1002, 1003)."""
    w = add_outliers(normal_weights((4096, 4096), 1002), 1003)
    return f32_to_bf16_bits(w)


def layer_seed(layer: int, proj: int) -> int:
    """seed of projection `proj` (index into LLAMA8B_LAYER) of decoder layer `layer`"""
    return 2000 + 7 * layer + proj


def normal_weights_device(shape, seed: int, std: float = WEIGHT_STD, device: str = "cuda"):
    """bf16 ~N(0, std^2) generated on the device, for the whole-model workload (7e9 weights are too many to draw
    on the host): torch's seeded device generator, fp32 draws scaled and cast once to bf16 (nearest even).  The
    values are fixed by the seed; checks copy the tensors they need back to the host as the oracle's input."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)


def activations_device(shape, seed: int, device: str = "cuda"):
    """bf16 ~N(0, 1) activations from torch's seeded device generator (see normal_weights_device)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)

