"""Seeded synthetic inputs for the theta-bundle path.

Both sides of every parity check draw their inputs from here: the CPU oracle
(``oracle/``) and the GPU library (``linear_theta_forward_b200``). This module
holds none of the method's arithmetic -- only random draws, the bf16 storage
encoding and the projection shapes -- so that the two implementations share
nothing but their inputs.

Weight model (stand-in for real decoder checkpoints, which are not available):
every projection family has a common base ``B ~ N(0, 0.02)`` and each layer
adds its own ``N_l ~ N(0, 0.005)``, so ``W_l = B + N_l``. Activations are
``X ~ N(0, 1)``; low-rank factors are ``U, V ~ N(0, 0.01)``. Shapes follow the
Gemma 3 1B and Gemma 4 31B decoders named on "Banded sharing" (Set G for
serving) and the seven projection families of "The theta bundle" (Projection
families).

Host draws use numpy's PCG64 with one child stream per (tag, key...) so that
every tensor is reproducible on its own. Device draws (for sizes too large to
build on the host quickly) use a seeded ``torch.Generator`` on the GPU.
"""
from __future__ import annotations

import zlib
from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "FAMILIES", "Model", "TINY", "GEMMA3_1B", "GEMMA4_31B",
    "np_generator", "f32_to_bf16_bits", "bf16_bits_to_f32", "as_dtype_values",
    "host_normal", "host_family_weights", "host_lowrank", "host_activations",
    "device_family_weights", "device_normal",
]

FAMILIES = ("q", "k", "v", "o", "gate", "up", "down")


@dataclass(frozen=True)
class Model:
    """Projection shapes of one decoder: family -> (out_dim, in_dim)."""
    name: str
    num_layers: int
    shapes: dict = field(default_factory=dict)


TINY = Model("tiny", 4, {"w": (256, 256)})

GEMMA3_1B = Model("gemma3-1b", 26, {
    "q": (1024, 1152), "k": (256, 1152), "v": (256, 1152), "o": (1152, 1024),
    "gate": (6912, 1152), "up": (6912, 1152), "down": (1152, 6912),
})

GEMMA4_31B = Model("gemma4-31b", 60, {
    "q": (8192, 5376), "k": (2048, 5376), "v": (2048, 5376), "o": (5376, 8192),
    "gate": (21504, 5376), "up": (21504, 5376), "down": (5376, 21504),
})

BASE_STD = 0.02
NOISE_STD = 0.005
LOWRANK_STD = 0.01


def _key(parts) -> tuple:
    out = []
    for p in parts:
        if isinstance(p, (int, np.integer)):
            out.append(int(p) & 0xFFFFFFFF)
        else:
            out.append(zlib.crc32(str(p).encode()))
    return tuple(out)


def np_generator(seed: int, *keys) -> np.random.Generator:
    """Independent PCG64 stream for (seed, keys...)."""
    ss = np.random.SeedSequence(entropy=int(seed), spawn_key=_key(keys))
    return np.random.Generator(np.random.PCG64(ss))


def f32_to_bf16_bits(x) -> np.ndarray:
    """Encode float32 values as bf16 bit patterns, round-to-nearest-even.

    This is the storage conversion torch and CUDA apply (``__float2bfloat16_rn``);
    NaNs stay NaNs.
    """
    a = np.ascontiguousarray(x, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(a)
    if nan.any():
        r[nan] = ((u[nan] >> 16) | 0x40).astype(np.uint16)
    return r.reshape(a.shape)


def bf16_bits_to_f32(bits) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).reshape(b.shape)


def as_dtype_values(x, dtype: str) -> np.ndarray:
    """float32 array whose values are exactly representable in ``dtype``."""
    a = np.asarray(x, dtype=np.float32)
    if dtype == "f32":
        return a
    if dtype == "bf16":
        return bf16_bits_to_f32(f32_to_bf16_bits(a))
    raise ValueError(f"unknown dtype {dtype!r}")


def host_normal(shape, std: float, seed: int, *keys, dtype: str = "f32") -> np.ndarray:
    g = np_generator(seed, *keys)
    a = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return as_dtype_values(a, dtype)


def host_family_weights(num_layers: int, out_dim: int, in_dim: int, *, seed: int = 0,
                        family: str = "w", dtype: str = "f32",
                        base_std: float = BASE_STD, noise_std: float = NOISE_STD,
                        layers=None) -> np.ndarray:
    """[L, O, I] float32 array of ``B + N_l`` rounded to ``dtype``.

    ``layers`` picks a subset of layer indices (each layer has its own stream,
    so a subset equals the same slice of the full draw).
    """
    base = host_normal((out_dim, in_dim), base_std, seed, "base", family)
    idx = range(num_layers) if layers is None else layers
    out = np.empty((len(idx), out_dim, in_dim), dtype=np.float32)
    for j, layer in enumerate(idx):
        noise = host_normal((out_dim, in_dim), noise_std, seed, "noise", family, layer)
        out[j] = as_dtype_values(base + noise, dtype)
    return out


def host_lowrank(out_dim: int, in_dim: int, rank: int, *, seed: int = 0, family: str = "w",
                 layer: int = 0, dtype: str = "f32", std: float = LOWRANK_STD):
    """(U [O, r], V [I, r]) drawn N(0, std)."""
    U = host_normal((out_dim, rank), std, seed, "U", family, layer, dtype=dtype)
    V = host_normal((in_dim, rank), std, seed, "V", family, layer, dtype=dtype)
    return U, V


def host_activations(m: int, in_dim: int, *, seed: int = 0, tag="x", dtype: str = "f32") -> np.ndarray:
    return host_normal((m, in_dim), 1.0, seed, "X", tag, dtype=dtype)


# ---------------------------------------------------------------- device draws
def _torch():
    import torch  # local import: the oracle tests never need torch
    return torch


def device_normal(shape, std: float, seed: int, *keys, dtype="bf16", device="cuda"):
    """Seeded normal draw made on the GPU (harness-side, for large sizes)."""
    torch = _torch()
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) * 1000003 + sum(_key(keys))) & 0x7FFFFFFFFFFFFFFF)
    a = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        a.mul_(std)
    return a.to(torch.bfloat16) if dtype == "bf16" else a


def device_family_weights(num_layers: int, out_dim: int, in_dim: int, *, seed: int = 0,
                          family: str = "w", dtype: str = "bf16", device="cuda",
                          base_std: float = BASE_STD, noise_std: float = NOISE_STD):
    """List of L device tensors [O, I]: ``B + N_l`` drawn on the GPU, rounded once."""
    torch = _torch()
    base = device_normal((out_dim, in_dim), base_std, seed, "base", family, dtype="f32", device=device)
    out = []
    for layer in range(num_layers):
        w = device_normal((out_dim, in_dim), noise_std, seed, "noise", family, layer, dtype="f32",
                          device=device)
        w.add_(base)
        out.append(w.to(torch.bfloat16) if dtype == "bf16" else w)
    del base
    return out
