"""Seeded synthetic inputs shared by the oracle tests and the CUDA path.

This module holds no arithmetic of the denoising method.  It only draws
numbers: every tensor is a function of ``(seed, name, shape, std)`` so the
oracle and the CUDA library can be fed bit-identical values without either
side importing the other.

Recipe (the same for every tensor):

* the tensor is cut into chunks of ``CHUNK`` elements in row-major order;
* chunk ``i`` is drawn from numpy's PCG64 seeded with
  ``SeedSequence([seed, crc32(name), i])`` as float32 standard normals,
  scaled by ``std``;
* for ``dtype="bf16"`` the float32 value is rounded to bfloat16 with
  round-to-nearest-even (the storage dtype of weights and activations) and
  returned as float32 holding the bf16 value (``bf16_bits`` gives the raw
  16-bit pattern that is uploaded to the GPU).

PCG64 + SeedSequence is platform independent, so a stored expected value
written by the oracle on one machine matches inputs drawn on another.
Chunks are drawn on a thread pool (numpy releases the GIL while filling),
which keeps multi-GB weight sets tractable on a host.
"""
from __future__ import annotations

import zlib
from concurrent.futures import ThreadPoolExecutor
import os

import numpy as np

CHUNK = 1 << 22
_POOL = None


def _pool():
    global _POOL
    if _POOL is None:
        _POOL = ThreadPoolExecutor(max_workers=max(1, min(32, os.cpu_count() or 1)))
    return _POOL


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); float32 out."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    # NaN stays NaN (never produced by the recipe, kept for completeness)
    r = np.where(np.isnan(x), u, r)
    return r.astype(np.uint32).view(np.float32).reshape(x.shape)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of float32 values that are already bf16-exact."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def normal(seed: int, name: str, shape, std: float = 1.0, dtype: str = "bf16") -> np.ndarray:
    """Seeded N(0, std^2) tensor of ``shape``; float32 array (bf16-exact if dtype='bf16')."""
    shape = tuple(int(s) for s in shape)
    n = int(np.prod(shape)) if shape else 1
    key = zlib.crc32(name.encode("utf-8"))
    out = np.empty(n, dtype=np.float32)
    nchunks = (n + CHUNK - 1) // CHUNK

    def fill(i):
        lo = i * CHUNK
        hi = min(n, lo + CHUNK)
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), key, i])))
        v = g.standard_normal(hi - lo, dtype=np.float32)
        v *= np.float32(std)
        if dtype == "bf16":
            v = bf16_round(v)
        elif dtype != "f32":
            raise ValueError(f"unknown dtype {dtype!r}")
        out[lo:hi] = v

    if nchunks <= 1:
        for i in range(nchunks):
            fill(i)
    else:
        list(_pool().map(fill, range(nchunks)))
    return out.reshape(shape)


def weight_std(name: str) -> float:
    """Standard deviation of the synthetic draw for a named parameter.

    Linear weights and biases use 0.02.  The learned position table uses 0.1
    and the register tokens 0.02, the scales the architecture description
    gives for their random initialisation (the AuraFlowTransformer2DModel
    article, sections "Patch Embedding" and "Register Tokens").
    """
    if name.endswith("pos_embed.pos_embed"):
        return 0.1
    return 0.02


def weights(seed: int, specs, dtype: str = "bf16") -> dict:
    """Draw every ``(name, shape)`` in ``specs``; returns {name: float32 array}."""
    return {name: normal(seed, name, shape, weight_std(name), dtype) for name, shape in specs}


def latents(seed: int, shape) -> np.ndarray:
    """Latent noise ~N(0,1), float32 (latents are kept in fp32)."""
    return normal(seed, "latents", shape, 1.0, "f32")


def text_embeddings(seed: int, shape) -> np.ndarray:
    """Synthetic text-encoder output ~N(0,1), bf16-exact float32."""
    return normal(seed, "text_embeddings", shape, 1.0, "bf16")


def activations(seed: int, name: str, shape) -> np.ndarray:
    """Synthetic hidden states ~N(0,1), bf16-exact float32."""
    return normal(seed, name, shape, 1.0, "bf16")


def conditioning(seed: int, shape) -> np.ndarray:
    """Synthetic conditioning vector (timestep embedding) ~N(0,1), float32."""
    return normal(seed, "temb", shape, 1.0, "f32")
