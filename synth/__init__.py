"""Seeded synthetic inputs shared by the oracle tests and the CUDA path.

This module holds no arithmetic of the denoising method.  It only draws
numbers: every tensor is a function of ``(seed, name, shape, std)`` so the
oracle and the CUDA library can be fed bit-identical values without either
side importing the other.

Recipe (the same for every tensor; the CUDA library's
``af_weights_init_random`` implements the same recipe on the device, from the
same published definitions, so a weight pack it fills holds these values):

* element ``j`` of a tensor (row-major) belongs to block ``j // 4``, lane
  ``j % 4``;
* block ``n`` is the output of the counter-based generator Philox4x32-10
  (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as 1, 2, 3",
  SC 2011) with key ``(seed mod 2^32, seed div 2^32)`` and counter
  ``(n mod 2^32, n div 2^32, crc32(name), 0)``; its four 32-bit words
  ``x0..x3`` become uniforms ``u = (x + 1/2) / 2^32`` in (0, 1);
* the Box-Muller transform turns ``(u0, u1)`` into lanes 0 and 1,
  ``r cos(2 pi u1)`` and ``r sin(2 pi u1)`` with ``r = sqrt(-2 ln u0)``, and
  ``(u2, u3)`` likewise into lanes 2 and 3 (float64 throughout);
* the value is ``float32(z * float32(std))`` (the product in float64, one
  rounding to float32, to nearest even);
* for ``dtype="bf16"`` that float32 value is rounded to bfloat16 with
  round-to-nearest-even (the storage dtype of weights and activations) and
  returned as float32 holding the bf16 value (``bf16_bits`` gives the raw
  16-bit pattern that is uploaded to the GPU).

Every element is a pure function of its index, so any slice can be drawn on
its own; chunks are drawn on a thread pool (numpy releases the GIL while it
works on large arrays), which keeps multi-GB weight sets tractable on a host.
"""
from __future__ import annotations

import os
import zlib
from concurrent.futures import ThreadPoolExecutor

import numpy as np

CHUNK = 1 << 22          # elements per work item (a multiple of 4: chunks hold whole blocks)
_POOL = None

# Philox4x32 constants (the published multipliers and Weyl key increments)
PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9
PHILOX_W1 = 0xBB67AE85
PHILOX_ROUNDS = 10
TWO_PI = 6.283185307179586476925286766559
_M32 = np.uint64(0xFFFFFFFF)
_S32 = np.uint64(32)


def _pool():
    global _POOL
    if _POOL is None:
        _POOL = ThreadPoolExecutor(max_workers=max(1, min(32, os.cpu_count() or 1)))
    return _POOL


def philox4x32(c0, c1, c2, c3, k0: int, k1: int, rounds: int = PHILOX_ROUNDS):
    """Philox4x32 bijection of the counter words (uint64 arrays holding
    32-bit values) under the key (k0, k1); returns the four output words.

    Each round multiplies c0 by M0 and c2 by M1 (64-bit products split into
    high and low halves) and mixes:  (hi(M1 c2) ^ c1 ^ k0, lo(M1 c2),
    hi(M0 c0) ^ c3 ^ k1, lo(M0 c0)); the key is bumped by the Weyl constants
    (W0, W1) before every round but the first.
    """
    m0, m1 = np.uint64(PHILOX_M0), np.uint64(PHILOX_M1)
    c0, c1, c2, c3 = (np.asarray(c, dtype=np.uint64) for c in (c0, c1, c2, c3))
    for r in range(rounds):
        kr0 = np.uint64((k0 + r * PHILOX_W0) & 0xFFFFFFFF)
        kr1 = np.uint64((k1 + r * PHILOX_W1) & 0xFFFFFFFF)
        p0 = m0 * c0
        p1 = m1 * c2
        c0, c1, c2, c3 = (p1 >> _S32) ^ c1 ^ kr0, p1 & _M32, (p0 >> _S32) ^ c3 ^ kr1, p0 & _M32
    return c0, c1, c2, c3


def name_key(name: str) -> int:
    """32-bit key of a tensor name: CRC-32 (IEEE 802.3 polynomial, reflected,
    initial and final XOR 0xFFFFFFFF) of its UTF-8 bytes."""
    return zlib.crc32(name.encode("utf-8")) & 0xFFFFFFFF


def standard_normal_blocks(seed: int, key: int, first_block: int, n_blocks: int) -> np.ndarray:
    """Standard normals of blocks [first_block, first_block + n_blocks):
    float64 array of 4 * n_blocks values in element order."""
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    n = np.arange(first_block, first_block + n_blocks, dtype=np.uint64)
    x0, x1, x2, x3 = philox4x32(n & _M32, n >> _S32, np.full(n.shape, key, np.uint64),
                                np.zeros(n.shape, np.uint64), seed & 0xFFFFFFFF, seed >> 32)
    out = np.empty((n_blocks, 4), dtype=np.float64)
    for (xa, xb), lane in (((x0, x1), 0), ((x2, x3), 2)):
        ua = (xa.astype(np.float64) + 0.5) * 2.0 ** -32
        ub = (xb.astype(np.float64) + 0.5) * 2.0 ** -32
        r = np.sqrt(-2.0 * np.log(ua))
        th = TWO_PI * ub
        out[:, lane] = r * np.cos(th)
        out[:, lane + 1] = r * np.sin(th)
    return out.reshape(-1)


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
    if dtype not in ("bf16", "f32"):
        raise ValueError(f"unknown dtype {dtype!r}")
    shape = tuple(int(s) for s in shape)
    n = int(np.prod(shape)) if shape else 1
    key = name_key(name)
    std32 = float(np.float32(std))
    out = np.empty(n, dtype=np.float32)
    nchunks = (n + CHUNK - 1) // CHUNK

    def fill(i):
        lo = i * CHUNK
        hi = min(n, lo + CHUNK)
        z = standard_normal_blocks(seed, key, lo // 4, (hi - lo + 3) // 4)[: hi - lo]
        v = (z * std32).astype(np.float32)
        if dtype == "bf16":
            v = bf16_round(v)
        out[lo:hi] = v

    if nchunks <= 1:
        for i in range(nchunks):
            fill(i)
    else:
        list(_pool().map(fill, range(nchunks)))
    return out.reshape(shape)


def weight_std(name: str, std: float = 0.02) -> float:
    """Standard deviation of the synthetic draw for a named parameter.

    Linear weights and biases use ``std`` (0.02 in every workload).  The
    learned position table uses 0.1 and the register tokens 0.02, the scales
    the architecture description gives for their random initialisation (the
    AuraFlowTransformer2DModel article, sections "Patch Embedding" and
    "Register Tokens").
    """
    if name.endswith("pos_embed.pos_embed"):
        return 0.1
    if name == "register_tokens":
        return 0.02
    return std


def weights(seed: int, specs, dtype: str = "bf16", std: float = 0.02) -> dict:
    """Draw every ``(name, shape)`` in ``specs``; returns {name: float32 array}."""
    return {name: normal(seed, name, shape, weight_std(name, std), dtype) for name, shape in specs}


def latents(seed: int, shape) -> np.ndarray:
    """Latent noise ~N(0,1), float32 (latents are kept in fp32)."""
    return normal(seed, "latents", shape, 1.0, "f32")


def text_embeddings(seed: int, shape, dtype: str = "bf16") -> np.ndarray:
    """Synthetic text-encoder output ~N(0,1), bf16-exact float32 (or plain float32)."""
    return normal(seed, "text_embeddings", shape, 1.0, dtype)


def activations(seed: int, name: str, shape) -> np.ndarray:
    """Synthetic hidden states ~N(0,1), bf16-exact float32."""
    return normal(seed, name, shape, 1.0, "bf16")


def conditioning(seed: int, shape) -> np.ndarray:
    """Synthetic conditioning vector (timestep embedding) ~N(0,1), float32."""
    return normal(seed, "temb", shape, 1.0, "f32")
