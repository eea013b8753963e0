"""Write the fp64 oracle's velocity for the two full-size workloads.

Calls only ``oracle`` and ``synth``.  The stored arrays are what the GPU
parity tests (``tests/test_gpu_full_forward.py``) compare the CUDA path's
forward and denoise step against:

* ``full_forward_1024.npy``: the AuraFlow forward at 1024 x 1024 (latent
  4 x 128 x 128 duplicated into a CFG batch of 2, text embeddings
  [2, 256, 2048] with the uncond prompt first, 64 x 64 position grid) at the
  first step of the 25-step, shift-1.73 schedule (model time t = sigma_0 = 1).
* ``full_forward_1536.npy``: the same at 1536 x 1536 (latent 4 x 192 x 192,
  96 x 96 position grid), also at sigma_0.

Weights are the full model (4 joint + 32 single blocks, D = 3072) drawn by
``synth.weights`` (linear weights and biases ~N(0, 0.02^2), positions
~N(0, 0.1^2), registers ~N(0, 0.02^2)); the forward streams them block by
block so only one block is held at a time.  The arrays are float32 copies of
the fp64 result; ``full_forward.json`` records the inputs.

    python tests/golden/make_full_forward.py [1024] [1536]
"""
from __future__ import annotations

import hashlib
import json
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle as O  # noqa: E402
import synth  # noqa: E402

WORKLOADS = {
    # name: (seed, latent side, position grid side, text tokens)
    "1024": (4, 128, 64, 256),
    "1536": (5, 192, 96, 256),
}
N_STEPS, SHIFT = 25, 1.73


def block_specs(cfg, prefix):
    return [s for s in O.weight_specs(cfg) if s[0].startswith(prefix)]


def streamed_forward(cfg, seed, lat, text, t, log=print):
    """O.transformer_forward with each block's weights drawn just before it
    runs (same calls in the same order, weights by name from synth)."""
    blocks = ("joint_transformer_blocks.", "single_transformer_blocks.")
    misc = synth.weights(seed, [s for s in O.weight_specs(cfg) if not s[0].startswith(blocks)])
    H, W = lat.shape[2], lat.shape[3]
    img, txt, temb = O.embed(lat, text, t, misc, cfg)
    for i in range(cfg.num_mmdit_layers):
        pre = f"joint_transformer_blocks.{i}."
        t0 = time.time()
        w = synth.weights(seed, block_specs(cfg, pre))
        txt, img = O.joint_block(img, txt, temb, w, pre, cfg)
        log(f"  joint {i}: {time.time() - t0:.1f} s")
    nt = txt.shape[1]
    x = np.concatenate([txt, img], axis=1)
    del txt, img
    for i in range(cfg.num_single_dit_layers):
        pre = f"single_transformer_blocks.{i}."
        t0 = time.time()
        w = synth.weights(seed, block_specs(cfg, pre))
        x = O.single_block(x, temb, w, pre, cfg)
        log(f"  single {i}: {time.time() - t0:.1f} s")
    return O.output_stage(x[:, nt:], temb, misc, cfg, H, W)


def oracle_sha1():
    h = hashlib.sha1()
    for name in ("auraflow.py", "__init__.py"):
        with open(os.path.join(ROOT, "oracle", name), "rb") as f:
            h.update(f.read())
    with open(os.path.join(ROOT, "synth", "__init__.py"), "rb") as f:
        h.update(f.read())
    return h.hexdigest()


def make(name):
    seed, side, G, L = WORKLOADS[name]
    cfg = O.Config(pos_embed_max_size=G * G)
    lat1 = synth.latents(seed, (1, 4, side, side))
    lat = np.concatenate([lat1, lat1])
    text = synth.text_embeddings(seed, (2, L, cfg.joint_attention_dim))
    sigma0 = float(np.float32(O.sigma_schedule(N_STEPS, SHIFT)[0]))
    t = np.full((2,), sigma0, dtype=np.float32)
    t0 = time.time()
    v = streamed_forward(cfg, seed, lat, text, t)
    secs = time.time() - t0
    out = os.path.join(HERE, f"full_forward_{name}.npy")
    np.save(out, v.astype(np.float32))
    meta_path = os.path.join(HERE, "full_forward.json")
    meta = {}
    if os.path.exists(meta_path):
        with open(meta_path) as f:
            meta = json.load(f)
    meta[name] = {
        "file": os.path.basename(out), "seed": seed, "latent": [1, 4, side, side], "cfg_batch": 2,
        "text": [2, L, cfg.joint_attention_dim], "pos_grid": [G, G], "t": sigma0, "weight_std": 0.02,
        "model": "4 joint + 32 single blocks, D = 3072 (12 x 256), FFN 8192",
        "oracle_and_synth_sha1": oracle_sha1(), "oracle_seconds": round(secs, 1),
        "velocity_rms": float(np.sqrt(np.mean(v ** 2))),
    }
    with open(meta_path, "w") as f:
        json.dump(meta, f, indent=1, sort_keys=True)
    print(f"{name}: wrote {out} ({secs:.0f} s)", flush=True)


if __name__ == "__main__":
    for name in sys.argv[1:] or sorted(WORKLOADS):
        make(name)
