"""Shared helpers for the parity tests: seeded inputs fed to both sides.

The oracle supplies parameter names and shapes (``oracle.weight_specs``), the
``synth`` module draws the values, and the same float32 (bf16-exact) arrays
go to the oracle (upcast to fp64) and, as bf16, to the CUDA library.
"""
from __future__ import annotations

import numpy as np

import oracle as O
import synth


def tiny_config(**kw) -> O.Config:
    """The tiny model: 1 joint + 1 single block, 4 heads x 8 (D = 32), F = 256, 8 x 8 grid."""
    c = dict(num_mmdit_layers=1, num_single_dit_layers=1, attention_head_dim=8, num_attention_heads=4,
             joint_attention_dim=32, pos_embed_max_size=64)
    c.update(kw)
    return O.Config(**c)


def full_config(**kw) -> O.Config:
    c = dict(pos_embed_max_size=64 * 64)
    c.update(kw)
    return O.Config(**c)


def af_config(cfg: O.Config, dtype: int = 0):
    """The library's configuration of an oracle configuration; dtype 1 makes
    an fp32 weight pack (fp32 arithmetic end to end)."""
    import diffusion_transformer_denoising_auraflow_b200 as af
    return af.Config.default(dtype=dtype,
        patch_size=cfg.patch_size, in_channels=cfg.in_channels, out_channels=cfg.out_channels,
        num_mmdit_layers=cfg.num_mmdit_layers, num_single_dit_layers=cfg.num_single_dit_layers,
        attention_head_dim=cfg.attention_head_dim, num_attention_heads=cfg.num_attention_heads,
        joint_attention_dim=cfg.joint_attention_dim, pos_embed_max_size=cfg.pos_embed_max_size,
        num_register_tokens=cfg.num_register_tokens, timestep_channels=cfg.timestep_channels,
        ffn_inner=0, ln_eps=cfg.ln_eps)


def draw_weights(cfg: O.Config, seed: int, names=None, dtype: str = "bf16") -> dict:
    specs = O.weight_specs(cfg)
    if names is not None:
        keep = set(names)
        specs = [s for s in specs if s[0] in keep]
    return synth.weights(seed, specs, dtype)


def block_names(cfg: O.Config, kind: str, i: int):
    pre = f"{kind}_transformer_blocks.{i}."
    return [n for n, _ in O.weight_specs(cfg) if n.startswith(pre)]


def to_bf16(arr, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32)).to(torch.bfloat16).to(device)


def to_f32(arr, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32)).to(device)


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def upload(weights_obj, w: dict):
    """Copy drawn arrays into the pack in its own dtype (bf16 or fp32)."""
    import torch
    conv = to_f32 if weights_obj.dtype == torch.float32 else to_bf16
    for name, arr in w.items():
        weights_obj.set(name, conv(arr))


def e4m3_lut():
    """Value of each of the 256 e4m3 codes (sign, 4 exponent bits with bias 7,
    3 mantissa bits; 0x7F / 0xFF NaN), from the format definition."""
    out = np.empty(256)
    for c in range(256):
        s = -1.0 if c & 0x80 else 1.0
        e, m = (c >> 3) & 0xF, c & 0x7
        if e == 0xF and m == 0x7:
            out[c] = np.nan
        elif e == 0:
            out[c] = s * m * 2.0 ** -9
        else:
            out[c] = s * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return out


def device_weights(af_module, w, seed: int, device="cuda"):
    """Fill every tensor of the pack on the device with the synthetic-input
    recipe (af_weights_init_random: the full 6.8 B-parameter model in well
    under a second); the values equal synth.weights(seed, ...) drawn on the host."""
    import torch
    w.init_random(seed, 0.02)
    torch.cuda.synchronize()
