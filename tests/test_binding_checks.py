"""Size checks of the Python binding (no GPU needed).

The C library receives raw device pointers, so it cannot see a buffer that
is smaller than the call implies; the binding compares every tensor's shape
with the shape the call implies and reports a mismatch as AF_ERR_SHAPE
before anything is launched.  On this CPU-only host, a call whose shapes are
right passes those checks and stops at the first device-pointer check
(TypeError: CPU tensors); a call with one wrong shape stops with AFError.
The valid shapes below are the ones the GPU tests use.
"""
import pytest
import torch

import diffusion_transformer_denoising_auraflow_b200 as af

BF, F32, U8 = torch.bfloat16, torch.float32, torch.uint8


class _Fake:
    """Stands in for Weights / Scratch: only .cfg and .handle are read before
    the library is called."""

    def __init__(self, **kw):
        self.cfg = af.Config.default(**kw)
        self.handle = None


def _tiny():
    return _Fake(num_mmdit_layers=1, num_single_dit_layers=1, attention_head_dim=8, num_attention_heads=4,
                 joint_attention_dim=32, pos_embed_max_size=64)


def _ok(fn, *a, **k):
    with pytest.raises(TypeError, match="CUDA tensor"):
        fn(*a, **k)


def _bad(fn, *a, **k):
    with pytest.raises(af.AFError) as ei:
        fn(*a, **k)
    assert ei.value.status == af.AF_ERR_SHAPE


def z(*shape, dtype=F32):
    return torch.zeros(*shape, dtype=dtype)


def test_timestep_embed():
    w, s = _tiny(), _Fake()
    _ok(af.timestep_embed, w, s, z(4), z(4, 32))
    _bad(af.timestep_embed, w, s, z(4), z(4, 31))
    _bad(af.timestep_embed, w, s, z(4), z(3, 32))
    _bad(af.timestep_embed_noalloc, w, z(4), z(4, 33))


def test_patch_embed():
    w, s = _tiny(), _Fake()
    _ok(af.patch_embed, w, s, z(2, 4, 16, 16), z(2, 64, 32, dtype=BF))
    _ok(af.patch_embed, w, s, z(2, 4, 12, 16), z(2, 48, 32, dtype=BF))
    _ok(af.patch_embed, w, s, z(1, 4, 15, 16), z(1, 64, 32, dtype=BF))   # odd height: the library rejects it
    _bad(af.patch_embed, w, s, z(2, 4, 16, 16), z(2, 63, 32, dtype=BF))
    _bad(af.patch_embed, w, s, z(2, 3, 16, 16), z(2, 64, 32, dtype=BF))


def test_blocks():
    w, s = _tiny(), _Fake()
    _ok(af.joint_block, w, s, 0, z(2, 64, 32, dtype=BF), z(2, 16, 32, dtype=BF), z(2, 32))
    _bad(af.joint_block, w, s, 0, z(2, 64, 32, dtype=BF), z(2, 16, 31, dtype=BF), z(2, 32))
    _bad(af.joint_block, w, s, 0, z(2, 64, 32, dtype=BF), z(1, 16, 32, dtype=BF), z(2, 32))
    _bad(af.joint_block, w, s, 0, z(2, 64, 32, dtype=BF), z(2, 16, 32, dtype=BF), z(1, 32))
    _ok(af.single_block, w, s, 0, z(2, 80, 32, dtype=BF), z(2, 32))
    _bad(af.single_block, w, s, 0, z(2, 80, 64, dtype=BF), z(2, 32))
    _bad(af.single_block, w, s, 0, z(2, 80, 32, dtype=BF), z(2, 31))


def test_forward_and_step():
    w, s = _tiny(), _Fake()
    _ok(af.transformer_forward, w, s, z(2, 4, 16, 16), z(2, 8, 32, dtype=BF), z(2), z(2, 4, 16, 16))
    _bad(af.transformer_forward, w, s, z(2, 4, 16, 16), z(2, 8, 32, dtype=BF), z(2), z(2, 4, 16, 15))
    _bad(af.transformer_forward, w, s, z(2, 4, 16, 16), z(2, 8, 31, dtype=BF), z(2), z(2, 4, 16, 16))
    _bad(af.transformer_forward, w, s, z(2, 4, 16, 16), z(2, 8, 32, dtype=BF), z(3), z(2, 4, 16, 16))
    _bad(af.transformer_forward, w, s, z(2, 3, 16, 16), z(2, 8, 32, dtype=BF), z(2), z(2, 3, 16, 16))
    _ok(af.denoise_step, w, s, z(1, 4, 16, 16), z(2, 8, 32, dtype=BF), 3.5, 0.8, 0.7)
    _bad(af.denoise_step, w, s, z(1, 4, 16, 16), z(2, 8, 33, dtype=BF), 3.5, 0.8, 0.7)
    _ok(af.Sampler, w, s, z(1, 4, 16, 16), z(2, 8, 32, dtype=BF), [1.0, 0.5, 0.0], 3.5)
    _bad(af.Sampler, w, s, z(1, 4, 16, 16), z(2, 8, 16, dtype=BF), [1.0, 0.5, 0.0], 3.5)


def test_building_blocks():
    D = 32
    md = z(2, 6 * D)
    _ok(af.ln_modulate, z(2, 37, D, dtype=BF), md[:, 3 * D:], md[:, 4 * D:], 6 * D, z(2, 37, D, dtype=BF), 1e-6)
    _bad(af.ln_modulate, z(2, 37, D, dtype=BF), md[:, 3 * D:], md[:, 4 * D:], 6 * D, z(2, 37, D - 1, dtype=BF),
         1e-6)
    _ok(af.ln_modulate_e4m3, z(2, 300, D, dtype=BF), md[:, 3 * D:], md[:, 4 * D:], 6 * D, z(600, D, dtype=U8),
        z(600), 1e-6)
    _bad(af.ln_modulate_e4m3, z(2, 300, D, dtype=BF), md[:, 3 * D:], md[:, 4 * D:], 6 * D,
         z(600, D - 1, dtype=U8), z(600), 1e-6)
    _ok(af.linear, z(300, 256, dtype=BF), z(520, 256, dtype=BF), z(300, 520, dtype=BF))
    _bad(af.linear, z(300, 256, dtype=BF), z(520, 248, dtype=BF), z(300, 520, dtype=BF))
    _bad(af.linear, z(300, 256, dtype=BF), z(520, 256, dtype=BF), z(300, 512, dtype=BF))
    q = z(1, 2, 7, 256, dtype=BF)
    _ok(af.attention, q, q, q, z(1, 7, 512, dtype=BF))
    _bad(af.attention, q, q, q, z(1, 7, 256, dtype=BF))
    _bad(af.attention, q, z(1, 2, 8, 256, dtype=BF), q, z(1, 7, 512, dtype=BF))
    _ok(af.quantize_rows_e4m3, z(37, 3072, dtype=BF), z(37, 3072, dtype=U8), z(37))
    _bad(af.quantize_rows_e4m3, z(37, 3072, dtype=BF), z(37, 3056, dtype=U8), z(37))
    _bad(af.quantize_rows_e4m3, z(37, 3072, dtype=BF), z(37, 3072, dtype=U8), z(36))
    _ok(af.linear_fp8, z(300, 256, dtype=U8), z(300), z(520, 256, dtype=U8), z(768), z(300, 520, dtype=BF))
    _bad(af.linear_fp8, z(300, 256, dtype=U8), z(300), z(520, 256, dtype=U8), z(768), z(300, 521, dtype=BF))
    _bad(af.linear_fp8, z(300, 256, dtype=U8), z(299), z(520, 256, dtype=U8), z(768), z(300, 520, dtype=BF))


def test_strided_modulation_views_reach_their_storage():
    """The LN calls read shift and scale as B rows, mod_stride apart, of a
    [B, 6 D] modulation table: a view cut at column 3 D reaches 6 D B - 3 D
    elements of its storage, enough for (B - 1) 6 D + D, and a view of a
    table with one row too few is short."""
    D, B = 32, 2
    md = z(B, 6 * D)
    assert af._elems_from_start(md[:, 3 * D:]) == 6 * D * B - 3 * D
    assert af._elems_from_start(md[:, 4 * D:]) == 6 * D * B - 4 * D
    assert (B - 1) * 6 * D + D <= af._elems_from_start(md[:, 5 * D:])
    short = z(B - 1, 6 * D)
    assert (B - 1) * 6 * D + D > af._elems_from_start(short[:, 3 * D:])


def test_device_mismatch_rule():
    """Every tensor must be on the weight pack's device and that device must be
    current (the library launches there); the first violation is named."""
    assert af.device_mismatch([("x", 0), ("temb", 0)], 0, 0) is None
    assert "temb is on cuda:1" in af.device_mismatch([("x", 0), ("temb", 1)], 0, 0)
    assert "current device is cuda:1" in af.device_mismatch([("x", 0)], 1, 0)
    assert af.device_mismatch([("x", 2)], 2, 2) is None
    assert "x is on cuda:0" in af.device_mismatch([("x", 0)], 2, 2)
