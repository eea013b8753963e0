"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every symbol include/af.h declares, derives the configuration like the
oracle, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "af.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(af_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    import diffusion_transformer_denoising_auraflow_b200 as af
    lib = ctypes.CDLL(af.LIB_PATH)
    names = _declared()
    assert "af_transformer_forward" in names and "af_euler_cfg_step" in names
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(af.EXPORTED)


def test_config_derivation_matches_oracle():
    import diffusion_transformer_denoising_auraflow_b200 as af
    for kw in ({}, dict(attention_head_dim=8, num_attention_heads=4, pos_embed_max_size=64),
               dict(pos_embed_max_size=9216)):
        c = af.Config.default(**kw)
        o = O.Config(**kw)
        assert c.derived() == (o.inner_dim, o.ffn_hidden, o.grid_side)
    bad = af.Config.default(pos_embed_max_size=1000)
    with pytest.raises(af.AFError):
        bad.derived()


def test_defaults_match_page_values():
    import diffusion_transformer_denoising_auraflow_b200 as af
    c = af.Config.default()
    o = O.Config()
    for f, _ in af.Config._fields_:
        if f in ("ffn_inner", "dtype"):
            continue
        assert getattr(c, f) == pytest.approx(getattr(o, f)), f


def test_argument_errors_are_host_side():
    import diffusion_transformer_denoising_auraflow_b200 as af
    L = af.lib
    assert L.af_linear(None, None, None, 4, 4, 4, None) == 1
    assert L.af_linear_grouped(None, None, None, 4, 4, 4, None, None, None, 4, 4, 4, None) == 1
    assert L.af_attention(None, None, None, None, 1, 1, 1, 256, 0, None, 0, 0, None) == 1
    assert L.af_euler_cfg_step(None, None, 1, 4, 8, 8, 3.5, 1.0, 0.9, None) == 1
    assert L.af_ln_modulate(None, None, None, 0, None, 1, 1, 32, 1e-6, None) == 1
    assert L.af_sync(None, None) == 1
    assert L.af_check_wait_timeout(None, 20_000_000, None) == 1
    assert L.af_transformer_forward(None, None, None, None, None, 1, 8, 8, 4, None, None, None) == 1
    assert L.af_status_string(6) == b"device wait timed out"
    out = ctypes.c_void_p()
    bad = af.Config.default(attention_head_dim=96)
    assert L.af_weights_create(ctypes.byref(bad), 0, ctypes.byref(out)) == 3
    # shapes the timestep / modulation GEMV cannot run are refused at creation
    assert L.af_weights_create(ctypes.byref(af.Config.default(timestep_channels=260)), 0, ctypes.byref(out)) == 3
    wide = af.Config.default(num_attention_heads=20)   # D = 5120 > 4096
    assert L.af_weights_create(ctypes.byref(wide), 0, ctypes.byref(out)) == 3
    f32_big_head = af.Config.default(dtype=af.AF_DTYPE_F32)   # the fp32 path covers head_dim <= 64
    assert L.af_weights_create(ctypes.byref(f32_big_head), 0, ctypes.byref(out)) == 3
    assert L.af_weights_create(ctypes.byref(af.Config.default(dtype=7)), 0, ctypes.byref(out)) == 1
    assert L.af_weights_set(None, 0, None, 0, 0, None) == 1
    assert L.af_weights_init_random(None, 1, 0.02, None) == 1


def test_sigma_schedule_matches_oracle():
    import numpy as np
    import diffusion_transformer_denoising_auraflow_b200 as af
    for n, k in ((25, 1.73), (10, 1.0), (1, 1.73), (50, 3.0)):
        got = np.array(af.sigma_schedule(n, k))
        ref = O.sigma_schedule(n, k)
        assert got.shape == ref.shape
        assert np.allclose(got, ref, rtol=1e-6, atol=1e-7)
