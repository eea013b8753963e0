"""Pins of the oracle's configuration, patch, position and timestep pieces.

Each check is tied to something other than the oracle itself: values the
pages state (tests/golden/config_defaults.json), hand-enumerated grids
(tests/golden/centre_crop.json, tests/golden/patch_order.json), closed forms
and identities.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- config

def test_find_multiple_closed_forms():
    assert O.find_multiple(85, 256) == 256
    assert O.find_multiple(8192, 256) == 8192
    assert O.find_multiple(256, 256) == 256
    assert O.find_multiple(257, 256) == 512
    assert O.find_multiple(1, 8) == 8
    assert O.find_multiple(0, 256) == 0


def test_config_defaults_match_page():
    g = _load("config_defaults.json")
    t = g["transformer"]
    c = O.Config()
    for k in ("patch_size", "in_channels", "out_channels", "num_mmdit_layers",
              "num_single_dit_layers", "attention_head_dim", "num_attention_heads",
              "joint_attention_dim", "pos_embed_max_size", "num_register_tokens"):
        assert getattr(c, k) == t[k], k
    assert c.inner_dim == t["inner_dim"] == t["caption_projection_dim"]
    assert c.num_train_timesteps == g["scheduler"]["num_train_timesteps"]
    for d, f in g["ffn_inner"].items():
        hd = int(d) // 4
        assert O.Config(attention_head_dim=hd, num_attention_heads=4).ffn_hidden == f


def test_grid_side():
    assert O.Config(pos_embed_max_size=1024).grid_side == 32
    assert O.Config(pos_embed_max_size=4096).grid_side == 64
    assert O.Config(pos_embed_max_size=9216).grid_side == 96
    with pytest.raises(ValueError):
        O.Config(pos_embed_max_size=1000).grid_side


def test_weight_specs_count_and_size():
    c = O.Config()
    specs = O.weight_specs(c)
    n = sum(int(np.prod(s)) for _, s in specs)
    # joint block: 2 x 6D^2 (adaLN) + 8 D^2 (q,k,v,add_q,add_k,add_v,out,add_out) + 2 x 3DF
    D, F = 3072, 8192
    joint = 12 * D * D + 8 * D * D + 6 * D * F
    single = 6 * D * D + 4 * D * D + 3 * D * F
    assert joint == 339_738_624 and single == 169_869_312
    assert 6.7e9 < n < 6.9e9
    assert len({name for name, _ in specs}) == len(specs)


# ---------------------------------------------------------------- patches

def test_centre_crop_hand_enumerated():
    g = _load("centre_crop.json")
    for case in g["cases"]:
        idx = O.pe_selection_index(case["G"], case["hp"], case["wp"])
        assert idx.tolist() == case["index"], case
    for case in g["errors"]:
        with pytest.raises(ValueError):
            O.pe_selection_index(case["G"], case["hp"], case["wp"])


def test_centre_crop_identity_when_grid_matches():
    for G in (8, 64, 96):
        assert O.pe_selection_index(G, G, G).tolist() == list(range(G * G))


def test_patch_order_worked_example():
    g = _load("patch_order.json")
    C, H, W, p = g["C"], g["H"], g["W"], g["p"]
    lat = np.zeros((1, C, H, W))
    for c in range(C):
        for y in range(H):
            for x in range(W):
                lat[0, c, y, x] = 100 * c + 10 * y + x
    tok = O.patchify(lat, p)
    assert tok.shape == (1, 4, 8)
    assert tok[0].tolist() == g["tokens"]
    # unpatchify is the inverse with the einsum order of the output stage
    back = O.unpatchify(tok, p, C, H // p, W // p)
    assert np.array_equal(back, lat)


@pytest.mark.parametrize("shape,p", [((2, 4, 16, 16), 2), ((1, 3, 6, 10), 2), ((1, 2, 9, 6), 3)])
def test_patchify_unpatchify_roundtrip(shape, p):
    x = np.random.default_rng(0).standard_normal(shape)
    t = O.patchify(x, p)
    B, C, H, W = shape
    assert np.array_equal(O.unpatchify(t, p, C, H // p, W // p), x)


def test_patchify_rejects_ragged():
    with pytest.raises(ValueError):
        O.patchify(np.zeros((1, 4, 5, 4)), 2)


def test_patch_embed_uses_cropped_positions():
    # Zero projection: the tokens are exactly the cropped position rows.
    G, D = 6, 5
    pe = np.arange(G * G * D, dtype=np.float64).reshape(G * G, D)
    lat = np.random.default_rng(1).standard_normal((1, 4, 4, 8))  # 2 x 4 patch grid
    tok = O.patch_embed(lat, np.zeros((D, 16)), pe, 2, G)
    rows = [(2 + i) * G + (1 + j) for i in range(2) for j in range(4)]
    assert np.array_equal(tok[0], pe[rows])


# ---------------------------------------------------------------- timestep

def test_timestep_features_closed_forms():
    e0 = O.timestep_features([0.0])
    assert e0.shape == (1, 256)
    assert np.array_equal(e0[0, :128], np.ones(128)) and np.array_equal(e0[0, 128:], np.zeros(128))
    t = 0.37
    e = O.timestep_features([t])[0]
    assert e[0] == pytest.approx(math.cos(1000 * t), abs=1e-12)
    assert e[128] == pytest.approx(math.sin(1000 * t), abs=1e-12)
    w127 = 10000.0 ** (-127 / 128)
    assert e[127] == pytest.approx(math.cos(1000 * t * w127), abs=1e-12)
    assert e[255] == pytest.approx(math.sin(1000 * t * w127), abs=1e-12)
    ts = np.linspace(0, 1, 7)
    E = O.timestep_features(ts)
    assert np.allclose(E[:, :128] ** 2 + E[:, 128:] ** 2, 1.0, atol=1e-14)


def test_timestep_mlp_zero_weight_cases():
    rng = np.random.default_rng(2)
    D = 6
    w1, b1 = rng.standard_normal((D, 256)), rng.standard_normal(D)
    w2, b2 = rng.standard_normal((D, D)), rng.standard_normal(D)
    t = [0.25, 0.9]
    out = O.timestep_embedding(t, w1, b1, np.zeros((D, D)), b2)
    assert np.array_equal(out, np.broadcast_to(b2, (2, D)))
    out = O.timestep_embedding(t, np.zeros((D, 256)), b1, w2, b2)
    s = b1 / (1 + np.exp(-b1))
    assert np.allclose(out, np.broadcast_to(w2 @ s + b2, (2, D)), rtol=1e-14, atol=1e-14)


def test_silu_closed_form():
    assert O.silu(np.array([0.0]))[0] == 0.0
    assert O.silu(np.array([1.0]))[0] == pytest.approx(1.0 / (1.0 + math.exp(-1.0)), rel=1e-15)
    assert O.silu(np.array([-40.0]))[0] == pytest.approx(-40.0 * math.exp(-40.0), rel=1e-9)


# ---------------------------------------------------------------- text stream

def test_text_stream_registers_first():
    rng = np.random.default_rng(3)
    B, L, Dj, D, R = 2, 3, 4, 5, 8
    e = rng.standard_normal((B, L, Dj))
    w = rng.standard_normal((D, Dj))
    reg = rng.standard_normal((R, D))
    t = O.text_stream(e, w, reg)
    assert t.shape == (B, R + L, D)
    for b in range(B):
        assert np.array_equal(t[b, :R], reg)
        for i in range(L):
            for d in range(D):
                assert t[b, R + i, d] == pytest.approx(sum(e[b, i, k] * w[d, k] for k in range(Dj)), rel=1e-12)
