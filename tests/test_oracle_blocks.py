"""Pins of the oracle's normalisation, attention, FFN and block definitions.

Invariants and closed forms chosen so that a plausible slip (a dropped term,
a wrong sign, a transposed weight, a swapped modulation chunk, the wrong
stream order) makes at least one of them fail.
"""
import math

import numpy as np
import pytest

import oracle as O


def tiny_cfg(**kw):
    c = dict(num_mmdit_layers=1, num_single_dit_layers=1, attention_head_dim=8,
             num_attention_heads=4, joint_attention_dim=32, pos_embed_max_size=64)
    c.update(kw)
    return O.Config(**c)


def rand_weights(cfg, seed=0, std=0.2):
    rng = np.random.default_rng(seed)
    return {n: rng.standard_normal(s) * std for n, s in O.weight_specs(cfg)}


def mods(B, D, rng, **fixed):
    m = {k: rng.standard_normal((B, D)) * 0.5 for k in O.MOD_CHUNKS}
    m.update(fixed)
    return m


# ---------------------------------------------------------------- layer norm

def test_layer_norm_moments_and_affine_invariance():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((3, 7, 50)) * 4 + 2
    y = O.layer_norm(x, 0.0)
    assert np.allclose(y.mean(-1), 0, atol=1e-13)
    assert np.allclose((y ** 2).mean(-1), 1, atol=1e-13)
    assert np.allclose(O.layer_norm(3.5 * x - 11.0, 0.0), y, atol=1e-12)
    # negative scale flips the sign (the map is odd under x -> -x)
    assert np.allclose(O.layer_norm(-x, 0.0), -y, atol=1e-12)
    # eps enters as var + eps: a constant row maps to 0, a 2-point row has closed form
    assert np.array_equal(O.layer_norm(np.full((1, 4), 3.0), 1e-6), np.zeros((1, 4)))
    r = O.layer_norm(np.array([[1.0, -1.0]]), 0.25)
    assert np.allclose(r, [[1 / math.sqrt(1.25), -1 / math.sqrt(1.25)]], rtol=1e-15)


def test_modulate_scale_minus_one_gives_shift():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((2, 5, 16))
    sh = rng.standard_normal((2, 16))
    out = O.modulate(x, sh, -np.ones((2, 16)), 1e-6)
    assert np.array_equal(out, np.broadcast_to(sh[:, None, :], out.shape))
    out0 = O.modulate(x, np.zeros((2, 16)), np.zeros((2, 16)), 1e-6)
    assert np.array_equal(out0, O.layer_norm(x, 1e-6))


# ---------------------------------------------------------------- attention

def brute_attention(q, k, v, scale):
    """Per-query loops with plain math.exp and no max shift (tiny N only)."""
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    out = np.zeros((B, H, Nq, v.shape[3]))
    for b in range(B):
        for h in range(H):
            for i in range(Nq):
                w = [math.exp(scale * sum(q[b, h, i, t] * k[b, h, j, t] for t in range(d))) for j in range(Nk)]
                z = sum(w)
                for j in range(Nk):
                    out[b, h, i] += (w[j] / z) * v[b, h, j]
    return out


def test_attention_single_token_returns_v():
    rng = np.random.default_rng(2)
    q, k, v = (rng.standard_normal((2, 3, 1, 8)) for _ in range(3))
    assert np.allclose(O.attention(q, k, v), v, rtol=0, atol=1e-15)


def test_attention_identical_keys_average_v():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, 2, 4, 8))
    k = np.broadcast_to(rng.standard_normal((1, 2, 1, 8)), (1, 2, 6, 8))
    v = rng.standard_normal((1, 2, 6, 8))
    o = O.attention(q, k, v)
    assert np.allclose(o, np.broadcast_to(v.mean(axis=2, keepdims=True), o.shape), atol=1e-14)


def test_attention_brute_force_and_scale():
    rng = np.random.default_rng(4)
    q, k, v = (rng.standard_normal((1, 2, 5, 4)) * 2 for _ in range(3))
    assert np.allclose(O.attention(q, k, v), brute_attention(q, k, v, 0.5), atol=1e-12)
    # head_dim 16 -> default scale 1/4
    q, k, v = (rng.standard_normal((1, 1, 3, 16)) for _ in range(3))
    assert np.allclose(O.attention(q, k, v), brute_attention(q, k, v, 0.25), atol=1e-12)


def test_attention_two_key_closed_form():
    q = np.array([[[[2.0, 0.0, 0.0, 0.0]]]])
    k = np.array([[[[1.0, 0, 0, 0], [-1.0, 0, 0, 0]]]])
    v = np.array([[[[1.0, 0, 0, 0], [0.0, 1, 0, 0]]]])
    # logits 2*1*0.5 = 1 and -1; weights e/(e+1/e), (1/e)/(e+1/e)
    o = O.attention(q, k, v)[0, 0, 0]
    a = math.e / (math.e + 1 / math.e)
    assert o[0] == pytest.approx(a, rel=1e-14) and o[1] == pytest.approx(1 - a, rel=1e-14)


def test_attention_permutation_equivariance():
    rng = np.random.default_rng(5)
    q, k, v = (rng.standard_normal((2, 2, 9, 8)) for _ in range(3))
    o = O.attention(q, k, v)
    perm = rng.permutation(9)
    assert np.allclose(O.attention(q, k[:, :, perm], v[:, :, perm]), o, atol=1e-13)
    assert np.allclose(O.attention(q[:, :, perm], k, v), o[:, :, perm], atol=1e-13)


# ---------------------------------------------------------------- FFN / closed-form single token blocks

def test_ffn_zero_gate_branch_and_closed_form():
    rng = np.random.default_rng(6)
    D, F = 6, 4
    y = rng.standard_normal((1, 3, D))
    w1, w2, w3 = rng.standard_normal((F, D)), rng.standard_normal((F, D)), rng.standard_normal((D, F))
    assert np.array_equal(O.feed_forward(y, w1, np.zeros((F, D)), w3), np.zeros((1, 3, D)))
    E = lambda r, c, shape: np.eye(1, shape[0] * shape[1], r * shape[1] + c).reshape(shape)
    out = O.feed_forward(y, E(2, 1, (F, D)), E(2, 4, (F, D)), E(5, 2, (D, F)))
    s = y[0, :, 1]
    expect = np.zeros((3, D))
    expect[:, 5] = s / (1 + np.exp(-s)) * y[0, :, 4]
    assert np.allclose(out[0], expect, atol=1e-15)


def _single_weights(D, F, rng, prefix="b."):
    return {prefix + "attn.to_q.weight": rng.standard_normal((D, D)),
            prefix + "attn.to_k.weight": rng.standard_normal((D, D)),
            prefix + "attn.to_v.weight": rng.standard_normal((D, D)),
            prefix + "attn.to_out.0.weight": rng.standard_normal((D, D)),
            prefix + "ff.linear_1.weight": rng.standard_normal((F, D)),
            prefix + "ff.linear_2.weight": rng.standard_normal((F, D)),
            prefix + "ff.out_projection.weight": rng.standard_normal((D, F))}


def test_single_block_one_token_closed_form_attention_branch():
    """N = 1, scale_msa = -1 => y = shift_msa, attention returns V, so
    x_out = x + gate_msa * (W_o W_v shift_msa); with W_v = I and W_o = E_ij
    only coordinate i moves, by gate[i] * shift[j]."""
    rng = np.random.default_rng(7)
    D, F, heads = 8, 4, 2
    w = _single_weights(D, F, rng)
    w["b.attn.to_v.weight"] = np.eye(D)
    Wo = np.zeros((D, D)); Wo[3, 6] = 1.0
    w["b.attn.to_out.0.weight"] = Wo
    x = rng.standard_normal((1, 1, D))
    m = mods(1, D, rng, scale_msa=-np.ones((1, D)), gate_mlp=np.zeros((1, D)))
    out = O.single_block_mod(x, m, w, "b.", heads, 1e-6)
    expect = x.copy()
    expect[0, 0, 3] += m["gate_msa"][0, 3] * m["shift_msa"][0, 6]
    assert np.allclose(out, expect, atol=1e-14)


def test_single_block_one_token_closed_form_ffn_branch():
    rng = np.random.default_rng(8)
    D, F, heads = 8, 4, 2
    w = _single_weights(D, F, rng)
    W1 = np.zeros((F, D)); W1[1, 2] = 1.0
    W2 = np.zeros((F, D)); W2[1, 5] = 1.0
    W3 = np.zeros((D, F)); W3[7, 1] = 1.0
    w.update({"b.ff.linear_1.weight": W1, "b.ff.linear_2.weight": W2, "b.ff.out_projection.weight": W3})
    x = rng.standard_normal((1, 1, D))
    m = mods(1, D, rng, gate_msa=np.zeros((1, D)), scale_mlp=-np.ones((1, D)))
    out = O.single_block_mod(x, m, w, "b.", heads, 1e-6)
    s = m["shift_mlp"][0]
    expect = x.copy()
    expect[0, 0, 7] += m["gate_mlp"][0, 7] * (s[2] / (1 + math.exp(-s[2]))) * s[5]
    assert np.allclose(out, expect, atol=1e-14)


# ---------------------------------------------------------------- block invariants

def test_zero_gates_make_blocks_identity():
    cfg = tiny_cfg()
    w = rand_weights(cfg)
    rng = np.random.default_rng(9)
    D = cfg.inner_dim
    for name in ("single_transformer_blocks.0.norm1.linear.weight",
                 "joint_transformer_blocks.0.norm1.linear.weight",
                 "joint_transformer_blocks.0.norm1_context.linear.weight"):
        W = w[name].copy()
        W[2 * D:3 * D] = 0.0   # gate_msa rows
        W[5 * D:6 * D] = 0.0   # gate_mlp rows
        w[name] = W
    temb = rng.standard_normal((2, D))
    x = rng.standard_normal((2, 11, D))
    assert np.array_equal(O.single_block(x, temb, w, "single_transformer_blocks.0.", cfg), x)
    img, txt = rng.standard_normal((2, 9, D)), rng.standard_normal((2, 5, D))
    t2, i2 = O.joint_block(img, txt, temb, w, "joint_transformer_blocks.0.", cfg)
    assert np.array_equal(t2, txt) and np.array_equal(i2, img)
    # sanity: with the gates back the block is not the identity
    w2 = rand_weights(cfg)
    assert not np.allclose(O.single_block(x, temb, w2, "single_transformer_blocks.0.", cfg), x)


def test_zero_msa_gate_removes_attention_dependence():
    cfg = tiny_cfg()
    rng = np.random.default_rng(10)
    D = cfg.inner_dim
    w = rand_weights(cfg)
    p = "single_transformer_blocks.0."
    W = w[p + "norm1.linear.weight"].copy(); W[2 * D:3 * D] = 0.0
    w[p + "norm1.linear.weight"] = W
    x, temb = rng.standard_normal((1, 7, D)), rng.standard_normal((1, D))
    a = O.single_block(x, temb, w, p, cfg)
    w2 = dict(w)
    for n in ("attn.to_q.weight", "attn.to_k.weight", "attn.to_v.weight", "attn.to_out.0.weight"):
        w2[p + n] = rng.standard_normal(w[p + n].shape)
    assert np.allclose(O.single_block(x, temb, w2, p, cfg), a, atol=1e-13)
    assert not np.allclose(a, x)


def test_qk_norm_scale_invariance():
    cfg = tiny_cfg()
    rng = np.random.default_rng(11)
    D = cfg.inner_dim
    w = rand_weights(cfg, std=0.5)
    p = "single_transformer_blocks.0."
    x, temb = rng.standard_normal((2, 10, D)), rng.standard_normal((2, D))
    ref = O.single_block(x, temb, w, p, cfg)
    w2 = dict(w)
    w2[p + "attn.to_q.weight"] = w[p + "attn.to_q.weight"] * 7.0
    w2[p + "attn.to_k.weight"] = w[p + "attn.to_k.weight"] * 0.3
    assert O.rel_l2(O.single_block(x, temb, w2, p, cfg), ref) < 1e-5
    w3 = dict(w)
    w3[p + "attn.to_v.weight"] = w[p + "attn.to_v.weight"] * 7.0   # V is not normalised
    assert O.rel_l2(O.single_block(x, temb, w3, p, cfg), ref) > 1e-2


def test_joint_with_tied_streams_equals_single_on_text_first_concat():
    cfg = tiny_cfg()
    rng = np.random.default_rng(12)
    D = cfg.inner_dim
    w = rand_weights(cfg)
    j, s = "joint_transformer_blocks.0.", "single_transformer_blocks.0."
    tie = {"norm1_context.linear.weight": "norm1.linear.weight",
           "attn.add_q_proj.weight": "attn.to_q.weight",
           "attn.add_k_proj.weight": "attn.to_k.weight",
           "attn.add_v_proj.weight": "attn.to_v.weight",
           "attn.to_add_out.weight": "attn.to_out.0.weight",
           "ff_context.linear_1.weight": "ff.linear_1.weight",
           "ff_context.linear_2.weight": "ff.linear_2.weight",
           "ff_context.out_projection.weight": "ff.out_projection.weight"}
    for a, b in tie.items():
        w[j + a] = w[j + b]
    for n in ("norm1.linear.weight", "attn.to_q.weight", "attn.to_k.weight", "attn.to_v.weight",
              "attn.to_out.0.weight", "ff.linear_1.weight", "ff.linear_2.weight", "ff.out_projection.weight"):
        w[s + n] = w[j + n]
    img, txt = rng.standard_normal((2, 12, D)), rng.standard_normal((2, 5, D))
    temb = rng.standard_normal((2, D))
    t2, i2 = O.joint_block(img, txt, temb, w, j, cfg)
    x2 = O.single_block(np.concatenate([txt, img], axis=1), temb, w, s, cfg)
    assert np.allclose(x2[:, :5], t2, atol=1e-12) and np.allclose(x2[:, 5:], i2, atol=1e-12)


def test_modulation_chunk_positions():
    """Only chunks 2 and 5 are gates: zeroing any other pair leaves a change."""
    cfg = tiny_cfg()
    rng = np.random.default_rng(13)
    D = cfg.inner_dim
    w = rand_weights(cfg)
    p = "single_transformer_blocks.0."
    x, temb = rng.standard_normal((1, 6, D)), rng.standard_normal((1, D))
    for a, b in [(0, 3), (1, 4), (0, 5), (2, 4), (2, 3)]:
        W = w[p + "norm1.linear.weight"].copy()
        W[a * D:(a + 1) * D] = 0.0
        W[b * D:(b + 1) * D] = 0.0
        w2 = dict(w); w2[p + "norm1.linear.weight"] = W
        assert not np.allclose(O.single_block(x, temb, w2, p, cfg), x)


def test_sampled_rows_match_full_blocks():
    cfg = tiny_cfg()
    rng = np.random.default_rng(14)
    D = cfg.inner_dim
    w = rand_weights(cfg)
    temb = rng.standard_normal((2, D))
    x = rng.standard_normal((2, 13, D))
    rows = [0, 4, 12]
    full = O.single_block(x, temb, w, "single_transformer_blocks.0.", cfg)
    part = O.single_block_rows(x, temb, w, "single_transformer_blocks.0.", cfg, rows)
    assert np.allclose(part, full[:, rows], atol=1e-12)
    img, txt = rng.standard_normal((2, 10, D)), rng.standard_normal((2, 6, D))
    t2, i2 = O.joint_block(img, txt, temb, w, "joint_transformer_blocks.0.", cfg)
    pt, pi = O.joint_block_rows(img, txt, temb, w, "joint_transformer_blocks.0.", cfg, [1, 9], [0, 5])
    assert np.allclose(pi, i2[:, [1, 9]], atol=1e-12) and np.allclose(pt, t2[:, [0, 5]], atol=1e-12)


# ---------------------------------------------------------------- whole forward

def test_forward_reduces_to_patch_roundtrip():
    """Zero adaLN and pre-final weights, W_pe = W_out = I (D = p*p*C = 16),
    zero positions: every block is the identity and the output is the input
    latent, which pins patchify/unpatchify consistency and the image slice."""
    cfg = O.Config(num_mmdit_layers=2, num_single_dit_layers=2, attention_head_dim=8,
                   num_attention_heads=2, joint_attention_dim=12, pos_embed_max_size=100)
    assert cfg.inner_dim == 16
    w = rand_weights(cfg)
    for n in list(w):
        if "norm1" in n or n == "norm_out.linear.weight":
            w[n] = np.zeros_like(w[n])
    w["pos_embed.proj.weight"] = np.eye(16)
    w["proj_out.weight"] = np.eye(16)
    w["pos_embed.pos_embed"] = np.zeros_like(w["pos_embed.pos_embed"])
    rng = np.random.default_rng(15)
    lat = rng.standard_normal((2, 4, 8, 12))
    text = rng.standard_normal((2, 3, 12))
    out = O.transformer_forward(lat, text, [0.3, 0.8], w, cfg)
    assert np.allclose(out, lat, atol=1e-14)
    # with positions on, the output gains the cropped grid, unpatchified
    pe = rng.standard_normal(w["pos_embed.pos_embed"].shape)
    w["pos_embed.pos_embed"] = pe
    out = O.transformer_forward(lat, text, [0.3, 0.8], w, cfg)
    idx = O.pe_selection_index(10, 4, 6)
    add = O.unpatchify(np.broadcast_to(pe[idx][None], (2, 24, 16)), 2, 4, 4, 6)
    assert np.allclose(out, lat + add, atol=1e-13)


def test_forward_batch_independence():
    cfg = tiny_cfg()
    w = rand_weights(cfg, std=0.1)
    rng = np.random.default_rng(16)
    lat = rng.standard_normal((2, 4, 8, 8))
    text = rng.standard_normal((2, 4, 32))
    t = [0.2, 0.7]
    both = O.transformer_forward(lat, text, t, w, cfg)
    for b in range(2):
        one = O.transformer_forward(lat[b:b + 1], text[b:b + 1], t[b:b + 1], w, cfg)
        assert np.allclose(both[b:b + 1], one, atol=1e-13)


def test_pre_final_order_scale_then_shift():
    rng = np.random.default_rng(17)
    D = 4
    x = rng.standard_normal((1, 3, D))
    temb = rng.standard_normal((1, D))
    W = np.zeros((2 * D, D))
    W[D:] = rng.standard_normal((D, D))    # only the second chunk (shift) is live
    sh = O.silu(temb) @ W[D:].T
    assert np.allclose(O.pre_final(x, temb, W), x + sh[:, None, :], atol=1e-15)
