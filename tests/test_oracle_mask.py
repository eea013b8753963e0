"""Pins of the oracle's padded-prompt extension: the key mask.

A masked key takes no part in any softmax, so (a) masked attention equals
plain attention over the kept keys, (b) an all-true mask changes nothing,
and (c) a forward over a prompt padded with arbitrary tokens, told the real
length, gives the image velocity of the unpadded prompt.
"""
import numpy as np

import oracle as O
import synth
from helpers import draw_weights, tiny_config


def test_masked_attention_is_attention_over_kept_keys():
    B, H, N, hd = 3, 2, 11, 8
    q = synth.normal(301, "mq", (B, H, 5, hd), 1.0).astype(np.float64)
    k = synth.normal(302, "mk", (B, H, N, hd), 1.0).astype(np.float64)
    v = synth.normal(303, "mv", (B, H, N, hd), 1.0).astype(np.float64)
    mask = np.zeros((B, N), bool)
    mask[0, :] = True
    mask[1, [0, 3, 4, 10]] = True
    mask[2, 7] = True                      # one key: the output is that value row
    got = O.attention(q, k, v, key_mask=mask)
    for b in range(B):
        keep = np.flatnonzero(mask[b])
        ref = O.attention(q[b:b + 1], k[b:b + 1, :, keep], v[b:b + 1, :, keep])
        assert np.allclose(got[b:b + 1], ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(got[2], np.broadcast_to(v[2, :, 7:8], got[2].shape), atol=1e-12)
    # brute force with loops on one (batch, head, query)
    b, h, i = 1, 1, 2
    logits = [(j, sum(q[b, h, i, d] * k[b, h, j, d] for d in range(hd)) / np.sqrt(hd)) for j in range(N) if mask[b, j]]
    mx = max(s for _, s in logits)
    wts = [(j, np.exp(s - mx)) for j, s in logits]
    z = sum(e for _, e in wts)
    ref = [sum(e * v[b, h, j, d] for j, e in wts) / z for d in range(hd)]
    assert np.allclose(got[b, h, i], ref, atol=1e-12)


def test_all_true_mask_changes_nothing():
    q = synth.normal(311, "aq", (2, 2, 6, 8), 1.0)
    k = synth.normal(312, "ak", (2, 2, 9, 8), 1.0)
    v = synth.normal(313, "av", (2, 2, 9, 8), 1.0)
    assert np.array_equal(O.attention(q, k, v, key_mask=np.ones((2, 9), bool)), O.attention(q, k, v))


def test_text_key_mask_layout():
    # registers 2, text 3, image 2; real lengths 3, 1, 0
    got = O.text_key_mask([3, 1, 0], 2, 3, 2)
    expect = np.array([[1, 1, 1, 1, 1, 1, 1],
                       [1, 1, 1, 0, 0, 1, 1],
                       [1, 1, 0, 0, 0, 1, 1]], bool)
    assert np.array_equal(got, expect)


def test_padded_prompt_forward_equals_unpadded():
    cfg = tiny_config()
    w = draw_weights(cfg, 321)
    L, lens = 8, [3, 8]
    lat = synth.latents(322, (2, 4, 16, 16))
    text = synth.text_embeddings(323, (2, L, cfg.joint_attention_dim)).astype(np.float64)
    text[0, 3:] = 50.0 * synth.normal(324, "junk", (L - 3, cfg.joint_attention_dim), 1.0)   # padding junk
    t = np.array([0.7, 0.2])
    got = O.transformer_forward(lat, text, t, w, cfg, text_len=lens)
    for b in range(2):
        ref = O.transformer_forward(lat[b:b + 1], text[b:b + 1, :lens[b]], t[b:b + 1], w, cfg)
        assert np.allclose(got[b:b + 1], ref, rtol=1e-9, atol=1e-11)
    # the mask matters: without it the junk reaches the image tokens
    plain = O.transformer_forward(lat, text, t, w, cfg)
    assert O.rel_l2(plain[:1], got[:1]) > 1e-8       # far above fp64 rounding (~1e-15)
    assert np.allclose(plain[1:], got[1:], rtol=1e-12, atol=1e-12)
