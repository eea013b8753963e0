"""The seeded input generator: determinism, chunk independence, bf16 rounding."""
import numpy as np
import torch

import synth


def test_deterministic_and_name_keyed():
    a = synth.normal(7, "w", (3, 5), 0.02)
    b = synth.normal(7, "w", (3, 5), 0.02)
    c = synth.normal(7, "w2", (3, 5), 0.02)
    d = synth.normal(8, "w", (3, 5), 0.02)
    assert np.array_equal(a, b)
    assert not np.array_equal(a, c) and not np.array_equal(a, d)


def test_multichunk_is_prefix_stable():
    n = synth.CHUNK * 2 + 17
    big = synth.normal(1, "x", (n,), 1.0, "f32")
    small = synth.normal(1, "x", (synth.CHUNK,), 1.0, "f32")
    assert np.array_equal(big[: synth.CHUNK], small)
    assert abs(big.std() - 1.0) < 0.01 and abs(big.mean()) < 0.01


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10,
                        np.array([1.0, 1.00390625, 1.005859375, -2.5, 0.0, 3e-39, 65504.0], np.float32)])
    ours = synth.bf16_round(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))
    bits = synth.bf16_bits(ours)
    assert np.array_equal(bits, torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
