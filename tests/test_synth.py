"""The seeded input generator: the Philox4x32-10 definition (published
known-answer vectors), Box-Muller moments, determinism, element
independence, bf16 rounding."""
import math

import numpy as np
import torch

import synth


def _one(ctr, key):
    out = synth.philox4x32(*[np.array([c], np.uint64) for c in ctr], *key)
    return tuple(int(x[0]) for x in out)


def test_philox4x32_10_known_answers():
    """Known-answer vectors of Philox4x32-10 from the authors' Random123
    distribution (counter, key) -> output: zeros, all ones, and the digits of
    pi; a dropped round, a swapped multiplier or a wrong key bump changes
    every word."""
    assert _one((0, 0, 0, 0), (0, 0)) == (0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8)
    ff = 0xFFFFFFFF
    assert _one((ff, ff, ff, ff), (ff, ff)) == (0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD)
    assert _one((0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344), (0xA4093822, 0x299F31D0)) == \
        (0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1)


def test_name_key_is_crc32():
    # CRC-32 check value of "123456789" (IEEE 802.3 polynomial, reflected)
    assert synth.name_key("123456789") == 0xCBF43926


def test_box_muller_lanes_follow_the_definition():
    """Lane values are the Box-Muller pair of the block's words, recomputed
    here in plain Python floats for a few blocks."""
    seed, key = 12345678901, synth.name_key("w")
    got = synth.standard_normal_blocks(seed, key, 5, 3)
    for i, n in enumerate(range(5, 8)):
        x = _one((n & 0xFFFFFFFF, n >> 32, key, 0), (seed & 0xFFFFFFFF, seed >> 32))
        u = [(xi + 0.5) / 2 ** 32 for xi in x]
        for lane, (a, b) in enumerate([(0, 1), (2, 3)]):
            r = math.sqrt(-2.0 * math.log(u[a]))
            th = 2 * math.pi * u[b]
            assert abs(got[4 * i + 2 * lane] - r * math.cos(th)) < 1e-12
            assert abs(got[4 * i + 2 * lane + 1] - r * math.sin(th)) < 1e-12


def test_moments_and_independence():
    z = synth.normal(3, "m", (1 << 20,), 1.0, "f32").astype(np.float64)
    n = z.size
    assert abs(z.mean()) < 4 / math.sqrt(n)
    assert abs(z.var() - 1.0) < 6 * math.sqrt(2.0 / n)
    assert abs(np.mean(z ** 3)) < 0.02 and abs(np.mean(z ** 4) - 3.0) < 0.05
    # neighbouring lanes (same block, cos / sin of one angle) are uncorrelated
    assert abs(np.corrcoef(z[0::2], z[1::2])[0, 1]) < 0.01


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
    small = synth.normal(1, "x", (synth.CHUNK + 3,), 1.0, "f32")
    assert np.array_equal(big[: synth.CHUNK + 3], small)
    assert abs(big.std() - 1.0) < 0.01 and abs(big.mean()) < 0.01


def test_value_is_rounded_product():
    z = synth.standard_normal_blocks(9, synth.name_key("p"), 0, 4)
    f = synth.normal(9, "p", (16,), 0.02, "f32")
    assert np.array_equal(f, (z * float(np.float32(0.02))).astype(np.float32))
    assert np.array_equal(synth.normal(9, "p", (16,), 0.02), synth.bf16_round(f))


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10,
                        np.array([1.0, 1.00390625, 1.005859375, -2.5, 0.0, 3e-39, 65504.0], np.float32)])
    ours = synth.bf16_round(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))
    bits = synth.bf16_bits(ours)
    assert np.array_equal(bits, torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))


def test_weight_stds():
    assert synth.weight_std("pos_embed.pos_embed") == 0.1
    assert synth.weight_std("register_tokens", 0.05) == 0.02
    assert synth.weight_std("single_transformer_blocks.0.attn.to_q.weight", 0.05) == 0.05
