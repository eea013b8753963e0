"""Pins of the oracle's 8-bit (e4m3) variant.

The e4m3 rounding is checked against the format's own definition, decoded
bit by bit here (sign, 4 exponent bits with bias 7, 3 mantissa bits, code
0x7F / 0xFF is NaN, no infinities): every finite code round-trips, every
midpoint between neighbours goes to the even code, values past 448 saturate.
The per-row quantiser is pinned by its invariants (the row maximum lands on
448 exactly, the error bound of a 3-bit mantissa, zero rows) and the 8-bit
linear by cases where quantisation is exact.
"""
import numpy as np

import oracle as O
import synth


def decode_e4m3(code: int) -> float:
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * m * 2.0 ** -9          # subnormal: m/8 * 2^(1-7)
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


FINITE = sorted({decode_e4m3(c) for c in range(256) if not np.isnan(decode_e4m3(c))})


def test_format_facts():
    pos = [v for v in FINITE if v > 0]
    assert max(FINITE) == 448.0 and min(FINITE) == -448.0
    assert min(pos) == 2.0 ** -9
    assert len(FINITE) == 253            # 254 finite codes, +0 and -0 coincide


def test_every_code_round_trips():
    v = np.array(FINITE)
    assert np.array_equal(O.e4m3_round(v), v)


def test_midpoints_round_to_even_code():
    pos = [v for v in FINITE if v >= 0]
    codes = {decode_e4m3(c): c for c in range(0x7F)}   # non-negative codes
    for a, b in zip(pos[:-1], pos[1:]):
        mid = 0.5 * (a + b)
        even = a if codes[a] % 2 == 0 else b
        assert O.e4m3_round(np.array([mid]))[0] == even, (a, b)
        assert O.e4m3_round(np.array([-mid]))[0] == -even
        # just off the midpoint goes to the nearer neighbour
        assert O.e4m3_round(np.array([mid - (b - a) * 1e-3]))[0] == a
        assert O.e4m3_round(np.array([mid + (b - a) * 1e-3]))[0] == b


def test_saturation_and_underflow():
    got = O.e4m3_round(np.array([448.0, 460.0, 1e6, -1e6, 2.0 ** -10, 3 * 2.0 ** -10, 2.0 ** -11, 0.0]))
    assert list(got) == [448.0, 448.0, 448.0, -448.0, 0.0, 2.0 ** -8, 0.0, 0.0]


def test_quantize_rows_invariants():
    x = synth.normal(601, "q8", (7, 96), 1.0).astype(np.float64)
    x[3] = 0.0
    x[5] *= 1e-3
    q, s = O.quantize_rows_e4m3(x)
    assert s.dtype == np.float32
    assert np.array_equal(O.e4m3_round(q), q)                     # codes are e4m3 values
    nz = [r for r in range(7) if r != 3]
    assert np.array_equal(np.max(np.abs(q[nz]), axis=1), np.full(6, 448.0))
    assert np.all(q[3] == 0) and s[3] == 1.0
    deq = O.dequantize_rows(q, s)
    # 3 mantissa bits: |x - deq| <= 2^-4 |x| in the normal range, plus the
    # subnormal step s 2^-10 near zero (fp32 scaling adds ~2^-23 relative)
    bound = 2.0 ** -4 * np.abs(x) * (1 + 1e-6) + s[:, None].astype(np.float64) * 2.0 ** -10
    assert np.all(np.abs(x - deq) <= bound)


def test_quantize_rows_exact_on_grid():
    # rows already on the e4m3 grid times a power of two, with the max at 448: exact
    rng = np.random.default_rng(602)
    vals = np.array(FINITE)
    rows = []
    for k in (-3, 0, 5):
        r = rng.choice(vals, size=40) * 2.0 ** k
        r[7] = 448.0 * 2.0 ** k
        rows.append(r)
    x = np.array(rows)
    assert np.array_equal(O.fake_quant_rows(x), x)


def test_linear_fp8_exact_when_inputs_are_representable():
    rng = np.random.default_rng(603)
    vals = np.array(FINITE)
    y = rng.choice(vals, size=(5, 64)) * 2.0 ** -4
    y[:, 0] = 448.0 * 2.0 ** -4
    w = rng.choice(vals, size=(12, 64)) * 2.0 ** -10
    w[:, 1] = -448.0 * 2.0 ** -10
    got = O.fake_quant_rows(y) @ O.fake_quant_rows(w).T
    assert np.array_equal(got, y @ w.T)


def test_fp8_forward_is_close_to_bf16_forward():
    """The 8-bit variant perturbs the forward by roughly the e4m3 rounding
    (~2^-5 relative per operand), not more; fp8=False is the plain forward."""
    from helpers import draw_weights, tiny_config
    cfg = tiny_config()
    w = draw_weights(cfg, 604)
    lat = synth.latents(605, (2, 4, 16, 16))
    text = synth.text_embeddings(606, (2, 8, cfg.joint_attention_dim))
    t = np.array([0.9, 0.4])
    ref = O.transformer_forward(lat, text, t, w, cfg)
    assert np.array_equal(O.transformer_forward(lat, text, t, w, cfg, fp8=False), ref)
    err = O.rel_l2(O.transformer_forward(lat, text, t, w, cfg, fp8=True), ref)
    assert 1e-8 < err < 5e-2      # nonzero, yet small


def test_round_bf16_matches_the_format():
    # bf16 keeps the top 16 bits of the fp32 pattern; ties go to the even pattern
    x = np.array([1.0, 1.0 + 2.0 ** -8, 1.0 + 2.0 ** -7, 1.0 + 3 * 2.0 ** -8, -2.5, 3.0e38, 1e-40])
    got = O.round_bf16(x)
    assert got[0] == 1.0
    assert got[1] == 1.0                    # halfway between 1 and 1 + 2^-7: even (1.0)
    assert got[2] == 1.0 + 2.0 ** -7        # representable
    assert got[3] == 1.0 + 2.0 ** -6        # halfway between 1 + 2^-7 (odd) and 1 + 2^-6 (even)
    assert got[4] == -2.5
    # every value is a bf16 (low 16 bits of its fp32 pattern are zero)
    bits = got.astype(np.float32).view(np.uint32)
    assert np.all((bits & 0xFFFF) == 0)
    r = np.random.default_rng(5).normal(size=1000)
    g = O.round_bf16(r)
    assert np.all(np.abs(g - r) <= 2.0 ** -8 * np.abs(r))
