"""GPU parity of the 8-bit (e4m3) variant against the oracle.

The variant's definition (a reading of the pipeline guide's 8-bit loading,
recorded with the other readings before any comparison): every projection of
the blocks multiplies e4m3 codes; each activation row and each weight row is
scaled by amax / 448; activations that the bf16 path stores in bf16 (the
attention output, the SwiGLU product) are quantised from that stored value;
the quantiser's division and product are fp32 steps.  A code is an integer
decision, so both sides take it in the same precision, and the weight and
activation quantiser is compared bit for bit.  Where the kernel's fp32
LayerNorm output differs from the oracle's fp64 one in the last bits, a code
may move by one step: at most 1% of codes, never by more than one step.
The 8-bit GEMM is compared with the exact product of the GPU's own codes
(bf16 output rounding, 3e-3).

Tolerances of the blocks and the forward, derived from the e4m3 format:

* e4m3 keeps 3 mantissa bits: a value with mantissa m in [1, 2) sits between
  codes 2^-3 / m apart (relative).  Over log-uniform mantissas the mean
  relative spacing is s = 2^-3 E[1/m] = 2^-3 / (2 ln 2) = 0.090, and the RMS
  relative rounding error of one quantisation is
  r = 2^-3 sqrt(E[1/m^2] / 12) = 2^-3 sqrt(3 / (8 ln 2) / 12) = 0.0265.
* Kernel vs the oracle's 8-bit block: two correct evaluations whose inputs to
  a quantiser differ by a relative delta put a value on the neighbouring code
  with probability delta / s, one spacing away, so the quantised tensor
  diverges by d(delta) = sqrt(delta s).  The kernel keeps the projections'
  outputs in bf16 where the oracle keeps fp64 (delta = 2^-9, the bf16 unit
  roundoff): d1 = sqrt(2^-9 s) = 1.3%.  The second quantiser of a chain (the
  attention output, the SwiGLU product) sees that divergence as its input
  difference: d2 = sqrt(d1 s) = 3.5%.  A block's update carries both,
  sqrt(d1^2 + d2^2) = 3.7%; BLOCK8_TOL = 5e-2.  Two blocks in sequence (the
  tiny forward) or three sampler steps add such divergences in quadrature:
  sqrt(2) * 3.7% = 5.2%; STACK8_TOL = 8e-2.
* Kernel vs the bf16 block: the variant's own rounding.  The FFN branch
  multiplies five independent quantisations (LN output, W1 and W2, SwiGLU
  product, W3), sqrt(5) r = 5.9% of the update; the attention branch has as
  many.  The 8-bit block must differ from the bf16 one by more than r / 2
  (the variant is in use) and by less than twice sqrt(5) r = 0.119.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import synth
from helpers import af_config, draw_weights, e4m3_lut, tiny_config, to_bf16, to_f32, to_np, upload

pytestmark = pytest.mark.gpu
LUT = e4m3_lut()

S_MEAN = 2.0 ** -3 / (2 * math.log(2))                       # mean relative code spacing, 0.090
R_RMS = 2.0 ** -3 * math.sqrt(3 / (8 * math.log(2)) / 12)    # RMS relative rounding error, 0.0265
D1 = math.sqrt(2.0 ** -9 * S_MEAN)                            # first quantiser of a chain, 1.3%
D2 = math.sqrt(D1 * S_MEAN)                                   # second quantiser of a chain, 3.5%
BLOCK8_EST = math.sqrt(D1 ** 2 + D2 ** 2)                     # 3.7%
BLOCK8_TOL = 5e-2
STACK8_TOL = 8e-2
VS_BF16_LO, VS_BF16_HI = R_RMS / 2, 2 * math.sqrt(5) * R_RMS  # 0.013, 0.119


@pytest.fixture(scope="module")
def af():
    import diffusion_transformer_denoising_auraflow_b200 as m
    return m


def _codes(t):
    return LUT[t.cpu().numpy().astype(np.int64)]


@pytest.mark.parametrize("rows,cols", [(37, 3072), (300, 520), (5, 8), (64, 96)])
def test_quantize_rows_bit_exact(af, rows, cols):
    x = synth.normal(701, f"q{rows}_{cols}", (rows, cols), 1.0)
    x[1] *= 1e-4
    x[2] = 0.0
    x[3, 5] = 300.0          # one outlier row
    x = synth.bf16_round(x.astype(np.float32))
    q = torch.empty(rows, cols, dtype=torch.uint8, device="cuda")
    s = torch.empty(rows, dtype=torch.float32, device="cuda")
    af.quantize_rows_e4m3(to_bf16(x), q, s)
    torch.cuda.synchronize()
    ref_q, ref_s = O.quantize_rows_e4m3(x)
    assert np.array_equal(s.cpu().numpy(), ref_s)
    assert np.array_equal(_codes(q), ref_q)


# (2, 37, 3072): an odd row count per sample, so the wide-row kernel's last
# two-row stage of each sample holds one row
@pytest.mark.parametrize("B,N,D", [(2, 300, 3072), (2, 37, 3072), (2, 37, 32), (1, 9, 256)])
def test_ln_modulate_e4m3_matches_oracle(af, B, N, D):
    x = synth.bf16_round((synth.normal(711, f"lx{N}_{D}", (B, N, D), 1.0) * 3 + 0.5).astype(np.float32))
    mods = synth.normal(712, f"lm{D}", (B, 6 * D), 0.5, "f32")
    y8 = torch.empty(B * N, D, dtype=torch.uint8, device="cuda")
    ys = torch.empty(B * N, dtype=torch.float32, device="cuda")
    md = to_f32(mods)
    af.ln_modulate_e4m3(to_bf16(x), md[:, 3 * D:], md[:, 4 * D:], 6 * D, y8, ys, 1e-6)
    torch.cuda.synchronize()
    y = O.modulate(x, mods[:, 3 * D:4 * D], mods[:, 4 * D:5 * D], 1e-6).reshape(B * N, D)
    ref_q, ref_s = O.quantize_rows_e4m3(y)
    got_s = ys.cpu().numpy()
    assert np.allclose(got_s, ref_s, rtol=1e-5)
    got_q = _codes(y8)
    same = np.mean(got_q == ref_q)
    assert same > 0.99
    # a differing code is a neighbour: within one e4m3 step (2^-3 relative, or the subnormal step)
    diff = np.abs(got_q - ref_q)
    assert np.all(diff <= np.maximum(np.abs(ref_q) * 2.0 ** -3, 2.0 ** -9) * (1 + 1e-9))
    deq = got_q * got_s[:, None]
    assert O.rel_l2(deq, y) < 4e-2          # the e4m3 rounding itself


@pytest.mark.parametrize("M,N,K", [(300, 520, 256), (64, 96, 32), (129, 256, 528),
                                   # M >= 1024 runs on CTA pairs
                                   (1100, 776, 528), (4096, 3072, 3072), (2304, 16, 64)])
def test_linear_fp8_matches_exact_product_of_codes(af, M, N, K):
    A = synth.bf16_round(synth.normal(721, f"fa{M}_{K}", (M, K), 1.0).astype(np.float32))
    W = synth.bf16_round(synth.normal(722, f"fw{N}_{K}", (N, K), 0.02).astype(np.float32))
    a8 = torch.empty(M, K, dtype=torch.uint8, device="cuda")
    w8 = torch.empty(N, K, dtype=torch.uint8, device="cuda")
    sa = torch.empty(M, dtype=torch.float32, device="cuda")
    sw = torch.zeros((N + 255) // 256 * 256, dtype=torch.float32, device="cuda")
    af.quantize_rows_e4m3(to_bf16(A), a8, sa)
    af.quantize_rows_e4m3(to_bf16(W), w8, sw[:N])
    C = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    af.linear_fp8(a8, sa, w8, sw, C)
    torch.cuda.synchronize()
    ref = (_codes(a8) * sa.cpu().numpy()[:, None].astype(np.float64)) @ \
          (_codes(w8) * sw[:N].cpu().numpy()[:, None].astype(np.float64)).T
    assert O.rel_l2(to_np(C), ref) < 3e-3
    # and the 8-bit product stays near the bf16 one
    assert O.rel_l2(to_np(C), A.astype(np.float64) @ W.astype(np.float64).T) < 1e-1


def _block_case(af, cfg, seed, names):
    w = af.Weights(af_config(cfg))
    drawn = draw_weights(cfg, seed, names)
    upload(w, drawn)
    w.quantize_fp8()
    return w, drawn


def test_single_block_fp8_matches_oracle(af):
    """Real width (D = 3072, F = 8192), B = 2, 300 tokens."""
    from helpers import block_names
    cfg = O.Config(num_mmdit_layers=0, num_single_dit_layers=1, pos_embed_max_size=64 * 64)
    pre = "single_transformer_blocks.0."
    w, drawn = _block_case(af, cfg, 731, block_names(cfg, "single", 0))
    s = af.Scratch(w, 2, 512, 64)
    x = synth.activations(732, "f8x", (2, 300, 3072))
    temb = synth.conditioning(733, (2, 3072))
    xt = to_bf16(x)
    af.single_block(w, s, 0, xt, to_f32(temb))
    s.sync()
    ref8 = O.single_block(x, temb, drawn, pre, cfg, fp8=True)
    got = to_np(xt)
    err = O.rel_l2(got - x, ref8 - x)
    print("single block, 8-bit vs oracle 8-bit: rel-L2", err)
    assert err < BLOCK8_TOL
    # the variant differs from the bf16 block by the e4m3 rounding, visibly but not grossly
    ref16 = O.single_block(x, temb, drawn, pre, cfg)
    err16 = O.rel_l2(got - x, ref16 - x)
    print("single block, 8-bit vs oracle bf16: rel-L2", err16)
    assert VS_BF16_LO < err16 < VS_BF16_HI


def test_joint_block_fp8_matches_oracle(af):
    from helpers import block_names
    cfg = O.Config(num_mmdit_layers=1, num_single_dit_layers=0, pos_embed_max_size=64 * 64)
    pre = "joint_transformer_blocks.0."
    w, drawn = _block_case(af, cfg, 741, block_names(cfg, "joint", 0))
    s = af.Scratch(w, 2, 256, 40)
    img = synth.activations(742, "f8i", (2, 256, 3072))
    txt = synth.activations(743, "f8t", (2, 48, 3072))
    temb = synth.conditioning(744, (2, 3072))
    it, tt = to_bf16(img), to_bf16(txt)
    af.joint_block(w, s, 0, it, tt, to_f32(temb))
    s.sync()
    rt, ri = O.joint_block(img, txt, temb, drawn, pre, cfg, fp8=True)
    ei, et = O.rel_l2(to_np(it) - img, ri - img), O.rel_l2(to_np(tt) - txt, rt - txt)
    print("joint block, 8-bit vs oracle 8-bit: rel-L2 image", ei, "text", et)
    assert ei < BLOCK8_TOL and et < BLOCK8_TOL
    rt16, ri16 = O.joint_block(img, txt, temb, drawn, pre, cfg)
    ei16, et16 = O.rel_l2(to_np(it) - img, ri16 - img), O.rel_l2(to_np(tt) - txt, rt16 - txt)
    print("joint block, 8-bit vs oracle bf16: rel-L2 image", ei16, "text", et16)
    assert VS_BF16_LO < ei16 < VS_BF16_HI and VS_BF16_LO < et16 < VS_BF16_HI


def test_tiny_forward_fp8_matches_oracle(af):
    cfg = tiny_config()
    w = af.Weights(af_config(cfg))
    drawn = draw_weights(cfg, 751)
    upload(w, drawn)
    w.quantize_fp8()
    s = af.Scratch(w, 2, 64, 8)
    lat = synth.latents(752, (2, 4, 16, 16))
    text = synth.text_embeddings(753, (2, 8, cfg.joint_attention_dim))
    t = np.array([0.8, 0.3], np.float32)
    vel = torch.empty(2, 4, 16, 16, device="cuda")
    af.transformer_forward(w, s, to_f32(lat), to_bf16(text), to_f32(t), vel)
    s.sync()
    ref = O.transformer_forward(lat, text, t, drawn, cfg, fp8=True)
    err = O.rel_l2(to_np(vel), ref)
    print("tiny forward, 8-bit vs oracle 8-bit: rel-L2", err)
    assert err < STACK8_TOL
    # switching back restores the bf16 path bit for bit
    w.quantize_fp8(False)
    vel16 = torch.empty_like(vel)
    af.transformer_forward(w, s, to_f32(lat), to_bf16(text), to_f32(t), vel16)
    w2 = af.Weights(af_config(cfg))
    upload(w2, drawn)
    s2 = af.Scratch(w2, 2, 64, 8)
    vel16b = torch.empty_like(vel)
    af.transformer_forward(w2, s2, to_f32(lat), to_bf16(text), to_f32(t), vel16b)
    s2.sync()
    assert torch.equal(vel16, vel16b)


def test_sampler_fp8_padded_prompts_match_oracle(af):
    """The 8-bit variant through the sampler plan (CUDA graphs) with padded
    prompts: three steps against the oracle's 8-bit, masked loop."""
    cfg = tiny_config()
    w = af.Weights(af_config(cfg))
    drawn = draw_weights(cfg, 761)
    upload(w, drawn)
    w.quantize_fp8()
    s = af.Scratch(w, 2, 64, 8)
    x0 = synth.latents(762, (1, 4, 16, 16))
    text = synth.text_embeddings(763, (2, 8, cfg.joint_attention_dim))
    lens = [3, 7]
    sig = af.sigma_schedule(3)
    xt, tt = to_f32(x0), to_bf16(text)
    stream = torch.cuda.Stream()
    smp = af.Sampler(w, s, xt, tt, sig, 3.5, use_graphs=True,
                     text_len=torch.tensor(lens, dtype=torch.int32, device="cuda"))
    with torch.cuda.stream(stream):
        smp.prepare(stream)
        for i in range(3):
            smp.step(i, stream)
    stream.synchronize()
    x = x0.astype(np.float64)
    for i in range(3):
        v = O.transformer_forward(np.concatenate([x, x]), text, np.full(2, sig[i]), drawn, cfg, text_len=lens,
                                  fp8=True)
        x = O.euler_cfg_step(x, v, 3.5, sig[i], sig[i + 1])
    err = O.rel_l2(to_np(xt) - x0, x - x0)
    print("sampler, 8-bit vs oracle 8-bit: rel-L2", err)
    assert err < STACK8_TOL
    smp.close()
