"""GPU parity of the whole forward (+ CFG / Euler step) against the oracle.

Tolerance for the full stack on the bf16 path: relative L2 <= 5e-2.

The tiny model is also run as the fp32 model its configuration states (an
fp32 weight pack: fp32 weights, activations and arithmetic end to end).  Its
bound, relative L2 <= 1e-4, comes from fp32 rounding: a dot product of
length K accumulates about sqrt(K) u relative error (u = 2^-24, K <= 256 here,
so ~1e-6 per step), and a dozen sequential steps with LayerNorm and softmax
in between leave two orders of magnitude of margin below 1e-4; the achieved
error is printed.  A latent update is a difference of two fp32 latents and is
known only to 2^-24 |x| / |dx| relative; that floor is added to the bound of
the step tests.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from helpers import af_config, draw_weights, tiny_config, to_bf16, to_f32, to_np, upload

pytestmark = pytest.mark.gpu

STACK_TOL = 5e-2
F32_TOL = 1e-4


@pytest.fixture(scope="module")
def af():
    import diffusion_transformer_denoising_auraflow_b200 as m
    return m


def _forward(af, cfg, seed, B, H, W, L, t, with_step=None):
    w = af.Weights(af_config(cfg))
    drawn = draw_weights(cfg, seed)
    upload(w, drawn)
    s = af.Scratch(w, B, (H // 2) * (W // 2), L)
    lat = synth.latents(seed, (B, 4, H, W))
    text = synth.text_embeddings(seed, (B, L, cfg.joint_attention_dim))
    tt = np.full((B,), t, dtype=np.float32)
    vel = torch.empty(B, 4, H, W, dtype=torch.float32, device="cuda")
    af.transformer_forward(w, s, to_f32(lat), to_bf16(text), to_f32(tt), vel)
    s.sync()
    ref = O.transformer_forward(lat, text, tt, drawn, cfg)
    return w, s, drawn, lat, text, to_np(vel), ref


def test_tiny_forward_matches_oracle(af):
    """Tiny model: 1 joint + 1 single block, D = 32 (4 x 8), F = 256, 8 x 8 grid,
    latent 4 x 16 x 16 (64 image tokens), 8 text tokens, timestep 500."""
    cfg = tiny_config()
    *_, got, ref = _forward(af, cfg, 1, 1, 16, 16, 8, 0.5)
    assert O.rel_l2(got, ref) < STACK_TOL


def _f32_floor(x_next, x):
    """fp32 storage floor of a latent update x_next - x, relative."""
    return 2.0 ** -24 * np.linalg.norm(x_next) / np.linalg.norm(np.asarray(x_next) - x)


def _tiny_f32(af, seed, B, L=8):
    cfg = tiny_config()
    w = af.Weights(af_config(cfg, dtype=af.AF_DTYPE_F32))
    drawn = draw_weights(cfg, seed, dtype="f32")
    upload(w, drawn)
    s = af.Scratch(w, B, 64, L)
    text = synth.text_embeddings(seed, (B, L, cfg.joint_attention_dim), "f32")
    return cfg, w, s, drawn, text


def test_tiny_fp32_forward_matches_oracle(af):
    """The tiny model as configured: fp32, batch 1, latent 4 x 16 x 16 (64 image
    tokens), 8 text tokens, timestep 500 (t = 0.5)."""
    cfg, w, s, drawn, text = _tiny_f32(af, 1, 1)
    lat = synth.latents(1, (1, 4, 16, 16))
    t = np.full((1,), 0.5, np.float32)
    vel = torch.empty(1, 4, 16, 16, device="cuda")
    af.transformer_forward(w, s, to_f32(lat), to_f32(text), to_f32(t), vel)
    s.sync()
    ref = O.transformer_forward(lat, text, t, drawn, cfg)
    err = O.rel_l2(to_np(vel), ref)
    print(f"\ntiny fp32 forward rel-L2 {err:.3e}")
    assert err < F32_TOL


def test_tiny_fp32_denoise_step_sampler_and_mask(af):
    """fp32 tiny model: one CFG denoise step per call and two through the
    sampler plan (CUDA graphs) against the oracle's loop, and padded prompts."""
    cfg, w, s, drawn, text = _tiny_f32(af, 12, 2)
    lat = synth.latents(12, (1, 4, 16, 16))
    sig = [float(np.float32(x)) for x in O.sigma_schedule(25, 1.73)]
    x = to_f32(lat)
    af.denoise_step(w, s, x, to_f32(text), 3.5, sig[0], sig[1])
    s.sync()
    v = O.transformer_forward(np.concatenate([lat, lat]), text, np.full((2,), sig[0], np.float32), drawn, cfg)
    ref = O.euler_cfg_step(lat, v, 3.5, sig[0], sig[1])
    err = O.rel_l2(to_np(x) - lat, ref - lat)
    floor = _f32_floor(ref, lat)
    print(f"\ntiny fp32 denoise step rel-L2 {err:.3e} (fp32 storage floor {floor:.1e})")
    assert err < F32_TOL + 4 * floor
    # the sampler plan: modulations of every step precomputed, steps as graphs
    xs = to_f32(lat)
    st = torch.cuda.Stream()
    smp = af.Sampler(w, s, xs, to_f32(text), sig[:3], 3.5, use_graphs=True)
    smp.prepare(st)
    smp.step(0, st)
    smp.step(1, st)
    st.synchronize()
    ref = lat.astype(np.float64)
    for i in range(2):
        v = O.transformer_forward(np.concatenate([ref, ref]), text, np.full((2,), sig[i], np.float32), drawn, cfg)
        ref = O.euler_cfg_step(ref, v, 3.5, sig[i], sig[i + 1])
    err = O.rel_l2(to_np(xs) - lat, ref - lat)
    floor = _f32_floor(ref, lat)
    print(f"tiny fp32 sampler (2 steps) rel-L2 {err:.3e} (fp32 storage floor {floor:.1e})")
    assert err < F32_TOL + 4 * floor
    smp.close()
    # padded prompts: real lengths 3 and 8
    lens = [3, 8]
    lat2 = synth.latents(13, (2, 4, 16, 16))
    t = np.array([0.8, 0.3], np.float32)
    vel = torch.empty(2, 4, 16, 16, device="cuda")
    af.transformer_forward(w, s, to_f32(lat2), to_f32(text), to_f32(t), vel,
                           text_len=torch.tensor(lens, dtype=torch.int32, device="cuda"))
    s.sync()
    ref = O.transformer_forward(lat2, text, t, drawn, cfg, text_len=lens)
    err = O.rel_l2(to_np(vel), ref)
    print(f"tiny fp32 padded-prompt forward rel-L2 {err:.3e}")
    assert err < F32_TOL


def test_fp32_pack_rejects_bf16_only_calls(af):
    cfg, w, s, drawn, text = _tiny_f32(af, 14, 1)
    with pytest.raises(af.AFError) as ei:
        af.single_block(w, s, 0, torch.zeros(1, 10, 32, device="cuda", dtype=torch.bfloat16),
                        torch.zeros(1, 32, device="cuda"))
    assert ei.value.status == 3
    with pytest.raises(af.AFError) as ei:
        w.quantize_fp8()
    assert ei.value.status == 3
    with pytest.raises(TypeError):   # an fp32 pack takes fp32 text embeddings
        af.transformer_forward(w, s, torch.zeros(1, 4, 16, 16, device="cuda"),
                               torch.zeros(1, 8, 32, device="cuda", dtype=torch.bfloat16),
                               torch.zeros(1, device="cuda"), torch.empty(1, 4, 16, 16, device="cuda"))


def test_tiny_forward_cfg_euler_step(af):
    cfg = tiny_config()
    w, s, drawn, lat, text, got, ref = _forward(af, cfg, 9, 2, 16, 16, 8, 1.0)
    x = synth.latents(10, (1, 4, 16, 16))
    xt = to_f32(x)
    sig = O.sigma_schedule(25, 1.73)
    af.euler_cfg_step(xt, to_f32(got.astype(np.float32)), 3.5, sig[0], sig[1])
    torch.cuda.synchronize()
    ref_x = O.euler_cfg_step(x, ref, 3.5, sig[0], sig[1])
    assert O.rel_l2(to_np(xt) - x, ref_x - x) < STACK_TOL


def test_tiny_forward_batch_independence(af):
    cfg = tiny_config()
    w = af.Weights(af_config(cfg))
    upload(w, draw_weights(cfg, 11))
    s = af.Scratch(w, 2, 64, 8)
    lat = to_f32(synth.latents(11, (2, 4, 16, 16)))
    text = to_bf16(synth.text_embeddings(11, (2, 8, 32)))
    t = to_f32(np.array([0.3, 0.9], np.float32))
    both = torch.empty(2, 4, 16, 16, device="cuda")
    af.transformer_forward(w, s, lat, text, t, both)
    for b in range(2):
        one = torch.empty(1, 4, 16, 16, device="cuda")
        af.transformer_forward(w, s, lat[b:b + 1].contiguous(), text[b:b + 1].contiguous(), t[b:b + 1].contiguous(),
                               one)
        s.sync()
        assert torch.equal(both[b:b + 1], one)


def test_forward_rejects_bad_shapes(af):
    cfg = tiny_config()
    w = af.Weights(af_config(cfg))
    s = af.Scratch(w, 1, 64, 8)
    vel = torch.empty(1, 4, 18, 18, device="cuda")
    with pytest.raises(af.AFError):
        af.transformer_forward(w, s, torch.zeros(1, 4, 18, 18, device="cuda"),
                               torch.zeros(1, 8, 32, dtype=torch.bfloat16, device="cuda"),
                               torch.zeros(1, device="cuda"), vel)
    with pytest.raises(af.AFError):   # text longer than the scratch was sized for
        af.transformer_forward(w, s, torch.zeros(1, 4, 16, 16, device="cuda"),
                               torch.zeros(1, 9, 32, dtype=torch.bfloat16, device="cuda"),
                               torch.zeros(1, device="cuda"), torch.empty(1, 4, 16, 16, device="cuda"))


def test_real_width_forward_small_latent(af):
    """Full model width and depth (4 joint + 32 single blocks, D = 3072) on a
    16 x 16 latent (64 image tokens) with 24 text tokens, CFG batch 2.  The
    oracle runs block by block so only one block's weights are held at a time."""
    from helpers import block_names
    cfg = O.Config(pos_embed_max_size=64 * 64)
    B, H, W, L, seed = 2, 16, 16, 24, 4
    w = af.Weights(af_config(cfg))
    blocks = set()
    for i in range(cfg.num_mmdit_layers):
        blocks |= set(block_names(cfg, "joint", i))
    for i in range(cfg.num_single_dit_layers):
        blocks |= set(block_names(cfg, "single", i))
    misc = draw_weights(cfg, seed, [n for n, _ in O.weight_specs(cfg) if n not in blocks])
    upload(w, misc)
    lat = synth.latents(seed, (B, 4, H, W))
    text = synth.text_embeddings(seed, (B, L, cfg.joint_attention_dim))
    tt = np.array([1.0, 1.0], dtype=np.float32)
    img, txt, temb = O.embed(lat, text, tt, misc, cfg)
    for i in range(cfg.num_mmdit_layers):
        blk = draw_weights(cfg, seed, block_names(cfg, "joint", i))
        upload(w, blk)
        txt, img = O.joint_block(img, txt, temb, blk, f"joint_transformer_blocks.{i}.", cfg)
    nt = txt.shape[1]
    x = np.concatenate([txt, img], axis=1)
    for i in range(cfg.num_single_dit_layers):
        blk = draw_weights(cfg, seed, block_names(cfg, "single", i))
        upload(w, blk)
        x = O.single_block(x, temb, blk, f"single_transformer_blocks.{i}.", cfg)
    ref = O.output_stage(x[:, nt:], temb, misc, cfg, H, W)
    s = af.Scratch(w, B, (H // 2) * (W // 2), L)
    vel = torch.empty(B, 4, H, W, dtype=torch.float32, device="cuda")
    af.transformer_forward(w, s, to_f32(lat), to_bf16(text), to_f32(tt), vel)
    s.sync()
    assert O.rel_l2(to_np(vel), ref) < STACK_TOL


def test_tiny_forward_padded_prompts_match_oracle(af):
    """Per-sample prompt lengths 3 and 8 of L = 8 (the first sample's last five
    text tokens are padding): GPU forward with text_len vs the oracle's masked
    forward, and the padding's values do not reach the velocity."""
    cfg = tiny_config()
    w = af.Weights(af_config(cfg))
    drawn = draw_weights(cfg, 21)
    upload(w, drawn)
    s = af.Scratch(w, 2, 64, 8)
    lat = synth.latents(21, (2, 4, 16, 16))
    text = synth.text_embeddings(22, (2, 8, cfg.joint_attention_dim))
    t = np.array([0.8, 0.3], np.float32)
    lens = [3, 8]
    tl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    vel = torch.empty(2, 4, 16, 16, device="cuda")
    af.transformer_forward(w, s, to_f32(lat), to_bf16(text), to_f32(t), vel, text_len=tl)
    s.sync()
    ref = O.transformer_forward(lat, text, t, drawn, cfg, text_len=lens)
    assert O.rel_l2(to_np(vel), ref) < STACK_TOL
    junk = text.copy()
    junk[0, 3:] = 7.0
    vel2 = torch.empty_like(vel)
    af.transformer_forward(w, s, to_f32(lat), to_bf16(junk), to_f32(t), vel2, text_len=tl)
    s.sync()
    assert torch.equal(vel, vel2)


def test_real_width_padded_prompts_match_oracle(af):
    """D = 3072 (12 x 256 heads), 1 joint + 2 single blocks, 64 image tokens,
    L = 40 text tokens with real lengths 17 and 40."""
    cfg = O.Config(num_mmdit_layers=1, num_single_dit_layers=2, pos_embed_max_size=64 * 64)
    w = af.Weights(af_config(cfg))
    drawn = draw_weights(cfg, 23)
    upload(w, drawn)
    s = af.Scratch(w, 2, 64, 40)
    lat = synth.latents(23, (2, 4, 16, 16))
    text = synth.text_embeddings(24, (2, 40, cfg.joint_attention_dim))
    t = np.array([1.0, 0.5], np.float32)
    lens = [17, 40]
    vel = torch.empty(2, 4, 16, 16, device="cuda")
    af.transformer_forward(w, s, to_f32(lat), to_bf16(text), to_f32(t), vel,
                           text_len=torch.tensor(lens, dtype=torch.int32, device="cuda"))
    s.sync()
    ref = O.transformer_forward(lat, text, t, drawn, cfg, text_len=lens)
    assert O.rel_l2(to_np(vel), ref) < STACK_TOL


@pytest.fixture(scope="module")
def full_model(af):
    """The full model (4 joint + 32 single blocks, D = 3072) with device-drawn
    weights, position grid 96 x 96 (room for the 1536^2 latent)."""
    from helpers import device_weights
    cfg = af.Config.default(pos_embed_max_size=96 * 96)
    w = af.Weights(cfg)
    device_weights(af, w, 31)
    s = af.Scratch(w, 2, 96 * 96, 256)
    yield w, s
    s.close()
    w.close()


@pytest.mark.parametrize("side", [128, 192])
def test_full_size_forward_batch_independence(af, full_model, side):
    """The 1024^2 and 1536^2 workloads (latent 4 x side x side, 256 text
    tokens, CFG batch 2) in the launch configuration the bench times: each
    sample of the batch equals its own B = 1 forward bit for bit (every
    kernel is row- or (sample, head)-local), and the output is finite."""
    w, s = full_model
    gen = torch.Generator(device="cuda")
    gen.manual_seed(side)
    lat = torch.randn(2, 4, side, side, generator=gen, device="cuda")
    text = torch.randn(2, 256, 2048, generator=gen, device="cuda").to(torch.bfloat16)
    t = torch.tensor([1.0, 0.37], device="cuda")
    both = torch.empty(2, 4, side, side, device="cuda")
    af.transformer_forward(w, s, lat, text, t, both)
    s.sync()
    assert torch.isfinite(both).all()
    for b in range(2):
        one = torch.empty(1, 4, side, side, device="cuda")
        af.transformer_forward(w, s, lat[b:b + 1].contiguous(), text[b:b + 1].contiguous(),
                               t[b:b + 1].contiguous(), one)
        s.sync()
        assert torch.equal(both[b:b + 1], one)


def test_full_size_guidance_one_is_the_text_half(af, full_model):
    """At the 1024^2 workload a denoise step with guidance 1 moves the latent
    by (sigma' - sigma) times the text-conditioned velocity alone."""
    w, s = full_model
    gen = torch.Generator(device="cuda")
    gen.manual_seed(7)
    lat = torch.randn(1, 4, 128, 128, generator=gen, device="cuda")
    text = torch.randn(2, 256, 2048, generator=gen, device="cuda").to(torch.bfloat16)
    sig, sig_next = 0.8, 0.75
    x = lat.clone()
    af.denoise_step(w, s, x, text, 1.0, sig, sig_next)
    v = torch.empty(1, 4, 128, 128, device="cuda")
    af.transformer_forward(w, s, lat, text[1:2].contiguous(), torch.tensor([sig], device="cuda"), v)
    s.sync()
    ref = lat + (sig_next - sig) * v
    assert torch.allclose(x, ref, rtol=1e-5, atol=1e-6)
