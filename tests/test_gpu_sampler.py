"""GPU parity of the sampling loop: af_denoise_step and the af_sampler plan
(modulations of every step precomputed, steps replayed as CUDA graphs)
against the oracle's CFG + flow-match Euler loop.

The compared quantity is the latent update x_final - x_0 (relative L2 <=
5e-2, the full-stack tolerance), so the check is not diluted by the part of
the latent that the steps leave alone.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from helpers import af_config, draw_weights, tiny_config, to_bf16, to_f32, to_np, upload

pytestmark = pytest.mark.gpu

STACK_TOL = 5e-2


@pytest.fixture(scope="module")
def af():
    import diffusion_transformer_denoising_auraflow_b200 as m
    return m


def _setup(af, cfg, seed, Bi, H, W, L):
    w = af.Weights(af_config(cfg))
    drawn = draw_weights(cfg, seed)
    upload(w, drawn)
    s = af.Scratch(w, 2 * Bi, (H // 2) * (W // 2), L)
    x0 = synth.latents(seed, (Bi, 4, H, W))
    text = synth.text_embeddings(seed + 1, (2 * Bi, L, cfg.joint_attention_dim))
    return w, s, drawn, x0, text


def _oracle_loop(x0, text, drawn, cfg, sig, guidance, n):
    x = x0.astype(np.float64)
    for i in range(n):
        v = O.transformer_forward(np.concatenate([x, x]), text, np.full(2 * x.shape[0], sig[i]), drawn, cfg)
        x = O.euler_cfg_step(x, v, guidance, sig[i], sig[i + 1])
    return x


def test_denoise_step_matches_oracle(af):
    cfg = tiny_config()
    w, s, drawn, x0, text = _setup(af, cfg, 71, 2, 16, 16, 8)
    sig = af.sigma_schedule(3)
    xt, tt = to_f32(x0), to_bf16(text)
    for i in range(3):
        af.denoise_step(w, s, xt, tt, 3.5, sig[i], sig[i + 1])
    s.sync()
    ref = _oracle_loop(x0, text, drawn, cfg, sig, 3.5, 3)
    assert O.rel_l2(to_np(xt) - x0, ref - x0) < STACK_TOL


@pytest.mark.parametrize("use_graphs", [False, True])
def test_sampler_matches_oracle(af, use_graphs):
    cfg = tiny_config()
    n = 4
    w, s, drawn, x0, text = _setup(af, cfg, 73, 1, 16, 16, 8)
    sig = af.sigma_schedule(n)
    xt, tt = to_f32(x0), to_bf16(text)
    stream = torch.cuda.Stream()
    smp = af.Sampler(w, s, xt, tt, sig, 3.5, use_graphs=use_graphs)
    with torch.cuda.stream(stream):
        smp.prepare(stream)
        for i in range(n):
            smp.step(i, stream)
    stream.synchronize()
    ref = _oracle_loop(x0, text, drawn, cfg, sig, 3.5, n)
    assert O.rel_l2(to_np(xt) - x0, ref - x0) < STACK_TOL
    smp.close()


def test_sampler_graph_replay_is_bit_identical(af):
    """Two runs of the same plan, the second replaying the captured graphs,
    and an uncaptured run give the same bits."""
    cfg = tiny_config()
    n = 3
    w, s, drawn, x0, text = _setup(af, cfg, 75, 2, 16, 12, 8)
    sig = af.sigma_schedule(n)
    tt = to_bf16(text)
    stream = torch.cuda.Stream()
    outs = []
    for graphs, runs in ((True, 2), (False, 1)):
        xt = to_f32(x0)
        smp = af.Sampler(w, s, xt, tt, sig, 2.0, use_graphs=graphs)
        for _ in range(runs):
            with torch.cuda.stream(stream):
                xt.copy_(to_f32(x0))
                smp.prepare(stream)
                for i in range(n):
                    smp.step(i, stream)
            stream.synchronize()
            outs.append(xt.clone())
        smp.close()
    assert torch.equal(outs[0], outs[1])
    assert torch.equal(outs[0], outs[2])


def test_sampler_close_to_direct_steps(af):
    """The plan precomputes every step's modulations; the per-step path
    computes the step's own with the same tensor-core GEMM (silu(temb)
    rounded to bf16 on both).  The two loops agree to well inside the stack
    tolerance."""
    cfg = tiny_config()
    n = 3
    w, s, drawn, x0, text = _setup(af, cfg, 77, 1, 16, 16, 8)
    sig = af.sigma_schedule(n)
    tt = to_bf16(text)
    direct = to_f32(x0)
    for i in range(n):
        af.denoise_step(w, s, direct, tt, 3.5, sig[i], sig[i + 1])
    planned = to_f32(x0)
    stream = torch.cuda.Stream()
    smp = af.Sampler(w, s, planned, tt, sig, 3.5, use_graphs=True)
    with torch.cuda.stream(stream):
        smp.prepare(stream)
        for i in range(n):
            smp.step(i, stream)
    stream.synchronize()
    d, p = to_np(direct) - x0, to_np(planned) - x0
    assert O.rel_l2(p, d) < 1e-2
    smp.close()


def test_sampler_real_width_two_steps(af):
    """Full width (D = 3072, 12 heads of 256) with one joint and two single blocks,
    64 image tokens, CFG batch 2, two steps."""
    cfg = O.Config(num_mmdit_layers=1, num_single_dit_layers=2, pos_embed_max_size=64 * 64)
    n = 2
    w, s, drawn, x0, text = _setup(af, cfg, 79, 1, 16, 16, 24)
    sig = af.sigma_schedule(n)
    xt, tt = to_f32(x0), to_bf16(text)
    stream = torch.cuda.Stream()
    smp = af.Sampler(w, s, xt, tt, sig, 3.5, use_graphs=True)
    with torch.cuda.stream(stream):
        smp.prepare(stream)
        for i in range(n):
            smp.step(i, stream)
    stream.synchronize()
    ref = _oracle_loop(x0, text, drawn, cfg, sig, 3.5, n)
    assert O.rel_l2(to_np(xt) - x0, ref - x0) < STACK_TOL
    smp.close()


def test_sampler_rejects_bad_args(af):
    cfg = tiny_config()
    w, s, drawn, x0, text = _setup(af, cfg, 81, 1, 16, 16, 8)
    xt, tt = to_f32(x0), to_bf16(text)
    with pytest.raises(af.AFError):          # no steps
        af.Sampler(w, s, xt, tt, [1.0], 3.5)
    smp = af.Sampler(w, s, xt, tt, af.sigma_schedule(2), 3.5, use_graphs=True)
    with pytest.raises(af.AFError):          # step out of range
        smp.step(2, torch.cuda.Stream())
    smp.close()


def test_sampler_padded_prompts_match_oracle(af):
    cfg = tiny_config()
    n = 3
    w, s, drawn, x0, text = _setup(af, cfg, 83, 1, 16, 16, 8)
    lens = [2, 6]                      # uncond prompt 2 tokens, text prompt 6 of 8
    sig = af.sigma_schedule(n)
    xt, tt = to_f32(x0), to_bf16(text)
    stream = torch.cuda.Stream()
    smp = af.Sampler(w, s, xt, tt, sig, 3.5, use_graphs=True,
                     text_len=torch.tensor(lens, dtype=torch.int32, device="cuda"))
    with torch.cuda.stream(stream):
        smp.prepare(stream)
        for i in range(n):
            smp.step(i, stream)
    stream.synchronize()
    x = x0.astype(np.float64)
    for i in range(n):
        v = O.transformer_forward(np.concatenate([x, x]), text, np.full(2, sig[i]), drawn, cfg, text_len=lens)
        x = O.euler_cfg_step(x, v, 3.5, sig[i], sig[i + 1])
    assert O.rel_l2(to_np(xt) - x0, x - x0) < STACK_TOL
    smp.close()
