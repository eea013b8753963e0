"""Full-stack parity at the two full-size workloads against the fp64 oracle.

The oracle's velocities for the 1024 x 1024 and 1536 x 1536 forwards (CFG
batch 2, text embeddings [2, 256, 2048], first step of the 25-step shift-1.73
schedule, t = sigma_0) are stored under ``tests/golden/`` by
``tests/golden/make_full_forward.py``, which calls only ``oracle`` and
``synth``.  Here the same weights are filled on the device by
``af_weights_init_random`` (the device form of synth's recipe,
``tests/test_gpu_init.py``), the same inputs are drawn by ``synth``, and the
CUDA path runs in the launch configuration the bench times.

Checked:

* the velocity of both CFG halves at the full-stack tolerance of the bf16
  path, relative L2 <= 5e-2;
* the latent update of one denoise step (guidance g = 3.5, sigma_0 ->
  sigma_1) against the oracle's guidance + Euler applied to the stored
  velocity ("Diffusers 中的 AuraFlowTransformer2DModel架构解析与源码级使用指南",
  §前向传播流程 and §在 AuraFlowPipeline 中的实际调用).  The guided velocity
  (1 - g) v_u + g v_c combines two halves whose errors are independent, so its
  error is sqrt((g - 1)^2 + g^2) = 4.30 times a half's, while with random
  weights the two halves nearly coincide and the guided velocity is no larger
  than either: the update is held to 4.30 x 5e-2;
* that same update against the oracle's guidance + Euler applied to the GPU's
  own velocities (the step's forward is the forward above, bit for bit), to
  the fp32 rounding of the stored latent: the update is a difference of fp32
  latents, known to 2^-24 |x| / |dx| relative.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
import synth
from helpers import to_bf16, to_f32, to_np

pytestmark = pytest.mark.gpu

STACK_TOL = 5e-2
GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
GUIDANCE, N_STEPS, SHIFT = 3.5, 25, 1.73
CFG_AMP = math.sqrt((GUIDANCE - 1) ** 2 + GUIDANCE ** 2)   # 4.30
STEP_TOL = CFG_AMP * STACK_TOL


@pytest.fixture(scope="module")
def af():
    import diffusion_transformer_denoising_auraflow_b200 as m
    return m


def _meta(name):
    with open(os.path.join(GOLD, "full_forward.json")) as f:
        return json.load(f)[name]


@pytest.mark.parametrize("name", ["1024", "1536"])
def test_full_forward_and_step_match_oracle(af, name):
    meta = _meta(name)
    seed, side, G, L = meta["seed"], meta["latent"][2], meta["pos_grid"][0], meta["text"][1]
    ref_v = np.load(os.path.join(GOLD, meta["file"])).astype(np.float64)
    cfg = af.Config.default(pos_embed_max_size=G * G)
    w = af.Weights(cfg)
    w.init_random(seed, meta["weight_std"])
    s = af.Scratch(w, 2, (side // 2) ** 2, L)
    lat1 = synth.latents(seed, (1, 4, side, side))
    lat = np.concatenate([lat1, lat1])
    text = synth.text_embeddings(seed, (2, L, cfg.joint_attention_dim))
    t = np.full((2,), meta["t"], np.float32)
    vel = torch.empty(2, 4, side, side, device="cuda")
    af.transformer_forward(w, s, to_f32(lat), to_bf16(text), to_f32(t), vel)
    s.sync()
    got_v = to_np(vel)
    err_v = O.rel_l2(got_v, ref_v)
    err_u = O.rel_l2(got_v[0], ref_v[0])
    err_c = O.rel_l2(got_v[1], ref_v[1])
    print(f"\n{name}: velocity rel-L2 {err_v:.3e} (uncond {err_u:.3e}, text {err_c:.3e})")
    assert err_v < STACK_TOL and err_u < STACK_TOL and err_c < STACK_TOL

    sig = [float(np.float32(x)) for x in O.sigma_schedule(N_STEPS, SHIFT)]
    assert sig[0] == meta["t"]
    x = to_f32(lat1)
    af.denoise_step(w, s, x, to_bf16(text), GUIDANCE, sig[0], sig[1])
    s.sync()
    got_dx = to_np(x) - lat1
    ref_x = O.euler_cfg_step(lat1, ref_v, GUIDANCE, sig[0], sig[1])
    err_x = O.rel_l2(got_dx, ref_x - lat1)
    comp_x = O.euler_cfg_step(lat1, got_v, GUIDANCE, sig[0], sig[1])
    floor = 2.0 ** -24 * np.linalg.norm(comp_x) / np.linalg.norm(comp_x - lat1)
    err_comp = O.rel_l2(got_dx, comp_x - lat1)
    print(f"{name}: denoise-step latent update rel-L2 {err_x:.3e} (bound {STEP_TOL:.3f}); "
          f"vs guidance + Euler of the GPU velocity {err_comp:.3e} (fp32 floor {floor:.1e})")
    assert err_x < STEP_TOL
    assert err_comp < 4 * floor + 1e-6
    s.close()
    w.close()
