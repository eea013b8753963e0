"""af_weights_init_random against the host draw of the same recipe, and the
typed weight set / get round trip.

The library's device generator (Philox4x32-10 + Box-Muller, keyed by seed and
tensor name) must reproduce ``synth.weights`` exactly: the full-size parity
goldens are written on the host from synth's draw and compared with forwards
whose weights were filled on the device.  Both sides evaluate log, sqrt, cos
and sin in fp64 and round once to fp32, so a value can differ only when an
fp64 result lands within a few fp64 ulps of an fp32 rounding boundary (about
one element in 10^8); the bf16 values then differ by one unit at most.  The
test allows that, and nothing else.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from helpers import af_config, full_config, tiny_config, to_bf16, to_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def af():
    import diffusion_transformer_denoising_auraflow_b200 as m
    return m


def _same(got: np.ndarray, ref: np.ndarray, ulp: float):
    """Equal, except for at most 1 in 10^6 elements one unit apart."""
    diff = got != ref
    n = int(diff.sum())
    if n:
        assert n <= max(1, got.size // 1_000_000), n
        assert np.all(np.abs(got[diff] - ref[diff]) <= ulp * np.abs(ref[diff]) * 1.01), n
    return n


def test_init_random_matches_host_draw_full_model(af):
    """The full model (D = 3072, 4 joint + 32 single blocks, 64 x 64 grid)
    filled on the device; a sample of tensors, including an interleaved FFN
    pair half, the position table (std 0.1), the registers (0.02) and a bias,
    read back and compared with the host draw."""
    cfg = full_config()
    w = af.Weights(af_config(cfg))
    w.init_random(4, 0.02)
    torch.cuda.synchronize()
    names = ["pos_embed.pos_embed", "register_tokens", "time_step_proj.linear_1.bias",
             "context_embedder.weight", "joint_transformer_blocks.0.norm1_context.linear.weight",
             "joint_transformer_blocks.3.ff_context.linear_2.weight", "single_transformer_blocks.31.ff.linear_1.weight",
             "single_transformer_blocks.17.attn.to_v.weight", "norm_out.linear.weight", "proj_out.weight"]
    specs = dict(O.weight_specs(cfg))
    for n in names:
        got = w.get(n).float().cpu().numpy()
        ref = synth.normal(4, n, specs[n], synth.weight_std(n))
        assert got.shape == ref.shape
        _same(got, ref, 2.0 ** -7)
    w.close()


def test_init_random_fp32_pack_and_seeds(af):
    cfg = tiny_config()
    w = af.Weights(af_config(cfg, dtype=af.AF_DTYPE_F32))
    w.init_random(123, 0.05)
    torch.cuda.synchronize()
    for n, shape in O.weight_specs(cfg):
        got = w.get(n).cpu().numpy()
        assert got.dtype == np.float32
        _same(got, synth.normal(123, n, shape, synth.weight_std(n, 0.05), "f32"), 2.0 ** -23)
    a = w.get("joint_transformer_blocks.0.ff.linear_1.weight").clone()
    w.init_random(123, 0.05)
    assert torch.equal(w.get("joint_transformer_blocks.0.ff.linear_1.weight"), a)
    w.init_random(124, 0.05)
    b = w.get("joint_transformer_blocks.0.ff.linear_1.weight")
    assert not torch.equal(a, b)
    w.close()


def test_init_random_moments(af):
    cfg = O.Config(num_mmdit_layers=0, num_single_dit_layers=1, pos_embed_max_size=64 * 64)
    w = af.Weights(af_config(cfg))
    w.init_random(9, 0.02)
    x = w.get("single_transformer_blocks.0.ff.linear_2.weight").double()
    assert abs(x.mean().item()) < 1e-4 and abs(x.std().item() / 0.02 - 1) < 2e-3
    p = w.get("pos_embed.pos_embed").double()
    assert abs(p.std().item() / 0.1 - 1) < 2e-3
    w.close()


@pytest.mark.parametrize("pack", ["bf16", "f32"])
def test_set_get_round_trip_and_conversion(af, pack):
    """set / get of an interleaved FFN half and a plain tensor, from bf16 and
    fp32 sources on the host and the device; fp32 into a bf16 pack rounds to
    nearest even."""
    cfg = tiny_config()
    dt = af.AF_DTYPE_F32 if pack == "f32" else af.AF_DTYPE_BF16
    w = af.Weights(af_config(cfg, dtype=dt))
    specs = dict(O.weight_specs(cfg))
    for n in ("joint_transformer_blocks.0.ff.linear_2.weight", "single_transformer_blocks.0.attn.to_k.weight"):
        v = synth.normal(77, n, specs[n], 0.3, "f32")
        for src in (torch.from_numpy(v), to_f32(v), torch.from_numpy(v).to(torch.bfloat16),
                    to_bf16(v)):
            w.set(n, src.contiguous())
            got = w.get(n).float().cpu().numpy()
            ref = synth.bf16_round(v) if (pack == "bf16" or src.dtype == torch.bfloat16) else v
            assert np.array_equal(got, ref), (n, src.dtype, src.device)
    w.close()
