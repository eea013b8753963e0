"""The bench's algorithmic FLOP count, checked against an independent count
(no GPU needed).

`bench.step_flops` is a closed form.  Here the same quantity is counted
from the oracle's list of weight matrices: every 2-D weight [out, in]
contributes 2 * rows * out * in, where rows is the number of tokens the
weight is applied to in one forward (the model's forward order,
"Diffusers 中的 AuraFlowTransformer2DModel架构解析与源码级使用指南",
§前向传播流程).  Each block's attention adds 4 * N^2 * D (QK^T and PV).
Position tables, register tokens, biases and the timestep MLP's weights
are gathers, copies, adds or single-row products; the closed form leaves
them out, so they are skipped here too.
"""
import os
import sys

import pytest

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _rows_for(name, Ni, Nt, N, L):
    """Tokens per sample that the weight `name` multiplies in one forward."""
    if name.startswith("pos_embed.proj"):
        return Ni                                   # patch projection
    if name.startswith("context_embedder"):
        return L                                    # text embedding
    if name.startswith("proj_out"):
        return Ni                                   # output projection
    if ".norm1" in name or name.startswith("norm_out") or ".norm1_context" in name:
        return 1                                    # adaLN / pre-final: one row per sample
    if name.startswith("joint_transformer_blocks."):
        text = (".add_" in name) or ("to_add_out" in name) or (".ff_context." in name)
        return Nt if text else Ni
    if name.startswith("single_transformer_blocks."):
        return N
    return None                                     # not a per-token product


@pytest.mark.parametrize("H,W,L", [(128, 128, 256), (192, 192, 256), (64, 96, 77)])
def test_step_flops_matches_count_from_weight_list(H, W, L):
    import bench
    grid = max(H, W) // 2
    cfg = O.Config(pos_embed_max_size=grid * grid)
    D = cfg.inner_dim
    Ni = (H // 2) * (W // 2)
    Nt = cfg.num_register_tokens + L
    N = Nt + Ni
    total = 0.0
    counted = set()
    for name, shape in O.weight_specs(cfg):
        if (len(shape) != 2 or name.endswith("pos_embed.pos_embed") or name.startswith("time_step_proj")
                or name == "register_tokens"):
            continue
        rows = _rows_for(name, Ni, Nt, N, L)
        assert rows is not None, name
        total += 2.0 * rows * shape[0] * shape[1]
        counted.add(name.split(".")[0])
    blocks = cfg.num_mmdit_layers + cfg.num_single_dit_layers
    total += blocks * 4.0 * N * N * D
    assert {"pos_embed", "context_embedder", "joint_transformer_blocks", "single_transformer_blocks",
            "norm_out", "proj_out"} <= counted
    B = 2
    assert bench.step_flops(H, W, L, B) == pytest.approx(B * total, rel=1e-12)


def test_step_flops_at_the_workload():
    """At 1024 x 1024 (latent 128 x 128, 256 text tokens, CFG batch 2): the
    36 blocks take 87.92 TFLOP (GEMM 71.1, attention 16.8) and the whole
    step 87.94 with the embeddings and modulations."""
    import bench
    D, F, _, _, _, R = bench.model_dims()
    N = R + 256 + 64 * 64
    gemm = 2 * 36 * 2.0 * N * (4 * D * D + 3 * D * F)
    attn = 2 * 36 * 4.0 * N * N * D
    assert gemm / 1e12 == pytest.approx(71.1, abs=0.05)
    assert attn / 1e12 == pytest.approx(16.8, abs=0.05)
    assert (gemm + attn) / 1e12 == pytest.approx(87.92, abs=0.005)
    assert bench.step_flops(128, 128, 256) / 1e12 == pytest.approx(87.94, abs=0.005)
