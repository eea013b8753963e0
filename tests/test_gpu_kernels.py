"""GPU parity of the individual kernels against the fp64 oracle.

Inputs are seeded (synth), bf16-exact, and identical on both sides.
Tolerances (relative L2 unless stated) follow from the arithmetic: outputs
stored as bf16 carry a relative rounding error of at most 2^-9 per element
(rel-L2 about 2^-9 / sqrt(3) ~ 1.1e-3 for random data); the attention
probabilities are also rounded to bf16 before the PV product, so it gets 1e-2.
Index and gather work is checked bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from helpers import to_bf16, to_f32, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def af():
    import diffusion_transformer_denoising_auraflow_b200 as m
    assert torch.cuda.is_available()
    return m


# ---------------------------------------------------------------- GEMM (tcgen05)

@pytest.mark.parametrize("M,N,K", [(300, 520, 200), (1000, 3072, 3072), (64, 96, 32), (129, 256, 64),
                                   (528, 9216, 3072), (8, 16, 2048),
                                   # M >= 1024 runs on CTA pairs (256-row tiles, cta_group::2)
                                   (1100, 776, 520), (4096, 3072, 3072), (2304, 16, 64), (8720, 1024, 8192)])
def test_linear_matches_fp64(af, M, N, K):
    A = synth.normal(11, f"A{M}_{N}_{K}", (M, K), 1.0)
    W = synth.normal(12, f"W{M}_{N}_{K}", (N, K), 0.02)
    C = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    af.linear(to_bf16(A), to_bf16(W), C)
    torch.cuda.synchronize()
    ref = A.astype(np.float64) @ W.astype(np.float64).T
    got = to_np(C)
    assert O.rel_l2(got, ref) < 3e-3
    # every element within bf16 rounding of the exact value (plus fp32 accumulation slack)
    assert np.all(np.abs(got - ref) <= 2 ** -8 * np.abs(ref) + 1e-4 * np.sqrt(K) * 0.02 * 4)


# The joint block's grouped form (image- and text-stream projections in one
# persistent launch) against the two products launched alone ("fused ==
# unfused"): every output element is one full-K chain of tensor-core MMAs
# in the same K order whichever tile, launch or CTA-group width computes it
# (a problem below 1024 rows runs on the 1-CTA kernel alone and on CTA pairs
# when grouped), so the two agree bit for bit; both are also held to fp64.
@pytest.mark.parametrize("M0,N0,K0,M1,N1,K1", [(8192, 3072, 3072, 528, 3072, 3072),
                                               (4096, 9216, 3072, 1030, 9216, 3072),
                                               (1100, 776, 520, 300, 520, 200),
                                               (300, 520, 200, 64, 96, 32)])
def test_linear_grouped_equals_separate(af, M0, N0, K0, M1, N1, K1):
    A0 = synth.normal(21, f"gA0_{M0}_{N0}_{K0}", (M0, K0), 1.0)
    W0 = synth.normal(22, f"gW0_{M0}_{N0}_{K0}", (N0, K0), 0.02)
    A1 = synth.normal(23, f"gA1_{M1}_{N1}_{K1}", (M1, K1), 1.0)
    W1 = synth.normal(24, f"gW1_{M1}_{N1}_{K1}", (N1, K1), 0.02)
    a0, w0, a1, w1 = to_bf16(A0), to_bf16(W0), to_bf16(A1), to_bf16(W1)
    G0 = torch.empty(M0, N0, dtype=torch.bfloat16, device="cuda")
    G1 = torch.empty(M1, N1, dtype=torch.bfloat16, device="cuda")
    S0 = torch.empty_like(G0)
    S1 = torch.empty_like(G1)
    af.linear_grouped(a0, w0, G0, a1, w1, G1)
    af.linear(a0, w0, S0)
    af.linear(a1, w1, S1)
    torch.cuda.synchronize()
    for G, S, A, W in ((G0, S0, A0, W0), (G1, S1, A1, W1)):
        assert torch.equal(G, S)
        ref = A.astype(np.float64) @ W.astype(np.float64).T
        assert O.rel_l2(to_np(G), ref) < 3e-3


def test_linear_rejects_unaligned_k(af):
    A = torch.zeros(4, 12, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(8, 12, dtype=torch.bfloat16, device="cuda")
    C = torch.zeros(4, 8, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(af.AFError):
        af.linear(A, W, C)


# ---------------------------------------------------------------- attention

ATTN_CASES = [(2, 2, 1, 256, 1.0), (1, 2, 7, 256, 1.0), (2, 1, 64, 256, 1.0), (1, 2, 129, 256, 1.0),
              (2, 2, 264, 256, 3.0), (1, 3, 600, 256, 1.0), (1, 4, 80, 8, 1.0), (2, 2, 33, 16, 1.0),
              # N >= 256 with QK-normalised inputs runs on CTA pairs (256 query rows, 128-key tiles)
              (1, 2, 256, 256, 1.0), (2, 1, 257, 256, 1.0), (1, 2, 1000, 256, 1.0), (1, 1, 4360, 256, 1.0)]


@pytest.mark.parametrize("qkn", [False, True])
@pytest.mark.parametrize("B,H,N,hd,qscale", ATTN_CASES)
def test_attention_matches_oracle(af, B, H, N, hd, qscale, qkn):
    if qkn and qscale != 1.0:
        pytest.skip("the fixed-shift kernel requires per-head LayerNorm-ed q and k")
    q = synth.normal(21, f"q{N}", (B, H, N, hd), 1.0)
    k = synth.normal(22, f"k{N}", (B, H, N, hd), 1.0)
    v = synth.normal(23, f"v{N}", (B, H, N, hd), 1.0)
    # per-head normalised q and k, like the QK-norm output, then scaled
    qn = synth.bf16_round((O.layer_norm(q, 1e-6) * qscale).astype(np.float32))
    kn = synth.bf16_round(O.layer_norm(k, 1e-6).astype(np.float32))
    o = torch.empty(B, N, H * hd, dtype=torch.bfloat16, device="cuda")
    af.attention(to_bf16(qn), to_bf16(kn), to_bf16(v), o, qk_normalized=qkn)
    torch.cuda.synchronize()
    ref = O.merge_heads(O.attention(qn, kn, v))
    assert O.rel_l2(to_np(o), ref) < 1e-2


@pytest.mark.parametrize("qkn", [False, True])
def test_attention_extreme_logits(af, qkn):
    """q = k (LayerNorm-ed): every diagonal logit is at the bound |q.k|/16 = 16."""
    B, H, N, hd = 1, 2, 300, 256
    q = synth.normal(26, "qe", (B, H, N, hd), 1.0)
    qn = synth.bf16_round(O.layer_norm(q, 1e-6).astype(np.float32))
    v = synth.normal(27, "ve", (B, H, N, hd), 1.0)
    o = torch.empty(B, N, H * hd, dtype=torch.bfloat16, device="cuda")
    af.attention(to_bf16(qn), to_bf16(qn), to_bf16(v), o, qk_normalized=qkn)
    torch.cuda.synchronize()
    ref = O.merge_heads(O.attention(qn, qn, v))
    assert O.rel_l2(to_np(o), ref) < 1e-2


def test_attention_single_token_is_v(af):
    v = synth.normal(24, "v1", (1, 2, 1, 256), 1.0)
    q = synth.normal(25, "q1", (1, 2, 1, 256), 1.0)
    o = torch.empty(1, 1, 512, dtype=torch.bfloat16, device="cuda")
    af.attention(to_bf16(q), to_bf16(q), to_bf16(v), o)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(o), O.merge_heads(v))


# ---------------------------------------------------------------- LN + modulate

@pytest.mark.parametrize("B,N,D", [(2, 37, 3072), (1, 5, 32), (2, 300, 3072), (3, 9, 256)])
def test_ln_modulate_matches_oracle(af, B, N, D):
    x = synth.normal(31, f"x{N}_{D}", (B, N, D), 1.0) * 3 + 0.5
    x = synth.bf16_round(x.astype(np.float32))
    mods = synth.normal(32, f"m{D}", (B, 6 * D), 0.5, "f32")
    y = torch.empty(B, N, D, dtype=torch.bfloat16, device="cuda")
    md = to_f32(mods)
    af.ln_modulate(to_bf16(x), md[:, 3 * D:], md[:, 4 * D:], 6 * D, y, 1e-6)
    torch.cuda.synchronize()
    ref = O.modulate(x, mods[:, 3 * D:4 * D], mods[:, 4 * D:5 * D], 1e-6)
    assert O.rel_l2(to_np(y), ref) < 3e-3


# ---------------------------------------------------------------- embeddings, sampler step

def _weights_for(af, cfg, seed, names):
    from helpers import af_config, draw_weights, upload
    w = af.Weights(af_config(cfg))
    drawn = draw_weights(cfg, seed, names)
    upload(w, drawn)
    return w, drawn


@pytest.mark.parametrize("G,H,W", [(8, 12, 8), (64, 128, 128), (8, 10, 14)])
def test_patch_embed_gather_bit_exact(af, G, H, W):
    from helpers import tiny_config
    cfg = tiny_config(pos_embed_max_size=G * G)
    w, drawn = _weights_for(af, cfg, 41, ["pos_embed.pos_embed"])   # projection stays zero
    s = af.Scratch(w, 2, (H // 2) * (W // 2), 8)
    lat = synth.latents(42, (2, 4, H, W))
    img = torch.empty(2, (H // 2) * (W // 2), cfg.inner_dim, dtype=torch.bfloat16, device="cuda")
    af.patch_embed(w, s, to_f32(lat), img)
    torch.cuda.synchronize()
    idx = O.pe_selection_index(G, H // 2, W // 2)
    expect = drawn["pos_embed.pos_embed"][idx]
    got = to_np(img)
    for b in range(2):
        assert np.array_equal(got[b], expect)


def test_patch_embed_matches_oracle(af):
    from helpers import tiny_config
    cfg = tiny_config(pos_embed_max_size=100)
    w, drawn = _weights_for(af, cfg, 43, ["pos_embed.pos_embed", "pos_embed.proj.weight"])
    s = af.Scratch(w, 2, 48, 8)
    lat = synth.latents(44, (2, 4, 12, 16))
    img = torch.empty(2, 48, cfg.inner_dim, dtype=torch.bfloat16, device="cuda")
    af.patch_embed(w, s, to_f32(lat), img)
    torch.cuda.synchronize()
    ref = O.patch_embed(lat, drawn["pos_embed.proj.weight"], drawn["pos_embed.pos_embed"], 2, 10)
    assert O.rel_l2(to_np(img), ref) < 3e-3


def test_patch_embed_rejects_bad_shapes(af):
    from helpers import tiny_config
    cfg = tiny_config()
    w, _ = _weights_for(af, cfg, 45, [])
    s = af.Scratch(w, 1, 64, 8)
    img = torch.empty(1, 64, 32, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(af.AFError):       # odd height
        af.patch_embed(w, s, torch.zeros(1, 4, 15, 16, device="cuda"), img)
    with pytest.raises(af.AFError):       # 9 x 9 patch grid > 8 x 8 position grid
        af.patch_embed(w, s, torch.zeros(1, 4, 18, 18, device="cuda"), img)


@pytest.mark.parametrize("D", [32, 3072])
def test_timestep_embed_matches_oracle(af, D):
    from helpers import tiny_config, full_config
    cfg = tiny_config() if D == 32 else full_config()
    names = [n for n, _ in O.weight_specs(cfg) if n.startswith("time_step_proj")]
    w, drawn = _weights_for(af, cfg, 51, names)
    s = af.Scratch(w, 4, 64, 8)
    t = np.array([0.0, 0.5, 0.731, 1.0], dtype=np.float32)
    temb = torch.empty(4, D, dtype=torch.float32, device="cuda")
    af.timestep_embed(w, s, to_f32(t), temb)
    torch.cuda.synchronize()
    ref = O.timestep_embedding(t, drawn["time_step_proj.linear_1.weight"], drawn["time_step_proj.linear_1.bias"],
                               drawn["time_step_proj.linear_2.weight"], drawn["time_step_proj.linear_2.bias"])
    assert O.rel_l2(to_np(temb), ref) < 1e-3


def test_euler_cfg_step_matches_oracle(af):
    x = synth.latents(61, (1, 4, 128, 128))
    v = synth.normal(62, "v", (2, 4, 128, 128), 1.0, "f32")
    xt = to_f32(x)
    af.euler_cfg_step(xt, to_f32(v), 3.5, 0.8, 0.75)
    torch.cuda.synchronize()
    ref = O.euler_cfg_step(x, v, 3.5, 0.8, 0.75)
    assert np.max(np.abs(to_np(xt) - ref)) < 1e-5
    xt = to_f32(x)
    af.euler_cfg_step(xt, to_f32(v), 3.5, 0.6, 0.6)    # sigma' = sigma: no-op, bit-exact
    torch.cuda.synchronize()
    assert np.array_equal(to_np(xt), x.astype(np.float64))


# ---------------------------------------------------------------- attention with a key mask (padded prompts)

MASK_CASES = [  # B, H, N, hd, key_base, key_end, key_len per sample
    (2, 2, 1000, 256, 8, 400, [5, 300]),      # CTA-pair kernel: masked range spans several key tiles
    (2, 1, 4360, 256, 8, 264, [0, 256]),      # the model's shape: 8 registers + 256 text tokens
    (2, 2, 200, 256, 8, 100, [0, 50]),        # one-CTA kernels (N < 256)
    (2, 2, 33, 16, 2, 20, [3, 18]),           # small heads (SIMT)
]


@pytest.mark.parametrize("qkn", [False, True])
@pytest.mark.parametrize("B,H,N,hd,base,end,lens", MASK_CASES)
def test_attention_key_mask_matches_oracle(af, B, H, N, hd, base, end, lens, qkn):
    q = synth.normal(401, f"mq{N}", (B, H, N, hd), 1.0)
    k = synth.normal(402, f"mk{N}", (B, H, N, hd), 1.0)
    v = synth.normal(403, f"mv{N}", (B, H, N, hd), 1.0)
    qn = synth.bf16_round(O.layer_norm(q, 1e-6).astype(np.float32))
    kn = synth.bf16_round(O.layer_norm(k, 1e-6).astype(np.float32))
    mask = np.ones((B, N), bool)
    for b, n in enumerate(lens):
        mask[b, base + n:end] = False
    o = torch.empty(B, N, H * hd, dtype=torch.bfloat16, device="cuda")
    kl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    af.attention(to_bf16(qn), to_bf16(kn), to_bf16(v), o, qk_normalized=qkn, key_len=kl, key_base=base, key_end=end)
    torch.cuda.synchronize()
    ref = O.merge_heads(O.attention(qn, kn, v, key_mask=mask))
    assert O.rel_l2(to_np(o), ref) < 1e-2
    # masked keys carry no weight: changing them leaves the output bit-identical
    k2 = kn.copy()
    v2 = v.copy()
    k2[~mask[:, None, :, None].repeat(H, 1).repeat(hd, 3)] = 0.5
    v2[~mask[:, None, :, None].repeat(H, 1).repeat(hd, 3)] = 100.0
    o2 = torch.empty_like(o)
    af.attention(to_bf16(qn), to_bf16(k2), to_bf16(v2), o2, qk_normalized=qkn, key_len=kl, key_base=base, key_end=end)
    torch.cuda.synchronize()
    assert torch.equal(o, o2)


def test_attention_rejects_bad_mask(af):
    q = torch.zeros(1, 1, 64, 256, dtype=torch.bfloat16, device="cuda")
    o = torch.empty(1, 64, 256, dtype=torch.bfloat16, device="cuda")
    kl = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(af.AFError):          # key_base 0 could mask every key
        af.attention(q, q, q, o, key_len=kl, key_base=0, key_end=10)
    with pytest.raises(af.AFError):          # end beyond N
        af.attention(q, q, q, o, key_len=kl, key_base=1, key_end=65)
