"""Plain fp64 CPU oracle of the AuraFlow denoising forward.

TEST INFRASTRUCTURE.  This file is the checker the CUDA path is compared
against; it is not part of the product.  Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import it.  It shares no code with the CUDA library.

Everything is numpy float64.  Inputs arrive as float32 arrays holding
bf16-exact (or fp32) values and are upcast once; no intermediate result is
rounded.  Library primitives used as single steps: ``@`` (matmul), ``exp``,
``sqrt``, ``cos``/``sin`` (and ``log2``/``exp2``/``floor``/``round`` for the
e4m3 rounding of the 8-bit variant).  Nothing is blocked, fused or reordered
beyond what the definitions below state.

Pages cited (title, then section):

* [ARCH]  "Diffusers 中的 AuraFlowTransformer2DModel架构解析与源码级使用指南"
  (mhpn.cn) -- the architecture description; its sections are 模型概述,
  构造参数详解, Patch Embedding, 联合注意力块, 单 DiT 块, FeedForward,
  调制与归一化, Register Tokens, 前向传播流程, 注意力处理器与 QKV 融合,
  在 AuraFlowPipeline 中的实际调用.
* [PIPE]  "Diffusers 中 AuraFlow 管线实战：从 bitsandbytes 量化到 torch.compile
  加速" (pwwt.cn) -- sections "AuraFlowPipeline 核心参数详解" and
  "深入源码：AuraFlowTransformer2DModel 的架构要点".
* [DEEP]  "【深度拆解】AuraFlow从基座到技术实现：开源文生图新范式" (csdn.net) --
  section "2.3 流匹配调度器：FlowMatchEulerDiscreteScheduler".

Where the pages leave a step open, the reading taken is marked READING.
Parity against the real diffusers model is unpinned for those readings (no
weights, source or golden tensors exist for it); each function below is
pinned instead by closed forms, invariants and brute force in
``tests/test_oracle_*.py``.
"""
from __future__ import annotations

from dataclasses import dataclass, field
import math

import numpy as np

F64 = np.float64


# --------------------------------------------------------------------------
# c1. Configuration
# --------------------------------------------------------------------------

def find_multiple(n: int, k: int) -> int:
    """Smallest multiple of ``k`` that is >= ``n``.

    [ARCH §FeedForward]: the FFN inner width is 2/3 of the hidden width,
    rounded up to a multiple of 256 with ``find_multiple``.
    """
    if n % k == 0:
        return n
    return n + k - (n % k)


@dataclass
class Config:
    """Constructor parameters, [ARCH §构造参数详解] (defaults are the page's)."""

    patch_size: int = 2
    in_channels: int = 4
    out_channels: int = 4
    num_mmdit_layers: int = 4
    num_single_dit_layers: int = 32
    attention_head_dim: int = 256
    num_attention_heads: int = 12
    joint_attention_dim: int = 2048
    pos_embed_max_size: int = 1024
    num_register_tokens: int = 8      # [ARCH §Register Tokens]
    timestep_channels: int = 256      # [ARCH §前向传播流程] Timesteps(256)
    ln_eps: float = 1e-6              # READING: eps not on the pages
    num_train_timesteps: int = 1000   # [DEEP §2.3]

    @property
    def inner_dim(self) -> int:
        """inner_dim = heads x head_dim ([ARCH §构造参数详解])."""
        return self.num_attention_heads * self.attention_head_dim

    @property
    def ffn_hidden(self) -> int:
        """FFN inner width: find_multiple(int(2 * hidden / 3), 256), hidden = 4 D.

        [ARCH §FeedForward] gives "2/3 x hidden_dim, then find_multiple to
        256".  READING: hidden_dim is 4 x inner_dim (the only value that
        gives the stated 8192 at D = 3072 and 256 at D = 32).
        """
        return find_multiple(int(2 * (4 * self.inner_dim) / 3), 256)

    @property
    def grid_side(self) -> int:
        """Side G of the square learned position grid (pos_embed_max_size = G*G).

        [ARCH §Patch Embedding]: the position table is viewed as a 2-D grid.
        """
        g = math.isqrt(self.pos_embed_max_size)
        if g * g != self.pos_embed_max_size:
            raise ValueError("pos_embed_max_size must be a perfect square")
        return g


def weight_specs(cfg: Config):
    """Names and shapes (nn.Linear layout [out, in]) of every parameter.

    Bias-free projections everywhere except the timestep MLP ([ARCH §模型概述]
    "注意力模块中不使用偏置", §联合注意力块 "bias=False", §前向传播流程
    context_embedder "bias=False", §调制与归一化 proj_out "bias=False").
    READING: the timestep MLP (TimestepEmbedding) carries biases.
    """
    D, F, p = cfg.inner_dim, cfg.ffn_hidden, cfg.patch_size
    s = [
        ("pos_embed.proj.weight", (D, p * p * cfg.in_channels)),
        ("pos_embed.pos_embed", (cfg.pos_embed_max_size, D)),
        ("time_step_proj.linear_1.weight", (D, cfg.timestep_channels)),
        ("time_step_proj.linear_1.bias", (D,)),
        ("time_step_proj.linear_2.weight", (D, D)),
        ("time_step_proj.linear_2.bias", (D,)),
        ("context_embedder.weight", (D, cfg.joint_attention_dim)),
        ("register_tokens", (cfg.num_register_tokens, D)),
    ]
    for i in range(cfg.num_mmdit_layers):
        b = f"joint_transformer_blocks.{i}."
        s += [
            (b + "norm1.linear.weight", (6 * D, D)),
            (b + "norm1_context.linear.weight", (6 * D, D)),
            (b + "attn.to_q.weight", (D, D)),
            (b + "attn.to_k.weight", (D, D)),
            (b + "attn.to_v.weight", (D, D)),
            (b + "attn.add_q_proj.weight", (D, D)),
            (b + "attn.add_k_proj.weight", (D, D)),
            (b + "attn.add_v_proj.weight", (D, D)),
            (b + "attn.to_out.0.weight", (D, D)),
            (b + "attn.to_add_out.weight", (D, D)),
            (b + "ff.linear_1.weight", (F, D)),
            (b + "ff.linear_2.weight", (F, D)),
            (b + "ff.out_projection.weight", (D, F)),
            (b + "ff_context.linear_1.weight", (F, D)),
            (b + "ff_context.linear_2.weight", (F, D)),
            (b + "ff_context.out_projection.weight", (D, F)),
        ]
    for i in range(cfg.num_single_dit_layers):
        b = f"single_transformer_blocks.{i}."
        s += [
            (b + "norm1.linear.weight", (6 * D, D)),
            (b + "attn.to_q.weight", (D, D)),
            (b + "attn.to_k.weight", (D, D)),
            (b + "attn.to_v.weight", (D, D)),
            (b + "attn.to_out.0.weight", (D, D)),
            (b + "ff.linear_1.weight", (F, D)),
            (b + "ff.linear_2.weight", (F, D)),
            (b + "ff.out_projection.weight", (D, F)),
        ]
    s += [
        ("norm_out.linear.weight", (2 * D, D)),
        ("proj_out.weight", (p * p * cfg.out_channels, D)),
    ]
    return s


def _f(x):
    return np.asarray(x, dtype=F64)


# --------------------------------------------------------------------------
# c2. Patchify / unpatchify
# --------------------------------------------------------------------------

def patchify(latents, p: int):
    """[B, C, H, W] -> [B, (H/p)(W/p), p*p*C].

    Token n = hp*(W/p) + wp (row-major patch grid).  Inside a patch the
    vector index is (py*p + px)*C + c, i.e. ordered (py, px, c).
    [ARCH §Patch Embedding]: latents are rearranged into patches and fed to
    nn.Linear(p*p*C, D).  READING: the inner order mirrors the (p, q, c)
    order that the unpatchify einsum fixes ([ARCH §前向传播流程]).
    """
    x = _f(latents)
    B, C, H, W = x.shape
    if H % p or W % p:
        raise ValueError("H and W must be multiples of the patch size")
    hp, wp = H // p, W // p
    out = np.empty((B, hp * wp, p * p * C), dtype=F64)
    for py in range(p):
        for px in range(p):
            for c in range(C):
                out[:, :, (py * p + px) * C + c] = x[:, c, py::p, px::p].reshape(B, hp * wp)
    return out


def unpatchify(o, p: int, c_out: int, hp: int, wp: int):
    """[B, hp*wp, p*p*c_out] -> [B, c_out, hp*p, wp*p].

    [ARCH §前向传播流程]: reshape to (patch_size, patch_size, out_channels)
    and apply einsum('nhwpqc->nchpwq').
    """
    o = _f(o)
    B = o.shape[0]
    x = o.reshape(B, hp, wp, p, p, c_out)
    x = np.einsum("nhwpqc->nchpwq", x)
    return x.reshape(B, c_out, hp * p, wp * p)


# --------------------------------------------------------------------------
# c3. Centre-cropped position table
# --------------------------------------------------------------------------

def pe_selection_index(G: int, hp: int, wp: int):
    """Flat indices of the centre hp x wp sub-grid of a G x G position grid.

    [ARCH §Patch Embedding] pe_selection_index_based_on_dim: the table is
    viewed as a 2-D grid, the centre block matching the patch grid is taken
    and flattened; the patch grid must not exceed the position grid.
    READING: an odd surplus is split with floor, top = (G - hp) // 2.
    """
    if hp > G or wp > G:
        raise ValueError("patch grid larger than the position grid")
    r0 = (G - hp) // 2
    c0 = (G - wp) // 2
    idx = []
    for i in range(hp):
        for j in range(wp):
            idx.append((r0 + i) * G + (c0 + j))
    return np.array(idx, dtype=np.int64)


def patch_embed(latents, w_proj, pos_table, p: int, G: int):
    """tokens = patchify(latents) @ W^T + PE[centre-crop index].

    [ARCH §Patch Embedding], [PIPE §深入源码] (linear projection, no conv,
    learned absolute positions).  READING: no projection bias.
    """
    lat = _f(latents)
    hp, wp = lat.shape[2] // p, lat.shape[3] // p
    tok = patchify(lat, p) @ _f(w_proj).T
    idx = pe_selection_index(G, hp, wp)
    return tok + _f(pos_table)[idx][None, :, :]


# --------------------------------------------------------------------------
# c4. Timestep embedding
# --------------------------------------------------------------------------

def timestep_features(t, n_channels: int = 256, scale: float = 1000.0):
    """Sinusoidal features of the model time t in [0, 1].

    [ARCH §前向传播流程]: Timesteps with 256 channels; [ARCH §在 AuraFlowPipeline
    中的实际调用]: the pipeline passes timestep/1000.
    READING: the argument is rescaled to the 1000-step training range
    ([DEEP §2.3] num_train_timesteps 1000), frequencies
    w_j = exp(-ln(10000) j / half), cosines first then sines.
    """
    t = _f(t).reshape(-1)
    half = n_channels // 2
    j = np.arange(half, dtype=F64)
    w = np.exp(-math.log(10000.0) * j / half)
    arg = (scale * t)[:, None] * w[None, :]
    return np.concatenate([np.cos(arg), np.sin(arg)], axis=1)


def silu(x):
    x = _f(x)
    return x / (1.0 + np.exp(-x))


def timestep_embedding(t, w1, b1, w2, b2, n_channels: int = 256):
    """temb = W2 silu(W1 e + b1) + b2 (TimestepEmbedding MLP, [ARCH §前向传播流程])."""
    e = timestep_features(t, n_channels)
    h = silu(e @ _f(w1).T + _f(b1))
    return h @ _f(w2).T + _f(b2)


# --------------------------------------------------------------------------
# c6/c7. adaLN-Zero, FP32 LayerNorm
# --------------------------------------------------------------------------

def layer_norm(x, eps: float):
    """LayerNorm over the last axis, biased variance, no affine parameters.

    [ARCH §调制与归一化]: FP32LayerNorm computes on inputs.float() and casts
    back (here everything is fp64).  READING: no affine weights, eps 1e-6.
    """
    x = _f(x)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps)


def modulate(x, shift, scale, eps: float):
    """LN(x) * (1 + scale) + shift, with per-sample shift/scale [B, D] on [B, N, D]."""
    return layer_norm(x, eps) * (1.0 + _f(scale)[:, None, :]) + _f(shift)[:, None, :]


MOD_CHUNKS = ("shift_msa", "scale_msa", "gate_msa", "shift_mlp", "scale_mlp", "gate_mlp")


def ada_ln_zero(temb, w_ada):
    """The six modulation vectors of one stream: W silu(temb), chunked in 6.

    [ARCH §联合注意力块] AdaLayerNormZero (bias=False); [ARCH §调制与归一化]
    "6 组调制系数".  READING: chunk order shift_msa, scale_msa, gate_msa,
    shift_mlp, scale_mlp, gate_mlp.
    """
    m = silu(temb) @ _f(w_ada).T
    return dict(zip(MOD_CHUNKS, np.split(m, 6, axis=-1)))


# --------------------------------------------------------------------------
# c8/c9. QK-norm and attention
# --------------------------------------------------------------------------

def split_heads(x, heads: int):
    B, N, D = x.shape
    return x.reshape(B, N, heads, D // heads).transpose(0, 2, 1, 3)


def merge_heads(x):
    B, H, N, hd = x.shape
    return x.transpose(0, 2, 1, 3).reshape(B, N, H * hd)


def attention(q, k, v, scale=None, key_mask=None):
    """softmax(q k^T * scale) v per (batch, head); non-causal, no dropout.

    [ARCH §注意力处理器与 QKV 融合]: F.scaled_dot_product_attention with
    dropout_p 0, is_causal False and an explicit scale.  READING: scale is
    head_dim^-1/2.  q, k, v: [B, H, N, hd].

    key_mask: optional bool [B, N_k], False = the key takes no part (its
    logit is -inf), like a boolean SDPA attn_mask broadcast over heads and
    queries.  The model's forward takes no mask ([ARCH §前向传播流程]); this
    is the padded-prompt extension (the pipeline pads prompts to a common
    length and builds an attention mask, [PIPE §AuraFlowPipeline 核心参数详解],
    [ARCH §在 AuraFlowPipeline 中的实际调用]).
    """
    q, k, v = _f(q), _f(k), _f(v)
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    B, H = q.shape[0], q.shape[1]
    out = np.empty(q.shape[:-1] + (v.shape[-1],), dtype=F64)
    # one (sample, head) at a time: the softmax of each is independent, and
    # the N x N logits of one head stay small enough for the 9480-token workload
    for b in range(B):
        for h in range(H):
            s = (q[b, h] @ k[b, h].T) * scale
            if key_mask is not None:
                s = np.where(np.asarray(key_mask, bool)[b][None, :], s, -np.inf)
            s = s - s.max(axis=-1, keepdims=True)
            p = np.exp(s)
            p = p / p.sum(axis=-1, keepdims=True)
            out[b, h] = p @ v[b, h]
    return out


def text_key_mask(text_len, n_registers: int, L: int, n_image: int):
    """Key mask [B, R + L + Ni] of the sequence [registers; text; image] when
    sample b's prompt has text_len[b] real tokens and L - text_len[b] padding
    tokens at its end.  Registers and image tokens are always attended.
    (Padded-prompt extension; see ``attention``.)"""
    tl = np.asarray(text_len, dtype=np.int64)
    B = tl.shape[0]
    m = np.ones((B, n_registers + L + n_image), dtype=bool)
    for b in range(B):
        m[b, n_registers + tl[b]:n_registers + L] = False
    return m


def _w8(w, fp8):
    """The weight as the GEMM sees it: as is, or per-output-row e4m3."""
    return fake_quant_rows(w) if fp8 else _f(w)


def _a8(x, fp8):
    """A GEMM's activation input as the GEMM sees it: as is, or per-token e4m3."""
    return fake_quant_rows(x) if fp8 else _f(x)


def round_bf16(x):
    """fp32 value of x, then rounded to bf16 (8 significant bits) to nearest even."""
    b = np.asarray(x, dtype=np.float64).astype(np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return b.astype(np.uint32).view(np.float32).astype(np.float64)


def _a8_stored(x, fp8):
    """Like _a8 for an activation the kernel path stores as bf16 before it is
    quantised (the attention output, the SwiGLU product): the per-token e4m3
    decision is taken on the bf16 value, in the kernel's precision."""
    return fake_quant_rows(round_bf16(x)) if fp8 else _f(x)


def qkv_normed(y, wq, wk, wv, heads: int, eps: float, fp8: bool = False):
    """Bias-free Q/K/V projections, then per-head LayerNorm of Q and K (not V).

    [ARCH §模型概述] QK Norm and no bias; [ARCH §注意力处理器与 QKV 融合]
    norm_q/norm_k (image) and norm_added_q/norm_added_k (text).
    READING: the QK-norm is the same affine-free fp32 LayerNorm, eps 1e-6.
    fp8: activations and weights pass through per-row e4m3 (8-bit variant).
    """
    if fp8:
        y = fake_quant_rows(y)
    q = split_heads(y @ _w8(wq, fp8).T, heads)
    k = split_heads(y @ _w8(wk, fp8).T, heads)
    v = split_heads(y @ _w8(wv, fp8).T, heads)
    return layer_norm(q, eps), layer_norm(k, eps), v


def feed_forward(y, w1, w2, w3, fp8: bool = False):
    """out_projection(silu(linear_1 y) * linear_2 y), all bias-free.

    [ARCH §FeedForward], [PIPE §深入源码] (SiLU-gated FFN).
    """
    y = _a8(y, fp8)
    h = silu(y @ _w8(w1, fp8).T) * (y @ _w8(w2, fp8).T)
    return _a8_stored(h, fp8) @ _w8(w3, fp8).T


# --------------------------------------------------------------------------
# 8-bit variant (extension): e4m3 weights and activations for the QKV and
# FFN up-projections
# --------------------------------------------------------------------------
# The pipeline guide loads the transformer with 8-bit weights
# ([PIPE] bitsandbytes quantisation sections).  The variant here is the
# tensor-core-native form of that idea: the operands of every projection in
# the blocks (fused QKV, output projection, FFN up and down) are rounded to
# the e4m3 format, each activation row (token) and each weight row (output
# channel) with its own fp32 scale, and the product is rescaled by both.
# READING: per-row absolute-maximum scaling, amax -> 448 (the largest finite
# e4m3 value); the attention itself, the LayerNorms, the modulations and the
# embedding / output stages stay as in the bf16 path.

E4M3_MAX = 448.0


def e4m3_round(x):
    """Nearest value of the 8-bit e4m3 format (1 sign bit, 4 exponent bits
    with bias 7, 3 mantissa bits, no infinities, largest finite 448, smallest
    subnormal 2^-9), ties to even, saturating at +-448.

    Normal binade [2^e, 2^(e+1)) for e >= -6 holds 8 values spaced 2^(e-3);
    below 2^-6 the spacing is the subnormal step 2^-9.
    """
    x = _f(x)
    a = np.abs(x)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -6.0)
    step = np.exp2(e - 3.0)
    q = np.round(a / step) * step          # np.round: half to even
    q = np.minimum(q, E4M3_MAX)
    return np.copysign(q, x)


def quantize_rows_e4m3(x):
    """Per-row e4m3 quantisation in the kernel's precision: with a = max |x|
    over the row (fp32), inv = 448 / a and s = a / 448 (fp32 divisions; 1
    for an all-zero row), the codes are e4m3(fp32(x * inv)).  Returns
    (codes as float64 values, s as float32)."""
    x32 = np.asarray(x, dtype=np.float64).astype(np.float32)
    amax = np.max(np.abs(x32), axis=-1)
    nz = amax > 0
    safe = np.where(nz, amax, np.float32(1.0)).astype(np.float32)
    inv = np.where(nz, np.float32(E4M3_MAX) / safe, np.float32(1.0)).astype(np.float32)
    scale = np.where(nz, safe / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    y = (x32 * inv[..., None]).astype(np.float32)
    return e4m3_round(y.astype(np.float64)), scale


def dequantize_rows(codes, scale):
    return _f(codes) * np.asarray(scale, dtype=np.float64)[..., None]


def fake_quant_rows(x):
    """x -> e4m3 codes x per-row scale, as the 8-bit GEMMs see it."""
    q, s = quantize_rows_e4m3(x)
    return dequantize_rows(q, s)


# --------------------------------------------------------------------------
# c10. Blocks
# --------------------------------------------------------------------------

def single_block_mod(x, mod, w, prefix, heads, eps, key_mask=None, fp8=False):
    """AuraFlowSingleTransformerBlock given its six modulation vectors.

    [ARCH §单 DiT 块]: adaLN-Zero DiT block on one (concatenated) sequence,
    self-attention with QK-norm, no bias, FP32 LayerNorm; then the gated
    SiLU FFN ([ARCH §FeedForward]).
      x += gate_msa * to_out(attn(QKV(LN(x)(1+scale_msa)+shift_msa)))
      x += gate_mlp * FFN(LN(x)(1+scale_mlp)+shift_mlp)
    """
    x = _f(x)
    y = modulate(x, mod["shift_msa"], mod["scale_msa"], eps)
    q, k, v = qkv_normed(y, w[prefix + "attn.to_q.weight"], w[prefix + "attn.to_k.weight"],
                         w[prefix + "attn.to_v.weight"], heads, eps, fp8)
    o = merge_heads(attention(q, k, v, key_mask=key_mask))
    x = x + mod["gate_msa"][:, None, :] * (_a8_stored(o, fp8) @ _w8(w[prefix + "attn.to_out.0.weight"], fp8).T)
    y = modulate(x, mod["shift_mlp"], mod["scale_mlp"], eps)
    f = feed_forward(y, w[prefix + "ff.linear_1.weight"], w[prefix + "ff.linear_2.weight"],
                     w[prefix + "ff.out_projection.weight"], fp8)
    return x + mod["gate_mlp"][:, None, :] * f


def single_block(x, temb, w, prefix, cfg: Config, key_mask=None, fp8=False):
    mod = ada_ln_zero(temb, w[prefix + "norm1.linear.weight"])
    return single_block_mod(x, mod, w, prefix, cfg.num_attention_heads, cfg.ln_eps, key_mask, fp8)


def joint_block_mod(img, txt, mod_i, mod_t, w, prefix, heads, eps, key_mask=None, fp8=False):
    """AuraFlowJointTransformerBlock given both streams' modulation vectors.

    [ARCH §联合注意力块]: two residual streams (image, text), each with its
    own adaLN-Zero, Q/K/V (text: add_q/k/v_proj, bias-free), output
    projection and FFN; one joint attention over the concatenated tokens.
    [ARCH §注意力处理器与 QKV 融合]: text and image tokens are concatenated,
    attended, and split back.  READING: text first in the concatenation
    (the single-block sequence is cat(text, image), [ARCH §前向传播流程]);
    the text stream's output projection is to_add_out.  Returns (txt, img)
    like the block's forward.
    """
    img, txt = _f(img), _f(txt)
    nt = txt.shape[1]
    yi = modulate(img, mod_i["shift_msa"], mod_i["scale_msa"], eps)
    yt = modulate(txt, mod_t["shift_msa"], mod_t["scale_msa"], eps)
    qi, ki, vi = qkv_normed(yi, w[prefix + "attn.to_q.weight"], w[prefix + "attn.to_k.weight"],
                            w[prefix + "attn.to_v.weight"], heads, eps, fp8)
    qt, kt, vt = qkv_normed(yt, w[prefix + "attn.add_q_proj.weight"], w[prefix + "attn.add_k_proj.weight"],
                            w[prefix + "attn.add_v_proj.weight"], heads, eps, fp8)
    q = np.concatenate([qt, qi], axis=2)
    k = np.concatenate([kt, ki], axis=2)
    v = np.concatenate([vt, vi], axis=2)
    o = merge_heads(attention(q, k, v, key_mask=key_mask))
    ot, oi = o[:, :nt], o[:, nt:]
    img = img + mod_i["gate_msa"][:, None, :] * (_a8_stored(oi, fp8) @ _w8(w[prefix + "attn.to_out.0.weight"], fp8).T)
    txt = txt + mod_t["gate_msa"][:, None, :] * (_a8_stored(ot, fp8) @ _w8(w[prefix + "attn.to_add_out.weight"], fp8).T)
    yi = modulate(img, mod_i["shift_mlp"], mod_i["scale_mlp"], eps)
    yt = modulate(txt, mod_t["shift_mlp"], mod_t["scale_mlp"], eps)
    img = img + mod_i["gate_mlp"][:, None, :] * feed_forward(
        yi, w[prefix + "ff.linear_1.weight"], w[prefix + "ff.linear_2.weight"],
        w[prefix + "ff.out_projection.weight"], fp8)
    txt = txt + mod_t["gate_mlp"][:, None, :] * feed_forward(
        yt, w[prefix + "ff_context.linear_1.weight"], w[prefix + "ff_context.linear_2.weight"],
        w[prefix + "ff_context.out_projection.weight"], fp8)
    return txt, img


def joint_block(img, txt, temb, w, prefix, cfg: Config, key_mask=None, fp8=False):
    mod_i = ada_ln_zero(temb, w[prefix + "norm1.linear.weight"])
    mod_t = ada_ln_zero(temb, w[prefix + "norm1_context.linear.weight"])
    return joint_block_mod(img, txt, mod_i, mod_t, w, prefix, cfg.num_attention_heads, cfg.ln_eps, key_mask, fp8)


# --------------------------------------------------------------------------
# Sampled-row evaluation of a block (same definition, fewer outputs)
# --------------------------------------------------------------------------

def single_block_rows(x, temb, w, prefix, cfg: Config, rows, key_mask=None):
    """Rows ``rows`` (indices into the sequence) of single_block's output.

    Same formula as ``single_block``: K and V need every token, while the
    query side, output projection and FFN act on each token independently,
    so only the listed tokens are carried through them.  Returns [B, len(rows), D].
    """
    x = _f(x)
    heads, eps = cfg.num_attention_heads, cfg.ln_eps
    mod = ada_ln_zero(temb, w[prefix + "norm1.linear.weight"])
    y = modulate(x, mod["shift_msa"], mod["scale_msa"], eps)
    k = layer_norm(split_heads(y @ _f(w[prefix + "attn.to_k.weight"]).T, heads), eps)
    v = split_heads(y @ _f(w[prefix + "attn.to_v.weight"]).T, heads)
    yr = y[:, rows]
    q = layer_norm(split_heads(yr @ _f(w[prefix + "attn.to_q.weight"]).T, heads), eps)
    o = merge_heads(attention(q, k, v, key_mask=key_mask))
    xr = x[:, rows] + mod["gate_msa"][:, None, :] * (o @ _f(w[prefix + "attn.to_out.0.weight"]).T)
    y2 = modulate(xr, mod["shift_mlp"], mod["scale_mlp"], eps)
    f = feed_forward(y2, w[prefix + "ff.linear_1.weight"], w[prefix + "ff.linear_2.weight"],
                     w[prefix + "ff.out_projection.weight"])
    return xr + mod["gate_mlp"][:, None, :] * f


def joint_block_rows(img, txt, temb, w, prefix, cfg: Config, img_rows, txt_rows, key_mask=None):
    """Rows of joint_block's outputs: (txt[:, txt_rows], img[:, img_rows])."""
    img, txt = _f(img), _f(txt)
    heads, eps = cfg.num_attention_heads, cfg.ln_eps
    mi = ada_ln_zero(temb, w[prefix + "norm1.linear.weight"])
    mt = ada_ln_zero(temb, w[prefix + "norm1_context.linear.weight"])
    yi = modulate(img, mi["shift_msa"], mi["scale_msa"], eps)
    yt = modulate(txt, mt["shift_msa"], mt["scale_msa"], eps)

    def kv(y, wk, wv):
        return (layer_norm(split_heads(y @ _f(w[prefix + wk]).T, heads), eps),
                split_heads(y @ _f(w[prefix + wv]).T, heads))

    ki, vi = kv(yi, "attn.to_k.weight", "attn.to_v.weight")
    kt, vt = kv(yt, "attn.add_k_proj.weight", "attn.add_v_proj.weight")
    k = np.concatenate([kt, ki], axis=2)
    v = np.concatenate([vt, vi], axis=2)
    qi = layer_norm(split_heads(yi[:, img_rows] @ _f(w[prefix + "attn.to_q.weight"]).T, heads), eps)
    qt = layer_norm(split_heads(yt[:, txt_rows] @ _f(w[prefix + "attn.add_q_proj.weight"]).T, heads), eps)
    oi = merge_heads(attention(qi, k, v, key_mask=key_mask))
    ot = merge_heads(attention(qt, k, v, key_mask=key_mask))
    xi = img[:, img_rows] + mi["gate_msa"][:, None, :] * (oi @ _f(w[prefix + "attn.to_out.0.weight"]).T)
    xt = txt[:, txt_rows] + mt["gate_msa"][:, None, :] * (ot @ _f(w[prefix + "attn.to_add_out.weight"]).T)
    y2i = modulate(xi, mi["shift_mlp"], mi["scale_mlp"], eps)
    y2t = modulate(xt, mt["shift_mlp"], mt["scale_mlp"], eps)
    xi = xi + mi["gate_mlp"][:, None, :] * feed_forward(
        y2i, w[prefix + "ff.linear_1.weight"], w[prefix + "ff.linear_2.weight"],
        w[prefix + "ff.out_projection.weight"])
    xt = xt + mt["gate_mlp"][:, None, :] * feed_forward(
        y2t, w[prefix + "ff_context.linear_1.weight"], w[prefix + "ff_context.linear_2.weight"],
        w[prefix + "ff_context.out_projection.weight"])
    return xt, xi


# --------------------------------------------------------------------------
# c5 / c11. Text stream entry, pre-final block, full forward
# --------------------------------------------------------------------------

def text_stream(text_emb, w_ctx, registers):
    """cat(register tokens, context_embedder(text)) along the sequence.

    [ARCH §前向传播流程]: context_embedder = Linear(2048, 3072, bias=False);
    [ARCH §Register Tokens]: 8 learned tokens are placed at the head of the
    encoder sequence.
    """
    e = _f(text_emb) @ _f(w_ctx).T
    B = e.shape[0]
    r = np.broadcast_to(_f(registers)[None], (B,) + tuple(registers.shape))
    return np.concatenate([r, e], axis=1)


def pre_final(x_img, temb, w_pf):
    """AuraFlowPreFinalBlock: x * (1 + scale) + shift with [scale, shift] = W silu(temb).

    [ARCH §调制与归一化], [PIPE §深入源码].  READING: chunk order scale then
    shift (the order of the page's formula), no LayerNorm, bias-free.
    """
    m = silu(temb) @ _f(w_pf).T
    scale, shift = np.split(m, 2, axis=-1)
    return _f(x_img) * (1.0 + scale[:, None, :]) + shift[:, None, :]


def embed(latents, text_emb, t, w, cfg: Config):
    """Entry stage: (image tokens, text tokens, temb) -- [ARCH §前向传播流程] 嵌入阶段."""
    img = patch_embed(latents, w["pos_embed.proj.weight"], w["pos_embed.pos_embed"],
                      cfg.patch_size, cfg.grid_side)
    temb = timestep_embedding(t, w["time_step_proj.linear_1.weight"], w["time_step_proj.linear_1.bias"],
                              w["time_step_proj.linear_2.weight"], w["time_step_proj.linear_2.bias"],
                              cfg.timestep_channels)
    txt = text_stream(text_emb, w["context_embedder.weight"], w["register_tokens"])
    return img, txt, temb


def output_stage(x_img, temb, w, cfg: Config, H: int, W: int):
    """Pre-final modulation, proj_out (bias-free) and unpatchify ([ARCH §前向传播流程] 输出阶段)."""
    p = cfg.patch_size
    z = pre_final(x_img, temb, w["norm_out.linear.weight"])
    o = z @ _f(w["proj_out.weight"]).T
    return unpatchify(o, p, cfg.out_channels, H // p, W // p)


def transformer_forward(latents, text_emb, t, w, cfg: Config, text_len=None, fp8=False):
    """AuraFlowTransformer2DModel.forward -> velocity [B, C_out, H, W].

    [ARCH §前向传播流程]: embed; num_mmdit_layers joint blocks updating both
    streams; cat(text, image); num_single_dit_layers single blocks; keep the
    image part combined[:, encoder_seq_len:]; pre-final; proj_out;
    unpatchify.  ``t`` is the model time in [0, 1] (timestep / 1000).
    ``text_len`` (optional, [B]): real prompt tokens per sample; the rest of
    the L text tokens are padding that no attention reads (``text_key_mask``).
    ``fp8``: the 8-bit variant (e4m3 operands for every projection in the blocks).
    """
    latents = _f(latents)
    H, W = latents.shape[2], latents.shape[3]
    img, txt, temb = embed(latents, text_emb, t, w, cfg)
    nt = txt.shape[1]
    mask = None
    if text_len is not None:
        mask = text_key_mask(text_len, cfg.num_register_tokens, nt - cfg.num_register_tokens, img.shape[1])
    for i in range(cfg.num_mmdit_layers):
        txt, img = joint_block(img, txt, temb, w, f"joint_transformer_blocks.{i}.", cfg, mask, fp8)
    x = np.concatenate([txt, img], axis=1)
    for i in range(cfg.num_single_dit_layers):
        x = single_block(x, temb, w, f"single_transformer_blocks.{i}.", cfg, mask, fp8)
    return output_stage(x[:, nt:], temb, w, cfg, H, W)


# --------------------------------------------------------------------------
# c12-c14. Sampler pieces: CFG combine, Euler step, sigma schedule
# --------------------------------------------------------------------------

def cfg_combine(v_uncond, v_text, guidance):
    """v_u + g (v_c - v_u) ([PIPE §AuraFlowPipeline 核心参数详解] CFG formula;
    [ARCH §在 AuraFlowPipeline 中的实际调用] chunk(2): uncond first)."""
    vu, vc = _f(v_uncond), _f(v_text)
    return vu + guidance * (vc - vu)


def euler_step(x, v, sigma, sigma_next):
    """Flow-matching Euler update x <- x + (sigma_next - sigma) v.

    [ARCH §在 AuraFlowPipeline 中的实际调用]: t = 1 is pure noise, t = 0 the
    image, and the scheduler steps back from the model's prediction; the
    scheduler is FlowMatchEulerDiscreteScheduler ([PIPE], [DEEP §2.3]).
    READING: x_sigma = (1 - sigma) x0 + sigma eps and the model returns
    v = eps - x0, so an Euler step in sigma is the update above.
    """
    return _f(x) + (float(sigma_next) - float(sigma)) * _f(v)


def euler_cfg_step(x, v_pair, guidance, sigma, sigma_next):
    """CFG combine of the [2B, ...] batch (uncond half first), then Euler."""
    v_pair = _f(v_pair)
    b = v_pair.shape[0] // 2
    return euler_step(x, cfg_combine(v_pair[:b], v_pair[b:], guidance), sigma, sigma_next)


def sigma_schedule(n_steps: int, shift: float = 1.73, num_train_timesteps: int = 1000):
    """n_steps + 1 sigmas, from 1 (noise) down to 0.

    [DEEP §2.3]: num_train_timesteps 1000, shift 1.73, 25 steps in use.
    READING: base s = linspace(1, 1/num_train_timesteps, n_steps), shifted
    sigma = k s / (1 + (k - 1) s), with a final 0 appended; the model time of
    step i is t_i = sigma_i.
    """
    s = np.linspace(1.0, 1.0 / num_train_timesteps, n_steps, dtype=F64)
    sig = shift * s / (1.0 + (shift - 1.0) * s)
    return np.append(sig, 0.0)


# --------------------------------------------------------------------------
# Utilities for comparisons
# --------------------------------------------------------------------------

def rel_l2(a, b) -> float:
    """||a - b||_2 / ||b||_2 in fp64 (b is the reference)."""
    a, b = _f(a), _f(b)
    return float(np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-300))
