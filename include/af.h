/*
 * af.h -- C ABI of the B200 (sm_100a) AuraFlow denoising forward.
 *
 * The library computes the AuraFlowTransformer2DModel forward and the
 * flow-match Euler + classifier-free-guidance step on one GPU with
 * hand-written CUDA kernels.  Citations name the page title and section of
 * the description the operation follows:
 *
 *   [ARCH] "Diffusers 中的 AuraFlowTransformer2DModel架构解析与源码级使用指南"
 *   [PIPE] "Diffusers 中 AuraFlow 管线实战：从 bitsandbytes 量化到 torch.compile 加速"
 *   [DEEP] "【深度拆解】AuraFlow从基座到技术实现：开源文生图新范式"
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Tensors are caller-owned, contiguous, row-major.  "device" pointers
 *    must be CUDA device memory of the device the weight pack lives on, and
 *    that device must be the current one when a call taking a weight pack
 *    or scratch handle is made (else AF_ERR_INVALID_ARG, nothing launched).
 *    bf16 tensors are passed as uint16_t bit patterns.
 *  - A weight pack stores bf16 (AF_DTYPE_BF16, the tensor-core path) or
 *    fp32 (AF_DTYPE_F32, plain fp32 arithmetic end to end for small
 *    configurations).  With an fp32 pack every activation a call takes or
 *    returns as bf16 below is fp32 instead (text_emb, which is declared
 *    const void*); the block-level, patch-embed and 8-bit calls take bf16
 *    packs only and return AF_ERR_UNSUPPORTED for an fp32 pack.
 *  - Compute calls are asynchronous on `stream` (a cudaStream_t passed as
 *    void*; NULL = legacy default stream).  They return once all work is
 *    enqueued.
 *  - Argument and shape errors are detected on the host, before anything is
 *    launched, and reported as AF_ERR_INVALID_ARG / AF_ERR_SHAPE /
 *    AF_ERR_UNSUPPORTED; nothing is modified in that case.
 *  - A CUDA launch or runtime failure returns AF_ERR_CUDA; af_last_error()
 *    then holds the CUDA error text.
 *  - Every device-side wait in the kernels is bounded.  A wait that runs out
 *    records an error word in the scratch handle; af_sync() reports it as
 *    AF_ERR_TIMEOUT.
 *  - Only *_create calls allocate device memory.  A scratch handle must not
 *    be used by two streams at once (calls on it would race).
 */
#ifndef AF_H_
#define AF_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  AF_OK = 0,
  AF_ERR_INVALID_ARG = 1,  /* null handle/pointer, bad enum, negative size */
  AF_ERR_SHAPE = 2,        /* sizes inconsistent with the model or over capacity */
  AF_ERR_UNSUPPORTED = 3,  /* configuration the kernels do not cover */
  AF_ERR_OOM = 4,          /* device allocation failed in a *_create call */
  AF_ERR_CUDA = 5,         /* CUDA runtime error (see af_last_error) */
  AF_ERR_TIMEOUT = 6,      /* a bounded device-side wait expired (from af_sync) */
  AF_ERR_NOT_FOUND = 7     /* unknown tensor name */
} af_status;

/* Storage / arithmetic type of a weight pack (af_config.dtype) and of the
 * tensors handed to af_weights_set / af_weights_get. */
#define AF_DTYPE_BF16 0
#define AF_DTYPE_F32 1

/* Model configuration: the constructor parameters of
 * AuraFlowTransformer2DModel ([ARCH] §构造参数详解).
 *   inner_dim D = num_attention_heads * attention_head_dim.
 *   ffn_inner  = 0 selects find_multiple(int(2 * 4D / 3), 256) ([ARCH]
 *                §FeedForward); any other value is used as given.
 *   pos_embed_max_size = G*G, the size of the learned position grid
 *                ([ARCH] §Patch Embedding); must be a perfect square.
 *   num_register_tokens: learned tokens at the head of the text sequence
 *                ([ARCH] §Register Tokens), 8 in the model.
 *   timestep_channels: sinusoidal timestep channels, 256 ([ARCH] §前向传播流程).
 *   ln_eps: epsilon of every LayerNorm (adaLN and QK-norm).
 *   dtype: AF_DTYPE_BF16 (bf16 weights and activations, fp32 accumulation
 *                and statistics, tcgen05 tensor cores) or AF_DTYPE_F32
 *                (fp32 weights, activations and arithmetic, SIMT kernels;
 *                head_dim 8, 16, 32 or 64). */
typedef struct {
  int patch_size;
  int in_channels;
  int out_channels;
  int num_mmdit_layers;
  int num_single_dit_layers;
  int attention_head_dim;
  int num_attention_heads;
  int joint_attention_dim;
  int pos_embed_max_size;
  int num_register_tokens;
  int timestep_channels;
  int ffn_inner;
  float ln_eps;
  int dtype;
} af_config;

typedef struct af_weights af_weights; /* device-resident weight pack (bf16) */
typedef struct af_scratch af_scratch; /* device work buffers + error word */

/* Fill *cfg with the page's defaults (patch 2, 4 -> 4 channels, 4 joint +
 * 32 single blocks, 12 heads x 256, joint_attention_dim 2048,
 * pos_embed_max_size 1024, 8 registers, 256 timestep channels, eps 1e-6),
 * dtype AF_DTYPE_BF16. */
af_status af_config_default(af_config* cfg);

/* Derived sizes: inner_dim D, FFN width F, position grid side G.
 * AF_ERR_INVALID_ARG if the configuration is malformed. */
af_status af_config_derive(const af_config* cfg, int* inner_dim, int* ffn_inner, int* grid_side);

/* ---- weight pack --------------------------------------------------------
 * One device allocation holding every parameter in cfg->dtype.  Tensors are
 * addressed by the diffusers-style names listed by af_weights_tensor_info
 * (e.g. "single_transformer_blocks.3.attn.to_q.weight"), each with the
 * nn.Linear layout [out, in].  Freshly created packs are zero-filled.
 * AF_ERR_UNSUPPORTED for shapes the kernels do not cover: for bf16 packs
 * D % 32, F % 128, joint_attention_dim % 8 or timestep_channels % 8 not 0,
 * D or timestep_channels above 4096, head_dim not in {8, 16, 32, 64, 256},
 * or p * p * in_channels above 64; for fp32 packs head_dim not in
 * {8, 16, 32, 64}. */
af_status af_weights_create(const af_config* cfg, int device, af_weights** out);
void af_weights_destroy(af_weights* w);
af_status af_weights_num_tensors(const af_weights* w, int* n);
/* name: written NUL-terminated into name[0..name_cap); shape: up to 2 dims
 * (ndim = 1 or 2). */
af_status af_weights_tensor_info(const af_weights* w, int id, char* name, size_t name_cap,
                                 int* ndim, int64_t shape[2]);
af_status af_weights_find(const af_weights* w, const char* name, int* id);
/* Copy one tensor (numel elements as listed) into the pack.  src_dtype:
 * AF_DTYPE_BF16 (uint16_t bit patterns) or AF_DTYPE_F32 (float); the values
 * are converted to the pack's dtype (fp32 -> bf16 rounds to nearest even).
 * src_is_device != 0: src is device memory on the pack's device, else host
 * memory.  Asynchronous on `stream` for device sources; host sources are
 * copied synchronously. */
af_status af_weights_set(af_weights* w, int id, const void* src, int src_is_device, int src_dtype, void* stream);
/* Copy one tensor out of the pack, in the pack's dtype (numel elements,
 * [out, in] row-major).  dst_is_device != 0: device memory on the pack's
 * device (asynchronous on `stream`), else host memory (synchronous). */
af_status af_weights_get(const af_weights* w, int id, void* dst, int dst_is_device, void* stream);
/* Fill every tensor of the pack with seeded synthetic values, on the device:
 * linear weights and biases ~N(0, std^2), the learned position table
 * ~N(0, 0.1^2) and the register tokens ~N(0, 0.02^2), the scales of their
 * random initialisation in [ARCH] §Patch Embedding and §Register Tokens.
 * Element j of tensor `name` takes lane j % 4 of the Philox4x32-10 block
 * j / 4 (Salmon et al., SC 2011) under key (seed mod 2^32, seed div 2^32)
 * and counter (block mod 2^32, block div 2^32, CRC-32(name), 0); the four
 * words become uniforms (x + 1/2) / 2^32 and the Box-Muller transform (in
 * fp64) turns pairs into normals; the stored value is float32(z * std),
 * rounded to bf16 (nearest even) in a bf16 pack.  Asynchronous on `stream`.
 * An 8-bit copy made by af_weights_quantize_fp8 is not refreshed. */
af_status af_weights_init_random(af_weights* w, uint64_t seed, float std, void* stream);
/* Total bytes of the pack (for reporting). */
af_status af_weights_bytes(const af_weights* w, size_t* bytes);

/* ---- scratch ------------------------------------------------------------
 * Work buffers for batches up to max_batch with at most max_img_tokens
 * image tokens ((H/p)*(W/p), so any latent shape, square or not, whose
 * patch grid has that many tokens fits) and at most max_text_len text
 * tokens (before the registers are prepended). */
af_status af_scratch_create(const af_weights* w, int max_batch, int max_img_tokens, int max_text_len,
                            af_scratch** out);
void af_scratch_destroy(af_scratch* s);
/* Synchronise `stream`, then read and clear the device error word.
 * Returns AF_ERR_TIMEOUT if a bounded device wait expired since the last
 * af_sync, AF_ERR_CUDA on a CUDA error, else AF_OK. */
af_status af_sync(af_scratch* s, void* stream);

/* ---- the forward path ---------------------------------------------------*/

/* Timestep embedding: temb[b] = W2 silu(W1 e(t_b) + b1) + b2 with e the
 * 256-channel sinusoid of 1000*t_b (cosines first).  [ARCH] §前向传播流程
 * (Timesteps -> TimestepEmbedding), §在 AuraFlowPipeline 中的实际调用 (the
 * model receives timestep/1000).
 *   t:    device float[B], model time in [0, 1] (1 = pure noise).
 *   temb: device float[B, D] (output). */
af_status af_timestep_embed(const af_weights* w, af_scratch* s, const float* t, int B, float* temb,
                            void* stream);

/* Same result as af_timestep_embed, for callers that cannot allocate device
 * memory (their device memory is owned and budgeted by another allocator,
 * they run a latency-critical loop where cudaMalloc/cudaFree may stall the
 * device, or they may only allocate at initialisation): no af_scratch is
 * needed and nothing is allocated.  The architecture description has no
 * counterpart of this call.  Its intermediates live in one fixed 256 KB
 * device array (65536 floats) that every GPU loading the library holds until
 * exit; a call needs B * (timestep_channels + inner_dim) floats of it and
 * larger requests return AF_ERR_SHAPE (text in af_last_error) before any
 * launch.  All calls on a device share that array and it keeps the last
 * call's contents (nothing in it needs to start at zero), so calls that
 * overlap on the GPU race and must be serialised by the caller.  The first
 * call on each device looks up the array's device address; make it before
 * any stream capture.
 *   t: device float[B]; temb: device float[B, D] (output). */
af_status af_timestep_embed_noalloc(const af_weights* w, const float* t, int B, float* temb, void* stream);
/* (AF_ERR_UNSUPPORTED for an fp32 pack; AF_ERR_INVALID_ARG when the current
 * device is not the pack's.) */

/* Patch embedding with centre-cropped learned positions ([ARCH] §Patch
 * Embedding): img[b, n] = W_pe patch(b, n) + PE[(r0 + n / wp) * G + c0 + n % wp]
 * with r0 = (G - H/p) / 2, c0 = (G - W/p) / 2 (floor); patch vector order
 * (row-in-patch, col-in-patch, channel); tokens row-major over the patch grid.
 *   latents:    device float[B, C_in, H, W].
 *   img_tokens: device bf16[B, (H/p)(W/p), D] (output).
 * AF_ERR_SHAPE if H or W is not a multiple of p or the patch grid exceeds
 * the G x G position grid ([PIPE] §AuraFlowPipeline 核心参数详解, the
 * resolution check). */
af_status af_patch_embed(const af_weights* w, af_scratch* s, const float* latents, int B, int H, int W,
                         uint16_t* img_tokens, void* stream);

/* One AuraFlowJointTransformerBlock ([ARCH] §联合注意力块, §注意力处理器与
 * QKV 融合), in place on both residual streams:
 *   per stream: adaLN-Zero (6 vectors from W silu(temb)), FP32 LayerNorm,
 *   bias-free Q/K/V with per-head LayerNorm on Q and K, joint attention over
 *   [text; image] (text first), gated output projection, gated SiLU FFN.
 *   img:  device bf16[B, Ni, D] in/out (image stream).
 *   txt:  device bf16[B, Nt, D] in/out (text stream incl. registers).
 *   temb: device float[B, D].
 *   layer in [0, num_mmdit_layers).
 *   text_len: NULL, or device int[B]: real prompt tokens of each sample
 *   (see "Padded prompts" below); text rows [num_register_tokens +
 *   text_len[b], Nt) are then masked as attention keys. */
af_status af_joint_block(const af_weights* w, af_scratch* s, int layer, uint16_t* img, uint16_t* txt,
                         const float* temb, int B, int Ni, int Nt, const int* text_len, void* stream);

/* One AuraFlowSingleTransformerBlock ([ARCH] §单 DiT 块) in place on the
 * concatenated sequence x = [text; image]:
 *   x: device bf16[B, N, D] in/out; temb: device float[B, D];
 *   layer in [0, num_single_dit_layers).
 *   Nt, text_len: the first Nt rows of x are the text stream (registers
 *   included); with text_len != NULL (device int[B]) rows
 *   [num_register_tokens + text_len[b], Nt) are masked as attention keys.
 *   Nt is ignored when text_len is NULL. */
af_status af_single_block(const af_weights* w, af_scratch* s, int layer, uint16_t* x, const float* temb,
                          int B, int N, int Nt, const int* text_len, void* stream);

/* The whole AuraFlowTransformer2DModel forward ([ARCH] §前向传播流程):
 * patch embed, timestep embed, context_embedder (bias-free 2048 -> D) with
 * the register tokens prepended, the joint blocks, concatenation
 * [text; image], the single blocks, the image slice, the pre-final
 * modulation x * (1 + scale) + shift, proj_out (bias-free) and unpatchify.
 *   latents:  device float[B, C_in, H, W]
 *   text_emb: device bf16[B, L, joint_attention_dim] (fp32 for an fp32 pack)
 *   t:        device float[B] (timestep / 1000)
 *   text_len: NULL (every text token is real, the model's own behaviour) or
 *             device int[B], see "Padded prompts"
 *   velocity: device float[B, C_out, H, W] (output)
 *
 * Padded prompts.  The pipeline pads every prompt of a batch to one length
 * and builds an attention mask ([PIPE] §AuraFlowPipeline 核心参数详解,
 * [ARCH] §在 AuraFlowPipeline 中的实际调用), but the transformer forward
 * itself takes no mask ([ARCH] §前向传播流程).  As an extension, text_len[b]
 * gives the real length of sample b's prompt: its last L - text_len[b] text
 * tokens then take no part as attention keys in any block (boolean key mask,
 * like an SDPA attn_mask); register tokens and image tokens always do.
 * Values are clamped to [0, L]. */
af_status af_transformer_forward(const af_weights* w, af_scratch* s, const float* latents,
                                 const void* text_emb, const float* t, int B, int H, int W, int L,
                                 const int* text_len, float* velocity, void* stream);

/* Classifier-free guidance combine and flow-match Euler step ([PIPE]
 * §AuraFlowPipeline 核心参数详解 (CFG formula), [ARCH] §在 AuraFlowPipeline
 * 中的实际调用 (uncond half first), [DEEP] §2.3 (FlowMatchEulerDiscreteScheduler)):
 *   v = v[uncond] + guidance (v[text] - v[uncond]);  x += (sigma_next - sigma) v
 *   latents:  device float[Bi, C, H, W] in/out
 *   velocity: device float[2 Bi, C, H, W], the uncond half first.
 * With guidance disabled pass the B = Bi velocity twice-concatenated or
 * guidance = 1 and any uncond half. */
af_status af_euler_cfg_step(float* latents, const float* velocity, int Bi, int C, int H, int W,
                            float guidance, float sigma, float sigma_next, void* stream);

/* ---- CFG split over two GPUs: the exchange fused into the update ---------
 * The CFG batch [uncond; text] is two independent forwards ([ARCH] §在
 * AuraFlowPipeline 中的实际调用), so two processes, one per GPU, can each run
 * one half.  Each writes its half of the velocity into an exchange buffer
 * that the other maps through CUDA IPC; af_euler_cfg_step2 then reads the
 * local half and the peer's half straight from the peer GPU's memory (plain
 * loads over NVLink) while it applies the guidance and the Euler step.
 *   af_exchange_create: a device buffer of `bytes` on `device` (zeroed).
 *   af_exchange_handle: its IPC handle (AF_IPC_HANDLE_BYTES opaque bytes), to
 *     be sent to the peer process by any host channel.
 *   af_exchange_open_peer: maps the peer's buffer (once per exchange).
 *   af_exchange_ptrs: device addresses of the local and the mapped peer
 *     buffer (peer NULL until opened).
 * Ordering is the caller's: launch the update only after both halves of the
 * step are complete on both GPUs (stream sync + host barrier), and do not
 * rewrite a buffer region while the peer may still read it (two slots,
 * alternating per step, need one barrier per step).  The current device must
 * be the exchange's device for handle / open. */
#define AF_IPC_HANDLE_BYTES 64
typedef struct af_exchange af_exchange;
af_status af_exchange_create(int device, size_t bytes, af_exchange** out);
af_status af_exchange_handle(const af_exchange* x, void* handle);
af_status af_exchange_open_peer(af_exchange* x, const void* peer_handle);
af_status af_exchange_ptrs(const af_exchange* x, void** local, void** peer);
void af_exchange_destroy(af_exchange* x);

/* af_euler_cfg_step with the two halves of the velocity given apart, so
 * either may be a mapped peer buffer ([PIPE] §AuraFlowPipeline 核心参数详解,
 * [DEEP] §2.3):  x += (sigma_next - sigma) (vu + guidance (vc - vu)).
 *   latents: device float[Bi, C, H, W] in/out; v_uncond, v_text: device (or
 *   peer-mapped) float[Bi, C, H, W].  Same arithmetic as af_euler_cfg_step. */
af_status af_euler_cfg_step2(float* latents, const float* v_uncond, const float* v_text, int Bi, int C, int H, int W,
                             float guidance, float sigma, float sigma_next, void* stream);

/* One step of the sampling loop ([ARCH] §在 AuraFlowPipeline 中的实际调用):
 * the latents are duplicated into a CFG batch [uncond; text], the forward
 * runs at model time t = sigma on the 2 Bi batch, and af_euler_cfg_step
 * updates the latents in place with sigma_next.
 *   latents:  device float[Bi, C_in, H, W] in/out
 *   text_emb: device bf16[2 Bi, L, joint_attention_dim], uncond rows first
 *             (fp32 for an fp32 pack).
 *   text_len: NULL or device int[2 Bi] (padded prompts, as for the forward).
 * Needs a scratch created with max_batch >= 2 Bi. */
af_status af_denoise_step(const af_weights* w, af_scratch* s, float* latents, const void* text_emb, int Bi,
                          int H, int W, int L, const int* text_len, float guidance, float sigma, float sigma_next,
                          void* stream);

/* ---- the sampling loop -----------------------------------------------------
 * The pipeline's denoising loop ([ARCH] §在 AuraFlowPipeline 中的实际调用,
 * [DEEP] §2.3: 25 flow-match Euler steps with CFG) as a reusable plan.  Every
 * adaLN-Zero and pre-final modulation depends only on the step's sigma, so
 * af_sampler_prepare computes them for all steps at once (one tensor-core
 * GEMM reading the modulation weights once); af_sampler_step then runs step
 * i exactly like af_denoise_step(sigma_i -> sigma_{i+1}) with those values.
 * With use_graphs != 0 each step is captured into a CUDA graph on first use
 * and replayed afterwards (needs a non-NULL stream; nothing may be captured
 * on the stream around these calls).
 *   latents:  device float[Bi, C, H, W], updated in place by every step
 *   text_emb: device bf16[2 Bi, L, joint_attention_dim] (uncond rows first;
 *             fp32 for an fp32 pack)
 *   text_len: NULL or device int[2 Bi] (padded prompts)
 *   sigmas:   host float[n_steps + 1] (e.g. from af_sigma_schedule)
 * The device buffers are bound to the sampler: change their contents, not
 * their addresses.  The scratch must fit a 2 Bi batch of this size. */
typedef struct af_sampler af_sampler;
af_status af_sampler_create(const af_weights* w, af_scratch* s, float* latents, const void* text_emb, int Bi,
                            int H, int W, int L, const int* text_len, int n_steps, const float* sigmas,
                            float guidance, int use_graphs, af_sampler** out);
af_status af_sampler_prepare(af_sampler* smp, void* stream);
af_status af_sampler_step(af_sampler* smp, int step, void* stream);
void af_sampler_destroy(af_sampler* smp);

/* ---- 8-bit variant ----------------------------------------------------------
 * The pipeline guide loads the transformer with 8-bit weights ([PIPE]
 * bitsandbytes sections).  This is the tensor-core form of that idea: every
 * projection of the blocks (fused QKV, output projection, FFN up pair, FFN
 * down) runs with e4m3 operands on tcgen05 kind::f8f6f4 MMAs, each
 * activation row (token) and each weight row (output channel) scaled by its
 * own fp32 factor amax / 448.  The LayerNorm+modulate kernel emits e4m3
 * directly; the attention output and the SwiGLU product are quantised per
 * token by a separate pass.  Attention, the LayerNorms, the modulations and
 * the embedding / output stages stay as in the bf16 path.
 *
 * af_weights_quantize_fp8(w, 1, stream) quantises the current bf16 values
 * of those weights into a second device pack (about a third of the bf16
 * pack) and switches every later forward, block and sampler step on `w` to
 * the 8-bit GEMMs; call it again after changing weights.  enable = 0 frees
 * the pack and returns to bf16.  Create samplers after switching. */
af_status af_weights_quantize_fp8(af_weights* w, int enable, void* stream);

/* Per-row e4m3 quantisation: for each row of x (device bf16 [rows, cols],
 * cols % 8 == 0) with a = max |x|: q = e4m3(x * (448 / a)) (round to nearest
 * even, saturating), scale = a / 448 (1 and zero codes for an all-zero row).
 *   q: device uint8 [rows, cols]; scale: device float [rows]. */
af_status af_quantize_rows_e4m3(const uint16_t* x, int rows, int cols, uint8_t* q, float* scale, void* stream);

/* af_ln_modulate with e4m3 output: y8 = per-row quantised LayerNorm+modulate
 * output (device uint8 [B*N, D]) and yscale its row scales (device float
 * [B*N]), with the rule of af_quantize_rows_e4m3. */
af_status af_ln_modulate_e4m3(const uint16_t* x, const float* shift, const float* scale, int mod_stride,
                              uint8_t* y8, float* yscale, int B, int N, int D, float eps, void* stream);

/* C[m, n] = a_scale[m] * w_scale[n] * sum_k A[m, k] W[n, k] with e4m3
 * operands on the tensor cores (fp32 accumulate, bf16 out).
 *   A: device uint8 [M, K]; W: device uint8 [N, K]; C: device bf16 [M, N];
 *   a_scale: device float [M]; w_scale: device float, readable for
 *   ceil(N / 256) * 256 entries.  K % 16 == 0, N % 8 == 0. */
af_status af_linear_fp8(const uint8_t* A, const float* a_scale, const uint8_t* W, const float* w_scale, uint16_t* C,
                        int M, int N, int K, void* stream);

/* Host-side sigma schedule of the flow-match Euler sampler ([DEEP] §2.3:
 * num_train_timesteps 1000, shift 1.73, 25 steps): n_steps + 1 values
 * sigma_i = k s_i / (1 + (k - 1) s_i) with s = linspace(1, 1/num_train,
 * n_steps), then a final 0.  The model time of step i is t_i = sigma_i.
 * out: host float[n_steps + 1].  No device work. */
af_status af_sigma_schedule(int n_steps, float shift, int num_train_timesteps, float* out);

/* ---- failure detection --------------------------------------------------
 * Every wait of the device code (mbarrier phases of the TMA / MMA / softmax
 * pipelines) is bounded: a wait that runs out records AF_ERR_TIMEOUT in the
 * scratch's error word, the kernel lets its in-flight copies and MMAs land
 * (bounded as well), frees its TMEM and returns, and the next af_sync
 * reports the timeout.  af_check_wait_timeout exercises that path without
 * any fault: one CTA takes 32 TMEM columns, waits on an mbarrier phase that
 * nothing completes, gives up after limit_ns nanoseconds (clamped to
 * [1 ms, 1 s]; the pipelines' own limit is 4 s), records the timeout in
 * s's error word, frees its TMEM and exits.  The next af_sync(s) then
 * returns AF_ERR_TIMEOUT and clears the word; the context stays usable.
 * Asynchronous on `stream`; AF_ERR_INVALID_ARG for a null scratch. */
af_status af_check_wait_timeout(af_scratch* s, int64_t limit_ns, void* stream);

/* ---- launch accounting and per-kernel-class timing ----------------------
 * Kernel classes: 0 tensor-core GEMM, 1 attention, 2 LayerNorm+modulate,
 * 3 other kernels (timestep/modulation GEMV, patch embed, output stage,
 * Euler/CFG).  af_launch_counts returns the number of this library's kernel
 * launches made through `s` since it was created (always counted).
 * Between af_profile_begin and af_profile_end, a CUDA event pair is
 * recorded around every launch; af_profile_end synchronises `stream` and
 * returns, per class, the summed device time (ms), the number of launches
 * and the algorithmic work (FLOPs for classes 0/1, bytes moved for 2/3). */
#define AF_NUM_KERNEL_CLASSES 4
af_status af_launch_counts(const af_scratch* s, int64_t counts[AF_NUM_KERNEL_CLASSES]);
af_status af_profile_begin(af_scratch* s);
af_status af_profile_end(af_scratch* s, void* stream, double ms[AF_NUM_KERNEL_CLASSES],
                         int64_t launches[AF_NUM_KERNEL_CLASSES], double work[AF_NUM_KERNEL_CLASSES]);

/* ---- building blocks (the kernels the forward is made of) --------------*/

/* y = LN(x) * (1 + scale[b]) + shift[b]: FP32 LayerNorm without affine
 * weights ([ARCH] §调制与归一化), then the adaLN modulation.
 *   x, y: device bf16[B*N, D];  shift, scale: device float, element (b, d)
 *   at shift[b * mod_stride + d]. */
af_status af_ln_modulate(const uint16_t* x, const float* shift, const float* scale, int mod_stride,
                         uint16_t* y, int B, int N, int D, float eps, void* stream);

/* C = A W^T on the tcgen05 tensor cores, bf16 in, fp32 accumulate, bf16 out.
 *   A: device bf16[M, K]; W: device bf16[N, K]; C: device bf16[M, N].
 *   K must be a multiple of 8 (16-byte rows for the TMA engine). */
af_status af_linear(const uint16_t* A, const uint16_t* W, uint16_t* C, int M, int N, int K, void* stream);

/* Two independent products C0 = A0 W0^T and C1 = A1 W1^T in one persistent
 * CTA-pair launch, the second problem's tiles after the first's: the form
 * the joint block gives its image- and text-stream projections ([ARCH]
 * §联合注意力块, one set of projections per stream).  Shapes, layout and
 * constraints as af_linear for each problem; when M0 + M1 < 1024 the two
 * products run as two af_linear launches. */
af_status af_linear_grouped(const uint16_t* A0, const uint16_t* W0, uint16_t* C0, int M0, int N0, int K0,
                            const uint16_t* A1, const uint16_t* W1, uint16_t* C1, int M1, int N1, int K1,
                            void* stream);

/* Non-causal softmax(q k^T / sqrt(hd)) v per (batch, head) ([ARCH]
 * §注意力处理器与 QKV 融合).
 *   q, k, v: device bf16[B, H, N, hd];  o: device bf16[B, N, H*hd].
 *   qk_normalized: nonzero promises that every q and k row has L2 norm at
 *   most sqrt(hd) (up to bf16 rounding), as the per-head LayerNorm (QK-norm)
 *   guarantees; the kernel then uses a fixed softmax shift instead of a
 *   running maximum.  Pass 0 for arbitrary inputs.
 *   key_len: NULL, or device int[B]: for sample b the keys
 *   [key_base + key_len[b], key_end) are masked (key_len[b] clamped to
 *   [0, key_end - key_base]); needs 1 <= key_base <= key_end <= N so that
 *   every row keeps at least one key. */
af_status af_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* o, int B,
                       int H, int N, int hd, int qk_normalized, const int* key_len, int key_base, int key_end,
                       void* stream);

const char* af_status_string(af_status st);
/* Text of the last CUDA error seen by this thread's calls ("" if none). */
const char* af_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* AF_H_ */
