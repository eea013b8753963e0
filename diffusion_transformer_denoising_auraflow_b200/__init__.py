"""Python binding of ``libaf.so``, the sm_100a AuraFlow denoising-forward library.

Argument marshalling only: every function below checks dtypes/devices of the
torch tensors it is given, passes ``data_ptr()`` and the current CUDA stream
to the C ABI declared in ``include/af.h`` and raises ``AFError`` on a non-OK
status.  All computation happens in the library's CUDA kernels; there is no
CPU or PyTorch fallback, and importing this package fails if the library has
not been built.
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libaf.so")

AF_OK = 0
STATUS = {0: "AF_OK", 1: "AF_ERR_INVALID_ARG", 2: "AF_ERR_SHAPE", 3: "AF_ERR_UNSUPPORTED",
          4: "AF_ERR_OOM", 5: "AF_ERR_CUDA", 6: "AF_ERR_TIMEOUT", 7: "AF_ERR_NOT_FOUND"}


class AFError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}" + (f" ({detail})" if detail else ""))


class Config(ctypes.Structure):
    """af_config (constructor parameters of AuraFlowTransformer2DModel)."""
    _fields_ = [(n, ctypes.c_int) for n in (
        "patch_size", "in_channels", "out_channels", "num_mmdit_layers", "num_single_dit_layers",
        "attention_head_dim", "num_attention_heads", "joint_attention_dim", "pos_embed_max_size",
        "num_register_tokens", "timestep_channels", "ffn_inner")] + [("ln_eps", ctypes.c_float)]

    @classmethod
    def default(cls, **overrides) -> "Config":
        c = cls()
        _check(lib.af_config_default(ctypes.byref(c)), "af_config_default")
        for k, v in overrides.items():
            setattr(c, k, v)
        return c

    def derived(self):
        d, f, g = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
        _check(lib.af_config_derive(ctypes.byref(self), ctypes.byref(d), ctypes.byref(f), ctypes.byref(g)),
               "af_config_derive")
        return d.value, f.value, g.value


_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float

_SIGS = {
    "af_config_default": [_P],
    "af_config_derive": [_P, _P, _P, _P],
    "af_weights_create": [_P, _I, _P],
    "af_weights_destroy": [_P],
    "af_weights_num_tensors": [_P, _P],
    "af_weights_tensor_info": [_P, _I, ctypes.c_char_p, ctypes.c_size_t, _P, _P],
    "af_weights_find": [_P, ctypes.c_char_p, _P],
    "af_weights_set": [_P, _I, _P, _I, _P],
    "af_weights_bytes": [_P, _P],
    "af_scratch_create": [_P, _I, _I, _I, _P],
    "af_scratch_destroy": [_P],
    "af_sync": [_P, _P],
    "af_timestep_embed": [_P, _P, _P, _I, _P, _P],
    "af_timestep_embed_noalloc": [_P, _P, _I, _P, _P],
    "af_patch_embed": [_P, _P, _P, _I, _I, _I, _P, _P],
    "af_joint_block": [_P, _P, _I, _P, _P, _P, _I, _I, _I, _P, _P],
    "af_single_block": [_P, _P, _I, _P, _P, _I, _I, _I, _P, _P],
    "af_transformer_forward": [_P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P],
    "af_euler_cfg_step": [_P, _P, _I, _I, _I, _I, _F, _F, _F, _P],
    "af_denoise_step": [_P, _P, _P, _P, _I, _I, _I, _I, _P, _F, _F, _F, _P],
    "af_sigma_schedule": [_I, _F, _I, _P],
    "af_sampler_create": [_P, _P, _P, _P, _I, _I, _I, _I, _P, _I, _P, _F, _I, _P],
    "af_sampler_prepare": [_P, _P],
    "af_sampler_step": [_P, _I, _P],
    "af_sampler_destroy": [_P],
    "af_launch_counts": [_P, _P],
    "af_profile_begin": [_P],
    "af_profile_end": [_P, _P, _P, _P, _P],
    "af_ln_modulate": [_P, _P, _P, _I, _P, _I, _I, _I, _F, _P],
    "af_linear": [_P, _P, _P, _I, _I, _I, _P],
    "af_attention": [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _I, _I, _P],
    "af_weights_quantize_fp8": [_P, _I, _P],
    "af_quantize_rows_e4m3": [_P, _I, _I, _P, _P, _P],
    "af_ln_modulate_e4m3": [_P, _P, _P, _I, _P, _P, _I, _I, _I, _F, _P],
    "af_linear_fp8": [_P, _P, _P, _P, _P, _I, _I, _I, _P],
    "af_status_string": [_I],
    "af_last_error": [],
}

EXPORTED = tuple(_SIGS)


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"{_LIB_PATH} is missing: build it with `python diffusion_transformer_denoising_auraflow_b200/build.py`")
    L = ctypes.CDLL(_LIB_PATH)
    for name, args in _SIGS.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = _I
    L.af_weights_destroy.restype = None
    L.af_scratch_destroy.restype = None
    L.af_sampler_destroy.restype = None
    L.af_status_string.restype = ctypes.c_char_p
    L.af_last_error.restype = ctypes.c_char_p
    return L


lib = _load()
LIB_PATH = _LIB_PATH


def _check(st: int, where: str):
    if st != AF_OK:
        detail = lib.af_last_error().decode() if st == 5 else ""
        raise AFError(st, where, detail)


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _lens(t, n: int, name: str):
    """Optional per-sample lengths: None, or a CUDA int32 tensor of n entries."""
    if t is None:
        return ctypes.c_void_p(0)
    if t.dim() != 1 or t.shape[0] != n:
        raise ValueError(f"{name} must hold {n} entries")
    return _dev(t, torch.int32, name)


def _dev(t: torch.Tensor, dtype, name: str):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


AF_ERR_SHAPE = 2


def _need(ok: bool, where: str, detail: str):
    """The library sees raw pointers only: a buffer whose size does not match
    the call is reported here, as the library reports its own shape errors,
    before anything is launched."""
    if not ok:
        raise AFError(AF_ERR_SHAPE, where, detail)


def _need_shape(t, shape, name: str, where: str):
    got = tuple(t.shape)
    _need(got == tuple(shape), where, f"{name} must have shape {tuple(shape)}, got {got}")


def _elems_from_start(t) -> int:
    """Elements of t's storage from t's first element on (a view may reach
    past its own shape into the storage it was cut from)."""
    return t.untyped_storage().nbytes() // t.element_size() - t.storage_offset()


def _dev_rows(t, dtype, name: str, rows: int, row_stride: int, row_len: int, where: str):
    """A CUDA tensor or strided view read as `rows` rows of `row_len`
    elements, `row_stride` elements apart, from its first element."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    need = (rows - 1) * row_stride + row_len if rows > 0 else 0
    avail = _elems_from_start(t)
    _need(need <= avail, where, f"{name} holds {avail} elements from its start, the call reads {need}")
    return ctypes.c_void_p(t.data_ptr())


def _width(w) -> int:
    return w.cfg.derived()[0]


class Weights:
    """Device-resident bf16 weight pack (af_weights)."""

    def __init__(self, cfg: Config, device: int = 0):
        self.cfg = cfg
        self.device = device
        h = ctypes.c_void_p()
        _check(lib.af_weights_create(ctypes.byref(cfg), device, ctypes.byref(h)), "af_weights_create")
        self.handle = h

    def tensors(self):
        n = ctypes.c_int()
        _check(lib.af_weights_num_tensors(self.handle, ctypes.byref(n)), "af_weights_num_tensors")
        out = []
        buf = ctypes.create_string_buffer(256)
        nd = ctypes.c_int()
        shp = (ctypes.c_int64 * 2)()
        for i in range(n.value):
            _check(lib.af_weights_tensor_info(self.handle, i, buf, 256, ctypes.byref(nd), shp),
                   "af_weights_tensor_info")
            out.append((buf.value.decode(), tuple(shp[: nd.value])))
        return out

    def find(self, name: str) -> int:
        i = ctypes.c_int()
        _check(lib.af_weights_find(self.handle, name.encode(), ctypes.byref(i)), f"af_weights_find({name})")
        return i.value

    def set(self, name: str, tensor: torch.Tensor, stream=None):
        """Copy a bf16 tensor (host or device, contiguous, listed numel) into the pack."""
        if tensor.dtype != torch.bfloat16 or not tensor.is_contiguous():
            raise TypeError("weights must be contiguous bfloat16")
        idx = self.find(name)
        buf = ctypes.create_string_buffer(256)
        nd = ctypes.c_int()
        shp = (ctypes.c_int64 * 2)()
        _check(lib.af_weights_tensor_info(self.handle, idx, buf, 256, ctypes.byref(nd), shp), "af_weights_tensor_info")
        numel = 1
        for d in shp[: nd.value]:
            numel *= d
        _need(tensor.numel() == numel, f"af_weights_set({name})",
              f"the pack holds {numel} elements, the tensor {tensor.numel()}")
        _check(lib.af_weights_set(self.handle, idx, ctypes.c_void_p(tensor.data_ptr()),
                                  1 if tensor.is_cuda else 0, _stream(stream) if tensor.is_cuda else None),
               f"af_weights_set({name})")

    def quantize_fp8(self, enable: bool = True, stream=None):
        """Switch every block projection to the 8-bit (e4m3) variant
        (re-quantising the current weights), or back to bf16."""
        _check(lib.af_weights_quantize_fp8(self.handle, 1 if enable else 0, _stream(stream)),
               "af_weights_quantize_fp8")

    def nbytes(self) -> int:
        b = ctypes.c_size_t()
        _check(lib.af_weights_bytes(self.handle, ctypes.byref(b)), "af_weights_bytes")
        return b.value

    def close(self):
        if self.handle:
            lib.af_weights_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class Scratch:
    """Device work buffers and the device error word (af_scratch)."""

    def __init__(self, weights: Weights, max_batch: int, max_img_tokens: int, max_text_len: int):
        self.weights = weights
        h = ctypes.c_void_p()
        _check(lib.af_scratch_create(weights.handle, max_batch, max_img_tokens, max_text_len, ctypes.byref(h)),
               "af_scratch_create")
        self.handle = h

    def sync(self, stream=None):
        _check(lib.af_sync(self.handle, _stream(stream)), "af_sync")

    def launch_counts(self):
        """Launches of this library's kernels through this scratch: [gemm, attention, ln, other]."""
        c = (ctypes.c_int64 * 4)()
        _check(lib.af_launch_counts(self.handle, c), "af_launch_counts")
        return list(c)

    def profile_begin(self):
        _check(lib.af_profile_begin(self.handle), "af_profile_begin")

    def profile_end(self, stream=None):
        """Per kernel class [gemm, attention, ln, other]: (device ms, launches, algorithmic work)."""
        ms = (ctypes.c_double * 4)()
        n = (ctypes.c_int64 * 4)()
        wk = (ctypes.c_double * 4)()
        _check(lib.af_profile_end(self.handle, _stream(stream), ms, n, wk), "af_profile_end")
        return list(ms), list(n), list(wk)

    def close(self):
        if self.handle:
            lib.af_scratch_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def timestep_embed(w: Weights, s: Scratch, t, temb, stream=None):
    _need_shape(temb, (t.numel(), _width(w)), "temb", "af_timestep_embed")
    _check(lib.af_timestep_embed(w.handle, s.handle, _dev(t, torch.float32, "t"), t.numel(),
                                 _dev(temb, torch.float32, "temb"), _stream(stream)), "af_timestep_embed")


def timestep_embed_noalloc(w: Weights, t, temb, stream=None):
    """af_timestep_embed without a scratch handle: nothing is allocated (fixed device array)."""
    _need_shape(temb, (t.numel(), _width(w)), "temb", "af_timestep_embed_noalloc")
    st = lib.af_timestep_embed_noalloc(w.handle, _dev(t, torch.float32, "t"), t.numel(),
                                       _dev(temb, torch.float32, "temb"), _stream(stream))
    if st != AF_OK:
        raise AFError(st, "af_timestep_embed_noalloc", lib.af_last_error().decode())


def patch_embed(w: Weights, s: Scratch, latents, img, stream=None):
    B, C, H, W = latents.shape
    p = w.cfg.patch_size
    _need(C == w.cfg.in_channels, "af_patch_embed", f"latents must have {w.cfg.in_channels} channels, got {C}")
    if H % p == 0 and W % p == 0:   # otherwise the library rejects the latent size itself
        _need_shape(img, (B, (H // p) * (W // p), _width(w)), "img", "af_patch_embed")
    _check(lib.af_patch_embed(w.handle, s.handle, _dev(latents, torch.float32, "latents"), B, H, W,
                              _dev(img, torch.bfloat16, "img"), _stream(stream)), "af_patch_embed")


def joint_block(w: Weights, s: Scratch, layer: int, img, txt, temb, text_len=None, stream=None):
    """text_len: optional CUDA int32 [B], real prompt tokens (padded prompts)."""
    B, Ni = img.shape[:2]
    Nt = txt.shape[1]
    D = _width(w)
    _need_shape(img, (B, Ni, D), "img", "af_joint_block")
    _need_shape(txt, (B, Nt, D), "txt", "af_joint_block")
    _need_shape(temb, (B, D), "temb", "af_joint_block")
    _check(lib.af_joint_block(w.handle, s.handle, layer, _dev(img, torch.bfloat16, "img"),
                              _dev(txt, torch.bfloat16, "txt"), _dev(temb, torch.float32, "temb"),
                              B, Ni, Nt, _lens(text_len, B, "text_len"), _stream(stream)), "af_joint_block")


def single_block(w: Weights, s: Scratch, layer: int, x, temb, n_text: int = 0, text_len=None, stream=None):
    """x = [text; image] per sample; with text_len the first n_text rows are the text stream."""
    B, N = x.shape[:2]
    D = _width(w)
    _need_shape(x, (B, N, D), "x", "af_single_block")
    _need_shape(temb, (B, D), "temb", "af_single_block")
    _check(lib.af_single_block(w.handle, s.handle, layer, _dev(x, torch.bfloat16, "x"),
                               _dev(temb, torch.float32, "temb"), B, N, int(n_text), _lens(text_len, B, "text_len"),
                               _stream(stream)), "af_single_block")


def transformer_forward(w: Weights, s: Scratch, latents, text_emb, t, velocity, text_len=None, stream=None):
    B, C, H, W = latents.shape
    L = text_emb.shape[1]
    where = "af_transformer_forward"
    _need(C == w.cfg.in_channels, where, f"latents must have {w.cfg.in_channels} channels, got {C}")
    _need_shape(text_emb, (B, L, w.cfg.joint_attention_dim), "text_emb", where)
    _need(t.numel() == B, where, f"t must hold {B} values, got {t.numel()}")
    _need_shape(velocity, (B, w.cfg.out_channels, H, W), "velocity", where)
    _check(lib.af_transformer_forward(w.handle, s.handle, _dev(latents, torch.float32, "latents"),
                                      _dev(text_emb, torch.bfloat16, "text_emb"), _dev(t, torch.float32, "t"),
                                      B, H, W, L, _lens(text_len, B, "text_len"),
                                      _dev(velocity, torch.float32, "velocity"), _stream(stream)),
           "af_transformer_forward")


def euler_cfg_step(latents, velocity, guidance: float, sigma: float, sigma_next: float, stream=None):
    Bi, C, H, W = latents.shape
    if velocity.shape[0] != 2 * Bi or tuple(velocity.shape[1:]) != (C, H, W):
        raise ValueError("velocity must be [2*Bi, C, H, W] (uncond half first)")
    _check(lib.af_euler_cfg_step(_dev(latents, torch.float32, "latents"), _dev(velocity, torch.float32, "velocity"),
                                 Bi, C, H, W, float(guidance), float(sigma), float(sigma_next), _stream(stream)),
           "af_euler_cfg_step")


def denoise_step(w: Weights, s: Scratch, latents, text_emb, guidance: float, sigma: float, sigma_next: float,
                 stream=None, text_len=None):
    """One sampling step: CFG batch [uncond; text] forward at t = sigma, guidance, Euler to sigma_next."""
    Bi, C, H, W = latents.shape
    if text_emb.shape[0] != 2 * Bi:
        raise ValueError("text_emb must hold 2*Bi rows (uncond first)")
    L = text_emb.shape[1]
    _need(C == w.cfg.in_channels, "af_denoise_step", f"latents must have {w.cfg.in_channels} channels, got {C}")
    _need_shape(text_emb, (2 * Bi, L, w.cfg.joint_attention_dim), "text_emb", "af_denoise_step")
    _check(lib.af_denoise_step(w.handle, s.handle, _dev(latents, torch.float32, "latents"),
                               _dev(text_emb, torch.bfloat16, "text_emb"), Bi, H, W, L,
                               _lens(text_len, 2 * Bi, "text_len"), float(guidance), float(sigma),
                               float(sigma_next), _stream(stream)), "af_denoise_step")


class Sampler:
    """The denoising loop as a plan (af_sampler): modulations of every step
    precomputed by prepare(), steps optionally replayed as CUDA graphs."""

    def __init__(self, w: Weights, s: Scratch, latents, text_emb, sigmas, guidance: float, use_graphs: bool = True,
                 text_len=None):
        Bi, C, H, W = latents.shape
        L = text_emb.shape[1]
        if text_emb.shape[0] != 2 * Bi:
            raise ValueError("text_emb must hold 2*Bi rows (uncond first)")
        _need(C == w.cfg.in_channels, "af_sampler_create", f"latents must have {w.cfg.in_channels} channels, got {C}")
        _need_shape(text_emb, (2 * Bi, L, w.cfg.joint_attention_dim), "text_emb", "af_sampler_create")
        self.n_steps = len(sigmas) - 1
        sig = (ctypes.c_float * len(sigmas))(*[float(x) for x in sigmas])
        h = ctypes.c_void_p()
        _check(lib.af_sampler_create(w.handle, s.handle, _dev(latents, torch.float32, "latents"),
                                     _dev(text_emb, torch.bfloat16, "text_emb"), Bi, H, W, L,
                                     _lens(text_len, 2 * Bi, "text_len"), self.n_steps, sig,
                                     float(guidance), 1 if use_graphs else 0, ctypes.byref(h)), "af_sampler_create")
        self.handle = h
        self._keep = (w, s, latents, text_emb, text_len)

    def prepare(self, stream=None):
        _check(lib.af_sampler_prepare(self.handle, _stream(stream)), "af_sampler_prepare")

    def step(self, i: int, stream=None):
        _check(lib.af_sampler_step(self.handle, int(i), _stream(stream)), "af_sampler_step")

    def close(self):
        if self.handle:
            lib.af_sampler_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def sigma_schedule(n_steps: int, shift: float = 1.73, num_train_timesteps: int = 1000):
    """Host-side shifted flow-match sigma schedule: list of n_steps + 1 floats ending in 0."""
    out = (ctypes.c_float * (n_steps + 1))()
    _check(lib.af_sigma_schedule(n_steps, float(shift), num_train_timesteps, out), "af_sigma_schedule")
    return list(out)


def ln_modulate(x, shift, scale, mod_stride: int, y, eps: float, stream=None):
    B, N, D = x.shape
    where = "af_ln_modulate"
    _need_shape(y, (B, N, D), "y", where)
    sh = _dev_rows(shift, torch.float32, "shift", B, mod_stride, D, where)
    sc = _dev_rows(scale, torch.float32, "scale", B, mod_stride, D, where)
    _check(lib.af_ln_modulate(_dev(x, torch.bfloat16, "x"), sh, sc, mod_stride, _dev(y, torch.bfloat16, "y"),
                              B, N, D, float(eps), _stream(stream)), "af_ln_modulate")


def linear(A, W, C, stream=None):
    M, K = A.shape
    N = W.shape[0]
    _need_shape(W, (N, K), "W", "af_linear")
    _need_shape(C, (M, N), "C", "af_linear")
    _check(lib.af_linear(_dev(A, torch.bfloat16, "A"), _dev(W, torch.bfloat16, "W"), _dev(C, torch.bfloat16, "C"),
                         M, N, K, _stream(stream)), "af_linear")


def attention(q, k, v, o, qk_normalized: bool = False, key_len=None, key_base: int = 0, key_end: int = 0,
              stream=None):
    """key_len: optional CUDA int32 [B]; keys [key_base + key_len[b], key_end) of sample b are masked."""
    B, H, N, hd = q.shape
    _need_shape(k, (B, H, N, hd), "k", "af_attention")
    _need_shape(v, (B, H, N, hd), "v", "af_attention")
    _need_shape(o, (B, N, H * hd), "o", "af_attention")
    _check(lib.af_attention(_dev(q, torch.bfloat16, "q"), _dev(k, torch.bfloat16, "k"), _dev(v, torch.bfloat16, "v"),
                            _dev(o, torch.bfloat16, "o"), B, H, N, hd, 1 if qk_normalized else 0,
                            _lens(key_len, B, "key_len"), int(key_base), int(key_end), _stream(stream)),
           "af_attention")


def quantize_rows_e4m3(x, q, scale, stream=None):
    """Per-row e4m3 codes of bf16 x [rows, cols] into uint8 q and float scale [rows]."""
    rows, cols = x.shape
    _need_shape(q, (rows, cols), "q", "af_quantize_rows_e4m3")
    _need(scale.numel() >= rows, "af_quantize_rows_e4m3", f"scale must hold {rows} values, got {scale.numel()}")
    _check(lib.af_quantize_rows_e4m3(_dev(x, torch.bfloat16, "x"), rows, cols, _dev(q, torch.uint8, "q"),
                                     _dev(scale, torch.float32, "scale"), _stream(stream)), "af_quantize_rows_e4m3")


def ln_modulate_e4m3(x, shift, scale, mod_stride: int, y8, yscale, eps: float, stream=None):
    B, N, D = x.shape
    where = "af_ln_modulate_e4m3"
    _need(y8.numel() == B * N * D, where, f"y8 must hold {B * N * D} codes, got {y8.numel()}")
    _need(yscale.numel() >= B * N, where, f"yscale must hold {B * N} values, got {yscale.numel()}")
    sh = _dev_rows(shift, torch.float32, "shift", B, mod_stride, D, where)
    sc = _dev_rows(scale, torch.float32, "scale", B, mod_stride, D, where)
    _check(lib.af_ln_modulate_e4m3(_dev(x, torch.bfloat16, "x"), sh, sc, mod_stride, _dev(y8, torch.uint8, "y8"),
                                   _dev(yscale, torch.float32, "yscale"), B, N, D, float(eps), _stream(stream)),
           "af_ln_modulate_e4m3")


def linear_fp8(A8, a_scale, W8, w_scale, C, stream=None):
    """C = diag(a_scale) (A8 W8^T) diag(w_scale) with e4m3 codes A8 [M, K], W8 [N, K]."""
    M, K = A8.shape
    N = W8.shape[0]
    if w_scale.numel() < (N + 255) // 256 * 256:
        raise ValueError("w_scale must hold ceil(N / 256) * 256 entries")
    _need_shape(W8, (N, K), "W8", "af_linear_fp8")
    _need_shape(C, (M, N), "C", "af_linear_fp8")
    _need(a_scale.numel() >= M, "af_linear_fp8", f"a_scale must hold {M} values, got {a_scale.numel()}")
    _check(lib.af_linear_fp8(_dev(A8, torch.uint8, "A8"), _dev(a_scale, torch.float32, "a_scale"),
                             _dev(W8, torch.uint8, "W8"), _dev(w_scale, torch.float32, "w_scale"),
                             _dev(C, torch.bfloat16, "C"), M, N, K, _stream(stream)), "af_linear_fp8")
