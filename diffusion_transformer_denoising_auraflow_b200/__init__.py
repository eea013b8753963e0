"""Python binding of ``libaf.so``, the sm_100a AuraFlow denoising-forward library.

Argument marshalling only: every function below checks the dtypes, shapes
and devices of the torch tensors it is given (each must live on the weight
pack's device, which must also be the current device, since the kernels
launch there), passes ``data_ptr()`` and the current CUDA stream to the C ABI
declared in ``include/af.h`` and raises ``AFError`` on a non-OK status.
All computation happens in the library's CUDA kernels; there is no CPU or
PyTorch fallback, and importing this package fails if the library has not
been built.
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
        "num_register_tokens", "timestep_channels", "ffn_inner")] + [("ln_eps", ctypes.c_float),
                                                                      ("dtype", ctypes.c_int)]

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
    "af_weights_set": [_P, _I, _P, _I, _I, _P],
    "af_weights_get": [_P, _I, _P, _I, _P],
    "af_weights_init_random": [_P, ctypes.c_uint64, _F, _P],
    "af_weights_bytes": [_P, _P],
    "af_scratch_create": [_P, _I, _I, _I, _P],
    "af_scratch_destroy": [_P],
    "af_sync": [_P, _P],
    "af_check_wait_timeout": [_P, ctypes.c_int64, _P],
    "af_timestep_embed": [_P, _P, _P, _I, _P, _P],
    "af_timestep_embed_noalloc": [_P, _P, _I, _P, _P],
    "af_patch_embed": [_P, _P, _P, _I, _I, _I, _P, _P],
    "af_joint_block": [_P, _P, _I, _P, _P, _P, _I, _I, _I, _P, _P],
    "af_single_block": [_P, _P, _I, _P, _P, _I, _I, _I, _P, _P],
    "af_transformer_forward": [_P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P],
    "af_euler_cfg_step": [_P, _P, _I, _I, _I, _I, _F, _F, _F, _P],
    "af_euler_cfg_step2": [_P, _P, _P, _I, _I, _I, _I, _F, _F, _F, _P],
    "af_exchange_create": [_I, ctypes.c_size_t, _P],
    "af_exchange_handle": [_P, _P],
    "af_exchange_open_peer": [_P, _P],
    "af_exchange_ptrs": [_P, _P, _P],
    "af_exchange_destroy": [_P],
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
    "af_linear_grouped": [_P, _P, _P, _I, _I, _I, _P, _P, _P, _I, _I, _I, _P],
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
    L.af_exchange_destroy.restype = None
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


AF_ERR_INVALID_ARG = 1
AF_ERR_SHAPE = 2
AF_DTYPE_BF16 = 0
AF_DTYPE_F32 = 1


def device_mismatch(tensor_devices, current: int, pack_device: int):
    """Why a call may not launch, or None: every tensor (given by its device
    index) must live on the weight pack's device, and that device must be the
    current one, because the library launches on the current device."""
    for name, dev in tensor_devices:
        if dev != pack_device:
            return f"{name} is on cuda:{dev}, the weight pack on cuda:{pack_device}"
    if current != pack_device:
        return f"the current device is cuda:{current}, the weight pack's is cuda:{pack_device}"
    return None


class _Call:
    """Collects the device tensors of one call and checks, before the library
    is entered, that they and the current device match the weight pack's."""

    def __init__(self, where: str, w=None):
        self.where = where
        self.w = w
        self.devs = []

    def dev(self, t, dtype, name: str):
        p = _dev(t, dtype, name)
        self.devs.append((name, t.device.index))
        return p

    def rows(self, t, dtype, name: str, rows: int, row_stride: int, row_len: int):
        p = _dev_rows(t, dtype, name, rows, row_stride, row_len, self.where)
        self.devs.append((name, t.device.index))
        return p

    def lens(self, t, n: int, name: str):
        p = _lens(t, n, name)
        if t is not None:
            self.devs.append((name, t.device.index))
        return p

    def check(self):
        pack = self.w.device if self.w is not None else torch.cuda.current_device()
        why = device_mismatch(self.devs, torch.cuda.current_device(), pack)
        if why:
            raise AFError(AF_ERR_INVALID_ARG, self.where, why)


def _dev(t: torch.Tensor, dtype, name: str):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


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


def _act(w):
    """Activation dtype of a pack: bf16, or fp32 for an fp32 pack."""
    return torch.float32 if getattr(w.cfg, "dtype", AF_DTYPE_BF16) == AF_DTYPE_F32 else torch.bfloat16


class Weights:
    """Device-resident weight pack (af_weights), bf16 or fp32 (cfg.dtype)."""

    def __init__(self, cfg: Config, device: int = 0):
        self.cfg = cfg
        self.device = device
        h = ctypes.c_void_p()
        _check(lib.af_weights_create(ctypes.byref(cfg), device, ctypes.byref(h)), "af_weights_create")
        self.handle = h

    @property
    def dtype(self):
        """torch dtype of the stored tensors and of the activations the calls take."""
        return _act(self)

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

    def _info(self, name: str):
        idx = self.find(name)
        buf = ctypes.create_string_buffer(256)
        nd = ctypes.c_int()
        shp = (ctypes.c_int64 * 2)()
        _check(lib.af_weights_tensor_info(self.handle, idx, buf, 256, ctypes.byref(nd), shp), "af_weights_tensor_info")
        return idx, tuple(shp[: nd.value])

    def _check_current(self, where: str, tensor=None):
        c = _Call(where, self)
        if tensor is not None and tensor.is_cuda:
            c.devs.append(("tensor", tensor.device.index))
        c.check()

    def set(self, name: str, tensor: torch.Tensor, stream=None):
        """Copy a bf16 or fp32 tensor (host or device, contiguous, listed numel)
        into the pack, converted to the pack's dtype."""
        if tensor.dtype not in (torch.bfloat16, torch.float32) or not tensor.is_contiguous():
            raise TypeError("weights must be contiguous bfloat16 or float32")
        idx, shape = self._info(name)
        numel = 1
        for d in shape:
            numel *= d
        where = f"af_weights_set({name})"
        _need(tensor.numel() == numel, where, f"the pack holds {numel} elements, the tensor {tensor.numel()}")
        self._check_current(where, tensor)
        src_dtype = AF_DTYPE_F32 if tensor.dtype == torch.float32 else AF_DTYPE_BF16
        _check(lib.af_weights_set(self.handle, idx, ctypes.c_void_p(tensor.data_ptr()), 1 if tensor.is_cuda else 0,
                                  src_dtype, _stream(stream) if tensor.is_cuda else None), where)

    def get(self, name: str, stream=None) -> torch.Tensor:
        """A device copy of one tensor, in the pack's dtype and [out, in] layout."""
        idx, shape = self._info(name)
        where = f"af_weights_get({name})"
        self._check_current(where)
        out = torch.empty(shape, dtype=self.dtype, device=torch.device("cuda", self.device))
        _check(lib.af_weights_get(self.handle, idx, ctypes.c_void_p(out.data_ptr()), 1, _stream(stream)), where)
        return out

    def init_random(self, seed: int, std: float = 0.02, stream=None):
        """Fill every tensor with seeded synthetic values on the device (linear
        weights ~N(0, std^2), positions ~N(0, 0.1^2), registers ~N(0, 0.02^2))."""
        self._check_current("af_weights_init_random")
        _check(lib.af_weights_init_random(self.handle, int(seed) & (2 ** 64 - 1), float(std), _stream(stream)),
               "af_weights_init_random")

    def quantize_fp8(self, enable: bool = True, stream=None):
        """Switch every block projection to the 8-bit (e4m3) variant
        (re-quantising the current weights), or back to bf16."""
        self._check_current("af_weights_quantize_fp8")
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
        _Call("af_scratch_create", weights).check()
        h = ctypes.c_void_p()
        _check(lib.af_scratch_create(weights.handle, max_batch, max_img_tokens, max_text_len, ctypes.byref(h)),
               "af_scratch_create")
        self.handle = h

    def sync(self, stream=None):
        _check(lib.af_sync(self.handle, _stream(stream)), "af_sync")

    def check_wait_timeout(self, limit_ns=20_000_000, stream=None):
        """Run the device timeout path on purpose (af_check_wait_timeout): the
        next sync() raises AFError with AF_ERR_TIMEOUT."""
        _check(lib.af_check_wait_timeout(self.handle, int(limit_ns), _stream(stream)), "af_check_wait_timeout")

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
    where = "af_timestep_embed"
    _need_shape(temb, (t.numel(), _width(w)), "temb", where)
    c = _Call(where, w)
    args = (c.dev(t, torch.float32, "t"), t.numel(), c.dev(temb, torch.float32, "temb"))
    c.check()
    _check(lib.af_timestep_embed(w.handle, s.handle, args[0], args[1], args[2], _stream(stream)), where)


def timestep_embed_noalloc(w: Weights, t, temb, stream=None):
    """af_timestep_embed without a scratch handle: nothing is allocated (fixed device array)."""
    where = "af_timestep_embed_noalloc"
    _need_shape(temb, (t.numel(), _width(w)), "temb", where)
    c = _Call(where, w)
    tp, tm = c.dev(t, torch.float32, "t"), c.dev(temb, torch.float32, "temb")
    c.check()
    st = lib.af_timestep_embed_noalloc(w.handle, tp, t.numel(), tm, _stream(stream))
    if st != AF_OK:
        raise AFError(st, where, lib.af_last_error().decode())


def patch_embed(w: Weights, s: Scratch, latents, img, stream=None):
    where = "af_patch_embed"
    B, C, H, W = latents.shape
    p = w.cfg.patch_size
    _need(C == w.cfg.in_channels, where, f"latents must have {w.cfg.in_channels} channels, got {C}")
    if H % p == 0 and W % p == 0:   # otherwise the library rejects the latent size itself
        _need_shape(img, (B, (H // p) * (W // p), _width(w)), "img", where)
    c = _Call(where, w)
    lp, ip = c.dev(latents, torch.float32, "latents"), c.dev(img, torch.bfloat16, "img")
    c.check()
    _check(lib.af_patch_embed(w.handle, s.handle, lp, B, H, W, ip, _stream(stream)), where)


def joint_block(w: Weights, s: Scratch, layer: int, img, txt, temb, text_len=None, stream=None):
    """text_len: optional CUDA int32 [B], real prompt tokens (padded prompts)."""
    where = "af_joint_block"
    B, Ni = img.shape[:2]
    Nt = txt.shape[1]
    D = _width(w)
    _need_shape(img, (B, Ni, D), "img", where)
    _need_shape(txt, (B, Nt, D), "txt", where)
    _need_shape(temb, (B, D), "temb", where)
    c = _Call(where, w)
    ip, tp = c.dev(img, torch.bfloat16, "img"), c.dev(txt, torch.bfloat16, "txt")
    ep, lp = c.dev(temb, torch.float32, "temb"), c.lens(text_len, B, "text_len")
    c.check()
    _check(lib.af_joint_block(w.handle, s.handle, layer, ip, tp, ep, B, Ni, Nt, lp, _stream(stream)), where)


def single_block(w: Weights, s: Scratch, layer: int, x, temb, n_text: int = 0, text_len=None, stream=None):
    """x = [text; image] per sample; with text_len the first n_text rows are the text stream."""
    where = "af_single_block"
    B, N = x.shape[:2]
    D = _width(w)
    _need_shape(x, (B, N, D), "x", where)
    _need_shape(temb, (B, D), "temb", where)
    c = _Call(where, w)
    xp, ep = c.dev(x, torch.bfloat16, "x"), c.dev(temb, torch.float32, "temb")
    lp = c.lens(text_len, B, "text_len")
    c.check()
    _check(lib.af_single_block(w.handle, s.handle, layer, xp, ep, B, N, int(n_text), lp, _stream(stream)), where)


def transformer_forward(w: Weights, s: Scratch, latents, text_emb, t, velocity, text_len=None, stream=None):
    """text_emb: bf16 (fp32 for an fp32 pack) [B, L, joint_attention_dim]."""
    where = "af_transformer_forward"
    B, C, H, W = latents.shape
    L = text_emb.shape[1]
    _need(C == w.cfg.in_channels, where, f"latents must have {w.cfg.in_channels} channels, got {C}")
    _need_shape(text_emb, (B, L, w.cfg.joint_attention_dim), "text_emb", where)
    _need(t.numel() == B, where, f"t must hold {B} values, got {t.numel()}")
    _need_shape(velocity, (B, w.cfg.out_channels, H, W), "velocity", where)
    c = _Call(where, w)
    lp, ep = c.dev(latents, torch.float32, "latents"), c.dev(text_emb, _act(w), "text_emb")
    tp, lnp = c.dev(t, torch.float32, "t"), c.lens(text_len, B, "text_len")
    vp = c.dev(velocity, torch.float32, "velocity")
    c.check()
    _check(lib.af_transformer_forward(w.handle, s.handle, lp, ep, tp, B, H, W, L, lnp, vp, _stream(stream)), where)


def euler_cfg_step(latents, velocity, guidance: float, sigma: float, sigma_next: float, stream=None):
    where = "af_euler_cfg_step"
    Bi, C, H, W = latents.shape
    if velocity.shape[0] != 2 * Bi or tuple(velocity.shape[1:]) != (C, H, W):
        raise ValueError("velocity must be [2*Bi, C, H, W] (uncond half first)")
    c = _Call(where)
    lp, vp = c.dev(latents, torch.float32, "latents"), c.dev(velocity, torch.float32, "velocity")
    c.check()
    _check(lib.af_euler_cfg_step(lp, vp, Bi, C, H, W, float(guidance), float(sigma), float(sigma_next),
                                 _stream(stream)), where)


def denoise_step(w: Weights, s: Scratch, latents, text_emb, guidance: float, sigma: float, sigma_next: float,
                 stream=None, text_len=None):
    """One sampling step: CFG batch [uncond; text] forward at t = sigma, guidance, Euler to sigma_next."""
    where = "af_denoise_step"
    Bi, C, H, W = latents.shape
    if text_emb.shape[0] != 2 * Bi:
        raise ValueError("text_emb must hold 2*Bi rows (uncond first)")
    L = text_emb.shape[1]
    _need(C == w.cfg.in_channels, where, f"latents must have {w.cfg.in_channels} channels, got {C}")
    _need_shape(text_emb, (2 * Bi, L, w.cfg.joint_attention_dim), "text_emb", where)
    c = _Call(where, w)
    lp, ep = c.dev(latents, torch.float32, "latents"), c.dev(text_emb, _act(w), "text_emb")
    lnp = c.lens(text_len, 2 * Bi, "text_len")
    c.check()
    _check(lib.af_denoise_step(w.handle, s.handle, lp, ep, Bi, H, W, L, lnp, float(guidance), float(sigma),
                               float(sigma_next), _stream(stream)), where)


class Sampler:
    """The denoising loop as a plan (af_sampler): modulations of every step
    precomputed by prepare(), steps optionally replayed as CUDA graphs."""

    def __init__(self, w: Weights, s: Scratch, latents, text_emb, sigmas, guidance: float, use_graphs: bool = True,
                 text_len=None):
        where = "af_sampler_create"
        Bi, C, H, W = latents.shape
        L = text_emb.shape[1]
        if text_emb.shape[0] != 2 * Bi:
            raise ValueError("text_emb must hold 2*Bi rows (uncond first)")
        _need(C == w.cfg.in_channels, where, f"latents must have {w.cfg.in_channels} channels, got {C}")
        _need_shape(text_emb, (2 * Bi, L, w.cfg.joint_attention_dim), "text_emb", where)
        self.n_steps = len(sigmas) - 1
        sig = (ctypes.c_float * len(sigmas))(*[float(x) for x in sigmas])
        c = _Call(where, w)
        lp, ep = c.dev(latents, torch.float32, "latents"), c.dev(text_emb, _act(w), "text_emb")
        lnp = c.lens(text_len, 2 * Bi, "text_len")
        c.check()
        h = ctypes.c_void_p()
        _check(lib.af_sampler_create(w.handle, s.handle, lp, ep, Bi, H, W, L, lnp, self.n_steps, sig,
                                     float(guidance), 1 if use_graphs else 0, ctypes.byref(h)), where)
        self.handle = h
        self._w = w
        self._keep = (w, s, latents, text_emb, text_len)

    def prepare(self, stream=None):
        _Call("af_sampler_prepare", self._w).check()
        _check(lib.af_sampler_prepare(self.handle, _stream(stream)), "af_sampler_prepare")

    def step(self, i: int, stream=None):
        _Call("af_sampler_step", self._w).check()
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
    c = _Call(where)
    sh = c.rows(shift, torch.float32, "shift", B, mod_stride, D)
    sc = c.rows(scale, torch.float32, "scale", B, mod_stride, D)
    xp, yp = c.dev(x, torch.bfloat16, "x"), c.dev(y, torch.bfloat16, "y")
    c.check()
    _check(lib.af_ln_modulate(xp, sh, sc, mod_stride, yp, B, N, D, float(eps), _stream(stream)), where)


def linear(A, W, C, stream=None):
    where = "af_linear"
    M, K = A.shape
    N = W.shape[0]
    _need_shape(W, (N, K), "W", where)
    _need_shape(C, (M, N), "C", where)
    c = _Call(where)
    ap, wp, cp = c.dev(A, torch.bfloat16, "A"), c.dev(W, torch.bfloat16, "W"), c.dev(C, torch.bfloat16, "C")
    c.check()
    _check(lib.af_linear(ap, wp, cp, M, N, K, _stream(stream)), where)


def linear_grouped(A0, W0, C0, A1, W1, C1, stream=None):
    """C0 = A0 W0^T and C1 = A1 W1^T in one launch (af_linear_grouped)."""
    where = "af_linear_grouped"
    M0, K0 = A0.shape
    N0 = W0.shape[0]
    M1, K1 = A1.shape
    N1 = W1.shape[0]
    _need_shape(W0, (N0, K0), "W0", where)
    _need_shape(C0, (M0, N0), "C0", where)
    _need_shape(W1, (N1, K1), "W1", where)
    _need_shape(C1, (M1, N1), "C1", where)
    c = _Call(where)
    a0, w0, c0 = c.dev(A0, torch.bfloat16, "A0"), c.dev(W0, torch.bfloat16, "W0"), c.dev(C0, torch.bfloat16, "C0")
    a1, w1, c1 = c.dev(A1, torch.bfloat16, "A1"), c.dev(W1, torch.bfloat16, "W1"), c.dev(C1, torch.bfloat16, "C1")
    c.check()
    _check(lib.af_linear_grouped(a0, w0, c0, M0, N0, K0, a1, w1, c1, M1, N1, K1, _stream(stream)), where)


def attention(q, k, v, o, qk_normalized: bool = False, key_len=None, key_base: int = 0, key_end: int = 0,
              stream=None):
    """key_len: optional CUDA int32 [B]; keys [key_base + key_len[b], key_end) of sample b are masked."""
    where = "af_attention"
    B, H, N, hd = q.shape
    _need_shape(k, (B, H, N, hd), "k", where)
    _need_shape(v, (B, H, N, hd), "v", where)
    _need_shape(o, (B, N, H * hd), "o", where)
    c = _Call(where)
    qp, kp = c.dev(q, torch.bfloat16, "q"), c.dev(k, torch.bfloat16, "k")
    vp, op = c.dev(v, torch.bfloat16, "v"), c.dev(o, torch.bfloat16, "o")
    lp = c.lens(key_len, B, "key_len")
    c.check()
    _check(lib.af_attention(qp, kp, vp, op, B, H, N, hd, 1 if qk_normalized else 0, lp, int(key_base), int(key_end),
                            _stream(stream)), where)


def quantize_rows_e4m3(x, q, scale, stream=None):
    """Per-row e4m3 codes of bf16 x [rows, cols] into uint8 q and float scale [rows]."""
    where = "af_quantize_rows_e4m3"
    rows, cols = x.shape
    _need_shape(q, (rows, cols), "q", where)
    _need(scale.numel() >= rows, where, f"scale must hold {rows} values, got {scale.numel()}")
    c = _Call(where)
    xp, qp, sp = c.dev(x, torch.bfloat16, "x"), c.dev(q, torch.uint8, "q"), c.dev(scale, torch.float32, "scale")
    c.check()
    _check(lib.af_quantize_rows_e4m3(xp, rows, cols, qp, sp, _stream(stream)), where)


def ln_modulate_e4m3(x, shift, scale, mod_stride: int, y8, yscale, eps: float, stream=None):
    B, N, D = x.shape
    where = "af_ln_modulate_e4m3"
    _need(y8.numel() == B * N * D, where, f"y8 must hold {B * N * D} codes, got {y8.numel()}")
    _need(yscale.numel() >= B * N, where, f"yscale must hold {B * N} values, got {yscale.numel()}")
    c = _Call(where)
    sh = c.rows(shift, torch.float32, "shift", B, mod_stride, D)
    sc = c.rows(scale, torch.float32, "scale", B, mod_stride, D)
    xp, yp, ysp = c.dev(x, torch.bfloat16, "x"), c.dev(y8, torch.uint8, "y8"), c.dev(yscale, torch.float32, "yscale")
    c.check()
    _check(lib.af_ln_modulate_e4m3(xp, sh, sc, mod_stride, yp, ysp, B, N, D, float(eps), _stream(stream)), where)


def linear_fp8(A8, a_scale, W8, w_scale, C, stream=None):
    """C = diag(a_scale) (A8 W8^T) diag(w_scale) with e4m3 codes A8 [M, K], W8 [N, K]."""
    where = "af_linear_fp8"
    M, K = A8.shape
    N = W8.shape[0]
    if w_scale.numel() < (N + 255) // 256 * 256:
        raise ValueError("w_scale must hold ceil(N / 256) * 256 entries")
    _need_shape(W8, (N, K), "W8", where)
    _need_shape(C, (M, N), "C", where)
    _need(a_scale.numel() >= M, where, f"a_scale must hold {M} values, got {a_scale.numel()}")
    c = _Call(where)
    ap, asp = c.dev(A8, torch.uint8, "A8"), c.dev(a_scale, torch.float32, "a_scale")
    wp, wsp = c.dev(W8, torch.uint8, "W8"), c.dev(w_scale, torch.float32, "w_scale")
    cp = c.dev(C, torch.bfloat16, "C")
    c.check()
    _check(lib.af_linear_fp8(ap, asp, wp, wsp, cp, M, N, K, _stream(stream)), where)


AF_IPC_HANDLE_BYTES = 64


class _DeviceView:
    """A device buffer seen by torch through the CUDA array interface (no copy)."""

    def __init__(self, ptr: int, shape):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": "<f4", "data": (int(ptr), False),
                                         "version": 3, "strides": None}


class Exchange:
    """Velocity exchange buffer of the two-GPU CFG split (af_exchange): `slots`
    float32 tensors of `shape` that the peer process maps through CUDA IPC."""

    def __init__(self, shape, slots: int = 2, device: int | None = None):
        self.shape = tuple(int(x) for x in shape)
        self.slots = int(slots)
        self.device = torch.cuda.current_device() if device is None else int(device)
        self.numel = 1
        for d in self.shape:
            self.numel *= d
        h = ctypes.c_void_p()
        _check(lib.af_exchange_create(self.device, self.slots * self.numel * 4, ctypes.byref(h)), "af_exchange_create")
        self.handle_ptr = h
        self._local = None

    def _ptrs(self):
        lp, pp = ctypes.c_void_p(), ctypes.c_void_p()
        _check(lib.af_exchange_ptrs(self.handle_ptr, ctypes.byref(lp), ctypes.byref(pp)), "af_exchange_ptrs")
        return lp.value, pp.value

    def handle(self) -> bytes:
        """Opaque IPC handle of this buffer, to send to the peer process."""
        buf = ctypes.create_string_buffer(AF_IPC_HANDLE_BYTES)
        _check(lib.af_exchange_handle(self.handle_ptr, buf), "af_exchange_handle")
        return buf.raw

    def open_peer(self, handle: bytes):
        _check(lib.af_exchange_open_peer(self.handle_ptr, ctypes.create_string_buffer(bytes(handle),
                                                                                     AF_IPC_HANDLE_BYTES)),
               "af_exchange_open_peer")

    def local(self, slot: int) -> torch.Tensor:
        """Slot `slot` of this process's buffer as a torch tensor (a view)."""
        if self._local is None:
            lp, _ = self._ptrs()
            view = torch.as_tensor(_DeviceView(lp, (self.slots,) + self.shape), device=torch.device("cuda", self.device))
            self._local = view
        return self._local[slot]

    def peer(self, slot: int) -> int:
        """Device address of slot `slot` of the peer's mapped buffer."""
        _, pp = self._ptrs()
        if not pp:
            raise AFError(AF_ERR_INVALID_ARG, "Exchange.peer", "the peer buffer is not open")
        return pp + slot * self.numel * 4

    def synchronize(self):
        torch.cuda.current_stream().synchronize()

    def close(self):
        if self.handle_ptr:
            self._local = None
            lib.af_exchange_destroy(self.handle_ptr)
            self.handle_ptr = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def euler_cfg_step2(latents, v_uncond, v_text, guidance: float, sigma: float, sigma_next: float, stream=None):
    """Guidance + Euler with the two velocity halves apart; either half may be
    a torch tensor on this device or the int device address of a peer buffer
    (Exchange.peer) holding latents.numel() floats."""
    where = "af_euler_cfg_step2"
    Bi, C, H, W = latents.shape
    c = _Call(where)
    lp = c.dev(latents, torch.float32, "latents")
    ptrs = []
    for name, v in (("v_uncond", v_uncond), ("v_text", v_text)):
        if isinstance(v, int):
            ptrs.append(ctypes.c_void_p(v))
        else:
            _need(v.numel() == latents.numel(), where, f"{name} must hold {latents.numel()} values, got {v.numel()}")
            ptrs.append(c.dev(v, torch.float32, name))
    c.check()
    _check(lib.af_euler_cfg_step2(lp, ptrs[0], ptrs[1], Bi, C, H, W, float(guidance), float(sigma), float(sigma_next),
                                  _stream(stream)), where)
