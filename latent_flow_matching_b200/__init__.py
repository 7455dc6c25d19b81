"""Python binding of libfluxdit.so, the sm_100a FLUX.2-klein / FLUX.3 Image Klein transformer library.

Argument marshalling only: every function forwards device pointers of torch
tensors (PyTorch owns the memory and the stream) to the C ABI declared in
``include/fluxdit.h``.  All computation happens in the library's CUDA kernels;
there is no CPU or PyTorch fallback.  Importing works without a GPU; calling a
compute function without the built library raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfluxdit.so")

FLUX_OK, FLUX_EIO, FLUX_ENOMEM, FLUX_EINVAL = 0, -5, -12, -22

EPI_BF16_BIAS, EPI_F32_BIAS, EPI_SWIGLU, EPI_RESID_GATE = 0, 1, 2, 3
PRECISION_BF16, PRECISION_FP8, PRECISION_NVFP4 = 0, 1, 2


class FluxConfig(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("n_double", "n_single", "hidden", "heads", "head_dim",
                                            "mlp_hidden", "in_ch", "txt_dim", "t_freq_dim")] + \
               [(n, ctypes.c_float) for n in ("rope_theta", "eps_ln", "eps_rms")]

    @classmethod
    def from_dims(cls, d):
        return cls(*(getattr(d, f) for f, _ in cls._fields_))


class Flux3Config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("n_mode", "n_joint", "hidden", "heads", "head_dim", "mlp_hidden",
                                            "in_ch", "txt_dim", "t_freq_dim", "flow_map")] + \
               [(n, ctypes.c_float) for n in ("rope_theta", "eps_ln", "eps_rms")]

    @classmethod
    def from_dims(cls, d):
        return cls(*(int(getattr(d, f)) if t is ctypes.c_int else getattr(d, f) for f, t in cls._fields_))


class FluxError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"fluxdit error {code}: {msg}")
        self.code = code


class FluxShapeError(FluxError, ValueError):
    """A buffer whose shape, size or dtype does not fit the call (found before anything is launched;
    code FLUX_EINVAL, like the library's own argument checks)."""

    def __init__(self, msg):
        super().__init__(FLUX_EINVAL, msg)


_P, _I, _F, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_SIGS = {
    "flux_get_error": (ctypes.c_char_p, []),
    "flux_get_error_code": (_I, []),
    "flux_blob_expected_bytes": (_Z, [ctypes.POINTER(FluxConfig)]),
    "flux_dit_create": (_P, [_P, _Z, ctypes.POINTER(FluxConfig), _P]),
    "flux_dit_destroy": (None, [_P]),
    "flux_dit_forward": (_I, [_P, _P, _I, _I, _P, _I, _P, _I, _I, _F, _P, _P]),
    "flux_dit_forward_refs": (_I, [_P, _P, _I, _I, _P, _I, _P, _I, ctypes.POINTER(ctypes.c_int), _F, _P, _P]),
    "flux_dit_forward_cfg": (_I, [_P, _P, _I, _I, _P, _P, _I, _P, _I, ctypes.POINTER(ctypes.c_int), _F, _P, _P,
                                  _P]),
    "flux_cfg_euler_step": (_I, [_P, _P, _P, _Z, _F, _F, _P]),
    "flux_cfg_euler_step_out": (_I, [_P, _P, _P, _P, _Z, _F, _F, _P]),
    "flux_selftest_bounded_wait": (_I, [ctypes.c_ulonglong, _I, _P]),
    "flux_test_fail_alloc_after": (None, [ctypes.c_longlong]),
    "flux_blend_latents": (_I, [_P, _P, _F, _P, _Z, _P]),
    "flux_dit_set_active_blocks": (_I, [_P, _I, _I]),
    "flux_dit_modulation_size": (_Z, [_P]),
    "flux_dit_modulation": (_I, [_P, _F, _P, _P]),
    "flux_euler_step": (_I, [_P, _P, _Z, _F, _P]),
    "flux_pack_latents": (_I, [_P, _P, _I, _I, _P]),
    "flux_unpack_latents": (_I, [_P, _P, _I, _I, _P]),
    "flux_joint_attention": (_I, [_P, _P, _P, _P, _I, _I, _I, _F, _P]),
    "flux_joint_attention_batch": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _F, _P]),
    "flux_linear": (_I, [_P, _I, _I, _I, _P, _I, _P, _I, _P, _I, _P, _P]),
    "flux_qkv_projection": (_I, [_P, _I, _I, _I, _P, _P, _I, _P, _P, _P, _I, _F, _P, _P]),
    "flux_layernorm_modulate": (_I, [_P, _P, _I, _I, _P, _P, _F, _P]),
    "flux_rope_table": (_I, [_P, _I, _I, _I, _I, _I, _F, _P]),
    "flux_qk_rmsnorm_rope": (_I, [_P, _I, _I, _I, _I, _P, _P, _P, _F, _P]),
    "flux_dit_profile": (_I, [_P, _I]),
    "flux_dit_profile_read": (_I, [_P, _I, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double),
                                   ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_longlong)]),
    "flux_kernel_launches": (ctypes.c_ulonglong, []),
    "flux_timestep_modulation_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _F, _P, _P]),
    "flux_device_error": (_I, [_P]),
    "flux3_blob_expected_bytes": (_Z, [ctypes.POINTER(Flux3Config)]),
    "flux3_dit_create": (_P, [_P, _Z, ctypes.POINTER(Flux3Config), _P]),
    "flux3_dit_destroy": (None, [_P]),
    "flux3_dit_forward": (_I, [_P, _P, _I, _I, _P, _I, _P, _I, ctypes.POINTER(ctypes.c_int), _F, _F, _P, _P]),
    "flux3_dit_forward_cfg": (_I, [_P, _P, _I, _I, _P, _P, _I, _P, _I, ctypes.POINTER(ctypes.c_int), _F, _F, _P,
                                   _P, _P]),
    "flux3_dit_set_active_blocks": (_I, [_P, _I, _I]),
    "flux3_dit_set_precision": (_I, [_P, _I]),
    "flux3_dit_modulation_size": (_Z, [_P]),
    "flux3_dit_modulation": (_I, [_P, _F, _F, _P, _P]),
    "flux3_dit_profile": (_I, [_P, _I]),
    "flux3_dit_profile_read": (_I, [_P, _I, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double),
                                    ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_longlong)]),
    "flux_joint_attention_segments": (_I, [_P, _P, _P, _P, _I, ctypes.POINTER(ctypes.c_int), _I, _I, _F, _P]),
    "flux_dit_set_precision": (_I, [_P, _I]),
    "flux_dit_prepare_timesteps": (_I, [_P, ctypes.POINTER(ctypes.c_float), _I, _P]),
    "flux_quantize_rows_e4m3": (_I, [_P, _I, _I, _I, _P, _I, _P, _P]),
    "flux_layernorm_modulate_fp8": (_I, [_P, _P, _P, _I, _I, _P, _P, _F, _P]),
    "flux_linear_fp8": (_I, [_P, _P, _I, _I, _I, _P, _P, _I, _P, _I, _P, _I, _P, _P]),
    "flux_nvfp4_scale_bytes": (_Z, [_I, _I]),
    "flux_quantize_rows_nvfp4": (_I, [_P, _I, _I, _I, _P, _I, _P, _P, _P]),
    "flux_linear_nvfp4": (_I, [_P, _P, _P, _I, _I, _I, _P, _P, _P, _I, _P, _I, _P, _I, _P, _P]),
    "flux_layernorm_modulate_nvfp4": (_I, [_P, _P, _P, _P, _I, _I, _P, _P, _F, _P]),
}
EXPORTED = tuple(_SIGS)

_lib = None


def lib():
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m latent_flow_matching_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def get_error() -> str:
    return lib().flux_get_error().decode()


def _check(rc):
    if rc != FLUX_OK:
        raise FluxError(rc, get_error())


def _stream(stream):
    if stream is not None:
        return ctypes.c_void_p(stream if isinstance(stream, int) else stream.cuda_stream)
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t, dtype=None, what="tensor"):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{what} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{what} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _bits(t, what):
    """bf16 tensors are passed as their raw 16-bit patterns."""
    import torch
    if t.dtype not in (torch.bfloat16, torch.uint16, torch.int16):
        raise ValueError(f"{what} must be bf16")
    return _ptr(t, None, what)


# Size checks: the C ABI takes plain pointers, so the binding checks every buffer against the
# sizes the call will touch before anything is launched (a short buffer would be read or written
# past its end on the device).
def _need_numel(t, n, what):
    if t is not None and t.numel() < n:
        raise FluxShapeError(f"{what} holds {t.numel()} elements; the call needs {n}")


def _need_same(t, ref, what):
    if t is None or tuple(t.shape) != tuple(ref.shape):
        raise FluxShapeError(f"{what} must have shape {tuple(ref.shape)}")


def _need_rows_cols(t, rows, cols, what):
    if t.dim() != 2 or t.shape[0] < rows or t.shape[1] < cols or t.stride(1) != 1:
        raise FluxShapeError(f"{what} must be 2-D with at least [{rows}, {cols}] and unit column stride, "
                         f"got {tuple(t.shape)}")


def _need_linear_out(out, gate, m, n, mode):
    import torch
    if mode not in (EPI_BF16_BIAS, EPI_F32_BIAS, EPI_SWIGLU, EPI_RESID_GATE):
        return                                  # the library rejects it
    bf = mode in (EPI_BF16_BIAS, EPI_SWIGLU)
    if bf and out.dtype not in (torch.bfloat16, torch.uint16, torch.int16):
        raise FluxShapeError("out must be bf16 for this mode")
    if not bf and out.dtype != torch.float32:
        raise FluxShapeError("out must be float32 for this mode")
    _need_rows_cols(out, m, n // 2 if mode == EPI_SWIGLU else n, "out")
    if mode == EPI_RESID_GATE:
        if gate is None:
            raise FluxShapeError("the gated residual mode needs gate")
        _need_numel(gate, n, "gate")


def _check_strided(t, kind, what):
    """A 2-D buffer whose rows may be strided (unit column stride); kind "bf16", "u8" or None
    (dtype checked elsewhere)."""
    import torch
    kinds = {"bf16": (torch.bfloat16, torch.uint16, torch.int16), "u8": (torch.uint8, torch.float8_e4m3fn)}
    if t.dim() != 2 or t.stride(1) != 1:
        raise FluxShapeError(f"{what} must be 2-D with unit column stride")
    if kind is not None and t.dtype not in kinds[kind]:
        raise FluxShapeError(f"{what} must be {kind}, got {t.dtype}")


def _strided(t, kind, what):
    """_check_strided, then the device pointer."""
    _check_strided(t, kind, what)
    if not t.is_cuda:
        raise ValueError(f"{what} must be a CUDA tensor")
    return ctypes.c_void_p(t.data_ptr())


def _need_tokens(t, rows, what, width=128):
    if t is None or t.numel() != rows * width:
        raise FluxShapeError(f"{what} must hold {rows} x {width} values")


def flux_blob_expected_bytes(dims) -> int:
    cfg = FluxConfig.from_dims(dims)
    return lib().flux_blob_expected_bytes(ctypes.byref(cfg))


def _check_forward_shapes(dims, img_tok, grid_hw, txts, hw_list, ref_tok, outs):
    """Token buffers of a forward: image tokens and every output [gh*gw, 128], each text
    [n_txt, txt_dim] (txt_dim checked when the model's dims are known), references [sum h*w, 128]."""
    n_img = int(grid_hw[0]) * int(grid_hw[1])
    _need_tokens(img_tok, n_img, "img_tok")
    for o in outs:
        _need_tokens(o, n_img, "velocity output")
    for txt in txts:
        if txt is not None and (txt.dim() != 2 or (dims is not None and txt.shape[1] != dims.txt_dim)):
            raise FluxShapeError("txt must be [n_txt, txt_dim]")
    n_ref = sum(int(h) * int(w) for h, w in hw_list)
    if n_ref:
        _need_tokens(ref_tok, n_ref, "ref_tok")


class FluxDiT:
    """A model created from a weight blob (host bytes); see flux_dit_create."""

    def __init__(self, blob: np.ndarray, dims=None, stream=None):
        blob = np.ascontiguousarray(blob)
        cfg = ctypes.byref(FluxConfig.from_dims(dims)) if dims is not None else None
        h = lib().flux_dit_create(ctypes.c_void_p(blob.ctypes.data), blob.nbytes, cfg, _stream(stream))
        if not h:
            raise FluxError(lib().flux_get_error_code() or FLUX_EINVAL, get_error())
        self._h = ctypes.c_void_p(h)
        self.dims = dims

    def close(self):
        if getattr(self, "_h", None):
            lib().flux_dit_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def forward(self, img_tok, grid_hw, txt, t, v_out, ref_tok=None, ref_hw=(0, 0), stream=None):
        """One forward.  ref_hw is one (h, w) or a list of them (then ref_tok holds every
        reference's packed tokens, concatenated in order)."""
        import torch
        n_txt = 0 if txt is None else txt.shape[0]
        hw_list = list(ref_hw) if ref_hw and isinstance(ref_hw[0], (tuple, list)) else \
            ([tuple(ref_hw)] if ref_hw and ref_hw[0] else [])
        self._check_shapes(img_tok, grid_hw, [txt], hw_list, ref_tok, [v_out])
        if ref_hw and isinstance(ref_hw[0], (tuple, list)):
            grids = (ctypes.c_int * (2 * len(ref_hw)))(*[v for hw in ref_hw for v in hw])
            _check(lib().flux_dit_forward_refs(self._h, _ptr(img_tok, torch.float32, "img_tok"), grid_hw[0],
                                               grid_hw[1], _ptr(txt, torch.float32, "txt"), n_txt,
                                               _ptr(ref_tok, torch.float32, "ref_tok"), len(ref_hw), grids,
                                               float(t), _ptr(v_out, torch.float32, "v_out"), _stream(stream)))
            return v_out
        _check(lib().flux_dit_forward(self._h, _ptr(img_tok, torch.float32, "img_tok"), grid_hw[0], grid_hw[1],
                                      _ptr(txt, torch.float32, "txt"), n_txt,
                                      _ptr(ref_tok, torch.float32, "ref_tok"), ref_hw[0], ref_hw[1],
                                      float(t), _ptr(v_out, torch.float32, "v_out"), _stream(stream)))
        return v_out

    def forward_cfg(self, img_tok, grid_hw, txt_cond, txt_uncond, t, v_cond, v_uncond, ref_tok=None, ref_hw=(),
                    stream=None):
        """Velocities for the prompt and the unconditional text in one batch-2 forward.
        ref_hw: a list of (h, w) (ref_tok holds every reference's packed tokens), or ()."""
        import torch
        n_txt = 0 if txt_cond is None else txt_cond.shape[0]
        if (0 if txt_uncond is None else txt_uncond.shape[0]) != n_txt:
            raise ValueError("txt_cond and txt_uncond must have the same token count")
        if ref_hw and not isinstance(ref_hw[0], (tuple, list)):
            ref_hw = [tuple(ref_hw)] if ref_hw[0] else []
        self._check_shapes(img_tok, grid_hw, [txt_cond, txt_uncond], list(ref_hw), ref_tok, [v_cond, v_uncond])
        grids = (ctypes.c_int * max(1, 2 * len(ref_hw)))(*[v for hw in ref_hw for v in hw])
        _check(lib().flux_dit_forward_cfg(self._h, _ptr(img_tok, torch.float32, "img_tok"), grid_hw[0], grid_hw[1],
                                          _ptr(txt_cond, torch.float32, "txt_cond"),
                                          _ptr(txt_uncond, torch.float32, "txt_uncond"), n_txt,
                                          _ptr(ref_tok, torch.float32, "ref_tok"), len(ref_hw), grids, float(t),
                                          _ptr(v_cond, torch.float32, "v_cond"),
                                          _ptr(v_uncond, torch.float32, "v_uncond"), _stream(stream)))
        return v_cond, v_uncond

    def _check_shapes(self, img_tok, grid_hw, txts, hw_list, ref_tok, outs):
        _check_forward_shapes(self.dims, img_tok, grid_hw, txts, hw_list, ref_tok, outs)

    def set_active_blocks(self, n_double=-1, n_single=-1):
        _check(lib().flux_dit_set_active_blocks(self._h, n_double, n_single))

    def set_precision(self, precision):
        """PRECISION_BF16, PRECISION_FP8 (row-wise e4m3) or PRECISION_NVFP4 (e2m1 with block scales) block
        linears; see flux_dit_set_precision."""
        _check(lib().flux_dit_set_precision(self._h, int(precision)))

    def prepare_timesteps(self, ts, stream=None):
        """Compute and keep the modulation vectors of these timesteps (see flux_dit_prepare_timesteps)."""
        arr = (ctypes.c_float * max(1, len(ts)))(*[float(t) for t in ts])
        _check(lib().flux_dit_prepare_timesteps(self._h, arr, len(ts), _stream(stream)))

    PROFILE_KINDS = ("gemm", "attention", "ln_mod", "qk_norm_rope", "gemv", "other")

    def profile(self, enable: bool):
        _check(lib().flux_dit_profile(self._h, 1 if enable else 0))

    def profile_read(self):
        """{kind: (ms, flops, bytes, launches)} accumulated since profile(True)."""
        out = {}
        for i, name in enumerate(self.PROFILE_KINDS):
            ms, fl, by, n = ctypes.c_double(), ctypes.c_double(), ctypes.c_double(), ctypes.c_longlong()
            _check(lib().flux_dit_profile_read(self._h, i, ctypes.byref(ms), ctypes.byref(fl), ctypes.byref(by),
                                               ctypes.byref(n)))
            out[name] = (ms.value, fl.value, by.value, n.value)
        return out

    def modulation_size(self) -> int:
        return lib().flux_dit_modulation_size(self._h)

    def modulation(self, t, out, stream=None):
        import torch
        _need_numel(out, self.modulation_size(), "out")
        _check(lib().flux_dit_modulation(self._h, float(t), _ptr(out, torch.float32, "mods"), _stream(stream)))
        return out


def flux3_blob_expected_bytes(dims) -> int:
    cfg = Flux3Config.from_dims(dims)
    return lib().flux3_blob_expected_bytes(ctypes.byref(cfg))


def _grids(ref_hw):
    """ref_hw: (), one (h, w), or a list of (h, w) -> (count, ctypes int array)."""
    if ref_hw and not isinstance(ref_hw[0], (tuple, list)):
        ref_hw = [tuple(ref_hw)] if ref_hw[0] else []
    ref_hw = list(ref_hw or [])
    return len(ref_hw), (ctypes.c_int * max(1, 2 * len(ref_hw)))(*[v for hw in ref_hw for v in hw])


class Flux3DiT:
    """A FLUX.3 Image Klein model created from a FLUX3DT weight blob (host bytes); see flux3_dit_create."""

    PROFILE_KINDS = FluxDiT.PROFILE_KINDS

    def __init__(self, blob: np.ndarray, dims=None, stream=None):
        blob = np.ascontiguousarray(blob)
        cfg = ctypes.byref(Flux3Config.from_dims(dims)) if dims is not None else None
        h = lib().flux3_dit_create(ctypes.c_void_p(blob.ctypes.data), blob.nbytes, cfg, _stream(stream))
        if not h:
            raise FluxError(lib().flux_get_error_code() or FLUX_EINVAL, get_error())
        self._h = ctypes.c_void_p(h)
        self.dims = dims
        self.flow_map = bool(dims.flow_map) if dims is not None else True

    def close(self):
        if getattr(self, "_h", None):
            lib().flux3_dit_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def forward(self, img_tok, grid_hw, txt, t, v_out, ref_tok=None, ref_hw=(), t_target=0.0, stream=None):
        """One forward.  ref_hw: (), one (h, w) or a list of them (ref_tok then holds every
        reference's packed tokens in order).  t_target: the step's target time (flow-map model)."""
        import torch
        n_txt = 0 if txt is None else txt.shape[0]
        n_refs, grids = _grids(ref_hw)
        _check_forward_shapes(self.dims, img_tok, grid_hw, [txt], list(zip(grids[0::2], grids[1::2]))[:n_refs],
                              ref_tok, [v_out])
        _check(lib().flux3_dit_forward(self._h, _ptr(img_tok, torch.float32, "img_tok"), grid_hw[0], grid_hw[1],
                                       _ptr(txt, torch.float32, "txt"), n_txt,
                                       _ptr(ref_tok, torch.float32, "ref_tok"), n_refs, grids, float(t),
                                       float(t_target), _ptr(v_out, torch.float32, "v_out"), _stream(stream)))
        return v_out

    def forward_cfg(self, img_tok, grid_hw, txt_cond, txt_uncond, t, v_cond, v_uncond, ref_tok=None, ref_hw=(),
                    t_target=0.0, stream=None):
        """Velocities for the prompt and the unconditional text in one batch-2 forward (the
        per-mode image and reference streams are computed once); see flux3_dit_forward_cfg."""
        import torch
        n_txt = 0 if txt_cond is None else txt_cond.shape[0]
        if (0 if txt_uncond is None else txt_uncond.shape[0]) != n_txt:
            raise ValueError("txt_cond and txt_uncond must have the same token count")
        n_refs, grids = _grids(ref_hw)
        _check_forward_shapes(self.dims, img_tok, grid_hw, [txt_cond, txt_uncond],
                              list(zip(grids[0::2], grids[1::2]))[:n_refs], ref_tok, [v_cond, v_uncond])
        _check(lib().flux3_dit_forward_cfg(self._h, _ptr(img_tok, torch.float32, "img_tok"), grid_hw[0], grid_hw[1],
                                           _ptr(txt_cond, torch.float32, "txt_cond"),
                                           _ptr(txt_uncond, torch.float32, "txt_uncond"), n_txt,
                                           _ptr(ref_tok, torch.float32, "ref_tok"), n_refs, grids, float(t),
                                           float(t_target), _ptr(v_cond, torch.float32, "v_cond"),
                                           _ptr(v_uncond, torch.float32, "v_uncond"), _stream(stream)))
        return v_cond, v_uncond

    def set_active_blocks(self, n_mode=-1, n_joint=-1):
        _check(lib().flux3_dit_set_active_blocks(self._h, n_mode, n_joint))

    def set_precision(self, precision):
        """PRECISION_BF16, PRECISION_FP8 or PRECISION_NVFP4 block linears; see flux3_dit_set_precision."""
        _check(lib().flux3_dit_set_precision(self._h, int(precision)))

    def modulation_size(self) -> int:
        return lib().flux3_dit_modulation_size(self._h)

    def modulation(self, t, t_target, out, stream=None):
        import torch
        _need_numel(out, self.modulation_size(), "out")
        _check(lib().flux3_dit_modulation(self._h, float(t), float(t_target), _ptr(out, torch.float32, "mods"),
                                          _stream(stream)))
        return out

    def profile(self, enable: bool):
        _check(lib().flux3_dit_profile(self._h, 1 if enable else 0))

    def profile_read(self):
        """{kind: (ms, flops, bytes, launches)} accumulated since profile(True)."""
        out = {}
        for i, name in enumerate(self.PROFILE_KINDS):
            ms, fl, by, n = ctypes.c_double(), ctypes.c_double(), ctypes.c_double(), ctypes.c_longlong()
            _check(lib().flux3_dit_profile_read(self._h, i, ctypes.byref(ms), ctypes.byref(fl), ctypes.byref(by),
                                                ctypes.byref(n)))
            out[name] = (ms.value, fl.value, by.value, n.value)
        return out


def euler_schedule(n_steps: int):
    """t_0 = 1 > ... > t_S = 0 evenly spaced (float32 values)."""
    return [float(np.float32(1.0 - i / n_steps)) for i in range(n_steps + 1)]


def img2img_first_step(n_steps: int, strength: float) -> int:
    """First schedule index run at img2img strength s: the last floor(S * s) steps are run."""
    return n_steps - min(int(n_steps * strength), n_steps)


def flux_blend_latents(x, noise, t, out, stream=None):
    """out = (1 - t) x + t noise (img2img start state)."""
    import torch
    _need_same(noise, x, "noise")
    _need_same(out, x, "out")
    _check(lib().flux_blend_latents(_ptr(x, torch.float32, "x"), _ptr(noise, torch.float32, "noise"), float(t),
                                    _ptr(out, torch.float32, "out"), x.numel(), _stream(stream)))
    return out


def flux_euler_step(x, v, dt, stream=None):
    import torch
    _need_same(v, x, "v")
    _check(lib().flux_euler_step(_ptr(x, torch.float32, "x"), _ptr(v, torch.float32, "v"), x.numel(),
                                 float(dt), _stream(stream)))
    return x


def flux_cfg_euler_step(x, v_cond, v_uncond, guidance, dt, stream=None, v_guided=None):
    """x += dt * (v_uncond + guidance * (v_cond - v_uncond)), in place; with ``v_guided`` (a tensor
    like x) the kernel also writes the guided velocity there."""
    import torch
    _need_same(v_cond, x, "v_cond")
    _need_same(v_uncond, x, "v_uncond")
    if v_guided is None:
        _check(lib().flux_cfg_euler_step(_ptr(x, torch.float32, "x"), _ptr(v_cond, torch.float32, "v_cond"),
                                         _ptr(v_uncond, torch.float32, "v_uncond"), x.numel(), float(guidance),
                                         float(dt), _stream(stream)))
        return x
    _need_same(v_guided, x, "v_guided")
    _check(lib().flux_cfg_euler_step_out(_ptr(x, torch.float32, "x"), _ptr(v_cond, torch.float32, "v_cond"),
                                         _ptr(v_uncond, torch.float32, "v_uncond"),
                                         _ptr(v_guided, torch.float32, "v_guided"), x.numel(), float(guidance),
                                         float(dt), _stream(stream)))
    return x


def _latent_tokens(lat, tok):
    if lat.dim() != 3 or lat.shape[0] != 32:
        raise FluxShapeError("lat must be [32, h8, w8]")
    _need_tokens(tok, (lat.shape[1] // 2) * (lat.shape[2] // 2), "tok")


def flux_pack_latents(lat, tok, stream=None):
    import torch
    _latent_tokens(lat, tok)
    _check(lib().flux_pack_latents(_ptr(lat, torch.float32, "lat"), _ptr(tok, torch.float32, "tok"),
                                   lat.shape[1], lat.shape[2], _stream(stream)))
    return tok


def flux_unpack_latents(tok, lat, stream=None):
    import torch
    _latent_tokens(lat, tok)
    _check(lib().flux_unpack_latents(_ptr(tok, torch.float32, "tok"), _ptr(lat, torch.float32, "lat"),
                                     lat.shape[1], lat.shape[2], _stream(stream)))
    return lat


def _qkvo(q, k, v, o):
    if q.dim() != 3:
        raise FluxShapeError("q must be [n, heads, head_dim]")
    for t, name in ((k, "k"), (v, "v"), (o, "o")):
        _need_same(t, q, name)


def flux_joint_attention(q, k, v, o, scale=None, stream=None):
    _qkvo(q, k, v, o)
    n, heads, hd = q.shape
    scale = hd ** -0.5 if scale is None else scale
    _check(lib().flux_joint_attention(_bits(q, "q"), _bits(k, "k"), _bits(v, "v"), _bits(o, "o"), n, heads, hd,
                                      float(scale), _stream(stream)))
    return o


def flux_joint_attention_batch(q, k, v, o, batch, scale=None, stream=None):
    """q, k, v, o bf16 [batch * n, heads, 128]; sequence b attends within rows [b n, (b + 1) n)."""
    _qkvo(q, k, v, o)
    rows, heads, hd = q.shape
    if rows % batch:
        raise ValueError("rows must be a multiple of batch")
    scale = hd ** -0.5 if scale is None else scale
    _check(lib().flux_joint_attention_batch(_bits(q, "q"), _bits(k, "k"), _bits(v, "v"), _bits(o, "o"), batch,
                                            rows // batch, heads, hd, float(scale), _stream(stream)))
    return o


def flux_joint_attention_segments(q, k, v, o, seg_len, scale=None, stream=None):
    """q, k, v, o bf16 [sum(seg_len), heads, 128]; each segment attends only within itself."""
    _qkvo(q, k, v, o)
    rows, heads, hd = q.shape
    if sum(seg_len) != rows:
        raise ValueError("segment lengths must add up to the row count")
    scale = hd ** -0.5 if scale is None else scale
    lens = (ctypes.c_int * len(seg_len))(*seg_len)
    _check(lib().flux_joint_attention_segments(_bits(q, "q"), _bits(k, "k"), _bits(v, "v"), _bits(o, "o"),
                                               len(seg_len), lens, heads, hd, float(scale), _stream(stream)))
    return o


def flux_linear(a, w, bias, mode, out, gate=None, stream=None):
    import torch
    m, k = a.shape
    n = w.shape[0]
    if w.dim() != 2 or w.shape[1] != k:
        raise FluxShapeError("w must be [n, k] with the k of a")
    _check_strided(a, "bf16", "a")
    _need_numel(bias, n, "bias")
    _need_linear_out(out, gate, m, n, mode)
    lda = a.stride(0)
    if a.stride(1) != 1:
        raise ValueError("a must have unit column stride")
    _check(lib().flux_linear(_strided(a, "bf16", "a"), m, k, lda, _bits(w, "w"), n, _bits(bias, "bias"), mode,
                             _strided(out, None, "out"), out.stride(0),
                             _ptr(gate, torch.float32, "gate"), _stream(stream)))
    return out


def _u8(t, what):
    import torch
    if t.dtype not in (torch.uint8, torch.float8_e4m3fn):
        raise ValueError(f"{what} must be uint8 e4m3 codes")
    return _ptr(t, None, what)


def flux_quantize_rows_e4m3(x, q, scale, stream=None):
    """Row-wise e4m3 codes q (uint8 [rows, cols]) and scales (fp32 [rows]) of bf16 x [rows, cols]."""
    import torch
    rows, cols = x.shape
    if x.stride(1) != 1 or q.stride(1) != 1:
        raise ValueError("x and q must have unit column stride")
    _check_strided(x, "bf16", "x")
    _check_strided(q, "u8", "q")
    _need_rows_cols(q, rows, cols, "q")
    _need_numel(scale, rows, "scale")
    _check(lib().flux_quantize_rows_e4m3(_strided(x, "bf16", "x"), rows, cols, x.stride(0),
                                         _strided(q, "u8", "q"), q.stride(0),
                                         _ptr(scale, torch.float32, "scale"), _stream(stream)))
    return q, scale


def flux_layernorm_modulate_fp8(x, q, q_scale, shift, scale, eps=1e-6, stream=None):
    import torch
    rows, dim = x.shape
    _need_numel(q, rows * dim, "q")
    _need_numel(q_scale, rows, "q_scale")
    _need_numel(shift, dim, "shift")
    _need_numel(scale, dim, "scale")
    _check(lib().flux_layernorm_modulate_fp8(_ptr(x, torch.float32, "x"), _u8(q, "q"),
                                             _ptr(q_scale, torch.float32, "q_scale"), rows, dim,
                                             _ptr(shift, torch.float32, "shift"), _ptr(scale, torch.float32, "scale"),
                                             float(eps), _stream(stream)))
    return q, q_scale


def flux_linear_fp8(a, a_scale, w, w_scale, bias, mode, out, gate=None, stream=None):
    """FP8 linear: a, w uint8 e4m3 codes [m, k] / [n, k] with row scales; epilogue modes as flux_linear."""
    import torch
    m, k = a.shape
    n = w.shape[0]
    if a.stride(1) != 1:
        raise ValueError("a must have unit column stride")
    if w.dim() != 2 or w.shape[1] != k:
        raise FluxShapeError("w must be [n, k] with the k of a")
    _check_strided(a, "u8", "a")
    _need_numel(a_scale, m, "a_scale")
    _need_numel(w_scale, n, "w_scale")
    _need_numel(bias, n, "bias")
    _need_linear_out(out, gate, m, n, mode)
    _check(lib().flux_linear_fp8(_strided(a, "u8", "a"), _ptr(a_scale, torch.float32, "a_scale"), m, k,
                                 a.stride(0), _u8(w, "w"), _ptr(w_scale, torch.float32, "w_scale"), n,
                                 _bits(bias, "bias"), mode, _strided(out, None, "out"), out.stride(0),
                                 _ptr(gate, torch.float32, "gate"), _stream(stream)))
    return out


def flux_nvfp4_scale_bytes(rows, k) -> int:
    """Bytes of the e4m3 block scales of an NVFP4 matrix [rows, k] (whole 128-row blocks)."""
    return int(lib().flux_nvfp4_scale_bytes(int(rows), int(k)))


def flux_quantize_rows_nvfp4(x, q, sf, row_scale, stream=None):
    """NVFP4 codes q (uint8 [rows, k/2], two per byte), block scales sf (uint8
    [flux_nvfp4_scale_bytes(rows, k)]) and row scales (fp32 [rows]) of bf16 x [rows, k]."""
    import torch
    rows, k = x.shape
    if x.stride(1) != 1 or q.stride(1) != 1:
        raise ValueError("x and q must have unit column stride")
    _check_strided(x, "bf16", "x")
    _check_strided(q, "u8", "q")
    _need_rows_cols(q, rows, k // 2, "q")
    _need_numel(sf, flux_nvfp4_scale_bytes(rows, k), "sf")
    _need_numel(row_scale, rows, "row_scale")
    _check(lib().flux_quantize_rows_nvfp4(_strided(x, "bf16", "x"), rows, k, x.stride(0),
                                          _strided(q, "u8", "q"), q.stride(0), _u8(sf, "sf"),
                                          _ptr(row_scale, torch.float32, "row_scale"), _stream(stream)))
    return q, sf, row_scale


def flux_layernorm_modulate_nvfp4(x, q, sf, row_scale, shift, scale, eps=1e-6, stream=None):
    """LN + modulation of fp32 x [rows, dim], the float32 results quantised to NVFP4 (q [rows, dim/2],
    sf [flux_nvfp4_scale_bytes(rows, dim)], row_scale [rows])."""
    import torch
    rows, dim = x.shape
    _need_numel(q, rows * dim // 2, "q")
    _need_numel(sf, flux_nvfp4_scale_bytes(rows, dim), "sf")
    _need_numel(row_scale, rows, "row_scale")
    _need_numel(shift, dim, "shift")
    _need_numel(scale, dim, "scale")
    _check(lib().flux_layernorm_modulate_nvfp4(_ptr(x, torch.float32, "x"), _u8(q, "q"), _u8(sf, "sf"),
                                               _ptr(row_scale, torch.float32, "row_scale"), rows, dim,
                                               _ptr(shift, torch.float32, "shift"), _ptr(scale, torch.float32, "scale"),
                                               float(eps), _stream(stream)))
    return q, sf, row_scale


def flux_linear_nvfp4(a, a_sf, a_scale, w, w_sf, w_scale, bias, mode, out, gate=None, stream=None):
    """NVFP4 linear: a, w packed codes [m, k/2] / [n, k/2] with block scales and row scales as
    written by flux_quantize_rows_nvfp4; epilogue modes as flux_linear."""
    import torch
    m, kh = a.shape
    n = w.shape[0]
    if a.stride(1) != 1:
        raise ValueError("a must have unit column stride")
    if w.dim() != 2 or w.shape[1] != kh:
        raise FluxShapeError("w must be [n, k/2] with the k of a")
    _check_strided(a, "u8", "a")
    _need_numel(a_sf, flux_nvfp4_scale_bytes(m, 2 * kh), "a_sf")
    _need_numel(w_sf, flux_nvfp4_scale_bytes(n, 2 * kh), "w_sf")
    _need_numel(a_scale, m, "a_scale")
    _need_numel(w_scale, n, "w_scale")
    _need_numel(bias, n, "bias")
    _need_linear_out(out, gate, m, n, mode)
    _check(lib().flux_linear_nvfp4(_strided(a, "u8", "a"), _u8(a_sf, "a_sf"),
                                   _ptr(a_scale, torch.float32, "a_scale"), m, 2 * kh, a.stride(0), _u8(w, "w"),
                                   _u8(w_sf, "w_sf"), _ptr(w_scale, torch.float32, "w_scale"), n,
                                   _bits(bias, "bias"), mode, _strided(out, None, "out"), out.stride(0),
                                   _ptr(gate, torch.float32, "gate"), _stream(stream)))
    return out


def flux_qkv_projection(a, w, bias, heads, q_gain, k_gain, table, qkv, table_row0=0, eps=1e-6, stream=None):
    """qkv = a w^T + bias with QK-RMSNorm + RoPE fused on the q and k heads (see fluxdit.h)."""
    import torch
    m, k = a.shape
    if a.stride(1) != 1:
        raise ValueError("a must have unit column stride")
    n = 3 * heads * 128
    _check_strided(a, "bf16", "a")
    if w.dim() != 2 or tuple(w.shape) != (n, k):
        raise FluxShapeError(f"w must be [{n}, {k}]")
    _need_numel(bias, n, "bias")
    _need_numel(q_gain, 128, "q_gain")
    _need_numel(k_gain, 128, "k_gain")
    _need_rows_cols(qkv, m, n, "qkv")
    _need_numel(table, (table_row0 + m) * 128, "table")
    _check(lib().flux_qkv_projection(_strided(a, "bf16", "a"), m, k, a.stride(0), _bits(w, "w"),
                                     _bits(bias, "bias"), heads, _bits(q_gain, "q_gain"), _bits(k_gain, "k_gain"),
                                     _ptr(table, torch.float32, "table"), table_row0, float(eps), _bits(qkv, "qkv"),
                                     _stream(stream)))
    return qkv


def flux_layernorm_modulate(x, y, shift, scale, eps=1e-6, stream=None):
    import torch
    rows, dim = x.shape
    _need_same(y, x, "y")
    _need_numel(shift, dim, "shift")
    _need_numel(scale, dim, "scale")
    _check(lib().flux_layernorm_modulate(_ptr(x, torch.float32, "x"), _bits(y, "y"), rows, dim,
                                         _ptr(shift, torch.float32, "shift"), _ptr(scale, torch.float32, "scale"),
                                         float(eps), _stream(stream)))
    return y


def flux_rope_table(table, n_txt, grid_hw, ref_hw=(0, 0), theta=1e4, stream=None):
    import torch
    _need_numel(table, (n_txt + grid_hw[0] * grid_hw[1] + ref_hw[0] * ref_hw[1]) * 128, "table")
    _check(lib().flux_rope_table(_ptr(table, torch.float32, "table"), n_txt, grid_hw[0], grid_hw[1], ref_hw[0],
                                 ref_hw[1], float(theta), _stream(stream)))
    return table


def flux_qk_rmsnorm_rope(qkv, k_col, heads, q_gain, k_gain, table, eps=1e-6, stream=None):
    import torch
    rows, ld = qkv.shape
    if heads * 128 > ld or k_col < 0 or k_col + heads * 128 > ld:
        raise FluxShapeError("q and k heads must lie inside the row")
    _need_numel(q_gain, 128, "q_gain")
    _need_numel(k_gain, 128, "k_gain")
    _need_numel(table, rows * 128, "table")
    _check(lib().flux_qk_rmsnorm_rope(_bits(qkv, "qkv"), rows, ld, k_col, heads, _bits(q_gain, "q_gain"),
                                      _bits(k_gain, "k_gain"), _ptr(table, torch.float32, "table"), float(eps),
                                      _stream(stream)))
    return qkv


def flux_timestep_modulation_noalloc(w1, b1, w2, b2, wmod, bmod, t, mods_out, stream=None):
    """Timestep conditioning with no device allocation (see fluxdit.h); weights bf16, mods_out fp32."""
    import torch
    hidden, t_freq_dim = w1.shape
    _check(lib().flux_timestep_modulation_noalloc(_bits(w1, "w1"), _bits(b1, "b1"), _bits(w2, "w2"), _bits(b2, "b2"),
                                                  _bits(wmod, "wmod"), _bits(bmod, "bmod"), hidden, t_freq_dim,
                                                  wmod.shape[0], float(t), _ptr(mods_out, torch.float32, "mods_out"),
                                                  _stream(stream)))
    return mods_out


def flux_kernel_launches() -> int:
    return lib().flux_kernel_launches()


def flux_device_error(stream=None) -> int:
    return lib().flux_device_error(_stream(stream))


DEVERR_TIMEOUT_SELFTEST = 6


def flux_selftest_bounded_wait(limit_ns: int, arrive: bool, stream=None):
    """One CTA waits on an mbarrier through the pipelines' bounded wait; with arrive=False nothing
    arrives and the kernel gives up after limit_ns, recording DEVERR_TIMEOUT_SELFTEST."""
    _check(lib().flux_selftest_bounded_wait(int(limit_ns), 1 if arrive else 0, _stream(stream)))


def flux_test_fail_alloc_after(n: int):
    """Test hook: the library's next n device allocations succeed and the one after them fails as
    if the device were out of memory (then the hook disarms itself); n < 0 disarms it."""
    lib().flux_test_fail_alloc_after(int(n))


def flux_sample(model: FluxDiT, latent, txt, n_steps, ref_latent=None, on_step=None, stream=None,
                init_latent=None, strength=1.0, txt_uncond=None, guidance=None):
    """Euler sampling on the device: pack -> S x (forward, Euler) -> unpack.

    latent fp32 [32, h8, w8] (device): the noise.  txt fp32 [n_txt, txt_dim] (device).
    ref_latent: one fp32 [32, r8, r8] latent, a list of them (context images), or None.
    init_latent (the latent of an image to edit) with strength s < 1: start from
    flux_blend_latents(init_latent, latent, t) at schedule step img2img_first_step(S, s).
    With ``guidance`` g (and ``txt_uncond``, the unconditional text of the same length) each
    step is one batch-2 forward and the fused guided Euler update; ``on_step(i, v)`` then sees
    the guided velocity (computed for it only when a callback is given).
    Returns the final latent (new tensor).  ``on_step(i, v)`` sees each velocity.
    """
    import torch
    c, h8, w8 = latent.shape
    gh, gw = h8 // 2, w8 // 2
    ts = euler_schedule(n_steps)
    start = 0
    if init_latent is not None:
        start = img2img_first_step(n_steps, strength)
        latent = flux_blend_latents(init_latent, latent, ts[start], torch.empty_like(latent), stream)
    tok = torch.empty(gh * gw, 4 * c, device=latent.device, dtype=torch.float32)
    flux_pack_latents(latent, tok, stream)
    ref_tok, ref_hw = None, (0, 0)
    if ref_latent is not None:
        refs = list(ref_latent) if isinstance(ref_latent, (list, tuple)) else [ref_latent]
        grids = [(r.shape[1] // 2, r.shape[2] // 2) for r in refs]
        ref_tok = torch.empty(sum(h * w for h, w in grids), 4 * c, device=latent.device, dtype=torch.float32)
        row = 0
        for r, (h, w) in zip(refs, grids):
            flux_pack_latents(r, ref_tok[row:row + h * w], stream)
            row += h * w
        ref_hw = grids if isinstance(ref_latent, (list, tuple)) else grids[0]
    v = torch.empty_like(tok)
    model.prepare_timesteps(ts[start:n_steps], stream)      # every step's modulation in one pass
    if guidance is not None:
        if txt_uncond is None:
            raise ValueError("guidance needs txt_uncond")
        v_u = torch.empty_like(tok)
        hw_list = ref_hw if (ref_hw and isinstance(ref_hw[0], (tuple, list))) else ([ref_hw] if ref_hw[0] else [])
        v_g = torch.empty_like(tok) if on_step is not None else None
        for i in range(start, n_steps):
            model.forward_cfg(tok, (gh, gw), txt, txt_uncond, ts[i], v, v_u, ref_tok, hw_list, stream)
            flux_cfg_euler_step(tok, v, v_u, guidance, ts[i + 1] - ts[i], stream, v_guided=v_g)
            if on_step is not None:
                on_step(i, v_g)
        out = torch.empty_like(latent)
        flux_unpack_latents(tok, out, stream)
        return out
    for i in range(start, n_steps):
        model.forward(tok, (gh, gw), txt, ts[i], v, ref_tok, ref_hw, stream)
        if on_step is not None:
            on_step(i, v)
        flux_euler_step(tok, v, ts[i + 1] - ts[i], stream)
    out = torch.empty_like(latent)
    flux_unpack_latents(tok, out, stream)
    return out


def flux3_sample(model: Flux3DiT, latent, txt, n_steps, ref_latent=None, on_step=None, stream=None,
                 init_latent=None, strength=1.0, txt_uncond=None, guidance=None):
    """Euler sampling with a FLUX.3 model on the device: pack -> S x (forward, Euler) -> unpack.

    The flow-map model receives t_{i+1} as the target time of step i.  latent fp32 [32, h8, w8]
    (device): the noise; txt fp32 [n_txt, txt_dim]; ref_latent: None, one latent or a list.
    init_latent / strength: image editing as in flux_sample.  With ``guidance`` g (and
    ``txt_uncond`` of the same length) each step is one batch-2 forward (flux3_dit_forward_cfg)
    and the fused guided Euler update; ``on_step(i, v)`` then sees the guided velocity.
    Returns the final latent (new tensor); ``on_step(i, v)`` sees each velocity.
    """
    import torch
    c, h8, w8 = latent.shape
    gh, gw = h8 // 2, w8 // 2
    ts = euler_schedule(n_steps)
    start = 0
    if init_latent is not None:
        start = img2img_first_step(n_steps, strength)
        latent = flux_blend_latents(init_latent, latent, ts[start], torch.empty_like(latent), stream)
    tok = torch.empty(gh * gw, 4 * c, device=latent.device, dtype=torch.float32)
    flux_pack_latents(latent, tok, stream)
    ref_tok, grids = None, []
    if ref_latent is not None:
        refs = list(ref_latent) if isinstance(ref_latent, (list, tuple)) else [ref_latent]
        grids = [(r.shape[1] // 2, r.shape[2] // 2) for r in refs]
        ref_tok = torch.empty(sum(h * w for h, w in grids), 4 * c, device=latent.device, dtype=torch.float32)
        row = 0
        for r, (h, w) in zip(refs, grids):
            flux_pack_latents(r, ref_tok[row:row + h * w], stream)
            row += h * w
    v = torch.empty_like(tok)
    if guidance is not None:
        if txt_uncond is None:
            raise ValueError("guidance needs txt_uncond")
        v_u = torch.empty_like(tok)
        v_g = torch.empty_like(tok) if on_step is not None else None
        for i in range(start, n_steps):
            model.forward_cfg(tok, (gh, gw), txt, txt_uncond, ts[i], v, v_u, ref_tok, grids, t_target=ts[i + 1],
                              stream=stream)
            flux_cfg_euler_step(tok, v, v_u, guidance, ts[i + 1] - ts[i], stream, v_guided=v_g)
            if on_step is not None:
                on_step(i, v_g)
    else:
        for i in range(start, n_steps):
            model.forward(tok, (gh, gw), txt, ts[i], v, ref_tok, grids, t_target=ts[i + 1], stream=stream)
            if on_step is not None:
                on_step(i, v)
            flux_euler_step(tok, v, ts[i + 1] - ts[i], stream)
    out = torch.empty_like(latent)
    flux_unpack_latents(tok, out, stream)
    return out
