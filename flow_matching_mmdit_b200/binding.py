"""ctypes binding of liblens_dit.so: the C ABI of include/lens_dit.h with the same
names, argument marshalling only.  Device tensors are torch CUDA tensors (their
data_ptr is passed); host arrays are numpy.  Every call raises LensError on a
non-zero status.  There is no fallback: without the built library on a CUDA
machine, loading fails loudly.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Mapping, Optional, Sequence

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liblens_dit.so")

STATUS = {0: "LENS_OK", 1: "LENS_ERR_INVALID_ARG", 2: "LENS_ERR_SHAPE", 3: "LENS_ERR_OOM", 4: "LENS_ERR_CUDA",
          5: "LENS_ERR_TIMEOUT", 6: "LENS_ERR_UNSUPPORTED"}

# every symbol include/lens_dit.h declares
EXPORTS = [
    "lens_dit_default_config", "lens_dit_create", "lens_dit_destroy", "lens_dit_forward", "lens_sample_euler",
    "lens_dit_debug_blocks", "lens_dit_debug_raise_abort", "lens_dit_sync", "lens_status_string",
    "lens_op_noise_tokens", "lens_op_patchify", "lens_op_unpatchify", "lens_op_rope_table", "lens_op_rmsnorm_modulate", "lens_op_gemm_bf16",
    "lens_op_attention", "lens_op_euler_cfg", "lens_dit_op_timestep", "lens_dit_op_text_input",
    "lens_device_sm_count", "lens_dit_profile_kernel", "lens_dit_profile_read", "lens_dit_launch_count",
    "lens_op_timestep_embed_noalloc", "lens_dit_forward_masked", "lens_sample_euler_masked",
    "lens_op_attention_masked", "lens_sampler_default_options", "lens_shift_mu", "lens_time_grid",
    "lens_sample_euler_ex", "lens_dit_op_euler_cfg_rescaled", "lens_sampler_prepare", "lens_sampler_velocity",
    "lens_sampler_update", "lens_sampler_finish", "lens_op_quantize_w4", "lens_op_gemm_w4",
]

KERNELS = {"none": 0, "attention": 1, "gemm_qkv": 2, "gemm_out": 3, "gemm_w13": 4, "gemm_w2": 5, "rmsnorm_mod": 6,
           "gemm_mod": 7}


class LensError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


class lens_dit_config(ctypes.Structure):
    _fields_ = [("num_blocks", ctypes.c_int), ("hidden", ctypes.c_int), ("heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("mlp_hidden", ctypes.c_int), ("in_channels", ctypes.c_int),
                ("latent_channels", ctypes.c_int), ("patch", ctypes.c_int), ("txt_layers", ctypes.c_int),
                ("txt_dim", ctypes.c_int), ("rope_axes", ctypes.c_int * 3), ("rope_theta", ctypes.c_float),
                ("eps", ctypes.c_float), ("freq_dim", ctypes.c_int), ("max_batch", ctypes.c_int),
                ("max_img_tokens", ctypes.c_int), ("max_txt_tokens", ctypes.c_int), ("max_timesteps", ctypes.c_int),
                ("weight_bits", ctypes.c_int)]


class lens_sampler_options(ctypes.Structure):
    _fields_ = [("guidance", ctypes.c_float), ("cfg_rescale", ctypes.c_float), ("time_shift", ctypes.c_int),
                ("shift_mu", ctypes.c_float)]


class lens_weight(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("data", ctypes.c_void_p), ("ndim", ctypes.c_int),
                ("shape", ctypes.c_int64 * 4)]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load (once) and type the shared library."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is not built; run `python -m flow_matching_mmdit_b200.build`")
    lib = ctypes.CDLL(path)
    P, I, F, L, U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_int64, ctypes.c_uint64
    sig = {
        "lens_dit_default_config": (I, [ctypes.POINTER(lens_dit_config)]),
        "lens_dit_create": (I, [ctypes.POINTER(lens_dit_config), ctypes.POINTER(lens_weight), I, P,
                                ctypes.POINTER(P)]),
        "lens_dit_destroy": (None, [P]),
        "lens_dit_forward": (I, [P, P, I, I, I, P, I, P, P, P]),
        "lens_sample_euler": (I, [P, P, P, I, I, I, I, I, F, U64, P, P]),
        "lens_dit_debug_blocks": (I, [P, I, I, P, P, I, I, I, I, P, P]),
        "lens_dit_debug_raise_abort": (I, [P, P]),
        "lens_dit_sync": (I, [P, P]),
        "lens_status_string": (ctypes.c_char_p, [I]),
        "lens_op_noise_tokens": (I, [U64, I, I, I, P, P]),
        "lens_op_patchify": (I, [P, I, I, I, P, P]),
        "lens_op_unpatchify": (I, [P, I, I, I, P, P]),
        "lens_op_rope_table": (I, [I, I, I, P, P]),
        "lens_op_rmsnorm_modulate": (I, [P, I, I, P, P, L, F, P, P]),
        "lens_op_gemm_bf16": (I, [P, P, P, P, I, I, I, P]),
        "lens_op_attention": (I, [P, P, P, I, I, I, P, P, P]),
        "lens_op_euler_cfg": (I, [P, P, P, L, F, F, P]),
        "lens_dit_op_timestep": (I, [P, P, I, P, P, P]),
        "lens_dit_op_text_input": (I, [P, P, I, I, P, P]),
        "lens_device_sm_count": (I, []),
        "lens_dit_profile_kernel": (I, [P, I, I]),
        "lens_dit_profile_read": (I, [P, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_double)]),
        "lens_dit_launch_count": (L, [P]),
        "lens_op_timestep_embed_noalloc": (I, [P, I, P, P, P, P, P, P]),
        "lens_dit_forward_masked": (I, [P, P, I, I, I, P, I, P, P, P, P]),
        "lens_sample_euler_masked": (I, [P, P, P, P, P, I, I, I, I, I, F, U64, P, P]),
        "lens_op_attention_masked": (I, [P, P, P, I, I, I, P, P, P, P]),
        "lens_sampler_default_options": (I, [ctypes.POINTER(lens_sampler_options)]),
        "lens_shift_mu": (ctypes.c_double, [I, I, ctypes.c_double, I, ctypes.c_double]),
        "lens_time_grid": (I, [I, I, ctypes.c_double, P]),
        "lens_sample_euler_ex": (I, [P, P, P, P, P, I, I, I, I, I, ctypes.POINTER(lens_sampler_options), U64, P,
                                     P]),
        "lens_dit_op_euler_cfg_rescaled": (I, [P, P, P, P, I, L, F, F, F, P]),
        "lens_sampler_prepare": (I, [P, P, P, I, I, I, I, I, ctypes.POINTER(lens_sampler_options), U64, P]),
        "lens_sampler_velocity": (I, [P, I, P, P]),
        "lens_sampler_update": (I, [P, I, P, P, P]),
        "lens_sampler_finish": (I, [P, P, P]),
        "lens_op_quantize_w4": (I, [P, L, L, P, P, P]),
        "lens_op_gemm_w4": (I, [P, P, P, P, P, I, I, I, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(status: int, where: str) -> None:
    if status != 0:
        raise LensError(status, where)


def _ptr(x) -> Optional[int]:
    """Device pointer of a torch tensor (None passes NULL)."""
    if x is None:
        return None
    return int(x.data_ptr())


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream or None
    if isinstance(stream, int):
        return stream or None
    return stream.cuda_stream or None


# ---------------------------------------------------------------- handle API
def lens_dit_default_config() -> lens_dit_config:
    c = lens_dit_config()
    _check(load_library().lens_dit_default_config(ctypes.byref(c)), "lens_dit_default_config")
    return c


class LensDit:
    """Owns a lens_dit handle; destroy() or garbage collection frees it."""

    def __init__(self, ptr: int, cfg: lens_dit_config):
        self.ptr = ptr
        self.cfg = cfg

    def destroy(self) -> None:
        if self.ptr:
            load_library().lens_dit_destroy(self.ptr)
            self.ptr = None

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass


def lens_dit_create(cfg: lens_dit_config, weights: Mapping[str, np.ndarray], stream=None) -> LensDit:
    """weights: name -> host bf16 bit patterns (np.uint16), shapes as in the header."""
    lib = load_library()
    items = list(weights.items())
    arr = (lens_weight * len(items))()
    keep = []
    for i, (name, w) in enumerate(items):
        w = np.ascontiguousarray(w)
        if w.dtype != np.uint16:
            raise TypeError(f"{name}: bf16 bit patterns (uint16) expected, got {w.dtype}")
        keep.append(w)
        arr[i].name = name.encode()
        arr[i].data = w.ctypes.data
        arr[i].ndim = w.ndim
        for d, s in enumerate(w.shape):
            arr[i].shape[d] = s
    out = ctypes.c_void_p()
    _check(lib.lens_dit_create(ctypes.byref(cfg), arr, len(items), _stream(stream), ctypes.byref(out)),
           "lens_dit_create")
    return LensDit(out.value, cfg)


def lens_dit_destroy(h: LensDit) -> None:
    h.destroy()


def lens_dit_forward(h: LensDit, img_tokens, B: int, grid_h: int, grid_w: int, txt, n_txt: int,
                     t: Sequence[float], v_out, stream=None) -> None:
    tt = np.ascontiguousarray(np.asarray(t, np.float32))
    _check(load_library().lens_dit_forward(h.ptr, _ptr(img_tokens), B, grid_h, grid_w, _ptr(txt), n_txt,
                                           tt.ctypes.data, _ptr(v_out), _stream(stream)), "lens_dit_forward")


def _ints(a) -> Optional[np.ndarray]:
    return None if a is None else np.ascontiguousarray(np.asarray(a, np.int32))


def _iptr(a) -> Optional[int]:
    return None if a is None else a.ctypes.data


def lens_dit_forward_masked(h: LensDit, img_tokens, B: int, grid_h: int, grid_w: int, txt, n_txt: int,
                            txt_len: Optional[Sequence[int]], t: Sequence[float], v_out, stream=None) -> None:
    tt = np.ascontiguousarray(np.asarray(t, np.float32))
    ln = _ints(txt_len)
    _check(load_library().lens_dit_forward_masked(h.ptr, _ptr(img_tokens), B, grid_h, grid_w, _ptr(txt), n_txt,
                                                  _iptr(ln), tt.ctypes.data, _ptr(v_out), _stream(stream)),
           "lens_dit_forward_masked")


def lens_sample_euler_masked(h: LensDit, txt_cond, len_cond, txt_uncond, len_uncond, B: int, n_txt: int,
                             height_px: int, width_px: int, steps: int, guidance: float, seed: int, latent_out,
                             stream=None) -> None:
    lc, lu = _ints(len_cond), _ints(len_uncond)
    _check(load_library().lens_sample_euler_masked(h.ptr, _ptr(txt_cond), _iptr(lc), _ptr(txt_uncond), _iptr(lu), B,
                                                   n_txt, height_px, width_px, steps, guidance, seed,
                                                   _ptr(latent_out), _stream(stream)), "lens_sample_euler_masked")


def lens_sampler_default_options() -> lens_sampler_options:
    o = lens_sampler_options()
    _check(load_library().lens_sampler_default_options(ctypes.byref(o)), "lens_sampler_default_options")
    return o


def lens_shift_mu(n_img_tokens: int, n1: int, mu1: float, n2: int, mu2: float) -> float:
    return load_library().lens_shift_mu(n_img_tokens, n1, mu1, n2, mu2)


def lens_time_grid(steps: int, time_shift: bool, mu: float) -> np.ndarray:
    t = np.empty(max(steps, 0) + 1, dtype=np.float64)
    _check(load_library().lens_time_grid(steps, 1 if time_shift else 0, mu, t.ctypes.data), "lens_time_grid")
    return t


def lens_sample_euler_ex(h: LensDit, txt_cond, len_cond, txt_uncond, len_uncond, B: int, n_txt: int,
                         height_px: int, width_px: int, steps: int, opt: lens_sampler_options, seed: int,
                         latent_out, stream=None) -> None:
    lc, lu = _ints(len_cond), _ints(len_uncond)
    _check(load_library().lens_sample_euler_ex(h.ptr, _ptr(txt_cond), _iptr(lc), _ptr(txt_uncond), _iptr(lu), B,
                                               n_txt, height_px, width_px, steps, ctypes.byref(opt), seed,
                                               _ptr(latent_out), _stream(stream)), "lens_sample_euler_ex")


def lens_dit_op_euler_cfg_rescaled(h: LensDit, x, v_cond, v_uncond, B: int, per_sample: int, dt: float,
                                   guidance: float, phi: float, stream=None) -> None:
    _check(load_library().lens_dit_op_euler_cfg_rescaled(h.ptr, _ptr(x), _ptr(v_cond), _ptr(v_uncond), B, per_sample,
                                                         dt, guidance, phi, _stream(stream)),
           "lens_dit_op_euler_cfg_rescaled")


def lens_sampler_prepare(h: LensDit, txt, txt_len, B: int, n_txt: int, height_px: int, width_px: int, steps: int,
                         opt: lens_sampler_options, seed: int, stream=None) -> None:
    tl = _ints(txt_len)
    _check(load_library().lens_sampler_prepare(h.ptr, _ptr(txt), _iptr(tl), B, n_txt, height_px, width_px, steps,
                                               ctypes.byref(opt), seed, _stream(stream)), "lens_sampler_prepare")


def lens_sampler_velocity(h: LensDit, k: int, v_out, stream=None) -> None:
    _check(load_library().lens_sampler_velocity(h.ptr, k, _ptr(v_out), _stream(stream)), "lens_sampler_velocity")


def lens_sampler_update(h: LensDit, k: int, v_cond, v_uncond, stream=None) -> None:
    _check(load_library().lens_sampler_update(h.ptr, k, _ptr(v_cond), _ptr(v_uncond), _stream(stream)),
           "lens_sampler_update")


def lens_sampler_finish(h: LensDit, latent_out, stream=None) -> None:
    _check(load_library().lens_sampler_finish(h.ptr, _ptr(latent_out), _stream(stream)), "lens_sampler_finish")


def lens_sample_euler(h: LensDit, txt_cond, txt_uncond, B: int, n_txt: int, height_px: int, width_px: int,
                      steps: int, guidance: float, seed: int, latent_out, stream=None) -> None:
    _check(load_library().lens_sample_euler(h.ptr, _ptr(txt_cond), _ptr(txt_uncond), B, n_txt, height_px, width_px,
                                            steps, guidance, seed, _ptr(latent_out), _stream(stream)),
           "lens_sample_euler")


def lens_dit_debug_blocks(h: LensDit, first: int, last: int, h_img, h_txt, B: int, grid_h: int, grid_w: int,
                          n_txt: int, t: Sequence[float], stream=None) -> None:
    tt = np.ascontiguousarray(np.asarray(t, np.float32))
    _check(load_library().lens_dit_debug_blocks(h.ptr, first, last, _ptr(h_img), _ptr(h_txt), B, grid_h, grid_w,
                                                 n_txt, tt.ctypes.data, _stream(stream)), "lens_dit_debug_blocks")


def lens_dit_debug_raise_abort(h: LensDit, stream=None) -> None:
    _check(load_library().lens_dit_debug_raise_abort(h.ptr, _stream(stream)), "lens_dit_debug_raise_abort")


def lens_dit_sync(h: LensDit, stream=None) -> None:
    _check(load_library().lens_dit_sync(h.ptr, _stream(stream)), "lens_dit_sync")


def lens_status_string(status: int) -> str:
    return load_library().lens_status_string(status).decode()


def lens_dit_op_timestep(h: LensDit, t: Sequence[float], temb, mod, stream=None) -> None:
    tt = np.ascontiguousarray(np.asarray(t, np.float32))
    _check(load_library().lens_dit_op_timestep(h.ptr, tt.ctypes.data, len(tt), _ptr(temb), _ptr(mod),
                                               _stream(stream)), "lens_dit_op_timestep")


def lens_dit_op_text_input(h: LensDit, txt, B: int, n_txt: int, c, stream=None) -> None:
    _check(load_library().lens_dit_op_text_input(h.ptr, _ptr(txt), B, n_txt, _ptr(c), _stream(stream)),
           "lens_dit_op_text_input")


# ---------------------------------------------------------------- single ops
def lens_op_noise_tokens(seed: int, B: int, grid_h: int, grid_w: int, tokens, stream=None) -> None:
    _check(load_library().lens_op_noise_tokens(seed, B, grid_h, grid_w, _ptr(tokens), _stream(stream)),
           "lens_op_noise_tokens")


def lens_op_patchify(latent, B: int, grid_h: int, grid_w: int, tokens, stream=None) -> None:
    _check(load_library().lens_op_patchify(_ptr(latent), B, grid_h, grid_w, _ptr(tokens), _stream(stream)),
           "lens_op_patchify")


def lens_op_unpatchify(tokens, B: int, grid_h: int, grid_w: int, latent, stream=None) -> None:
    _check(load_library().lens_op_unpatchify(_ptr(tokens), B, grid_h, grid_w, _ptr(latent), _stream(stream)),
           "lens_op_unpatchify")


def lens_op_rope_table(grid_h: int, grid_w: int, n_txt: int, cos_sin, stream=None) -> None:
    _check(load_library().lens_op_rope_table(grid_h, grid_w, n_txt, _ptr(cos_sin), _stream(stream)),
           "lens_op_rope_table")


def lens_op_rmsnorm_modulate(x, M: int, rows_per_batch: int, shift, scale, mod_stride: int, eps: float, y,
                             stream=None) -> None:
    _check(load_library().lens_op_rmsnorm_modulate(_ptr(x), M, rows_per_batch, _ptr(shift), _ptr(scale), mod_stride,
                                                   eps, _ptr(y), _stream(stream)), "lens_op_rmsnorm_modulate")


def lens_op_gemm_bf16(A, Bm, bias, C, M: int, N: int, K: int, stream=None) -> None:
    _check(load_library().lens_op_gemm_bf16(_ptr(A), _ptr(Bm), _ptr(bias), _ptr(C), M, N, K, _stream(stream)),
           "lens_op_gemm_bf16")


def lens_op_attention(q, k, v, B: int, n_txt: int, n_img: int, out_txt, out_img, stream=None) -> None:
    _check(load_library().lens_op_attention(_ptr(q), _ptr(k), _ptr(v), B, n_txt, n_img, _ptr(out_txt),
                                            _ptr(out_img), _stream(stream)), "lens_op_attention")


def lens_op_attention_masked(q, k, v, B: int, n_txt: int, n_img: int, txt_len, out_txt, out_img,
                             stream=None) -> None:
    ln = _ints(txt_len)
    _check(load_library().lens_op_attention_masked(_ptr(q), _ptr(k), _ptr(v), B, n_txt, n_img, _iptr(ln),
                                                   _ptr(out_txt), _ptr(out_img), _stream(stream)),
           "lens_op_attention_masked")


def lens_op_quantize_w4(w, rows: int, k: int, codes, scales, stream=None) -> None:
    _check(load_library().lens_op_quantize_w4(_ptr(w), rows, k, _ptr(codes), _ptr(scales), _stream(stream)),
           "lens_op_quantize_w4")


def lens_op_gemm_w4(A, codes, scales, bias, C, M: int, N: int, K: int, stream=None) -> None:
    _check(load_library().lens_op_gemm_w4(_ptr(A), _ptr(codes), _ptr(scales), _ptr(bias), _ptr(C), M, N, K,
                                          _stream(stream)), "lens_op_gemm_w4")


def lens_op_euler_cfg(x, v_cond, v_uncond, n: int, dt: float, guidance: float, stream=None) -> None:
    _check(load_library().lens_op_euler_cfg(_ptr(x), _ptr(v_cond), _ptr(v_uncond), n, dt, guidance,
                                            _stream(stream)), "lens_op_euler_cfg")


def lens_dit_profile_kernel(h: LensDit, kernel, capacity: int) -> None:
    k = KERNELS[kernel] if isinstance(kernel, str) else int(kernel)
    _check(load_library().lens_dit_profile_kernel(h.ptr, k, capacity), "lens_dit_profile_kernel")


def lens_dit_profile_read(h: LensDit):
    """-> (timed launches, total device milliseconds)"""
    n, ms = ctypes.c_int(), ctypes.c_double()
    _check(load_library().lens_dit_profile_read(h.ptr, ctypes.byref(n), ctypes.byref(ms)), "lens_dit_profile_read")
    return n.value, ms.value


def lens_dit_launch_count(h: LensDit) -> int:
    return int(load_library().lens_dit_launch_count(h.ptr))


def lens_op_timestep_embed_noalloc(t: Sequence[float], w1, b1, w2, b2, temb, stream=None) -> None:
    """Timestep embedding for callers that cannot allocate device memory: all
    intermediates stay in a fixed array inside the library (at most 64 timesteps)."""
    tt = np.ascontiguousarray(np.asarray(t, np.float32))
    _check(load_library().lens_op_timestep_embed_noalloc(tt.ctypes.data, len(tt), _ptr(w1), _ptr(b1), _ptr(w2),
                                                         _ptr(b2), _ptr(temb), _stream(stream)),
           "lens_op_timestep_embed_noalloc")


def lens_device_sm_count() -> int:
    return int(load_library().lens_device_sm_count())
