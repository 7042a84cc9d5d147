"""ctypes binding of the DiT chunk-denoise calls of libm3.so (include/m3_dit.h),
under the same names.

Argument marshalling only: every step runs in the library's CUDA kernels.
Tensors are torch tensors on the GPU (fp16 / fp32), or on the host for the
weight sources.  There is no CPU fallback.
"""
from __future__ import annotations

import ctypes as C

import torch

from .m3 import M3_MEM_DEVICE, M3_MEM_HOST, _check, _ptr, _stream, lib

EXPORTED = ("m3_dit_create", "m3_dit_load", "m3_dit_step", "m3_dit_denoise", "m3_dit_forward",
            "m3_dit_blocks", "m3_dit_time_gemm", "m3_dit_sync_status", "m3_dit_destroy")

LAYER_FIELDS = ("ln1_g", "ln1_b", "wqkv", "wo", "ln2_g", "ln2_b", "wg", "wu", "wd")


class m3_dit_config(C.Structure):
    _fields_ = [("width", C.c_int), ("n_layers", C.c_int), ("n_heads", C.c_int),
                ("head_dim", C.c_int), ("ffn", C.c_int), ("latent", C.c_int), ("cond", C.c_int),
                ("temb", C.c_int), ("rope_dims", C.c_int), ("rope_theta", C.c_double),
                ("ln_eps", C.c_float), ("max_tokens", C.c_int)]


class m3_dit_layer_src(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in LAYER_FIELDS]


class m3_dit_src(C.Structure):
    _fields_ = [("first_layer", C.c_int), ("n_layers", C.c_int),
                ("layers", C.POINTER(m3_dit_layer_src)), ("w_in", C.c_void_p),
                ("w_t1", C.c_void_p), ("w_t2", C.c_void_p), ("lnf_g", C.c_void_p),
                ("lnf_b", C.c_void_p), ("w_out", C.c_void_p), ("mem", C.c_int)]


def _setup():
    vp, i32, f32 = C.c_void_p, C.c_int, C.c_float
    lib.m3_dit_create.argtypes = [C.POINTER(m3_dit_config), vp, C.POINTER(vp)]
    lib.m3_dit_load.argtypes = [vp, C.POINTER(m3_dit_src)]
    lib.m3_dit_step.argtypes = [vp, i32, vp, vp, vp, f32, f32, f32, vp, vp]
    lib.m3_dit_denoise.argtypes = [vp, i32, vp, vp, vp, vp, i32, f32]
    lib.m3_dit_forward.argtypes = [vp, i32, i32, vp, f32, vp]
    lib.m3_dit_blocks.argtypes = [vp, i32, i32, vp, i32, i32]
    lib.m3_dit_time_gemm.argtypes = [vp, i32, i32, i32, C.POINTER(C.c_float),
                                     C.POINTER(C.c_double)]
    lib.m3_dit_sync_status.argtypes = [vp]
    lib.m3_dit_destroy.argtypes = [vp]
    lib.m3_dit_destroy.restype = None
    for n in EXPORTED:
        if n != "m3_dit_destroy":
            getattr(lib, n).restype = C.c_int


_setup()


def config_from_shape(s, max_tokens: int) -> m3_dit_config:
    return m3_dit_config(s.width, s.n_layers, s.n_heads, s.head_dim, s.ffn, s.latent, s.cond,
                         s.temb, s.rope_dims, s.rope_theta, s.ln_eps, max_tokens)


def m3_dit_create(cfg: m3_dit_config, stream=None) -> int:
    d = C.c_void_p()
    _check(lib.m3_dit_create(C.byref(cfg), _stream(stream), C.byref(d)))
    return d.value


def m3_dit_load(d: int, w: dict, first_layer: int = 0, outer: bool = True) -> None:
    """w: synth.dit_weights-style dict of fp16 tensors (all on the host or all
    on the GPU); w["layers"] go to blocks first_layer..; outer=False skips
    the input / time / output tensors."""
    keep = []
    layers = w.get("layers", [])
    arr = (m3_dit_layer_src * max(1, len(layers)))()
    dev = None
    for i, Lw in enumerate(layers):
        vals = []
        for n in LAYER_FIELDS:
            t = Lw[n].contiguous()
            keep.append(t)
            vals.append(t.data_ptr())
            dev = t.is_cuda
        arr[i] = m3_dit_layer_src(*vals)
    outs = {}
    for n in ("w_in", "w_t1", "w_t2", "lnf_g", "lnf_b", "w_out"):
        if outer:
            t = w[n].contiguous()
            keep.append(t)
            outs[n] = t.data_ptr()
            dev = t.is_cuda if dev is None else dev
        else:
            outs[n] = None
    src = m3_dit_src(first_layer, len(layers), arr, outs["w_in"], outs["w_t1"], outs["w_t2"],
                     outs["lnf_g"], outs["lnf_b"], outs["w_out"],
                     M3_MEM_DEVICE if dev else M3_MEM_HOST)
    _check(lib.m3_dit_load(d, C.byref(src)))
    if dev:
        torch.cuda.current_stream().synchronize()


def m3_dit_step(d: int, x: torch.Tensor, ctx: torch.Tensor, cond: torch.Tensor, sigma: float,
                sigma_next: float, cfg_scale: float, v_guided=None, v_pair=None) -> None:
    _check(lib.m3_dit_step(d, x.shape[0], _ptr(x), _ptr(ctx), _ptr(cond), sigma, sigma_next,
                           cfg_scale, _ptr(v_guided), _ptr(v_pair)))


def m3_dit_denoise(d: int, x: torch.Tensor, ctx: torch.Tensor, cond: torch.Tensor, sigmas,
                   cfg_scale: float) -> None:
    s = (C.c_float * len(sigmas))(*[float(v) for v in sigmas])
    _check(lib.m3_dit_denoise(d, x.shape[0], _ptr(x), _ptr(ctx), _ptr(cond),
                              C.cast(s, C.c_void_p), len(sigmas) - 1, cfg_scale))


def m3_dit_forward(d: int, h_in: torch.Tensor, B: int, T: int, t: float,
                   v: torch.Tensor) -> None:
    _check(lib.m3_dit_forward(d, B, T, _ptr(h_in), t, _ptr(v)))


def m3_dit_blocks(d: int, h: torch.Tensor, B: int, T: int, first: int = 0, n: int = 1) -> None:
    _check(lib.m3_dit_blocks(d, B, T, _ptr(h), first, n))


def m3_dit_time_gemm(d: int, which: int, T: int, iters: int):
    """(mean ms per launch, FLOPs per launch) of one block GEMM kind."""
    ms = C.c_float()
    fl = C.c_double()
    _check(lib.m3_dit_time_gemm(d, which, T, iters, C.byref(ms), C.byref(fl)))
    return ms.value, fl.value


def m3_dit_sync_status(d: int) -> None:
    _check(lib.m3_dit_sync_status(d))


def m3_dit_destroy(d: int) -> None:
    lib.m3_dit_destroy(d)
