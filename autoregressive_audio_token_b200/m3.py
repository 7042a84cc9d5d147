"""ctypes binding of libm3.so: the C ABI of include/m3.h under the same names.

Argument marshalling only -- every step of the decode runs in the library's
CUDA kernels.  Tensors are torch tensors (device memory and streams come
from torch); the library keeps its own copies of weights and KV cache.
There is no CPU fallback: importing this module fails if the library is
missing or does not load.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libm3.so")

M3_OK, M3_EINVAL, M3_ENOMEM, M3_ECUDA, M3_ESTATE, M3_ECAPACITY, M3_ETIMEOUT, M3_EDEVICE = \
    0, -1, -2, -3, -4, -5, -6, -7
M3_EEMPTY = -8
M3_W_BF16, M3_W_INT8 = 0, 1
M3_KV_BF16, M3_KV_F16 = 0, 1
M3_MEM_HOST, M3_MEM_DEVICE = 0, 1
M3_FAULT_NONE, M3_FAULT_ALLOC, M3_FAULT_H2D, M3_FAULT_GRAPH = 0, 1, 2, 3

EXPORTED = ("m3_create", "m3_load_weights", "m3_load_depth_weights", "m3_kv_alloc", "m3_kv_set",
            "m3_kv_get", "m3_decode_frame", "m3_depth_decode", "m3_embed", "m3_quantize_int8",
            "m3_export_weight", "m3_frame_bytes", "m3_frame_kernels", "m3_depth_kernels", "m3_time_gemv", "m3_sample_noalloc", "m3_set_top_k",
            "m3_load_feedback", "m3_generate", "m3_prefill", "m3_gumbel_fill", "m3_inject_fault",
            "m3_stalled_wait", "m3_sync_status", "m3_last_error", "m3_destroy")


class M3Error(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"m3 status {code}: {msg}")
        self.code = code


class m3_config(C.Structure):
    _fields_ = [("hidden", C.c_int), ("n_layers", C.c_int), ("n_q_heads", C.c_int),
                ("n_kv_heads", C.c_int), ("head_dim", C.c_int), ("ffn", C.c_int),
                ("vocab", C.c_int), ("slice_start", C.c_int), ("slice_len", C.c_int),
                ("rope_theta", C.c_double), ("rms_eps", C.c_float), ("max_rows", C.c_int),
                ("depth_layers", C.c_int), ("depth_hidden", C.c_int), ("depth_heads", C.c_int),
                ("depth_head_dim", C.c_int), ("depth_ffn", C.c_int),
                ("depth_codebooks", C.c_int), ("depth_vocab", C.c_int),
                ("depth_rope_theta", C.c_double), ("has_end_token", C.c_int),
                ("end_token", C.c_int)]


LAYER_FIELDS = ("attn_norm", "wq", "wk", "wv", "q_norm", "k_norm", "wo", "mlp_norm", "wg",
                "wu", "wd")


class m3_layer_src(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in LAYER_FIELDS]


class m3_weight_src(C.Structure):
    _fields_ = [("first_layer", C.c_int), ("n_layers", C.c_int),
                ("layers", C.POINTER(m3_layer_src)), ("final_norm", C.c_void_p),
                ("lm_head", C.c_void_p), ("mem", C.c_int), ("lm_end_row", C.c_void_p)]


class m3_depth_src(C.Structure):
    _fields_ = [("layers", C.POINTER(m3_layer_src)), ("proj", C.c_void_p),
                ("emb", C.POINTER(C.c_void_p)), ("final_norm", C.c_void_p),
                ("heads", C.POINTER(C.c_void_p)), ("mem", C.c_int)]


def load_library() -> C.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m autoregressive_audio_token_b200.build` (no CPU fallback)")
    L = C.CDLL(LIB_PATH)
    vp, i32, i64, u64, f32 = C.c_void_p, C.c_int, C.c_int64, C.c_uint64, C.c_float
    L.m3_create.argtypes = [C.POINTER(m3_config), vp, C.POINTER(vp)]
    L.m3_load_weights.argtypes = [vp, C.POINTER(m3_weight_src), i32]
    L.m3_load_depth_weights.argtypes = [vp, C.POINTER(m3_depth_src)]
    L.m3_kv_alloc.argtypes = [vp, i32, i32, i32, i32]
    L.m3_set_top_k.argtypes = [vp, i32]
    L.m3_kv_set.argtypes = [vp, i32, i32, vp, vp, i32]
    L.m3_kv_get.argtypes = [vp, i32, i32, vp, vp]
    L.m3_decode_frame.argtypes = [vp, i32, vp, u64, u64, vp, f32, f32, vp, vp, vp]
    L.m3_depth_decode.argtypes = [vp, i32, vp, vp, u64, u64, f32, f32, vp, vp, vp]
    L.m3_embed.argtypes = [vp, i32, vp, vp, i32, vp]
    L.m3_quantize_int8.argtypes = [vp, i64, i64, i64, vp, vp, vp]
    L.m3_export_weight.argtypes = [vp, i32, i32, vp, vp]
    L.m3_frame_bytes.argtypes = [vp, i32, i32]
    L.m3_frame_bytes.restype = C.c_double
    L.m3_frame_kernels.argtypes = [vp, i32]
    L.m3_depth_kernels.argtypes = [vp, i32]
    L.m3_time_gemv.argtypes = [vp, i32, i32, i32, C.POINTER(C.c_float), C.POINTER(C.c_double)]
    L.m3_sample_noalloc.argtypes = [vp, i32, vp, u64, u64, f32, f32, vp, vp]
    L.m3_load_feedback.argtypes = [vp, vp, C.POINTER(vp), i32]
    L.m3_prefill.argtypes = [vp, i32, i32, i32, vp, vp]
    L.m3_generate.argtypes = [vp, i32, vp, u64, u64, vp, f32, f32, i32, vp, vp, vp]
    L.m3_gumbel_fill.argtypes = [u64, u64, u64, u64, i64, vp, vp]
    L.m3_inject_fault.argtypes = [vp, i32, i64]
    L.m3_stalled_wait.argtypes = [vp, i64]
    L.m3_sync_status.argtypes = [vp]
    L.m3_last_error.restype = C.c_char_p
    L.m3_destroy.argtypes = [vp]
    L.m3_destroy.restype = None
    for n in EXPORTED:
        if n not in ("m3_frame_bytes", "m3_last_error", "m3_destroy"):
            getattr(L, n).restype = C.c_int
    return L


lib = load_library()


def _check(rc: int) -> None:
    if rc != M3_OK:
        raise M3Error(rc, lib.m3_last_error().decode())


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        assert t.is_contiguous(), "tensors passed to libm3 must be contiguous"
        return t.data_ptr()
    return t


def _stream(stream=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


# ----------------------------------------------------- the ABI, by name ----

def m3_create(cfg: m3_config, stream=None) -> int:
    ctx = C.c_void_p()
    _check(lib.m3_create(C.byref(cfg), _stream(stream), C.byref(ctx)))
    return ctx.value


def _layer_src(t: dict, keep: list) -> m3_layer_src:
    s = m3_layer_src()
    for n in LAYER_FIELDS:
        v = t[n].contiguous()
        keep.append(v)
        setattr(s, n, v.data_ptr())
    return s


def m3_load_weights(ctx: int, layers: list, first_layer: int = 0, final_norm=None, lm_head=None,
                    wdtype: int = M3_W_BF16, lm_end_row=None) -> None:
    """layers: list of dicts of bf16 tensors (all on the host or all on the GPU);
    lm_end_row: the end token's lm_head row [H] when the config has one."""
    keep = []
    arr = (m3_layer_src * max(1, len(layers)))()
    dev = None
    for i, t in enumerate(layers):
        arr[i] = _layer_src(t, keep)
        dev = t["wq"].is_cuda
    for t in (final_norm, lm_head, lm_end_row):
        if t is not None:
            keep.append(t.contiguous())
            dev = t.is_cuda if dev is None else dev
    src = m3_weight_src(first_layer, len(layers), arr,
                        _ptr(final_norm.contiguous()) if final_norm is not None else None,
                        _ptr(lm_head.contiguous()) if lm_head is not None else None,
                        M3_MEM_DEVICE if dev else M3_MEM_HOST,
                        _ptr(lm_end_row.contiguous()) if lm_end_row is not None else None)
    if final_norm is not None:
        keep.append(final_norm)
    _check(lib.m3_load_weights(ctx, C.byref(src), wdtype))


def m3_load_depth_weights(ctx: int, w: dict) -> None:
    keep = []
    nl = len(w["layers"])
    arr = (m3_layer_src * nl)()
    for i, t in enumerate(w["layers"]):
        arr[i] = _layer_src(t, keep)
    emb = (C.c_void_p * len(w["emb"]))(*[keep.append(e.contiguous()) or keep[-1].data_ptr()
                                         for e in w["emb"]])
    heads = (C.c_void_p * len(w["heads"]))(*[keep.append(h.contiguous()) or keep[-1].data_ptr()
                                             for h in w["heads"]])
    proj = w["proj"].contiguous()
    fn = w["final_norm"].contiguous()
    keep += [proj, fn]
    src = m3_depth_src(arr, proj.data_ptr(), emb, fn.data_ptr(), heads,
                       M3_MEM_DEVICE if proj.is_cuda else M3_MEM_HOST)
    _check(lib.m3_load_depth_weights(ctx, C.byref(src)))


def m3_kv_alloc(ctx: int, rows: int, max_positions: int, kvdtype: int = M3_KV_BF16,
                bucket: int = 256) -> None:
    _check(lib.m3_kv_alloc(ctx, rows, max_positions, kvdtype, bucket))


def m3_kv_set(ctx: int, row: int, k: torch.Tensor, v: torch.Tensor) -> None:
    """k, v: bf16 [n_layers, n_positions, Hkv, d] on the host or the GPU."""
    k, v = k.contiguous(), v.contiguous()
    _check(lib.m3_kv_set(ctx, row, k.shape[1], k.data_ptr(), v.data_ptr(),
                         M3_MEM_DEVICE if k.is_cuda else M3_MEM_HOST))


def m3_kv_get(ctx: int, row: int, n_layers: int, n_positions: int, hkv: int, d: int):
    k = torch.empty((n_layers, n_positions, hkv, d), dtype=torch.int16)
    v = torch.empty_like(k)
    _check(lib.m3_kv_get(ctx, row, n_positions, k.data_ptr(), v.data_ptr()))
    return k, v


def m3_decode_frame(ctx: int, positions, seed: int, frame: int, x_in: torch.Tensor,
                    cfg_scale: float, temperature: float, codes: torch.Tensor,
                    h_out: torch.Tensor | None = None, logits: torch.Tensor | None = None) -> None:
    rows = x_in.shape[0]
    pos = (C.c_int32 * rows)(*[int(p) for p in positions])
    _check(lib.m3_decode_frame(ctx, rows, C.cast(pos, C.c_void_p), seed, frame, _ptr(x_in),
                               cfg_scale, temperature, _ptr(codes), _ptr(h_out), _ptr(logits)))


def m3_depth_decode(ctx: int, h_frame: torch.Tensor, code0: torch.Tensor, seed: int, frame: int,
                    cfg_scale: float, temperature: float, codes: torch.Tensor,
                    forced: torch.Tensor | None = None, logits: torch.Tensor | None = None) -> None:
    rows = h_frame.shape[0]
    _check(lib.m3_depth_decode(ctx, rows, _ptr(h_frame), _ptr(code0), seed, frame, cfg_scale,
                               temperature, _ptr(forced), _ptr(codes), _ptr(logits)))


def m3_embed(ctx: int, codes: torch.Tensor, table: torch.Tensor, offset: int,
             x_out: torch.Tensor) -> None:
    _check(lib.m3_embed(ctx, codes.shape[0], _ptr(codes), _ptr(table), offset, _ptr(x_out)))


def m3_quantize_int8(w: torch.Tensor, group: int | None = None, stream=None):
    rows, cols = w.shape
    g = cols if group is None else group
    q = torch.empty((rows, cols), dtype=torch.int8, device=w.device)
    s = torch.empty((rows, cols // g), dtype=torch.float32, device=w.device)
    _check(lib.m3_quantize_int8(_ptr(w.contiguous()), rows, cols, g, _ptr(q), _ptr(s),
                                _stream(stream)))
    return q, s


def m3_export_weight(ctx: int, which: int, layer: int, rows: int, cols: int, int8: bool,
                     nscales: int = 1):
    q = torch.empty((rows, cols), dtype=torch.int8 if int8 else torch.int16)
    s = torch.empty((rows, nscales), dtype=torch.float32)
    _check(lib.m3_export_weight(ctx, which, layer, q.data_ptr(), s.data_ptr()))
    return q, s


def m3_frame_bytes(ctx: int, rows: int, ctx_len: int) -> float:
    return lib.m3_frame_bytes(ctx, rows, ctx_len)


def m3_frame_kernels(ctx: int, rows: int) -> int:
    n = lib.m3_frame_kernels(ctx, rows)
    if n < 0:
        _check(n)
    return n


def m3_depth_kernels(ctx: int, rows: int) -> int:
    n = lib.m3_depth_kernels(ctx, rows)
    if n < 0:
        _check(n)
    return n


def m3_time_gemv(ctx: int, which: int, rows: int, iters: int):
    """(mean ms per launch, algorithmic bytes per launch) of one GEMV kind."""
    ms = C.c_float()
    b = C.c_double()
    _check(lib.m3_time_gemv(ctx, which, rows, iters, C.byref(ms), C.byref(b)))
    return ms.value, b.value


def m3_sample_noalloc(ctx: int, h: torch.Tensor, seed: int, frame: int, cfg_scale: float,
                      temperature: float, codes: torch.Tensor,
                      logits: torch.Tensor | None = None) -> None:
    """The allocation-free draw on a final-normed hidden state (see m3.h)."""
    _check(lib.m3_sample_noalloc(ctx, h.shape[0], _ptr(h), seed, frame, cfg_scale, temperature,
                                 _ptr(codes), _ptr(logits)))


def m3_set_top_k(ctx: int, top_k: int) -> None:
    """Top-k filter of the frame draw (0 keeps every logit); see m3.h."""
    _check(lib.m3_set_top_k(ctx, top_k))


def m3_load_feedback(ctx: int, tok_emb: torch.Tensor, audio_emb=None) -> None:
    """The generation loop's feedback tables (see m3.h): tok_emb [slice_len, H]
    and the residual codebooks' audio_emb tables [depth_vocab, H], bf16."""
    keep = [tok_emb.contiguous()] + [a.contiguous() for a in (audio_emb or [])]
    arr = (C.c_void_p * max(1, len(keep) - 1))(*[t.data_ptr() for t in keep[1:]])
    _check(lib.m3_load_feedback(ctx, keep[0].data_ptr(), arr if audio_emb else None,
                                M3_MEM_DEVICE if tok_emb.is_cuda else M3_MEM_HOST))


def m3_generate(ctx: int, positions, seed: int, frame0: int, x_in: torch.Tensor,
                cfg_scale: float, temperature: float, max_frames: int, codes: torch.Tensor,
                h_hist: torch.Tensor | None = None):
    """The GPU generation loop (see m3.h).  codes: int32 [max_frames, rows, 1 + NC]
    on the GPU.  Returns (status, n_frames per key): status is M3_OK or M3_EEMPTY;
    any other status raises."""
    rows = x_in.shape[0]
    keys = rows // 2 if cfg_scale > 0 else rows
    pos = (C.c_int32 * rows)(*[int(p) for p in positions])
    nf = (C.c_int32 * keys)()
    rc = lib.m3_generate(ctx, rows, C.cast(pos, C.c_void_p), seed, frame0, _ptr(x_in), cfg_scale,
                         temperature, max_frames, _ptr(codes), _ptr(h_hist),
                         C.cast(nf, C.c_void_p))
    if rc not in (M3_OK, M3_EEMPTY):
        _check(rc)
    return rc, [int(v) for v in nf]


def m3_prefill(ctx: int, row: int, start: int, x: torch.Tensor,
               h_last: torch.Tensor | None = None) -> None:
    """Prompt prefill of cache row `row` (see m3.h): x bf16 [n_tokens, H] on the GPU."""
    _check(lib.m3_prefill(ctx, row, start, x.shape[0], _ptr(x.contiguous()), _ptr(h_last)))


def m3_gumbel_fill(seed: int, frame: int, row: int, index0: int, n: int,
                   stream=None) -> torch.Tensor:
    """The device's Gumbel noise G(seed, frame, row, index0 + i), i < n (see m3.h)."""
    out = torch.empty(n, dtype=torch.float32, device="cuda")
    _check(lib.m3_gumbel_fill(seed, frame, row, index0, n, _ptr(out), _stream(stream)))
    return out


def m3_inject_fault(ctx: int, kind: int, nth: int = 1) -> None:
    """Make the nth next call of `kind` fail on the host (see m3.h)."""
    _check(lib.m3_inject_fault(ctx, kind, nth))


def m3_stalled_wait(ctx: int, polls: int) -> None:
    """A kernel whose bounded wait is never satisfied (see m3.h); the next
    m3_sync_status raises M3_ETIMEOUT."""
    _check(lib.m3_stalled_wait(ctx, polls))


def m3_sync_status(ctx: int) -> None:
    _check(lib.m3_sync_status(ctx))


def m3_destroy(ctx: int) -> None:
    lib.m3_destroy(ctx)


def config_from_shapes(body, depth=None, max_rows: int = 2) -> m3_config:
    c = m3_config()
    c.hidden, c.n_layers = body.hidden, body.n_layers
    c.n_q_heads, c.n_kv_heads, c.head_dim, c.ffn = (body.n_q_heads, body.n_kv_heads,
                                                    body.head_dim, body.ffn)
    c.vocab, c.slice_start, c.slice_len = body.vocab, body.slice_start, body.slice_len
    c.rope_theta, c.rms_eps, c.max_rows = body.rope_theta, body.rms_eps, max_rows
    end = getattr(body, "end_token", -1)
    c.has_end_token, c.end_token = (1, end) if end >= 0 else (0, 0)
    if depth is not None:
        c.depth_layers, c.depth_hidden, c.depth_heads = depth.n_layers, depth.hidden, depth.n_heads
        c.depth_head_dim, c.depth_ffn = depth.head_dim, depth.ffn
        c.depth_codebooks, c.depth_vocab = depth.codebooks, depth.vocab
        c.depth_rope_theta = depth.rope_theta
    return c


def m3_last_error() -> str:
    return lib.m3_last_error().decode()
