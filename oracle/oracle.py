"""ctypes wrapper around the CPU oracle (oracle/m3_oracle.cpp).

TEST INFRASTRUCTURE ONLY: the test-suite, the package smoke check and the
benchmark's CPU-baseline leg may import this module; the product path never
does.  Arrays cross as numpy buffers of raw bits: bf16 / f16 as uint16.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from . import build as _build

_lib = None


class OraMat(C.Structure):
    _fields_ = [("w", C.c_void_p), ("q", C.c_void_p), ("s", C.c_void_p), ("wfmt", C.c_int)]


class OraCfg(C.Structure):
    _fields_ = [("hidden", C.c_int), ("n_layers", C.c_int), ("n_q_heads", C.c_int),
                ("n_kv_heads", C.c_int), ("head_dim", C.c_int), ("ffn", C.c_int),
                ("slice_start", C.c_int), ("slice_len", C.c_int), ("rope_theta", C.c_double),
                ("rms_eps", C.c_float), ("wfmt", C.c_int), ("kv_f16", C.c_int),
                ("has_end", C.c_int), ("end_token", C.c_int)]


class OraLayer(C.Structure):
    _fields_ = [("attn_norm", C.c_void_p), ("wq", OraMat), ("wk", OraMat), ("wv", OraMat),
                ("q_norm", C.c_void_p), ("k_norm", C.c_void_p), ("wo", OraMat),
                ("mlp_norm", C.c_void_p), ("wg", OraMat), ("wu", OraMat), ("wd", OraMat)]


class OraDepth(C.Structure):
    _fields_ = [("hidden", C.c_int), ("n_layers", C.c_int), ("n_heads", C.c_int),
                ("head_dim", C.c_int), ("ffn", C.c_int), ("codebooks", C.c_int),
                ("vocab", C.c_int), ("in_hidden", C.c_int), ("rope_theta", C.c_double),
                ("rms_eps", C.c_float), ("layers", C.POINTER(OraLayer)), ("proj", OraMat),
                ("emb", C.POINTER(C.c_void_p)), ("final_norm", C.c_void_p),
                ("heads", C.POINTER(OraMat)), ("sem_vocab", C.c_int)]


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        u64, f32, f64, i64, vp = C.c_uint64, C.c_float, C.c_double, C.c_int64, C.c_void_p
        L.ora_f2bf.restype = C.c_uint16
        L.ora_f2bf.argtypes = [f32]
        L.ora_bf2f.restype = f32
        L.ora_bf2f.argtypes = [C.c_uint16]
        L.ora_f2h.restype = C.c_uint16
        L.ora_f2h.argtypes = [f32]
        L.ora_mix64.restype = u64
        L.ora_mix64.argtypes = [u64]
        L.ora_noise_bits.restype = u64
        L.ora_noise_bits.argtypes = [u64, u64, u64, u64]
        L.ora_uniform.restype = f64
        L.ora_uniform.argtypes = [u64]
        L.ora_ln.restype = f64
        L.ora_ln.argtypes = [f64]
        L.ora_gumbel.restype = f32
        L.ora_gumbel.argtypes = [u64, u64, u64, u64]
        L.ora_quantize.restype = None
        L.ora_quantize.argtypes = [vp, i64, i64, i64, vp, vp]
        L.ora_gemv.restype = None
        L.ora_gemv.argtypes = [vp, vp, vp, C.c_int, i64, i64, vp, vp]
        L.ora_rmsnorm.restype = None
        L.ora_rmsnorm.argtypes = [vp, vp, i64, f32, vp]
        L.ora_rope.restype = None
        L.ora_rope.argtypes = [vp, C.c_int, i64, f64]
        L.ora_attention.restype = None
        L.ora_attention.argtypes = [vp, vp, vp, i64, C.c_int, vp]
        L.ora_sample.restype = C.c_int
        L.ora_sample.argtypes = [C.POINTER(OraCfg), OraMat, C.c_int, vp, u64, u64, f32, f32,
                                 C.c_int, vp, vp, vp]
        L.ora_sample_full_masked.restype = C.c_int
        L.ora_sample_full_masked.argtypes = [C.POINTER(OraCfg), vp, C.c_int, C.c_int, vp, u64,
                                             u64, f32, f32, C.c_int, vp]
        L.ora_generate.restype = C.c_int
        L.ora_generate.argtypes = [C.POINTER(OraCfg), C.POINTER(OraLayer), vp, OraMat,
                                   C.POINTER(OraDepth), vp, C.POINTER(C.c_void_p), C.c_int, i64,
                                   vp, vp, vp, u64, u64, vp, f32, f32, C.c_int, C.c_int, vp, vp,
                                   vp, vp]
        L.ora_decode_frame.restype = C.c_int
        L.ora_decode_frame.argtypes = [C.POINTER(OraCfg), C.POINTER(OraLayer), vp, OraMat,
                                       C.c_int, i64, vp, vp, vp, u64, u64, vp, f32, f32, C.c_int,
                                       vp, vp, vp]
        L.ora_body.restype = C.c_int
        L.ora_body.argtypes = [C.POINTER(OraCfg), C.POINTER(OraLayer), C.c_int, i64, vp, vp, vp,
                               vp, vp]
        L.ora_depth_decode.restype = C.c_int
        L.ora_depth_decode.argtypes = [C.POINTER(OraDepth), C.c_int, vp, vp, u64, u64, f32, f32,
                                       vp, vp, vp]
        L.ora_gumbel_argmax_draws.restype = None
        L.ora_gumbel_argmax_draws.argtypes = [vp, i64, f32, u64, u64, i64, vp]
        L.ora_topk_draw.restype = C.c_int32
        L.ora_topk_draw.argtypes = [vp, i64, i64, f32, u64, u64, u64, u64]
        L.ora_topk_draws.restype = None
        L.ora_topk_draws.argtypes = [vp, i64, i64, f32, u64, u64, i64, vp]
        L.ora_set_accum64.restype = None
        L.ora_set_accum64.argtypes = [C.c_int]
        L.ora_gumbel_fill.restype = None
        L.ora_gumbel_fill.argtypes = [u64, u64, u64, u64, i64, vp]
        L.ora_draw.restype = C.c_int
        L.ora_draw.argtypes = [vp, C.c_int, i64, f32, f32, C.c_int, u64, u64, u64, i64, u64, vp,
                               vp]
        L.ora_num_threads.restype = C.c_int
        L.ora_set_num_threads.argtypes = [C.c_int]
        _lib = L
    return _lib


# ------------------------------------------------------------ helpers -------

def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(C.c_void_p)


def bits(t) -> np.ndarray:
    """A torch bf16/f16 tensor (or uint16 ndarray) as a C-contiguous uint16 ndarray."""
    if isinstance(t, np.ndarray):
        return np.ascontiguousarray(t.view(np.uint16) if t.dtype != np.uint16 else t)
    import torch
    return np.ascontiguousarray(t.detach().cpu().contiguous().view(torch.int16).numpy()
                                .view(np.uint16))


def bf16_to_f32(u16: np.ndarray) -> np.ndarray:
    return (u16.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    L = lib()
    flat = np.asarray(x, np.float32).ravel()
    return np.array([L.ora_f2bf(float(v)) for v in flat], np.uint16).reshape(np.shape(x))


def quantize(w_bits: np.ndarray, group: int | None = None):
    """int8 weight-only quantisation; group None = one scale per row."""
    w_bits = np.ascontiguousarray(w_bits, np.uint16)
    rows, cols = w_bits.shape
    g = cols if group is None else group
    q = np.empty((rows, cols), np.int8)
    s = np.empty((rows, cols // g), np.float32)
    lib().ora_quantize(_p(w_bits), rows, cols, g, _p(q), _p(s))
    return q, (s[:, 0].copy() if group is None else s)


def gemv(w=None, q=None, s=None, wfmt=0, x=None):
    x = np.ascontiguousarray(x, np.float32)
    ref = w if wfmt == 0 else q
    rows, cols = ref.shape
    y = np.empty(rows, np.float32)
    lib().ora_gemv(_p(w) if w is not None else None, _p(q) if q is not None else None,
                   _p(s) if s is not None else None, wfmt, rows, cols, _p(x), _p(y))
    return y


def rmsnorm(x: np.ndarray, gamma_bits: np.ndarray, eps: float) -> np.ndarray:
    x = np.ascontiguousarray(x, np.float32)
    g = np.ascontiguousarray(gamma_bits, np.uint16)
    out = np.empty_like(x)
    lib().ora_rmsnorm(_p(x), _p(g), x.size, eps, _p(out))
    return out


def rope(v: np.ndarray, pos: int, theta: float) -> np.ndarray:
    v = np.array(v, np.float32, copy=True)
    lib().ora_rope(_p(v), v.size, pos, theta)
    return v


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, np.float32)
    k = np.ascontiguousarray(k, np.float32)
    v = np.ascontiguousarray(v, np.float32)
    out = np.empty(q.size, np.float32)
    lib().ora_attention(_p(q), _p(k), _p(v), k.shape[0], q.size, _p(out))
    return out


def gumbel(seed, frame, row, index) -> float:
    return lib().ora_gumbel(seed, frame, row, index)


def gumbel_argmax_draws(logits, temperature, seed, frame0, ndraws) -> np.ndarray:
    lg = np.ascontiguousarray(logits, np.float32)
    out = np.empty(ndraws, np.int32)
    lib().ora_gumbel_argmax_draws(_p(lg), lg.size, temperature, seed, frame0, ndraws, _p(out))
    return out


def topk_draw(g, k, temperature, seed, frame, key_row, index_base) -> int:
    gg = np.ascontiguousarray(g, np.float32)
    return int(lib().ora_topk_draw(_p(gg), gg.size, k, temperature, seed, frame, key_row,
                                   index_base))


def topk_draws(logits, k, temperature, seed, frame0, ndraws) -> np.ndarray:
    lg = np.ascontiguousarray(logits, np.float32)
    out = np.empty(ndraws, np.int32)
    lib().ora_topk_draws(_p(lg), lg.size, k, temperature, seed, frame0, ndraws, _p(out))
    return out


def gumbel_fill(seed, frame, row, index0, n) -> np.ndarray:
    """G(seed, frame, row, index0 + i) for i < n, fp32."""
    out = np.empty(n, np.float32)
    lib().ora_gumbel_fill(seed, frame, row, index0, n, _p(out))
    return out


def draw(logits, seed, frame, cfg_scale=0.0, temperature=1.0, top_k=0, index_base=0,
         end_i=-1, end_index=0):
    """The oracle's draw on given per-row logits [rows, n] (CFG pairs when
    cfg_scale > 0): (codes [rows], margins [rows])."""
    lg = np.ascontiguousarray(logits, np.float32)
    rows, n = lg.shape
    codes = np.empty(rows, np.int32)
    mg = np.empty(rows, np.float32)
    rc = lib().ora_draw(_p(lg), rows, n, cfg_scale, temperature, top_k, seed, frame, index_base,
                        end_i, end_index, _p(codes), _p(mg))
    if rc != 0:
        raise RuntimeError(f"ora_draw: {rc}")
    return codes, mg


class accum64:
    """Context manager: the oracle's GEMV sums in fp64 (the summation-order
    comparator) inside the block, the fp32 definition outside."""

    def __enter__(self):
        lib().ora_set_accum64(1)
        return self

    def __exit__(self, *exc):
        lib().ora_set_accum64(0)
        return False


def set_threads(n: int) -> None:
    lib().ora_set_num_threads(int(n))


def num_threads() -> int:
    return lib().ora_num_threads()


# -------------------------------------------------------- model objects -----

class _Keep:
    """Holds numpy arrays alive for as long as the ctypes structs point at them."""

    def __init__(self):
        self.arrs = []

    def __call__(self, a):
        self.arrs.append(a)
        return _p(a)


def _mat(keep, w_bits, wfmt, group=128):
    if wfmt == 0:
        return OraMat(keep(np.ascontiguousarray(w_bits, np.uint16)), None, None, 0)
    q, s = quantize(w_bits, None if wfmt == 1 else group)
    return OraMat(None, keep(q), keep(np.ascontiguousarray(s)), wfmt)


class Body:
    """The oracle's copy of a body: weights as raw bits, optionally int8-quantised
    by the oracle's own quantiser (wfmt 1 = one scale per row)."""

    def __init__(self, shape, layers: list, final_norm, lm_slice, wfmt=0, kv_f16=False,
                 lm_end_row=None):
        """lm_end_row: the end token's lm_head row [H] when shape.end_token >= 0
        (drawn as code slice_len)."""
        self.shape = shape
        self.keep = _Keep()
        k = self.keep
        self.has_end = getattr(shape, "end_token", -1) >= 0
        self.n_cand = shape.slice_len + (1 if self.has_end else 0)
        self.cfg = OraCfg(shape.hidden, shape.n_layers, shape.n_q_heads, shape.n_kv_heads,
                          shape.head_dim, shape.ffn, shape.slice_start, shape.slice_len,
                          shape.rope_theta, shape.rms_eps, wfmt, int(kv_f16),
                          int(self.has_end), int(getattr(shape, "end_token", -1)))
        if self.has_end and lm_slice is not None:
            assert lm_end_row is not None, "the end token needs its lm_head row"
            lm_slice = np.concatenate([bits(lm_slice), bits(lm_end_row).reshape(1, -1)], 0)
        arr = (OraLayer * len(layers))()
        for i, Lw in enumerate(layers):
            b = {n: bits(t) for n, t in Lw.items()}
            arr[i] = OraLayer(k(b["attn_norm"]), _mat(k, b["wq"], wfmt), _mat(k, b["wk"], wfmt),
                              _mat(k, b["wv"], wfmt), k(b["q_norm"]), k(b["k_norm"]),
                              _mat(k, b["wo"], wfmt), k(b["mlp_norm"]), _mat(k, b["wg"], wfmt),
                              _mat(k, b["wu"], wfmt), _mat(k, b["wd"], wfmt))
        self.layers = arr
        self.final_norm = bits(final_norm) if final_norm is not None else None
        self.lm = _mat(k, bits(lm_slice), wfmt) if lm_slice is not None else None

    def new_cache(self, rows: int, max_pos: int):
        s = self.shape
        shp = (rows, s.n_layers, max_pos, s.n_kv_heads, s.head_dim)
        return np.zeros(shp, np.uint16), np.zeros(shp, np.uint16)

    def decode_frame(self, kc, vc, positions, seed, frame, x_in_bits, cfg_scale=0.0,
                     temperature=1.0, top_k=0):
        rows = x_in_bits.shape[0]
        pos = np.ascontiguousarray(positions, np.int32)
        x = np.ascontiguousarray(x_in_bits, np.uint16)
        codes = np.empty(rows, np.int32)
        h = np.empty((rows, self.shape.hidden), np.uint16)
        lg = np.empty((rows, self.n_cand), np.float32)
        rc = lib().ora_decode_frame(C.byref(self.cfg), self.layers, _p(self.final_norm), self.lm,
                                    rows, kc.shape[2], _p(kc), _p(vc), _p(pos), seed, frame,
                                    _p(x), cfg_scale, temperature, top_k, _p(codes), _p(h),
                                    _p(lg))
        if rc != 0:
            raise RuntimeError(f"ora_decode_frame: {rc}")
        return codes, h, lg

    def body(self, kc, vc, positions, x_in_bits):
        rows = x_in_bits.shape[0]
        pos = np.ascontiguousarray(positions, np.int32)
        x = np.ascontiguousarray(x_in_bits, np.uint16)
        out = np.empty_like(x)
        lib().ora_body(C.byref(self.cfg), self.layers, rows, kc.shape[2], _p(kc), _p(vc),
                       _p(pos), _p(x), _p(out))
        return out

    def sample(self, h_bits, seed, frame, cfg_scale=0.0, temperature=1.0, with_margin=False,
               top_k=0):
        h = np.ascontiguousarray(h_bits, np.uint16)
        rows = h.shape[0]
        codes = np.empty(rows, np.int32)
        lg = np.empty((rows, self.n_cand), np.float32)
        mg = np.empty(rows, np.float32)
        rc = lib().ora_sample(C.byref(self.cfg), self.lm, rows, _p(h), seed, frame, cfg_scale,
                              temperature, top_k, _p(codes), _p(lg),
                              _p(mg) if with_margin else None)
        if rc != 0:
            raise RuntimeError(f"ora_sample: {rc}")
        return (codes, lg, mg) if with_margin else (codes, lg)

    def sample_full_masked(self, lm_full_bits, h_bits, seed, frame, cfg_scale=0.0,
                           temperature=1.0, top_k=0):
        h = np.ascontiguousarray(h_bits, np.uint16)
        W = np.ascontiguousarray(lm_full_bits, np.uint16)
        rows = h.shape[0]
        codes = np.empty(rows, np.int32)
        rc = lib().ora_sample_full_masked(C.byref(self.cfg), _p(W), W.shape[0], rows, _p(h), seed,
                                          frame, cfg_scale, temperature, top_k, _p(codes))
        if rc != 0:
            raise RuntimeError(f"ora_sample_full_masked: {rc}")
        return codes

    def generate(self, kc, vc, positions, seed, frame0, x_in_bits, max_frames, tok_emb,
                 depth=None, audio_emb=None, cfg_scale=0.0, temperature=1.0, top_k=0,
                 forced=None, with_h=False):
        """The multi-frame loop (ora_generate).  Returns (rc, codes [F, rows, 1+NC],
        n_frames [keys], h_hist [F, rows, H] bf16 bits or None); rc is 0 or -8
        (a key stopped at frame 0)."""
        s = self.shape
        rows = x_in_bits.shape[0]
        nc = depth.shape.codebooks if depth is not None else 0
        keys = rows // 2 if cfg_scale > 0 else rows
        pos = np.ascontiguousarray(positions, np.int32)
        x = np.ascontiguousarray(x_in_bits, np.uint16)
        te = np.ascontiguousarray(bits(tok_emb), np.uint16)
        ae = [np.ascontiguousarray(bits(a), np.uint16) for a in (audio_emb or [])]
        ap = (C.c_void_p * max(1, len(ae)))()
        for j, a in enumerate(ae):
            ap[j] = _p(a).value
        codes = np.empty((max_frames, rows, 1 + nc), np.int32)
        nf = np.empty(keys, np.int32)
        hh = np.empty((max_frames, rows, s.hidden), np.uint16) if with_h else None
        fc = None if forced is None else np.ascontiguousarray(forced, np.int32)
        rc = lib().ora_generate(C.byref(self.cfg), self.layers, _p(self.final_norm), self.lm,
                                C.byref(depth.D) if depth is not None else None, _p(te), ap,
                                rows, kc.shape[2], _p(kc), _p(vc), _p(pos), seed, frame0, _p(x),
                                cfg_scale, temperature, top_k, max_frames,
                                _p(fc) if fc is not None else None, _p(codes),
                                _p(hh) if hh is not None else None, _p(nf))
        if rc not in (0, -8):
            raise RuntimeError(f"ora_generate: {rc}")
        return rc, codes, nf, hh


class Depth:
    """The oracle's depth decoder; weights int8 with one scale per group of 128,
    quantised by the oracle's quantiser from the bf16 tensors."""

    def __init__(self, shape, w: dict):
        self.shape = shape
        self.keep = _Keep()
        k = self.keep
        arr = (OraLayer * shape.n_layers)()
        for i, Lw in enumerate(w["layers"]):
            b = {n: bits(t) for n, t in Lw.items()}
            arr[i] = OraLayer(k(b["attn_norm"]), _mat(k, b["wq"], 2), _mat(k, b["wk"], 2),
                              _mat(k, b["wv"], 2), k(b["q_norm"]), k(b["k_norm"]),
                              _mat(k, b["wo"], 2), k(b["mlp_norm"]), _mat(k, b["wg"], 2),
                              _mat(k, b["wu"], 2), _mat(k, b["wd"], 2))
        self.layers = arr
        emb = (C.c_void_p * shape.codebooks)()
        for j, e in enumerate(w["emb"]):
            emb[j] = k(bits(e)).value
        self.emb = emb
        heads = (OraMat * shape.codebooks)()
        for j, hw in enumerate(w["heads"]):
            heads[j] = _mat(k, bits(hw), 2)
        self.heads = heads
        self.D = OraDepth(shape.hidden, shape.n_layers, shape.n_heads, shape.head_dim, shape.ffn,
                          shape.codebooks, shape.vocab, shape.in_hidden, shape.rope_theta,
                          shape.rms_eps, arr, _mat(k, bits(w["proj"]), 2), emb,
                          k(bits(w["final_norm"])), heads, shape.sem_vocab)

    def decode(self, h_frame_bits, code0, seed, frame, cfg_scale=0.0, temperature=1.0,
               forced=None):
        h = np.ascontiguousarray(h_frame_bits, np.uint16)
        rows = h.shape[0]
        c0 = np.ascontiguousarray(code0, np.int32)
        codes = np.empty((rows, self.shape.codebooks), np.int32)
        lg = np.empty((rows, self.shape.codebooks, self.shape.vocab), np.float32)
        fc = None if forced is None else np.ascontiguousarray(forced, np.int32)
        rc = lib().ora_depth_decode(C.byref(self.D), rows, _p(h), _p(c0), seed, frame, cfg_scale,
                                    temperature, _p(fc) if fc is not None else None, _p(codes),
                                    _p(lg))
        if rc != 0:
            raise RuntimeError(f"ora_depth_decode: {rc}")
        return codes, lg


# ------------------------------------------------------------------- DiT ----
# The chunk-denoise DiT (oracle/dit_oracle.cpp); fp16 values cross as uint16 bits.

class OraDitCfg(C.Structure):
    _fields_ = [("width", C.c_int), ("n_layers", C.c_int), ("n_heads", C.c_int),
                ("head_dim", C.c_int), ("ffn", C.c_int), ("latent", C.c_int), ("cond", C.c_int),
                ("temb", C.c_int), ("rope_dims", C.c_int), ("rope_theta", C.c_double),
                ("ln_eps", C.c_float)]


DIT_LAYER_FIELDS = ("ln1_g", "ln1_b", "wqkv", "wo", "ln2_g", "ln2_b", "wg", "wu", "wd")


class OraDitLayer(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in DIT_LAYER_FIELDS]


class OraDitWeights(C.Structure):
    _fields_ = [("w_in", C.c_void_p), ("w_t1", C.c_void_p), ("w_t2", C.c_void_p),
                ("layers", C.POINTER(OraDitLayer)), ("lnf_g", C.c_void_p), ("lnf_b", C.c_void_p),
                ("w_out", C.c_void_p)]


def _dit_lib():
    L = lib()
    if not getattr(L, "_dit_ready", False):
        vp, i64, f32, f64 = C.c_void_p, C.c_int64, C.c_float, C.c_double
        L.ora_dit_layernorm.restype = None
        L.ora_dit_layernorm.argtypes = [vp, vp, vp, i64, f32, vp]
        L.ora_dit_rope.restype = None
        L.ora_dit_rope.argtypes = [vp, C.c_int, i64, f64]
        L.ora_dit_attention.restype = None
        L.ora_dit_attention.argtypes = [vp, vp, vp, i64, C.c_int, vp]
        L.ora_dit_time_features.restype = None
        L.ora_dit_time_features.argtypes = [f32, C.c_int, vp]
        L.ora_dit_layers.restype = C.c_int
        L.ora_dit_layers.argtypes = [C.POINTER(OraDitCfg), C.POINTER(OraDitLayer), C.c_int,
                                     C.c_int, C.c_int, vp]
        L.ora_dit_forward.restype = C.c_int
        L.ora_dit_forward.argtypes = [C.POINTER(OraDitCfg), C.POINTER(OraDitWeights), C.c_int,
                                      C.c_int, vp, f32, vp, vp]
        L.ora_dit_guide_step.restype = None
        L.ora_dit_guide_step.argtypes = [i64, vp, vp, vp, f32, f32, f32, vp, vp]
        L.ora_dit_step.restype = C.c_int
        L.ora_dit_step.argtypes = [C.POINTER(OraDitCfg), C.POINTER(OraDitWeights), C.c_int, vp,
                                   vp, vp, f32, f32, f32, vp, vp, vp]
        L._dit_ready = True
    return L


def h16(t) -> np.ndarray:
    """fp16 tensor / array as C-contiguous uint16 bits."""
    return bits(t)


def f16_to_f32(u16: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(u16, np.uint16).view(np.float16).astype(np.float32)


def dit_layernorm(x, g_bits, b_bits, eps) -> np.ndarray:
    x = np.ascontiguousarray(x, np.float32)
    out = np.empty_like(x)
    _dit_lib().ora_dit_layernorm(_p(x), _p(np.ascontiguousarray(g_bits, np.uint16)),
                                 _p(np.ascontiguousarray(b_bits, np.uint16)), x.size, eps, _p(out))
    return out


def dit_rope(v, rot, pos, theta) -> np.ndarray:
    v = np.array(v, np.float32, copy=True)
    _dit_lib().ora_dit_rope(_p(v), rot, pos, theta)
    return v


def dit_attention(q, k, v) -> np.ndarray:
    q, k, v = (np.ascontiguousarray(a, np.float32) for a in (q, k, v))
    T, d = q.shape
    out = np.empty((T, d), np.float32)
    _dit_lib().ora_dit_attention(_p(q), _p(k), _p(v), T, d, _p(out))
    return out


def dit_time_features(t, temb) -> np.ndarray:
    out = np.empty(temb, np.float32)
    _dit_lib().ora_dit_time_features(t, temb, _p(out))
    return out


def dit_guide_step(x, vc_bits, vu_bits, cfg_scale, sigma, sigma_next):
    x = np.ascontiguousarray(x, np.float32)
    xn = np.empty_like(x)
    vg = np.empty_like(x)
    _dit_lib().ora_dit_guide_step(x.size, _p(x), _p(np.ascontiguousarray(vc_bits, np.uint16)),
                                  _p(np.ascontiguousarray(vu_bits, np.uint16)), cfg_scale, sigma,
                                  sigma_next, _p(xn), _p(vg))
    return xn, vg


class Dit:
    """The oracle's DiT: fp16 weights (synth.dit_weights) as raw bits."""

    def __init__(self, shape, w: dict):
        self.shape = shape
        self.keep = _Keep()
        k = self.keep
        self.cfg = OraDitCfg(shape.width, shape.n_layers, shape.n_heads, shape.head_dim,
                             shape.ffn, shape.latent, shape.cond, shape.temb, shape.rope_dims,
                             shape.rope_theta, shape.ln_eps)
        arr = (OraDitLayer * max(1, len(w["layers"])))()
        for i, Lw in enumerate(w["layers"]):
            arr[i] = OraDitLayer(*[k(h16(Lw[n])) for n in DIT_LAYER_FIELDS])
        self.layers = arr
        self.W = OraDitWeights(k(h16(w["w_in"])), k(h16(w["w_t1"])), k(h16(w["w_t2"])), arr,
                               k(h16(w["lnf_g"])), k(h16(w["lnf_b"])), k(h16(w["w_out"])))

    def layers_forward(self, h_bits, B, T, first=0, n=None):
        """Blocks first..first+n on h [B, T, W] (fp16 bits); returns the new bits."""
        h = np.ascontiguousarray(h_bits, np.uint16).copy()
        n = self.shape.n_layers - first if n is None else n
        sub = C.cast(C.byref(self.layers, first * C.sizeof(OraDitLayer)), C.POINTER(OraDitLayer))
        rc = _dit_lib().ora_dit_layers(C.byref(self.cfg), sub, n, B, T, _p(h))
        if rc:
            raise RuntimeError(f"ora_dit_layers: {rc}")
        return h

    def forward(self, h_in_bits, B, T, t, with_h=False):
        s = self.shape
        hin = np.ascontiguousarray(h_in_bits, np.uint16)
        v = np.empty((B, T, s.latent), np.uint16)
        hl = np.empty((B, T, s.width), np.uint16) if with_h else None
        rc = _dit_lib().ora_dit_forward(C.byref(self.cfg), C.byref(self.W), B, T, _p(hin), t,
                                        _p(v), _p(hl) if with_h else None)
        if rc:
            raise RuntimeError(f"ora_dit_forward: {rc}")
        return (v, hl) if with_h else v

    def step(self, x, ctx_bits, cond_bits, sigma, sigma_next, cfg_scale):
        """One denoising step: (x_next fp32 [T, latent], guided v fp32, v_pair f16 bits)."""
        s = self.shape
        x = np.ascontiguousarray(x, np.float32)
        T = x.shape[0]
        xn = np.empty_like(x)
        vg = np.empty_like(x)
        vp = np.empty((2, T, s.latent), np.uint16)
        rc = _dit_lib().ora_dit_step(C.byref(self.cfg), C.byref(self.W), T, _p(x),
                                     _p(np.ascontiguousarray(ctx_bits, np.uint16)),
                                     _p(np.ascontiguousarray(cond_bits, np.uint16)), sigma,
                                     sigma_next, cfg_scale, _p(xn), _p(vg), _p(vp))
        if rc:
            raise RuntimeError(f"ora_dit_step: {rc}")
        return xn, vg, vp
