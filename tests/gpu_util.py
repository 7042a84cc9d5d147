"""Shared set-up for the GPU parity tests: the same seeded tensors go to the
CUDA library (through the C ABI) and to the CPU oracle."""
from __future__ import annotations

import numpy as np
import torch

import synth


def bits(t) -> np.ndarray:
    from oracle.oracle import bits as _b
    return _b(t)


def f32(bits_u16: np.ndarray) -> np.ndarray:
    return (bits_u16.astype(np.uint32) << 16).view(np.float32)


def rel_err(got: np.ndarray, ref: np.ndarray) -> float:
    return float(np.max(np.abs(got.astype(np.float64) - ref.astype(np.float64))) /
                 max(np.max(np.abs(ref.astype(np.float64))), 1e-30))


class Model:
    """Body weights drawn once; handed to the library and to the oracle."""

    def __init__(self, shape, seed=0, device="cpu", wdtype=0, kv_f16=False, max_rows=2,
                 depth=None, depth_seed=None, layers=None, oracle=True, end_row=None):
        from autoregressive_audio_token_b200 import m3
        self.m3 = m3
        self.shape = shape
        self.layers = layers if layers is not None else \
            [synth.layer_weights(shape, seed, l, device=device) for l in range(shape.n_layers)]
        self.final_norm = synth.final_norm(shape, seed, device=device)
        self.lm = synth.lm_head_slice(shape, seed, device=device)
        self.has_end = getattr(shape, "end_token", -1) >= 0
        self.n_cand = shape.slice_len + (1 if self.has_end else 0)
        self.lm_end = (end_row if end_row is not None else
                       synth.lm_head_end_row(shape, seed, device=device)) if self.has_end else None
        self.wdtype = wdtype
        self.kv_f16 = kv_f16
        self.depth_shape = depth
        self.dw = synth.depth_weights(depth, depth_seed if depth_seed is not None else seed + 7,
                                      device=device) if depth is not None else None
        cfg = m3.config_from_shapes(shape, depth, max_rows=max_rows)
        self.ctx = m3.m3_create(cfg)
        m3.m3_load_weights(self.ctx, [{k: v.cuda() for k, v in L.items()} for L in self.layers]
                           if device == "cpu" else self.layers, 0, self.final_norm.cuda(),
                           self.lm.cuda(), wdtype=wdtype,
                           lm_end_row=self.lm_end.cuda() if self.has_end else None)
        if self.dw is not None:
            dwc = {"layers": [{k: v.cuda() for k, v in L.items()} for L in self.dw["layers"]],
                   "proj": self.dw["proj"].cuda(), "emb": [e.cuda() for e in self.dw["emb"]],
                   "final_norm": self.dw["final_norm"].cuda(),
                   "heads": [h.cuda() for h in self.dw["heads"]]}
            m3.m3_load_depth_weights(self.ctx, dwc)
        self.ora = None
        if oracle:
            from oracle import oracle as O
            self.ora = O.Body(shape, [{k: v.cpu() for k, v in L.items()} for L in self.layers],
                              self.final_norm.cpu(), self.lm.cpu(), wfmt=1 if wdtype else 0,
                              kv_f16=kv_f16,
                              lm_end_row=self.lm_end.cpu() if self.has_end else None)
            self.ora_depth = O.Depth(depth, {"layers": [{k: v.cpu() for k, v in L.items()}
                                                        for L in self.dw["layers"]],
                                             "proj": self.dw["proj"].cpu(),
                                             "emb": [e.cpu() for e in self.dw["emb"]],
                                             "final_norm": self.dw["final_norm"].cpu(),
                                             "heads": [h.cpu() for h in self.dw["heads"]]}) \
                if self.dw is not None else None

    def close(self):
        if self.ctx:
            self.m3.m3_destroy(self.ctx)
            self.ctx = None

    def kv_setup(self, rows, n_prefill, max_pos, seed=0, bucket=256):
        m3 = self.m3
        m3.m3_kv_alloc(self.ctx, rows, max_pos, 1 if self.kv_f16 else 0, bucket)
        K, V = synth.kv_prefill(self.shape, rows, n_prefill, seed)
        kc = vc = None
        if self.ora is not None:
            kc, vc = self.ora.new_cache(rows, max_pos)
        for r in range(rows):
            if n_prefill:
                m3.m3_kv_set(self.ctx, r, K[r].cuda(), V[r].cuda())
            if kc is not None and n_prefill:
                kb, vb = bits(K[r]), bits(V[r])
                if self.kv_f16:
                    kb = f32(kb).astype(np.float16).view(np.uint16)
                    vb = f32(vb).astype(np.float16).view(np.uint16)
                kc[r, :, :n_prefill] = kb
                vc[r, :, :n_prefill] = vb
        return kc, vc

    def decode(self, positions, seed, frame, x_in, cfg_scale=0.0, temperature=1.0):
        rows = x_in.shape[0]
        s = self.shape
        codes = torch.empty(rows, dtype=torch.int32, device="cuda")
        h = torch.empty((rows, s.hidden), dtype=torch.bfloat16, device="cuda")
        lg = torch.empty((rows, self.n_cand), dtype=torch.float32, device="cuda")
        self.m3.m3_decode_frame(self.ctx, positions, seed, frame, x_in.cuda().contiguous(),
                                cfg_scale, temperature, codes, h, lg)
        torch.cuda.synchronize()
        self.m3.m3_sync_status(self.ctx)
        return codes.cpu().numpy(), bits(h), lg.cpu().numpy()


def check_codes_teacher_forced(model, h_bits, gpu_codes, seed, frame, cfg_scale=0.0,
                               temperature=1.0, margin_tol=1e-3):
    """Run the oracle's sampler on the GPU's own final hidden state; codes must
    agree by the draw rule of check_draws."""
    codes, _lg, margin = model.ora.sample(h_bits, seed, frame, cfg_scale, temperature,
                                          with_margin=True)
    return check_draws(codes, margin, gpu_codes, margin_tol)


def check_draws(codes_ora, margins, gpu_codes, margin_tol=1e-3):
    """The code rule of the parity tests: codes identical on >= 99.9 % of the
    draws, and every mismatch with an oracle top-2 perturbed-logit margin
    below margin_tol.  Returns the number of mismatches."""
    codes_ora = np.asarray(codes_ora).ravel()
    gpu_codes = np.asarray(gpu_codes).ravel()
    margins = np.asarray(margins).ravel()
    mism = codes_ora != gpu_codes
    assert np.all(margins[mism] < margin_tol), (codes_ora[mism], gpu_codes[mism], margins[mism])
    assert mism.sum() <= int(0.001 * mism.size), (int(mism.sum()), mism.size)
    return int(mism.sum())


def check_depth_draws(glg, gpu_codes, seed, frame, cfg_scale=0.0, temperature=1.0):
    """The depth decoder's draws, teacher-forced: codebook j (1-based) of every
    row drawn by the oracle's sampler from the GPU's own logits glg
    [rows, codebooks, vocab] with noise index (j << 32) | i, against the GPU's
    codes [rows, codebooks]."""
    from oracle import oracle as O
    rows, nc, _ = glg.shape
    oc = np.empty((rows, nc), np.int32)
    om = np.empty((rows, nc), np.float32)
    for j in range(nc):
        oc[:, j], om[:, j] = O.draw(np.ascontiguousarray(glg[:, j]), seed, frame,
                                    cfg_scale=cfg_scale, temperature=temperature,
                                    index_base=(j + 1) << 32)
    return check_draws(oc, om, gpu_codes)
