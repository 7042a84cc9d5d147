"""GPU parity of the DiT chunk-denoise step (include/m3_dit.h) against the CPU
oracle (oracle/dit_oracle.cpp), through the C ABI, on the same seeded fp16
weights and inputs.

Tolerances (fp16 activations with fp32 sums on both sides, different
summation orders and softmax blocking): blocks and the tiny forward within
1e-2 of the largest value (max-abs relative error), the velocities and the
Euler-stepped latent within 2e-2.  At full depth (36 blocks) rounding is
amplified; there the GPU's deviation must stay within max(2e-2, 1.5 x the
oracle's own response to a one-step change of one input element), and the
numbers are printed (-s).

Shapes: a tiny DiT (width 256, 4 heads of 64, FFN 512) over 40 and 200
latent frames (ragged 128-token tiles), one full-size block (width 2048,
32 heads, FFN 8192) over a whole 200-frame chunk (689 latent frames, batch
2 = 1378 tokens), and the full 36-block model over 16 frames.
"""
import dataclasses

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def _rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


def _f16(u16):
    return np.ascontiguousarray(u16).view(np.float16).astype(np.float32)


class DitPair:
    """The same weights in the library and in the oracle."""

    def __init__(self, shape, seed, max_tokens, n_layers=None, device="cpu"):
        from autoregressive_audio_token_b200 import dit as D
        from oracle import oracle as O
        self.D, self.O = D, O
        s = shape if n_layers is None else dataclasses.replace(shape, n_layers=n_layers)
        self.s = s
        w = synth.dit_weights(s, seed, device=device)
        self.h = D.m3_dit_create(D.config_from_shape(s, max_tokens))
        D.m3_dit_load(self.h, {k: ([{n: t.cuda() for n, t in L.items()} for L in v]
                                   if k == "layers" else v.cuda()) for k, v in w.items()})
        wc = {k: ([{n: t.cpu() for n, t in L.items()} for L in v] if k == "layers" else v.cpu())
              for k, v in w.items()}
        self.ora = O.Dit(s, wc)

    def close(self):
        if self.h:
            self.D.m3_dit_destroy(self.h)
            self.h = None

    def sync(self):
        torch.cuda.synchronize()
        self.D.m3_dit_sync_status(self.h)


@pytest.mark.parametrize("T,n", [(40, 1), (200, 2)])
def test_tiny_blocks(ora, T, n):
    p = DitPair(synth.DIT_TINY, 11, 256)
    try:
        B, W = 2, p.s.width
        h = synth.normal((B * T, W), 11, "gpu/h", dtype=torch.float16)
        hg = h.cuda()
        p.D.m3_dit_blocks(p.h, hg, B, T, 0, n)
        p.sync()
        ref = ora.f16_to_f32(p.ora.layers_forward(ora.h16(h), B, T, 0, n))
        err = _rel(hg.float().cpu().numpy(), ref)
        assert err <= 1e-2, err
    finally:
        p.close()


@pytest.mark.parametrize("B,T", [(2, 40), (1, 13), (2, 200)])
def test_tiny_forward(ora, B, T):
    p = DitPair(synth.DIT_TINY, 12, 256)
    try:
        s = p.s
        hin = synth.normal((B * T, 2 * s.latent + s.cond), 12, "gpu/hin", dtype=torch.float16)
        v = torch.empty((B * T, s.latent), dtype=torch.float16, device="cuda")
        p.D.m3_dit_forward(p.h, hin.cuda(), B, T, 640.0, v)
        p.sync()
        ref = ora.f16_to_f32(p.ora.forward(ora.h16(hin), B, T, 640.0))
        err = _rel(v.float().cpu().numpy(), ref.reshape(B * T, -1))
        assert err <= 2e-2, err
    finally:
        p.close()


def test_tiny_step_and_denoise(ora):
    p = DitPair(synth.DIT_TINY, 13, 256)
    try:
        s, T = p.s, 57
        x, ctx, cond = synth.dit_inputs(s, T, 13)
        xg = x.clone().cuda()
        vg = torch.empty((T, s.latent), dtype=torch.float32, device="cuda")
        vp = torch.empty((2, T, s.latent), dtype=torch.float16, device="cuda")
        p.D.m3_dit_step(p.h, xg, ctx.cuda(), cond.cuda(), 0.9, 0.85, 1.7, vg, vp)
        p.sync()
        xn, ovg, ovp = p.ora.step(x.numpy(), ora.h16(ctx), ora.h16(cond), 0.9, 0.85, 1.7)
        assert _rel(vp.float().cpu().numpy(), _f16(ovp)) <= 2e-2
        assert _rel(vg.cpu().numpy(), ovg) <= 2e-2
        assert _rel(xg.cpu().numpy() - x.numpy(), xn - x.numpy()) <= 2e-2
        # the cond and uncond predictions differ (the zero condition is used)
        assert not np.array_equal(ovp[0], ovp[1])
        # four steps of a schedule, as one call
        sig = [1.0, 0.75, 0.5, 0.25, 0.0]
        xg = x.clone().cuda()
        p.D.m3_dit_denoise(p.h, xg, ctx.cuda(), cond.cuda(), sig, 1.7)
        p.sync()
        xo = x.numpy()
        for i in range(4):
            xo, _, _ = p.ora.step(xo, ora.h16(ctx), ora.h16(cond), sig[i], sig[i + 1], 1.7)
        assert _rel(xg.cpu().numpy(), xo) <= 2e-2, _rel(xg.cpu().numpy(), xo)
        # a second T uses its own graph; the first one still runs
        x2, c2, d2 = synth.dit_inputs(s, 33, 14)
        x2g = x2.clone().cuda()
        p.D.m3_dit_step(p.h, x2g, c2.cuda(), d2.cuda(), 0.5, 0.4, 1.7)
        p.sync()
        xo2, _, _ = p.ora.step(x2.numpy(), ora.h16(c2), ora.h16(d2), 0.5, 0.4, 1.7)
        assert _rel(x2g.cpu().numpy() - x2.numpy(), xo2 - x2.numpy()) <= 2e-2
    finally:
        p.close()


def test_full_size_block_one_chunk(ora):
    # one full-size block over a whole chunk: 689 latent frames x (cond, uncond)
    T, B = synth.DIT_CHUNK_T, 2
    p = DitPair(synth.DIT, 21, T, n_layers=1, device="cuda")
    try:
        W = p.s.width
        h = synth.normal((B * T, W), 21, "gpu/h", dtype=torch.float16)
        hg = h.cuda()
        p.D.m3_dit_blocks(p.h, hg, B, T, 0, 1)
        p.sync()
        ref = ora.f16_to_f32(p.ora.layers_forward(ora.h16(h), B, T, 0, 1))
        got = hg.float().cpu().numpy()
        err = _rel(got, ref)
        print(f"\n[full-size block, T={T}] max-abs relative error {err:.2e}")
        assert err <= 1e-2, err
        # the update (h' - h) itself, which carries all of the block's arithmetic
        hv = h.float().numpy()
        assert _rel(got - hv, ref - hv) <= 2e-2
    finally:
        p.close()


@pytest.mark.slow
def test_full_depth_forward(ora):
    # all 36 blocks at full width over 16 latent frames, batch 2
    T, B = 16, 2
    p = DitPair(synth.DIT, 22, T, device="cuda")
    try:
        s = p.s
        hin = synth.normal((B * T, 2 * s.latent + s.cond), 22, "gpu/hin", dtype=torch.float16)
        v = torch.empty((B * T, s.latent), dtype=torch.float16, device="cuda")
        p.D.m3_dit_forward(p.h, hin.cuda(), B, T, 500.0, v)
        p.sync()
        hb = ora.h16(hin)
        ref = ora.f16_to_f32(p.ora.forward(hb, B, T, 500.0)).reshape(B * T, -1)
        hp = hb.copy()
        hp.reshape(-1)[0] += 1  # one input element one fp16 step up
        refp = ora.f16_to_f32(p.ora.forward(hp, B, T, 500.0)).reshape(B * T, -1)
        err = _rel(v.float().cpu().numpy(), ref)
        sens = _rel(refp, ref)
        print(f"\n[full depth, T={T}] velocity rel err {err:.4f}, oracle one-step "
              f"sensitivity {sens:.4f}")
        assert err <= max(2e-2, 1.5 * sens), (err, sens)
    finally:
        p.close()
