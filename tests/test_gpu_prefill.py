"""GPU parity of the prompt prefill (m3_prefill) against the CPU oracle.

Prefilling tokens at positions start .. start + n - 1 is defined as decoding
them one by one (each token attends to every earlier position of its row and
to itself); the oracle runs exactly that, token by token, through its
single-row layers.  With M3_PREFILL_TC=1 (the default for bf16 weights) the
GPU runs the prompt in chunks (2048 tokens by default for bf16 weights, 256
for int8) whose projections are tcgen05 GEMMs -- for bf16 the TMA-fed kernel
over a row-major copy of the weights, single CTAs or CTA pairs by shape --
with a causal attention over the row's cache; M3_PREFILL_TC=0 (the default
for int8) selects the decode GEMV kernels over chunks of up to max_rows
tokens.  Compared:
  * the K/V the prefill leaves in the row's cache (every layer, position);
  * the final-normed hidden state of the last token;
  * the other rows' caches, untouched;
  * a decode frame on the prefilled cache (logits, teacher-forced codes).
Tolerance: the bf16 logit bar, 2e-2 of the largest magnitude.
"""
import dataclasses

import numpy as np
import pytest
import torch

import synth
from gpu_util import Model, bits, check_codes_teacher_forced, f32, rel_err

pytestmark = pytest.mark.gpu

TWO_LAYERS = dataclasses.replace(synth.TINY, n_layers=2)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


@pytest.mark.parametrize("start,n,max_rows,wdtype,tc,chunk", [
    (3, 37, 16, 0, "1", 256), (0, 1, 2, 0, "1", 256), (5, 20, 8, 1, "1", 256),
    (2, 70, 4, 0, "1", 32),     # three chunks, the last one ragged
    (0, 200, 16, 0, "1", 256),  # two token tiles of the GEMM, the second ragged
    (0, 600, 16, 0, "1", 2048),  # one chunk on CTA pairs: 256-token tiles, the last ragged
    (1, 150, 4, 1, "1", 64),    # int8, chunks of 64
    (3, 37, 16, 0, "0", 256), (5, 20, 8, 1, "0", 256)])  # the GEMV prefill
def test_prefill_matches_sequential_decode(ora, start, n, max_rows, wdtype, tc, chunk,
                                           monkeypatch):
    monkeypatch.setenv("M3_PREFILL_TC", tc)
    monkeypatch.setenv("M3_PREFILL_CHUNK", str(chunk))
    s = TWO_LAYERS
    m = Model(s, seed=21, max_rows=max_rows, wdtype=wdtype)
    try:
        kc, vc = m.kv_setup(rows=2, n_prefill=start, max_pos=start + n + 8, bucket=32)
        xs = synth.normal((n, s.hidden), 21, "prompt", std=0.02)
        h_last = torch.empty(s.hidden, dtype=torch.bfloat16, device="cuda")
        m.m3.m3_prefill(m.ctx, 1, start, xs.cuda(), h_last)
        torch.cuda.synchronize()
        m.m3.m3_sync_status(m.ctx)
        # the oracle: the tokens one by one into row 1
        k1, v1 = kc[1:2], vc[1:2]
        xb = bits(xs)
        x_out = None
        for t in range(n):
            x_out = m.ora.body(k1, v1, [start + t], xb[t:t + 1].copy())
        npos = start + n
        gk, gv = m.m3.m3_kv_get(m.ctx, 1, s.n_layers, npos, s.n_kv_heads, s.head_dim)
        gk = gk.numpy().view(np.uint16)
        gv = gv.numpy().view(np.uint16)
        for l in range(s.n_layers):
            assert rel_err(f32(gk[l]), f32(kc[1, l, :npos])) <= 2e-2, ("K", l)
            assert rel_err(f32(gv[l]), f32(vc[1, l, :npos])) <= 2e-2, ("V", l)
        # the last token's final-normed hidden state
        href = ora.rmsnorm(f32(x_out[0]), bits(m.final_norm), s.rms_eps)
        assert rel_err(f32(bits(h_last)), href) <= 2e-2
        # row 0 untouched
        if start:
            g0, _ = m.m3.m3_kv_get(m.ctx, 0, s.n_layers, start, s.n_kv_heads, s.head_dim)
            assert np.array_equal(g0.numpy().view(np.uint16), kc[0, :, :start])
        # a frame decoded on the prefilled cache
        pos = [start, npos]
        x = synth.frame_input(s, 2, 22, 0)
        codes, h, lg = m.decode(pos, seed=4, frame=7, x_in=x)
        oc, oh, olg = m.ora.decode_frame(kc, vc, pos, 4, 7, bits(x))
        assert rel_err(lg, olg) <= (2e-2 if wdtype == 0 else 5e-2)
        check_codes_teacher_forced(m, h, codes, 4, 7)
    finally:
        m.close()


@pytest.mark.parametrize("wdtype", [0, 1])
def test_prefill_8b_layer(ora, wdtype, monkeypatch):
    # one Qwen3-8B layer, 160 prompt tokens: the GEMMs at full width (K up to
    # 12288, 48 to 192 weight blocks), two token tiles with a ragged second
    monkeypatch.setenv("M3_PREFILL_TC", "1")
    s = synth.LAYER8B
    m = Model(s, seed=23, device="cuda", wdtype=wdtype, max_rows=2)
    try:
        start, n = 8, 160
        kc, vc = m.kv_setup(rows=1, n_prefill=start, max_pos=start + n + 4, bucket=64)
        xs = synth.normal((n, s.hidden), 23, "prompt8b", std=0.02)
        h_last = torch.empty(s.hidden, dtype=torch.bfloat16, device="cuda")
        m.m3.m3_prefill(m.ctx, 0, start, xs.cuda(), h_last)
        torch.cuda.synchronize()
        m.m3.m3_sync_status(m.ctx)
        xb = bits(xs)
        x_out = None
        for t in range(n):
            x_out = m.ora.body(kc, vc, [start + t], xb[t:t + 1].copy())
        npos = start + n
        gk, gv = m.m3.m3_kv_get(m.ctx, 0, s.n_layers, npos, s.n_kv_heads, s.head_dim)
        tol = 2e-2 if wdtype == 0 else 5e-2
        assert rel_err(f32(gk.numpy().view(np.uint16)[0]), f32(kc[0, 0, :npos])) <= tol
        assert rel_err(f32(gv.numpy().view(np.uint16)[0]), f32(vc[0, 0, :npos])) <= tol
        href = ora.rmsnorm(f32(x_out[0]), bits(m.final_norm), s.rms_eps)
        assert rel_err(f32(bits(h_last)), href) <= tol
    finally:
        m.close()


def test_prefill_argument_errors(ora):
    from autoregressive_audio_token_b200 import m3
    s = TWO_LAYERS
    m = Model(s, seed=2, max_rows=4, oracle=False)
    try:
        x = synth.normal((10, s.hidden), 2, "p", std=0.02).cuda()
        with pytest.raises(m3.M3Error) as e:  # no KV cache yet
            m3.m3_prefill(m.ctx, 0, 0, x)
        assert e.value.code == m3.M3_ESTATE
        m3.m3_kv_alloc(m.ctx, 1, 16, 0, 32)
        with pytest.raises(m3.M3Error) as e:  # 10 + 10 > 16 positions
            m3.m3_prefill(m.ctx, 0, 10, x)
        assert e.value.code == m3.M3_ECAPACITY
        with pytest.raises(m3.M3Error) as e:
            m3.m3_prefill(m.ctx, 1, 0, x)  # row 1 of a one-row cache
        assert e.value.code == m3.M3_EINVAL
        m3.m3_sync_status(m.ctx)
    finally:
        m.close()


def test_prefill_after_reloading_a_layer(ora):
    # the GEMM prefill reads a row-major copy of the bf16 weights made at the
    # first prefill; reloading a layer must retire that layer's copy
    s = TWO_LAYERS
    m = Model(s, seed=31, max_rows=2)
    try:
        m.m3.m3_kv_alloc(m.ctx, 1, 64, 0, 32)
        xs = synth.normal((24, s.hidden), 31, "prompt", std=0.02)
        h1 = torch.empty(s.hidden, dtype=torch.bfloat16, device="cuda")
        m.m3.m3_prefill(m.ctx, 0, 0, xs.cuda(), h1)
        new = synth.layer_weights(s, 32, 1)
        m.m3.m3_load_weights(m.ctx, [{k: v.cuda() for k, v in new.items()}], first_layer=1)
        h2 = torch.empty_like(h1)
        m.m3.m3_prefill(m.ctx, 0, 0, xs.cuda(), h2)
        torch.cuda.synchronize()
        m.m3.m3_sync_status(m.ctx)
        body = ora.Body(s, [m.layers[0], new], m.final_norm, m.lm)
        kc, vc = body.new_cache(1, 64)
        xb = bits(xs)
        for t in range(24):
            x_out = body.body(kc, vc, [t], xb[t:t + 1].copy())
        href = ora.rmsnorm(f32(x_out[0]), bits(m.final_norm), s.rms_eps)
        assert rel_err(f32(bits(h2)), href) <= 2e-2
        assert not np.array_equal(bits(h1), bits(h2))
    finally:
        m.close()
