"""Pins for the DiT chunk-denoise oracle (oracle/dit_oracle.cpp).

Each pin checks a part of the oracle against something other than itself:
closed forms, fp64 restatements of the pages' definitions, invariants, and
compositions that must agree bit for bit.

* Batch-2 == two batch-1 forwards (the diffusers issue, finding 3: the
  cond/uncond pair as one batch-2 forward is formula-identical).
* Guided velocity uncond + c (cond - uncond) and the Euler step
  (DiffSynth-Studio article, "第三阶段"): c = 1 gives cond, c = 0 uncond;
  30 steps of a constant field over sigma 1 -> 0 move x by -v.
* LayerNorm, partial RoPE, bidirectional attention, Fourier timestep
  features, the GLU block: fp64 restatements and invariants.
* Wiring: with every block's output projections zero the forward reduces to
  W_out LN(W_in h_in + temb), checked in fp64; the input concatenation order;
  L blocks == L one-block calls chained.
"""
import numpy as np
import pytest
import torch

import synth

S = synth.DIT_TINY


def _f16(x):
    """fp64 -> fp32 -> fp16 (RNE) -> fp64."""
    return np.asarray(x, np.float64).astype(np.float32).astype(np.float16).astype(np.float64)


def _bits16(x):
    return np.asarray(x, np.float32).astype(np.float16).view(np.uint16)


def _vals(t):
    return t.float().numpy().astype(np.float64)


def _hin(T, B, seed):
    Cin = 2 * S.latent + S.cond
    return synth.normal((B, T, Cin), seed, "pin/hin", dtype=torch.float16)


# ------------------------------------------------------------- the pieces ----

def test_layernorm_fp64(ora):
    rng = np.random.default_rng(0)
    for n in (128, 2048):
        x = _f16(rng.standard_normal(n) * 3 + 1.5).astype(np.float32)
        g = _f16(1 + 0.1 * rng.standard_normal(n))
        b = _f16(0.1 * rng.standard_normal(n))
        got = ora.dit_layernorm(x, _bits16(g), _bits16(b), 1e-5).astype(np.float64)
        xd = x.astype(np.float64)
        ref = (xd - xd.mean()) / np.sqrt(xd.var() + 1e-5) * g + b
        assert np.all(np.abs(got - ref) <= 2.0 ** -10 * np.abs(ref) + 1e-6)
        # gain 1, bias 0: zero mean, unit variance (to f16 rounding)
        one, zero = _bits16(np.ones(n)), _bits16(np.zeros(n))
        y = ora.dit_layernorm(x, one, zero, 1e-5).astype(np.float64)
        assert abs(y.mean()) < 1e-3 and abs(y.var() - 1) < 2e-3
        # shift invariance by an exactly representable constant
        y2 = ora.dit_layernorm((x + np.float32(4.0)), one, zero, 1e-5)
        assert np.max(np.abs(y2 - y)) <= 2.0 ** -9


def test_partial_rope(ora):
    rng = np.random.default_rng(1)
    d, rot, theta = 64, 32, 1e4
    v = _f16(rng.standard_normal(d)).astype(np.float32)
    assert np.array_equal(ora.dit_rope(v, rot, 0, theta), v)  # position 0: identity
    for pos in (1, 7, 688):
        r = ora.dit_rope(v, rot, pos, theta).astype(np.float64)
        assert np.array_equal(r[rot:], v[rot:])  # the unrotated dims pass through
        h = rot // 2
        ang = pos * theta ** (-2.0 * np.arange(h) / rot)
        a, b = v[:h].astype(np.float64), v[h:rot].astype(np.float64)
        ref = np.concatenate([a * np.cos(ang) - b * np.sin(ang), b * np.cos(ang) + a * np.sin(ang)])
        assert np.all(np.abs(r[:rot] - ref) <= 2.0 ** -10 * np.abs(ref) + 1e-4)
        assert abs(np.linalg.norm(r[:rot]) - np.linalg.norm(v[:rot])) < 2e-3 * np.linalg.norm(v)
    # relative positions: <R_m q, R_n k> depends on m - n only
    q = _f16(rng.standard_normal(d)).astype(np.float32)
    k = _f16(rng.standard_normal(d)).astype(np.float32)
    dots = [float(ora.dit_rope(q, rot, m, theta).astype(np.float64) @
                  ora.dit_rope(k, rot, m - 3, theta).astype(np.float64)) for m in (3, 10, 50)]
    assert max(dots) - min(dots) < 2e-2


def test_attention_fp64_and_bidirectional(ora):
    rng = np.random.default_rng(2)
    T, d = 37, 64
    q, k, v = (_f16(rng.standard_normal((T, d))).astype(np.float32) for _ in range(3))
    got = ora.dit_attention(q, k, v).astype(np.float64)
    s = q.astype(np.float64) @ k.astype(np.float64).T / 8.0
    p = np.exp(s - s.max(1, keepdims=True))
    ref = (p / p.sum(1, keepdims=True)) @ v.astype(np.float64)
    assert np.max(np.abs(got - ref)) <= 4e-3 * np.max(np.abs(ref))
    # one token: o = v_0; equal keys: the mean of V
    assert np.array_equal(ora.dit_attention(q[:1], k[:1], v[:1]), _f16(v[:1]).astype(np.float32))
    eq = ora.dit_attention(q, np.repeat(k[:1], T, 0), v).astype(np.float64)
    assert np.max(np.abs(eq - v.astype(np.float64).mean(0))) < 2e-3
    # not causal: the first token sees the last one
    v2 = v.copy()
    v2[-1] += 1.0
    assert not np.array_equal(ora.dit_attention(q, k, v2)[0], got[0].astype(np.float32))


def test_time_features(ora):
    f0 = ora.dit_time_features(0.0, 256)
    assert np.array_equal(f0[:128], np.ones(128, np.float32))
    assert np.array_equal(f0[128:], np.zeros(128, np.float32))
    t = 734.0
    f = ora.dit_time_features(t, 256).astype(np.float64)
    k = np.arange(128)
    fr = np.exp(-np.log(10000.0) * k / 128)
    assert np.max(np.abs(f - np.concatenate([np.cos(t * fr), np.sin(t * fr)]))) < 1e-3
    assert f[0] == _f16(np.cos(t)) and f[128] == _f16(np.sin(t))  # frequency 1 first


def test_guide_and_euler_closed_forms(ora):
    rng = np.random.default_rng(3)
    n = 64
    x = rng.standard_normal(n).astype(np.float32)
    vc, vu = _bits16(rng.standard_normal(n)), _bits16(rng.standard_normal(n))
    xc, gc = ora.dit_guide_step(x, vc, vu, 1.0, 0.5, 0.25)
    assert np.array_equal(gc, vc.view(np.float16).astype(np.float32))  # c = 1: cond
    xu, gu = ora.dit_guide_step(x, vc, vu, 0.0, 0.5, 0.25)
    assert np.array_equal(gu, vu.view(np.float16).astype(np.float32))  # c = 0: uncond
    assert np.array_equal(xc, (x + np.float32(-0.25) * gc).astype(np.float32))
    # a constant field integrated over a 30-step schedule from sigma 1 to 0: x - v
    sig = np.linspace(1.0, 0.0, 31).astype(np.float32)
    xs = x.copy()
    for i in range(30):
        xs, _ = ora.dit_guide_step(xs, vc, vc, 1.7, sig[i], sig[i + 1])
    ref = x.astype(np.float64) - vc.view(np.float16).astype(np.float64)
    assert np.max(np.abs(xs - ref)) < 1e-5 * 30 * (np.abs(ref).max() + 1)


# -------------------------------------------------------------- the block ----

def test_glu_block_wiring(ora):
    # W_o = 0: attention adds nothing; h' = h + W_d (silu(W_g n) * W_u n), n = LN2(h)
    L = synth.dit_layer_weights(S, 0, 0)
    L["wo"] = torch.zeros_like(L["wo"])
    w = synth.dit_weights(S, 0, layers=[L])
    dit = ora.Dit(S, w)
    T = 5
    h = synth.normal((1, T, S.width), 0, "pin/h", dtype=torch.float16)
    out = ora.f16_to_f32(dit.layers_forward(ora.h16(h), 1, T, 0, 1)).astype(np.float64)
    Lv = {k: _vals(v) for k, v in L.items()}
    hv = _vals(h)[0]
    mu = hv.mean(1, keepdims=True)
    n = (hv - mu) / np.sqrt(hv.var(1, keepdims=True) + S.ln_eps) * Lv["ln2_g"] + Lv["ln2_b"]
    g, u = n @ Lv["wg"].T, n @ Lv["wu"].T
    ref = hv + (g / (1 + np.exp(-g)) * u) @ Lv["wd"].T
    err = np.abs(out[0] - ref)
    upd = np.abs(ref - hv).max()
    assert err.max() < 0.03 * upd + 2.0 ** -10 * np.abs(ref).max()
    swapped = hv + (u / (1 + np.exp(-u)) * g) @ Lv["wd"].T
    assert np.abs(out[0] - swapped).max() > 5 * err.max()


def test_attention_block_wiring(ora):
    # W_d = 0 and W_o = I: h' = h + attn(LN1 h) with partial RoPE on q, k
    L = synth.dit_layer_weights(S, 1, 0)
    L["wd"] = torch.zeros_like(L["wd"])
    L["wo"] = torch.eye(S.width, dtype=torch.float16)
    w = synth.dit_weights(S, 1, layers=[L])
    dit = ora.Dit(S, w)
    T, d, W = 9, S.head_dim, S.width
    h = synth.normal((1, T, W), 1, "pin/h", dtype=torch.float16)
    out = ora.f16_to_f32(dit.layers_forward(ora.h16(h), 1, T, 0, 1)).astype(np.float64)[0]
    Lv = {k: _vals(v) for k, v in L.items()}
    hv = _vals(h)[0]
    n = (hv - hv.mean(1, keepdims=True)) / np.sqrt(hv.var(1, keepdims=True) + S.ln_eps)
    n = n * Lv["ln1_g"] + Lv["ln1_b"]
    qkv = n @ Lv["wqkv"].T
    o = np.zeros((T, W))
    h2, rot = S.rope_dims // 2, S.rope_dims
    ang = np.arange(T)[:, None] * S.rope_theta ** (-2.0 * np.arange(h2) / rot)
    c, s_ = np.cos(ang), np.sin(ang)

    def rope(x):
        a, b = x[:, :h2], x[:, h2:rot]
        return np.concatenate([a * c - b * s_, b * c + a * s_, x[:, rot:]], 1)

    for hd in range(S.n_heads):
        q = rope(qkv[:, hd * d:(hd + 1) * d])
        k = rope(qkv[:, W + hd * d:W + (hd + 1) * d])
        v = qkv[:, 2 * W + hd * d:2 * W + (hd + 1) * d]
        sc = q @ k.T / np.sqrt(d)
        p = np.exp(sc - sc.max(1, keepdims=True))
        o[:, hd * d:(hd + 1) * d] = (p / p.sum(1, keepdims=True)) @ v
    ref = hv + o
    err = np.abs(out - ref).max()
    assert err < 0.03 * np.abs(o).max() + 2.0 ** -10 * np.abs(ref).max(), err
    # without the rotation the answer moves
    o2 = np.zeros((T, W))
    for hd in range(S.n_heads):
        q, k = qkv[:, hd * d:(hd + 1) * d], qkv[:, W + hd * d:W + (hd + 1) * d]
        v = qkv[:, 2 * W + hd * d:2 * W + (hd + 1) * d]
        sc = q @ k.T / np.sqrt(d)
        p = np.exp(sc - sc.max(1, keepdims=True))
        o2[:, hd * d:(hd + 1) * d] = (p / p.sum(1, keepdims=True)) @ v
    assert np.abs(out - (hv + o2)).max() > 3 * err


def test_forward_with_zero_blocks_closed_form(ora):
    # W_o = W_d = 0 in every block: v = W_out LN_f(f16(f16(W_in h_in) + temb(t)))
    layers = [synth.dit_layer_weights(S, 2, l) for l in range(S.n_layers)]
    for L in layers:
        L["wo"] = torch.zeros_like(L["wo"])
        L["wd"] = torch.zeros_like(L["wd"])
    w = synth.dit_weights(S, 2, layers=layers)
    dit = ora.Dit(S, w)
    T, B, t = 6, 2, 910.0
    hin = _hin(T, B, 2)
    v = ora.f16_to_f32(dit.forward(ora.h16(hin), B, T, t)).astype(np.float64)
    W = {k: _vals(w[k]) for k in ("w_in", "w_t1", "w_t2", "lnf_g", "lnf_b", "w_out")}
    k = np.arange(S.temb // 2)
    fr = np.exp(-np.log(10000.0) * k / (S.temb // 2))
    feat = np.concatenate([np.cos(t * fr), np.sin(t * fr)])
    a1 = W["w_t1"] @ feat
    temb = W["w_t2"] @ (a1 / (1 + np.exp(-a1)))
    h = _vals(hin) @ W["w_in"].T + temb
    n = (h - h.mean(-1, keepdims=True)) / np.sqrt(h.var(-1, keepdims=True) + S.ln_eps)
    ref = (n * W["lnf_g"] + W["lnf_b"]) @ W["w_out"].T
    assert np.max(np.abs(v - ref)) < 0.02 * np.abs(ref).max()
    # the concatenation order: moving the condition channels changes the answer
    hin2 = hin.clone()
    hin2[..., :S.latent], hin2[..., 2 * S.latent:3 * S.latent] = \
        hin[..., 2 * S.latent:3 * S.latent], hin[..., :S.latent]
    v2 = ora.f16_to_f32(dit.forward(ora.h16(hin2), B, T, t)).astype(np.float64)
    assert np.max(np.abs(v2 - v)) > 0.05 * np.abs(ref).max()


def test_batch2_equals_two_batch1(ora):
    w = synth.dit_weights(S, 3)
    dit = ora.Dit(S, w)
    T = 11
    hin = ora.h16(_hin(T, 2, 3))
    both = dit.forward(hin, 2, T, 500.0)
    for b in range(2):
        one = dit.forward(np.ascontiguousarray(hin[b:b + 1]), 1, T, 500.0)
        assert np.array_equal(both[b], one[0])
    # attention over the two batch elements together would differ
    joined = dit.forward(np.ascontiguousarray(hin.reshape(1, 2 * T, -1)), 1, 2 * T, 500.0)
    assert not np.array_equal(joined[0, :T], both[0])


def test_layer_stack_equals_chained_blocks(ora):
    w = synth.dit_weights(S, 4)
    dit = ora.Dit(S, w)
    T = 7
    h = ora.h16(synth.normal((2, T, S.width), 4, "pin/h", dtype=torch.float16))
    full = dit.layers_forward(h, 2, T)
    chain = h
    for l in range(S.n_layers):
        chain = dit.layers_forward(chain, 2, T, l, 1)
    assert np.array_equal(full, chain)
    # the blocks in the other order differ
    rev = h
    for l in reversed(range(S.n_layers)):
        rev = dit.layers_forward(rev, 2, T, l, 1)
    assert not np.array_equal(full, rev)


def test_step_is_forward_guide_euler(ora):
    # ora_dit_step == the batch-2 forward on [x | ctx | cond] and [x | ctx | 0],
    # then the guided Euler step, t = 1000 sigma
    w = synth.dit_weights(S, 5)
    dit = ora.Dit(S, w)
    T = 13
    x, ctx, cond = synth.dit_inputs(S, T, 5)
    xn, vg, vp = dit.step(x.numpy(), ora.h16(ctx), ora.h16(cond), 0.8, 0.75, 1.7)
    hin = torch.cat([torch.cat([x.half(), ctx, cond], 1)[None],
                     torch.cat([x.half(), ctx, torch.zeros_like(cond)], 1)[None]], 0)
    v = dit.forward(ora.h16(hin), 2, T, np.float32(0.8) * np.float32(1000.0))
    assert np.array_equal(vp, v)
    xr, gr = ora.dit_guide_step(x.numpy(), v[0], v[1], 1.7, 0.8, 0.75)
    assert np.array_equal(xn, xr) and np.array_equal(vg, gr)
