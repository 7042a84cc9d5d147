"""Pins for the oracle's composed decode step and sampler.

* Sliced lm_head == full lm_head with every non-sampleable row at -inf
  (diffusers issue "MiniMax Music 3 modular pipeline", finding 3).
* CFG guided = uncond + c * (cond - uncond) (DiffSynth-Studio article, "第二阶段"):
  c = 1 reproduces the cond row, c = 0 the uncond row.
* Residual wiring, GQA head mapping, the inclusive attention range and the
  KV write are pinned with weights chosen so that the layer has a closed form.
"""
import numpy as np
import pytest
import torch

import synth


def _bits(t):
    from oracle.oracle import bits
    return bits(t)


def _f(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


def _tiny_body(ora, seed=0, zero=(), eye=(), wfmt=0, kv_f16=False, shape=synth.TINY):
    Ls = [synth.layer_weights(shape, seed, l) for l in range(shape.n_layers)]
    for Lw in Ls:
        for n in zero:
            Lw[n] = torch.zeros_like(Lw[n])
        for n in eye:
            Lw[n] = torch.eye(*Lw[n].shape, dtype=torch.bfloat16)
    fn = synth.final_norm(shape, seed)
    lm = synth.lm_head_slice(shape, seed)
    return ora.Body(shape, Ls, fn, lm, wfmt=wfmt, kv_f16=kv_f16), Ls, fn, lm


def _prefill(body, rows, n_pos, max_pos, seed=0):
    s = body.shape
    K, V = synth.kv_prefill(s, rows, n_pos, seed)
    kc, vc = body.new_cache(rows, max_pos)
    kc[:, :, :n_pos] = _bits(K)
    vc[:, :, :n_pos] = _bits(V)
    return kc, vc


# ----------------------------------------------------------------- sampler --

@pytest.mark.parametrize("cfg_scale", [0.0, 1.5])
def test_slice_equals_masked_full(ora, cfg_scale):
    s = synth.TINY
    body, *_ = _tiny_body(ora)
    full = _bits(synth.lm_head_full(s, 0))
    assert np.array_equal(full[s.slice_start:s.slice_start + s.slice_len], _bits(synth.lm_head_slice(s, 0)))
    rng = np.random.default_rng(0)
    for trial in range(25):
        h = ((rng.standard_normal((4, s.hidden)).astype(np.float32).view(np.uint32)) >> 16).astype(np.uint16)
        a, _ = body.sample(h, seed=trial, frame=trial * 3, cfg_scale=cfg_scale)
        b = body.sample_full_masked(full, h, seed=trial, frame=trial * 3, cfg_scale=cfg_scale)
        assert np.array_equal(a, b)


def test_cfg_closed_forms(ora):
    s = synth.TINY
    body, *_ = _tiny_body(ora)
    rng = np.random.default_rng(1)
    for trial in range(10):
        hc = ((rng.standard_normal((1, s.hidden)).astype(np.float32).view(np.uint32)) >> 16).astype(np.uint16)
        hz = np.zeros_like(hc)  # uncond row with exactly zero logits
        pair = np.concatenate([hc, hz], 0)
        c_cond, _ = body.sample(hc, seed=trial, frame=5)
        c1, _ = body.sample(pair, seed=trial, frame=5, cfg_scale=1.0)  # g = 0 + 1*(l_c - 0) = l_c
        assert c1[0] == c1[1] == c_cond[0]
        c2, _ = body.sample(pair, seed=trial, frame=5, cfg_scale=2.0)  # g = 2 l_c = l_c at T = 2
        ct, _ = body.sample(hc, seed=trial, frame=5, temperature=0.5)
        assert c2[0] == ct[0]
    # c -> 0 (but > 0, so the pair path runs) draws from the uncond row's logits
    pair = np.concatenate([hz, hc], 0)
    for trial in range(5):
        c0, _ = body.sample(pair, seed=trial, frame=9, cfg_scale=1e-30)
        cu, _ = body.sample(hc, seed=trial, frame=9)
        assert c0[0] == cu[0]


def test_sampler_logits_are_unrounded_fp32(ora):
    s = synth.TINY
    body, Ls, fn, lm = _tiny_body(ora)
    rng = np.random.default_rng(2)
    h = ((rng.standard_normal((2, s.hidden)).astype(np.float32).view(np.uint32)) >> 16).astype(np.uint16)
    _, lg = body.sample(h, seed=1, frame=1)
    ref = _f(h).astype(np.float64) @ _f(_bits(lm)).astype(np.float64).T
    assert np.allclose(lg, ref, rtol=0, atol=1e-5 * np.abs(ref).max())
    assert np.mean(((lg.view(np.uint32)) & 0xFFFF) != 0) > 0.9  # not bf16-rounded


# ------------------------------------------------------------ composition --

def test_zero_output_projections_leave_residual_unchanged(ora):
    body, *_ = _tiny_body(ora, zero=("wo", "wd"))
    kc, vc = _prefill(body, 2, 64, 80)
    x = _bits(synth.frame_input(body.shape, 2, 0, 0))
    out = body.body(kc, vc, [64, 70], x)
    assert np.array_equal(out, x)


def test_attention_wiring_uniform_scores(ora):
    # Wq = 0 -> every score is 0 -> o_h = mean of V[0..pos] of KV head h // group;
    # Wv = 0 -> the new value is 0; Wo = I -> x' = bf16(x + o); Wd = 0.
    s = synth.TINY
    body, *_ = _tiny_body(ora, zero=("wq", "wv", "wd"), eye=("wo",))
    rows, npos, maxp = 2, 64, 100
    kc, vc = _prefill(body, rows, npos, maxp)
    positions = [64, 90]  # row 1 attends over a gap of zero-initialised slots 64..89
    x = _bits(synth.frame_input(s, rows, 0, 0))
    out = body.body(kc, vc, positions, x)
    grp = s.n_q_heads // s.n_kv_heads
    for r in range(rows):
        pos = positions[r]
        V = _f(vc[r, 0, :pos + 1]).astype(np.float64)  # [pos+1, Hkv, d] incl. the new zero value
        assert (V[pos] == 0).all()
        o = np.concatenate([V[:, h // grp].mean(0) for h in range(s.n_q_heads)])
        ref = _f(x[r]).astype(np.float64) + o
        got = _f(out[r]).astype(np.float64)
        # two bf16 roundings on values of size |x| + |o|
        tol = (np.abs(_f(x[r])) + np.abs(o)) * 2.0 ** -7 + 1e-6
        assert np.all(np.abs(got - ref) <= tol)


def test_kv_write_at_position(ora):
    # Wk = 0 -> the new key is RoPE(norm(0)) = 0; Wv = I-like picks n = norm(x)*g1.
    s = synth.TINY
    body, Ls, *_ = _tiny_body(ora, zero=("wk",), eye=("wv",))
    rows, maxp = 1, 80
    kc, vc = _prefill(body, rows, 64, maxp)
    before_k, before_v = kc.copy(), vc.copy()
    x = _bits(synth.frame_input(s, rows, 0, 3))
    body.body(kc, vc, [70], x)
    assert (_f(kc[0, 0, 70]) == 0).all()  # +-0
    n = ora.rmsnorm(_f(x[0]), _bits(Ls[0]["attn_norm"]), s.rms_eps)
    assert np.array_equal(_f(vc[0, 0, 70]).ravel(), n[: s.n_kv_heads * s.head_dim])
    # nothing else was written
    mask = np.ones(maxp, bool)
    mask[70] = False
    assert np.array_equal(kc[0, 0, mask], before_k[0, 0, mask])
    assert np.array_equal(vc[0, 0, mask], before_v[0, 0, mask])


def test_mlp_wiring(ora):
    # attention contributes nothing (Wo = 0); x' = x + Wd (silu(Wg n2) * (Wu n2))
    s = synth.TINY
    body, Ls, *_ = _tiny_body(ora, zero=("wo",))
    kc, vc = _prefill(body, 1, 16, 32)
    x = _bits(synth.frame_input(s, 1, 0, 1))
    out = body.body(kc, vc, [16], x)
    L0 = {k: _f(_bits(v)).astype(np.float64) for k, v in Ls[0].items()}
    xf = _f(x[0]).astype(np.float64)
    n2 = L0["mlp_norm"] * xf / np.sqrt(np.mean(xf * xf) + s.rms_eps)
    g = L0["wg"] @ n2
    u = L0["wu"] @ n2
    a = g / (1 + np.exp(-g)) * u
    ref = xf + L0["wd"] @ a
    got = _f(out[0]).astype(np.float64)
    err = np.abs(got - ref)
    # bf16 roundings at each stage: a few bf16 ulps of the update
    assert np.max(err) < 0.05 * np.max(np.abs(ref - xf)) + 2.0 ** -7 * np.max(np.abs(ref))
    # swapping the gate and the up projection would change the answer
    a_sw = u / (1 + np.exp(-u)) * g
    ref_sw = xf + L0["wd"] @ a_sw
    assert np.max(np.abs(got - ref_sw)) > 5 * np.max(err)


def test_gqa_identical_queries_identical_outputs(ora):
    # heads of one group see the same keys; with equal q rows they must agree
    s = synth.TINY
    Ls = [synth.layer_weights(s, 0, 0)]
    wq = Ls[0]["wq"].clone()
    d = s.head_dim
    grp = s.n_q_heads // s.n_kv_heads
    for h in range(s.n_q_heads):
        wq[h * d:(h + 1) * d] = wq[(h // grp) * grp * d:((h // grp) * grp + 1) * d]
    Ls[0]["wq"] = wq
    Ls[0]["wo"] = torch.eye(s.hidden, dtype=torch.bfloat16)
    Ls[0]["wd"] = torch.zeros_like(Ls[0]["wd"])
    body = ora.Body(s, Ls, synth.final_norm(s, 0), synth.lm_head_slice(s, 0))
    kc, vc = _prefill(body, 1, 40, 64)
    x = np.zeros((1, s.hidden), np.uint16)  # x = 0 -> x' = o exactly representable
    out = body.body(kc, vc, [40], x)
    o = _f(out[0]).reshape(s.n_q_heads, d)
    for h in range(s.n_q_heads):
        assert np.array_equal(o[h], o[(h // grp) * grp])
    assert not np.array_equal(o[0], o[grp])


def test_thread_count_independence(ora):
    s = synth.TINY
    body, *_ = _tiny_body(ora)
    x = _bits(synth.frame_input(s, 2, 0, 0))
    res = []
    for nt in (1, 3):
        ora.set_threads(nt)
        kc, vc = _prefill(body, 2, 64, 80)
        codes, h, lg = body.decode_frame(kc, vc, [64, 64], 5, 0, x, cfg_scale=1.5)
        res.append((codes, h, lg, kc))
    ora.set_threads(max(1, __import__("os").cpu_count() or 1))
    for a, b in zip(res[0], res[1]):
        assert np.array_equal(a, b)


def test_f16_cache_stores_rne_of_value(ora):
    s = synth.TINY
    body, Ls, *_ = _tiny_body(ora, zero=("wk",), eye=("wv",), kv_f16=True)
    kc, vc = _prefill(body, 1, 8, 16)
    x = _bits(synth.frame_input(s, 1, 0, 3))
    body.body(kc, vc, [8], x)
    n = ora.rmsnorm(_f(x[0]), _bits(Ls[0]["attn_norm"]), s.rms_eps)[: s.n_kv_heads * s.head_dim]
    assert np.array_equal(vc[0, 0, 8].ravel(), n.astype(np.float16).view(np.uint16))


def test_decode_frame_rejects_out_of_range_position(ora):
    body, *_ = _tiny_body(ora)
    kc, vc = _prefill(body, 1, 8, 16)
    x = _bits(synth.frame_input(body.shape, 1, 0, 0))
    with pytest.raises(RuntimeError):
        body.decode_frame(kc, vc, [16], 1, 0, x)


# ------------------------------------------------------------ depth decoder --

def test_depth_structure_with_zero_block_outputs(ora):
    # W_o = W_d = 0 in every layer: each position's state is its input, so the
    # logits of codebook j are head_j . norm(E_{j-1}[c_{j-1}]) (c_0 = semantic code).
    D = synth.DepthShape(hidden=256, n_layers=2, n_heads=4, head_dim=64, ffn=384,
                         codebooks=7, vocab=128, sem_vocab=512, in_hidden=512)
    w = synth.depth_weights(D, 0)
    for Lw in w["layers"]:
        Lw["wo"] = torch.zeros_like(Lw["wo"])
        Lw["wd"] = torch.zeros_like(Lw["wd"])
    dep = ora.Depth(D, w)
    rows = 2
    h = _bits(synth.normal((rows, D.in_hidden), 0, "hf"))
    code0 = np.array([5, 300], np.int32)
    codes, lg = dep.decode(h, code0, seed=3, frame=7)
    fn = _bits(w["final_norm"])
    for r in range(rows):
        prev = code0[r]
        for j in range(D.codebooks):
            e = _f(_bits(w["emb"][j]))[prev]
            n = ora.rmsnorm(e, fn, D.rms_eps)
            q, sc = ora.quantize(_bits(w["heads"][j]), 128)
            ref = ora.gemv(q=q, s=sc, wfmt=2, x=n)
            assert np.array_equal(lg[r, j], ref)
            prev = codes[r, j]
    # teacher forcing with the model's own codes changes nothing
    codes2, lg2 = dep.decode(h, code0, seed=3, frame=7, forced=codes)
    assert np.array_equal(codes, codes2) and np.array_equal(lg, lg2)


def test_depth_noise_index_per_codebook(ora):
    # identical logits in two codebooks must still be drawn with different noise
    D = synth.DepthShape(hidden=256, n_layers=1, n_heads=4, head_dim=64, ffn=384,
                         codebooks=7, vocab=128, sem_vocab=512, in_hidden=512)
    w = synth.depth_weights(D, 1)
    w["heads"] = [torch.zeros_like(w["heads"][0])] * D.codebooks  # all logits 0
    dep = ora.Depth(D, w)
    h = _bits(synth.normal((1, D.in_hidden), 1, "hf"))
    codes, _ = dep.decode(h, np.array([0], np.int32), seed=9, frame=0)
    L = ora.lib()
    for j in range(D.codebooks):
        z = [L.ora_gumbel(9, 0, 0, ((j + 1) << 32) | i) for i in range(D.vocab)]
        assert codes[0, j] == int(np.argmax(z))


# ------------------------------------------------ the q/k norm -> RoPE chain --

def _rbf(x):
    """fp64 -> fp32 -> bf16 (round to nearest even) -> fp64, in numpy."""
    b = np.asarray(x, np.float64).astype(np.float32).view(np.uint32).astype(np.uint64)
    b = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16) << 16
    return b.astype(np.uint32).view(np.float32).astype(np.float64)


def _to_bits(x):
    return (np.asarray(_rbf(x), np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _head_chain(v, gamma, pos, theta, eps):
    """The reading of the head step (DiffSynth-Studio article, "各子模型的结构要点":
    Qwen3 q/k RMSNorm, then rope_theta 1e6 rotary embedding, half rotation):
    bf16(RoPE_pos(bf16(gamma * bf16(v / rms(v))))), here in fp64."""
    d = v.size
    n = _rbf(v / np.sqrt(np.mean(v * v) + eps))
    n = _rbf(gamma * n)
    i = np.arange(d // 2)
    ang = pos * theta ** (-2.0 * i / d)
    c, s = np.cos(ang), np.sin(ang)
    a, b = n[: d // 2], n[d // 2:]
    return _rbf(np.concatenate([a * c - b * s, b * c + a * s]))


def test_qk_norm_rope_chain_and_score(ora):
    """Pins the order of the head step inside the layer, which the function
    pins of RMSNorm and RoPE alone cannot: x = e_a makes the normalised input
    16 e_a exactly, so q, k and v are 16 x (column a of Wq, Wk, Wv), chosen
    bf16 values.  The key stored at `pos` must be the rotated, normalised,
    gained key of the closed form; a norm after the rotation, an unrotated
    key, the angle of pos + 1 or the q gain on k each move it by far more
    than one bf16 step.  The attention output (Wo = I) then exposes the two
    softmax weights of a two-position context, whose log ratio must be the
    fp64 score difference q'.(k'_1 - k_0)/sqrt(d) of the same closed form."""
    s = synth.TINY
    d, Hq, Hkv, H = s.head_dim, s.n_q_heads, s.n_kv_heads, s.hidden
    grp = Hq // Hkv
    rng = np.random.default_rng(11)
    a = 5                                     # the one non-zero input column
    bq, bk = 7, 9                             # value dims that carry p0 and p1

    def bf(x):
        return torch.from_numpy(_to_bits(x).view(np.int16)).view(torch.bfloat16)

    Lw = synth.layer_weights(s, 0, 0)
    wq = np.zeros((Hq * d, H)); wq[:, a] = rng.standard_normal(Hq * d) * 0.25
    wk = np.zeros((Hkv * d, H)); wk[:, a] = rng.standard_normal(Hkv * d) * 0.25
    wv = np.zeros((Hkv * d, H))
    for g in range(Hkv):
        wv[g * d + bk, a] = 1.0 / 16.0       # v_1 = e_bk in every KV head
    Lw.update(wq=bf(wq), wk=bf(wk), wv=bf(wv), wo=torch.eye(H, dtype=torch.bfloat16),
              wd=torch.zeros_like(Lw["wd"]), attn_norm=bf(np.ones(H)),
              q_norm=bf(1.0 + 0.5 * np.sign(np.sin(np.arange(d) * 1.7))),
              k_norm=bf(np.where(np.arange(d) < d // 2, 1.75, 0.375)))
    body = ora.Body(s, [Lw], synth.final_norm(s, 0), synth.lm_head_slice(s, 0))
    gq = _f(_bits(Lw["q_norm"])).astype(np.float64)
    gk = _f(_bits(Lw["k_norm"])).astype(np.float64)
    theta, eps = s.rope_theta, s.rms_eps

    rows, maxp = 2, 64
    positions = [1, 37]
    kc, vc = body.new_cache(rows, maxp)
    k0 = rng.standard_normal((Hkv, d)) * 1.5
    kc[0, 0, 0] = _to_bits(k0)
    v0 = np.zeros((Hkv, d)); v0[:, bq] = 1.0  # v_0 = e_bq
    vc[0, 0, 0] = _to_bits(v0)
    K, V = synth.kv_prefill(s, 1, 37, 3)
    kc[1, 0, :37] = _bits(K[0])
    vc[1, 0, :37] = _bits(V[0])
    x = np.zeros((rows, H), np.uint16)
    x[:, a] = 0x3F80                          # 1.0
    out = body.body(kc, vc, positions, x)

    q = _f(_bits(Lw["wq"]))[:, a].astype(np.float64) * 16.0
    k = _f(_bits(Lw["wk"]))[:, a].astype(np.float64) * 16.0
    ulp = 2.0 ** -7                           # one bf16 step, relative
    for r, pos in enumerate(positions):
        got = _f(kc[r, 0, pos]).astype(np.float64)
        for g in range(Hkv):
            ref = _head_chain(k[g * d:(g + 1) * d], gk, pos, theta, eps)
            dev = np.abs(got[g] - ref)
            assert np.all(dev <= ulp * np.abs(ref) + 1e-30), (r, g, dev.max())
            assert np.mean(dev == 0) >= 0.95
            # the plausible misreadings all land far away
            n = _rbf(k[g * d:(g + 1) * d] / np.sqrt(np.mean(k[g * d:(g + 1) * d] ** 2) + eps))
            wrong = {
                "unrotated": _rbf(gk * n),
                "pos+1": _head_chain(k[g * d:(g + 1) * d], gk, pos + 1, theta, eps),
                "q gain": _head_chain(k[g * d:(g + 1) * d], gq, pos, theta, eps),
                "rope first": _rbf(gk * _rbf(_head_chain(k[g * d:(g + 1) * d], np.ones(d), pos,
                                                         theta, eps))),
            }
            for name, w in wrong.items():
                assert np.max(np.abs(got[g] - w)) > 0.05, name
        assert (_f(vc[r, 0, pos]).reshape(Hkv, d)[:, bk] == 1.0).all()

    # row 0: context {0, 1}; o_h = p0 e_bq + p1 e_bk, and Wo = I puts o_h at x[h d + .]
    xo = _f(out[0]).astype(np.float64)
    for h in range(Hq):
        g = h // grp
        qh = _head_chain(q[h * d:(h + 1) * d], gq, 1, theta, eps)
        k1 = _f(kc[0, 0, 1, g]).astype(np.float64)
        ds = qh @ (k1 - _f(kc[0, 0, 0, g]).astype(np.float64)) / np.sqrt(d)
        p0, p1 = xo[h * d + bq], xo[h * d + bk]
        assert abs(p0 + p1 - 1.0) < 2e-2
        # p0, p1 are bf16 values: ln(p1/p0) holds them to about 2 x 2^-8
        assert abs(np.log(p1 / p0) - ds) < 2e-2 + 0.01 * abs(ds), (h, np.log(p1 / p0), ds)
