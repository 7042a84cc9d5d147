"""Pins for the oracle's end-token draw and its multi-frame generation loop.

Sources (page title, section):
* DiffSynth-Studio article on MiniMax-Music3, "第二阶段": the vocab mask keeps
  the audio codes and the end token sampleable; each frame's codes are
  embedded back (token embedding plus the audio embeddings, times 8^-0.5) as
  the next input; the end token stops the loop early, and stopping before the
  first frame is an error.
* "MiniMax Music 3 on Metal": position, step and count advance per frame.

What pins what:
* slice + end row == the full lm_head with every other row at -inf (with and
  without CFG and top-k), on logits where the end token is drawn sometimes;
* the loop's bookkeeping (positions + f, noise frame frame0 + f, codes fed
  forward, the stop rule and the -1 fill) against frame-by-frame calls of the
  oracle's single-frame functions;
* the feedback embedding by closed forms: with no depth decoder it is the
  token embedding row itself; with 7 residual codebooks and every table row
  equal to 1/8 it is bf16(1/sqrt(8)) in every element;
* teacher forcing with the loop's own codes is the identity, and a forced end
  code stops that key at that frame;
* an end token drawn at frame 0 gives status -8 with empty counts.
"""
import dataclasses

import numpy as np
import pytest
import torch

import synth

S_END = synth.TINY_END
DEPTH = synth.DepthShape(hidden=256, n_layers=1, n_heads=4, head_dim=64, ffn=384, codebooks=7,
                         vocab=128, sem_vocab=S_END.slice_len, in_hidden=S_END.hidden)


def _bits(t):
    from oracle.oracle import bits
    return bits(t)


def _f(b):
    return (b.astype(np.uint32) << 16).view(np.float32)


def _body(ora, shape=S_END, seed=0, end_row=None):
    Ls = [synth.layer_weights(shape, seed, l) for l in range(shape.n_layers)]
    fn = synth.final_norm(shape, seed)
    lm = synth.lm_head_slice(shape, seed)
    er = None
    if shape.end_token >= 0:
        er = synth.lm_head_end_row(shape, seed) if end_row is None else end_row
    return ora.Body(shape, Ls, fn, lm, lm_end_row=er), Ls, fn, lm, er


def _cache(body, rows, n_pos, max_pos, seed=0):
    K, V = synth.kv_prefill(body.shape, rows, n_pos, seed)
    kc, vc = body.new_cache(rows, max_pos)
    kc[:, :, :n_pos] = _bits(K)
    vc[:, :, :n_pos] = _bits(V)
    return kc, vc


# ------------------------------------------------------- end-token draw ----

@pytest.mark.parametrize("cfg_scale,top_k", [(0.0, 0), (1.5, 0), (1.5, 50), (0.0, 7)])
def test_end_token_slice_equals_masked_full(ora, cfg_scale, top_k):
    s = S_END
    rng = np.random.default_rng(3)
    u = rng.standard_normal(s.hidden).astype(np.float32)
    # an end row whose logit on h ~ u is about 5.4: competitive with the
    # Gumbel-perturbed maximum over 512 codes, so it is drawn sometimes
    end_row = torch.from_numpy(5.4 * u / float(u @ u)).to(torch.bfloat16)
    body, *_ = _body(ora, end_row=end_row)
    full = _bits(synth.lm_head_full(s, 0)).copy()
    full[s.end_token] = _bits(end_row)
    drawn_end = 0
    for trial in range(40):
        h = u[None, :] + 0.3 * rng.standard_normal((4, s.hidden)).astype(np.float32)
        hb = ((h.view(np.uint32)) >> 16).astype(np.uint16)
        a, lg = body.sample(hb, seed=trial, frame=trial * 5, cfg_scale=cfg_scale, top_k=top_k)
        b = body.sample_full_masked(full, hb, seed=trial, frame=trial * 5, cfg_scale=cfg_scale,
                                    top_k=top_k)
        assert np.array_equal(a, b), (trial, a, b)
        assert lg.shape == (4, s.slice_len + 1)
        drawn_end += int(np.sum(a == s.slice_len))
    assert 0 < drawn_end < 40 * 4  # both outcomes occur


def test_end_row_logit_and_noise_index(ora):
    # the end candidate's logit is its row's dot product, and its noise is keyed
    # by the end token's vocab row: with every logit 0 the draw is the argmax of
    # the noise over [slice_start, +S) and {end_token}
    s = S_END
    body, Ls, fn, lm, er = _body(ora, end_row=torch.zeros(s.hidden, dtype=torch.bfloat16))
    body0 = ora.Body(s, Ls, fn, torch.zeros_like(lm), lm_end_row=torch.zeros_like(er))
    h = np.zeros((1, s.hidden), np.uint16)
    L = ora.lib()
    for seed in range(30):
        c, lg = body0.sample(h, seed=seed, frame=2)
        assert np.all(lg == 0.0)
        z = [L.ora_gumbel(seed, 2, 0, s.slice_start + i) for i in range(s.slice_len)]
        z.append(L.ora_gumbel(seed, 2, 0, s.end_token))
        assert c[0] == int(np.argmax(z))
    # non-zero h: the last logit column is the end row's dot product
    hb = _bits(synth.normal((1, s.hidden), 4, "h"))
    er2 = synth.lm_head_end_row(s, 0)
    b2, *_ = _body(ora, end_row=er2)
    _, lg = b2.sample(hb, seed=0, frame=0)
    ref = ora.gemv(w=_bits(er2).reshape(1, -1), x=_f(hb[0]))
    assert np.array_equal(lg[0, -1:], ref)


# ------------------------------------------------------------------ loop ----

def _feedback_tables(shape, depth, seed=5):
    tok = synth.embedding_slice(shape, seed)
    aud = synth.audio_embeddings(depth, shape.hidden, seed) if depth is not None else None
    return tok, aud


def _depth(ora, seed=2):
    w = synth.depth_weights(DEPTH, seed)
    return ora.Depth(DEPTH, w), w


def _boosted_end_row(shape, seed, logit):
    # the end row = logit * (final-norm gains)^-1 / H: its logit on a hidden
    # state of all ones would be `logit`; on the real states it is a fixed,
    # modest pull that makes the end token come out within a few frames
    rng = np.random.default_rng(seed)
    v = rng.standard_normal(shape.hidden).astype(np.float32) * (logit / np.sqrt(shape.hidden))
    return torch.from_numpy(v).to(torch.bfloat16)


@pytest.mark.parametrize("rows,cfg,with_depth,top_k", [(2, 1.5, True, 0), (3, 0.0, True, 50),
                                                       (2, 0.0, False, 0)])
def test_generate_matches_frame_by_frame(ora, rows, cfg, with_depth, top_k):
    s = S_END
    body, *_ = _body(ora, end_row=_boosted_end_row(s, 1, 40.0))
    dep, _w = _depth(ora) if with_depth else (None, None)
    tok, aud = _feedback_tables(s, DEPTH if with_depth else None)
    NC = DEPTH.codebooks if with_depth else 0
    F, n0, max_pos = 12, 20, 48
    pos0 = [n0 + 2 * r for r in range(rows)]
    x0 = _bits(synth.frame_input(s, rows, 3, 0))
    kc, vc = _cache(body, rows, n0 + 2 * rows, max_pos)
    kc2, vc2 = kc.copy(), vc.copy()
    rc, codes, nf, hh = body.generate(kc, vc, pos0, 11, 100, x0, F, tok, depth=dep,
                                      audio_emb=aud, cfg_scale=cfg, top_k=top_k, with_h=True)
    assert codes.shape == (F, rows, 1 + NC)
    # the same loop, frame by frame, from the single-frame functions
    keys = rows // 2 if cfg > 0 else rows
    key = [r // 2 if cfg > 0 else r for r in range(rows)]
    active = [True] * keys
    cnt = [0] * keys
    x = x0.copy()
    tokf = _f(_bits(tok))
    audf = [_f(_bits(a)) for a in aud] if aud else []
    sc = np.float32(1.0 / np.sqrt(1.0 + NC))
    for f in range(F):
        if not any(active):
            assert np.all(codes[f:] == -1)
            break
        pos = [p + f for p in pos0]
        c0, h, _ = body.decode_frame(kc2, vc2, pos, 11, 100 + f, x, cfg_scale=cfg, top_k=top_k)
        dc = np.zeros((rows, NC), np.int32)
        if NC:
            dc, _ = dep.decode(h, c0, 11, 100 + f, cfg_scale=cfg)
        for r in range(rows):
            if not active[key[r]]:
                assert np.all(codes[f, r] == -1)
                continue
            assert codes[f, r, 0] == c0[r]
            assert np.array_equal(hh[f, r], h[r])
            if c0[r] == s.slice_len:
                assert np.all(codes[f, r, 1:] == -1)
            else:
                assert np.array_equal(codes[f, r, 1:], dc[r])
        for k in range(keys):
            if active[k]:
                r = 2 * k if cfg > 0 else k
                if c0[r] == s.slice_len:
                    active[k] = False
                else:
                    cnt[k] += 1
        xn = np.zeros_like(x)
        for r in range(rows):
            if active[key[r]]:
                t = tokf[c0[r]].copy()
                for j in range(NC):
                    t = t + audf[j][dc[r, j]]
                xn[r] = _bits(torch.from_numpy(t * sc).to(torch.bfloat16))
        x = xn
    assert list(nf) == cnt
    assert rc == (-8 if min(cnt) == 0 else 0)
    assert any(c < F for c in cnt), "the boosted end row should stop some key"


def test_feedback_closed_forms(ora):
    s = S_END
    body, *_ = _body(ora, end_row=torch.zeros(s.hidden, dtype=torch.bfloat16))
    rows, n0, max_pos = 1, 10, 16
    x0 = _bits(synth.frame_input(s, rows, 4, 0))
    # (a) no depth decoder: the next input is the token embedding row itself
    tok = synth.embedding_slice(s, 6)
    kc, vc = _cache(body, rows, n0, max_pos)
    kref, vref = kc.copy(), vc.copy()
    rc, codes, nf, hh = body.generate(kc, vc, [n0], 2, 0, x0, 2, tok, with_h=True)
    assert rc == 0 and list(nf) == [2]
    c0, h0, _ = body.decode_frame(kref, vref, [n0], 2, 0, x0)
    x1 = _bits(tok[int(c0[0])]).reshape(1, -1)
    _, h1, _ = body.decode_frame(kref, vref, [n0 + 1], 2, 1, x1)
    assert np.array_equal(hh[0], h0) and np.array_equal(hh[1], h1)
    # (b) 7 residual codebooks, every table row 1/8: the 8-term sum is 1 and
    # the next input is bf16(8^-0.5) in every element
    dep, _w = _depth(ora)
    eighth = torch.full((s.slice_len, s.hidden), 0.125, dtype=torch.bfloat16)
    aud = [torch.full((DEPTH.vocab, s.hidden), 0.125, dtype=torch.bfloat16)] * DEPTH.codebooks
    kc, vc = _cache(body, rows, n0, max_pos)
    kref, vref = kc.copy(), vc.copy()
    rc, codes, nf, hh = body.generate(kc, vc, [n0], 2, 0, x0, 2, eighth, depth=dep,
                                      audio_emb=aud, with_h=True)
    assert rc == 0
    body.decode_frame(kref, vref, [n0], 2, 0, x0)
    x1 = np.full((1, s.hidden), _bits(torch.tensor([8.0 ** -0.5]).to(torch.bfloat16))[0],
                 np.uint16)
    assert x1[0, 0] == 0x3EB5  # bf16(0.35355...) = 0.353515625
    _, h1, _ = body.decode_frame(kref, vref, [n0 + 1], 2, 1, x1)
    assert np.array_equal(hh[1], h1)
    # a dropped term (7 of 8 summed) would give a different input
    x7 = np.full((1, s.hidden), _bits(torch.tensor([7 / 8 * 8.0 ** -0.5]).to(torch.bfloat16))[0],
                 np.uint16)
    assert x7[0, 0] != x1[0, 0]


def test_teacher_forcing_and_forced_stop(ora):
    s = S_END
    body, *_ = _body(ora, end_row=torch.zeros(s.hidden, dtype=torch.bfloat16))
    dep, _w = _depth(ora)
    tok, aud = _feedback_tables(s, DEPTH)
    rows, F, n0, max_pos = 2, 6, 8, 16
    x0 = _bits(synth.frame_input(s, rows, 5, 0))
    kc, vc = _cache(body, rows, n0, max_pos)
    k2, v2, k3, v3 = kc.copy(), vc.copy(), kc.copy(), vc.copy()
    rc, codes, nf, hh = body.generate(kc, vc, [n0, n0], 7, 3, x0, F, tok, depth=dep,
                                      audio_emb=aud, with_h=True)
    assert rc == 0 and list(nf) == [F, F]
    rc2, codes2, nf2, hh2 = body.generate(k2, v2, [n0, n0], 7, 3, x0, F, tok, depth=dep,
                                          audio_emb=aud, forced=codes, with_h=True)
    assert np.array_equal(codes, codes2) and np.array_equal(hh, hh2) and list(nf2) == [F, F]
    forced = codes.copy()
    forced[3, 0, 0] = s.slice_len  # row 0 (its own key, no CFG) ends at frame 3
    rc3, codes3, nf3, hh3 = body.generate(k3, v3, [n0, n0], 7, 3, x0, F, tok, depth=dep,
                                          audio_emb=aud, forced=forced, with_h=True)
    assert list(nf3) == [3, F]
    assert np.array_equal(codes3[:3], codes[:3])
    assert np.all(codes3[3, 0, 1:] == -1) and np.all(codes3[4:, 0] == -1)
    assert np.all(hh3[4:, 0] == 0)
    # row 1 is independent of row 0's stop
    assert np.array_equal(codes3[:, 1], codes[:, 1]) and np.array_equal(hh3[:, 1], hh[:, 1])


def test_end_at_first_frame_is_an_error(ora):
    s = S_END
    rng = np.random.default_rng(8)
    body, *_ = _body(ora)
    x0 = _bits(synth.frame_input(s, 1, 6, 0))
    kc, vc = _cache(body, 1, 4, 16)
    # find the hidden state of frame 0, then make the end row dominate on it
    k0, v0 = kc.copy(), vc.copy()
    _, h, _ = body.decode_frame(k0, v0, [4], 1, 0, x0)
    hf = _f(h[0])
    end_row = torch.from_numpy(1000.0 * hf / float(hf @ hf)).to(torch.bfloat16)
    body2, *_ = _body(ora, end_row=end_row)
    tok = synth.embedding_slice(s, 1)
    rc, codes, nf, _ = body2.generate(kc, vc, [4], 1, 0, x0, 5, tok)
    assert rc == -8 and list(nf) == [0]
    assert codes[0, 0, 0] == s.slice_len and np.all(codes[1:] == -1)
    # capacity: positions + frames beyond the cache are refused
    with pytest.raises(RuntimeError):
        body2.generate(kc, vc, [12], 1, 0, x0, 5, tok)
    del rng
