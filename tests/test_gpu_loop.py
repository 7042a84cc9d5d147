"""GPU parity of the end-token draw and the GPU generation loop (m3_generate)
against the CPU oracle, through the C ABI.

The loop is checked teacher-forced, as the single frame is: the oracle's loop
is fed the GPU's own codes (ora_generate's forcing), so one near-tie draw
cannot send the two runs down different songs.  Then
  * every recorded hidden state agrees within the bf16 logit tolerance,
  * the GPU's semantic codes equal the oracle sampler's draw on the GPU's own
    hidden state on >= 99.9 % of the draws, every mismatch with an oracle
    top-2 margin below 1e-3,
  * the residual codes, re-run through m3_depth_decode on the recorded hidden
    states, equal the oracle sampler's draws on the GPU's own depth logits by
    the same rule (>= 99.9 % identical, every mismatch with a margin < 1e-3),
  * the counts follow the stop rule on the GPU's codes and equal the oracle's,
  * entries after a key's end are -1 and its hidden states zero.
"""
import numpy as np
import pytest
import torch

import synth
from gpu_util import Model, bits, check_draws, f32, rel_err

pytestmark = pytest.mark.gpu

S_END = synth.TINY_END
DEPTH = synth.DepthShape(hidden=256, n_layers=1, n_heads=4, head_dim=64, ffn=384, codebooks=7,
                         vocab=128, sem_vocab=S_END.slice_len, in_hidden=S_END.hidden)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def _end_row(shape, seed, logit):
    # a random end row with entries N(0, (logit / sqrt(H))^2): its logit on a
    # final-normed state is a few units, so the end token comes out within a
    # few frames for some keys and not for others
    g = torch.Generator().manual_seed(seed)
    v = torch.randn(shape.hidden, generator=g) * (logit / shape.hidden ** 0.5)
    return v.to(torch.bfloat16)


# ------------------------------------------------------- end-token draw ----

@pytest.mark.parametrize("rows,cfg,k", [(2, 1.5, 0), (1, 0.0, 0), (2, 1.5, 50), (3, 0.0, 7)])
def test_end_token_draw(ora, rows, cfg, k):
    s = S_END
    m = Model(s, seed=3, max_rows=4, end_row=_end_row(s, 1, 40.0))
    try:
        m.m3.m3_set_top_k(m.ctx, k)
        kc, vc = m.kv_setup(rows=rows, n_prefill=30, max_pos=64)
        drawn_end = 0
        for f in range(6):
            pos = [30 + f] * rows
            x = synth.frame_input(s, rows, 3, f)
            codes, h, lg = m.decode(pos, seed=9, frame=f, x_in=x, cfg_scale=cfg)
            oc, oh, olg = m.ora.decode_frame(kc, vc, pos, 9, f, bits(x), cfg_scale=cfg, top_k=k)
            assert lg.shape == (rows, s.slice_len + 1)
            assert rel_err(lg, olg) <= 2e-2
            assert rel_err(lg[:, -1], olg[:, -1]) <= 2e-2  # the end row's own logit
            oc2, _lg, margin = m.ora.sample(h, 9, f, cfg, 1.0, with_margin=True, top_k=k)
            check_draws(oc2, margin, codes)
            drawn_end += int(np.sum(codes == s.slice_len))
        assert drawn_end > 0  # the end candidate is reachable
    finally:
        m.close()


def test_end_token_config_checks(ora):
    from autoregressive_audio_token_b200 import m3
    import dataclasses
    bad = dataclasses.replace(S_END, end_token=S_END.slice_start + 3)  # inside the slice
    with pytest.raises(m3.M3Error) as e:
        m3.m3_create(m3.config_from_shapes(bad))
    assert e.value.code == m3.M3_EINVAL
    cfg = m3.config_from_shapes(S_END)
    ctx = m3.m3_create(cfg)
    try:
        Ls = [synth.layer_weights(S_END, 0, 0)]
        with pytest.raises(m3.M3Error) as e:  # lm_head without the end row
            m3.m3_load_weights(ctx, Ls, 0, synth.final_norm(S_END, 0),
                               synth.lm_head_slice(S_END, 0))
        assert e.value.code == m3.M3_EINVAL
    finally:
        m3.m3_destroy(ctx)


# ------------------------------------------------------------------ loop ----

def _loop_case(ora, rows, cfg, k, with_depth, F, bucket, end_logit, n_prefill=20, seed=4):
    s = S_END
    m = Model(s, seed=seed, max_rows=max(2, rows), depth=DEPTH if with_depth else None,
              end_row=_end_row(s, seed, end_logit))
    try:
        nc = DEPTH.codebooks if with_depth else 0
        tok = synth.embedding_slice(s, 5)
        aud = synth.audio_embeddings(DEPTH, s.hidden, 5) if with_depth else None
        m.m3.m3_load_feedback(m.ctx, tok.cuda(), [a.cuda() for a in aud] if aud else None)
        m.m3.m3_set_top_k(m.ctx, k)
        max_pos = n_prefill + 2 * rows + F + 1
        kc, vc = m.kv_setup(rows=rows, n_prefill=n_prefill, max_pos=max_pos, bucket=bucket)
        pos0 = [n_prefill + 2 * r for r in range(rows)]
        x0 = synth.frame_input(s, rows, 6, 0)
        codes = torch.empty((F, rows, 1 + nc), dtype=torch.int32, device="cuda")
        hh = torch.empty((F, rows, s.hidden), dtype=torch.bfloat16, device="cuda")
        rc, nf = m.m3.m3_generate(m.ctx, pos0, 21, 500, x0.cuda(), cfg, 1.0, F, codes, hh)
        torch.cuda.synchronize()
        m.m3.m3_sync_status(m.ctx)
        gc = codes.cpu().numpy()
        gh = bits(hh)
        orc, oc, onf, oh = m.ora.generate(kc, vc, pos0, 21, 500, bits(x0), F, tok,
                                          depth=m.ora_depth, audio_emb=aud, cfg_scale=cfg,
                                          top_k=k, forced=gc, with_h=True)
        keys = rows // 2 if cfg > 0 else rows
        key_rows = [[2 * q, 2 * q + 1] if cfg > 0 else [q] for q in range(keys)]
        # the stop rule on the GPU's own codes
        for q in range(keys):
            r0 = key_rows[q][0]
            col = gc[:, r0, 0]
            ends = np.nonzero(col == s.slice_len)[0]
            want = int(ends[0]) if len(ends) else F
            assert nf[q] == want == onf[q], (q, nf, onf, col)
            for r in key_rows[q]:
                last = want + 1 if want < F else F
                assert np.all(gc[last:, r] == -1)
                assert np.all(gh[last:, r] == 0)
                if want < F:
                    assert gc[want, r, 0] == s.slice_len and np.all(gc[want, r, 1:] == -1)
                if cfg > 0:
                    assert np.array_equal(gc[:last, key_rows[q][0]], gc[:last, key_rows[q][1]])
                # the recorded frames
                for f in range(last):
                    assert rel_err(f32(gh[f, r]), f32(oh[f, r])) <= 2e-2, (f, r)
        assert rc == (m.m3.M3_EEMPTY if min(nf) == 0 else m.m3.M3_OK)
        assert orc == (-8 if min(nf) == 0 else 0)
        # semantic codes: the oracle sampler on the GPU's hidden state of each frame
        mism_total = 0
        for f in range(F):
            live = [r for q in range(keys) for r in key_rows[q] if f < nf[q] + 1 and f < F]
            if not live:
                break
            c2, _lg, margin = m.ora.sample(gh[f], 21, 500 + f, cfg, 1.0, with_margin=True,
                                           top_k=k)
            for r in live:
                if c2[r] != gc[f, r, 0]:
                    assert margin[r] < 1e-3, (f, r, c2[r], gc[f, r, 0], margin[r])
                    mism_total += 1
        n_sem = sum(1 for f in range(F) for q in range(keys) if f < nf[q] + 1)
        assert mism_total <= int(0.001 * n_sem), (mism_total, n_sem)
        # residual codes: each frame's depth decoder run again through the ABI on
        # the loop's recorded hidden state and code (bit-identical codes: the
        # same kernels on the same inputs), then every draw against the
        # oracle's sampler on those GPU logits
        if nc:
            V = DEPTH.vocab
            all_o, all_m, all_g = [], [], []
            for f in range(F):
                live = gc[f, :, 1] >= 0  # rows whose key drew residual codes this frame
                if not live.any():
                    continue
                # rows are independent in the depth decoder (CFG pairs stop together),
                # so stopped rows ride along on any valid code
                c0 = torch.from_numpy(np.where(gc[f, :, 0] < 0, 0, gc[f, :, 0]).astype(np.int32))
                dc = torch.empty((rows, nc), dtype=torch.int32, device="cuda")
                dl = torch.empty((rows, nc, V), dtype=torch.float32, device="cuda")
                m.m3.m3_depth_decode(m.ctx, hh[f].contiguous(), c0.cuda(), 21, 500 + f, cfg, 1.0,
                                     dc, logits=dl)
                torch.cuda.synchronize()
                m.m3.m3_sync_status(m.ctx)
                dcn = dc.cpu().numpy()
                assert np.array_equal(dcn[live], gc[f, live, 1:]), f
                glg = dl.cpu().numpy()
                for j in range(nc):
                    o, mg = ora.draw(np.ascontiguousarray(glg[:, j]), 21, 500 + f,
                                     cfg_scale=cfg, index_base=(j + 1) << 32)
                    all_o.append(o[live])
                    all_m.append(mg[live])
                    all_g.append(dcn[live, j])
            assert all_o, "no frame drew residual codes"
            check_draws(np.concatenate(all_o), np.concatenate(all_m), np.concatenate(all_g))
        return nf
    finally:
        m.close()


@pytest.mark.parametrize("rows,cfg,k,with_depth", [(2, 1.5, 0, True), (3, 0.0, 50, True),
                                                   (4, 1.5, 0, False)])
def test_generate_teacher_forced(ora, rows, cfg, k, with_depth):
    _loop_case(ora, rows, cfg, k, with_depth, F=12, bucket=256, end_logit=1.5)


def test_generate_many_chunks_and_pages(ora):
    # 40 frames: three 16-frame chunks, across 32-position KV pages; the end
    # token made rare so most keys run to the frame cap
    nf = _loop_case(ora, 2, 0.0, 0, True, F=40, bucket=32, end_logit=4.0)
    assert max(nf) > 16


def test_generate_zero_frames_is_empty(ora):
    s = S_END
    m = Model(s, seed=8, max_rows=2, oracle=False,
              end_row=torch.zeros(s.hidden, dtype=torch.bfloat16))
    try:
        # end row = 1000 * the first frame's hidden state direction: drawn at frame 0
        m.m3.m3_kv_alloc(m.ctx, 1, 32, 0, 32)
        x0 = synth.frame_input(s, 1, 2, 0).cuda()
        codes1 = torch.empty(1, dtype=torch.int32, device="cuda")
        h = torch.empty((1, s.hidden), dtype=torch.bfloat16, device="cuda")
        m.m3.m3_decode_frame(m.ctx, [4], 1, 0, x0, 0.0, 1.0, codes1, h)
        torch.cuda.synchronize()
        hf = h.float().cpu()[0]
        m.close()
        m = Model(s, seed=8, max_rows=2, oracle=False,
                  end_row=(1000.0 * hf / float(hf @ hf)).to(torch.bfloat16))
        m.m3.m3_kv_alloc(m.ctx, 1, 32, 0, 32)
        m.m3.m3_load_feedback(m.ctx, synth.embedding_slice(s, 1).cuda())
        codes = torch.empty((5, 1, 1), dtype=torch.int32, device="cuda")
        rc, nf = m.m3.m3_generate(m.ctx, [4], 1, 0, x0, 0.0, 1.0, 5, codes)
        assert rc == m.m3.M3_EEMPTY and nf == [0]
        gc = codes.cpu().numpy()
        assert gc[0, 0, 0] == s.slice_len and np.all(gc[1:] == -1)
    finally:
        m.close()


def test_generate_argument_errors(ora):
    from autoregressive_audio_token_b200 import m3
    s = S_END
    m = Model(s, seed=1, max_rows=2, oracle=False)
    try:
        m.m3.m3_kv_alloc(m.ctx, 2, 40, 0, 32)
        x0 = synth.frame_input(s, 2, 2, 0).cuda()
        codes = torch.empty((8, 2, 1), dtype=torch.int32, device="cuda")
        with pytest.raises(m3.M3Error) as e:  # no feedback tables yet
            m3.m3_generate(m.ctx, [4, 4], 1, 0, x0, 0.0, 1.0, 8, codes)
        assert e.value.code == m3.M3_ESTATE
        m3.m3_load_feedback(m.ctx, synth.embedding_slice(s, 1).cuda())
        with pytest.raises(m3.M3Error) as e:  # 35 + 8 frames > 40 positions
            m3.m3_generate(m.ctx, [4, 35], 1, 0, x0, 0.0, 1.0, 8, codes)
        assert e.value.code == m3.M3_ECAPACITY
        with pytest.raises(m3.M3Error) as e:  # CFG needs row pairs
            m3.m3_generate(m.ctx, [4], 1, 0, x0[:1], 1.5, 1.0, 8, codes)
        assert e.value.code == m3.M3_EINVAL
        with pytest.raises(m3.M3Error) as e:
            m3.m3_generate(m.ctx, [4, 4], 1, 0, x0, 0.0, 1.0, 0, codes)
        assert e.value.code == m3.M3_EINVAL
        m3.m3_sync_status(m.ctx)
    finally:
        m.close()
