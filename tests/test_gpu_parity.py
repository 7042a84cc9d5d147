"""GPU parity: the CUDA library (through the C ABI) against the CPU oracle on
the same seeded inputs.

Tolerances (the workload's stated bar):
  * int8 codes and scales, Gumbel noise: bit-exact;
  * logits: max |l_gpu - l_ora| / max |l_ora| <= 2e-2 (bf16 weights),
    <= 5e-2 (int8 weights);
  * drawn codes: teacher-forced -- the oracle's sampler on the GPU's own final
    hidden state -- identical, every mismatch having a top-2 margin < 1e-3.
"""
import numpy as np
import pytest
import torch

import synth
from gpu_util import check_depth_draws, Model, bits, check_codes_teacher_forced, f32, rel_err

pytestmark = pytest.mark.gpu

TOL = {0: 2e-2, 1: 5e-2}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


# ------------------------------------------------------------ quantiser ----

@pytest.mark.parametrize("rows,cols,group", [(1, 256, None), (37, 4096, None), (5, 12288, None),
                                             (64, 1024, 128), (33, 2816, 128), (3, 4096, 128)])
def test_quantize_bit_exact(ora, rows, cols, group):
    from autoregressive_audio_token_b200 import m3
    w = synth.normal((rows, cols), rows * 7 + cols, "qw", std=0.02)
    w[0, :] = 0  # a zero row / group
    q, s = m3.m3_quantize_int8(w.cuda(), group)
    torch.cuda.synchronize()
    qo, so = ora.quantize(bits(w), group)
    assert np.array_equal(q.cpu().numpy(), qo)
    assert np.array_equal(s.cpu().numpy().reshape(so.shape), so)


# ---------------------------------------------------------- tiny decode ----

def test_tiny_16_frames_teacher_forced(ora):
    s = synth.TINY
    m = Model(s, seed=0)
    try:
        E = synth.embedding(s, 0)
        kc, vc = m.kv_setup(rows=1, n_prefill=64, max_pos=128)
        x = E[s.slice_start:s.slice_start + 1].clone()  # first input: code 0
        for f in range(16):
            pos = 64 + f
            codes, h, lg = m.decode([pos], seed=123, frame=f, x_in=x)
            oc, oh, olg = m.ora.decode_frame(kc, vc, [pos], 123, f, bits(x))
            assert rel_err(lg, olg) <= TOL[0], (f, rel_err(lg, olg))
            assert rel_err(f32(h), f32(oh)) <= 2e-2
            check_codes_teacher_forced(m, h, codes, 123, f)
            # feed the GPU's own draw back (teacher forcing for the oracle too)
            x = E[s.slice_start + int(codes[0]):s.slice_start + int(codes[0]) + 1].clone()
    finally:
        m.close()


@pytest.mark.parametrize("rows,cfg", [(1, 0.0), (2, 0.0), (2, 1.5), (4, 1.5), (3, 0.0), (6, 1.5)])
def test_tiny_rows_and_cfg(ora, rows, cfg):
    s = synth.TINY
    m = Model(s, seed=1, max_rows=8)
    try:
        kc, vc = m.kv_setup(rows=rows, n_prefill=40, max_pos=300)
        pos = [40 + 3 * r for r in range(rows)]  # ragged positions per row
        x = synth.frame_input(s, rows, 1, 0)
        codes, h, lg = m.decode(pos, seed=5, frame=9, x_in=x, cfg_scale=cfg)
        oc, oh, olg = m.ora.decode_frame(kc, vc, pos, 5, 9, bits(x), cfg_scale=cfg)
        assert rel_err(lg, olg) <= TOL[0]
        check_codes_teacher_forced(m, h, codes, 5, 9, cfg_scale=cfg)
        if cfg > 0:
            assert np.array_equal(codes[0::2], codes[1::2])
    finally:
        m.close()


@pytest.mark.parametrize("rows,cfg,wdtype", [(9, 0.0, 0), (16, 1.5, 0), (16, 0.0, 1),
                                              (12, 1.5, 1)])
def test_tiny_many_rows(ora, rows, cfg, wdtype):
    # 9..16 activation rows: the MMA's second row half (rows 8..15) in use
    s = synth.TINY
    m = Model(s, seed=12, max_rows=16, wdtype=wdtype)
    try:
        kc, vc = m.kv_setup(rows=rows, n_prefill=33, max_pos=100)
        pos = [33 + (r % 5) for r in range(rows)]
        x = synth.frame_input(s, rows, 12, 0)
        codes, h, lg = m.decode(pos, seed=8, frame=2, x_in=x, cfg_scale=cfg)
        oc, oh, olg = m.ora.decode_frame(kc, vc, pos, 8, 2, bits(x), cfg_scale=cfg)
        assert rel_err(lg, olg) <= TOL[wdtype], rel_err(lg, olg)
        check_codes_teacher_forced(m, h, codes, 8, 2, cfg_scale=cfg)
    finally:
        m.close()


@pytest.mark.parametrize("rows", [2, 9])
def test_int8_activation_beyond_f16_range(ora, rows):
    # int8 weights take f16 activations; a norm gain of 4e5 on two inputs
    # puts normalised activations far beyond 2^15, so those rows are staged
    # again with a power-of-two scale (the QKV and gate/up launches)
    s = synth.TINY
    Ls = [synth.layer_weights(s, 13, 0)]
    for name in ("attn_norm", "mlp_norm"):
        g = Ls[0][name].clone()
        g[3] = 4.0e5
        g[200] = -4.0e5
        Ls[0][name] = g
    m = Model(s, seed=13, max_rows=16, wdtype=1, layers=Ls)
    try:
        kc, vc = m.kv_setup(rows=rows, n_prefill=20, max_pos=64)
        pos = [20] * rows
        x = synth.frame_input(s, rows, 13, 0)
        codes, h, lg = m.decode(pos, seed=3, frame=1, x_in=x)
        oc, oh, olg = m.ora.decode_frame(kc, vc, pos, 3, 1, bits(x))
        assert np.all(np.isfinite(lg))
        assert rel_err(lg, olg) <= TOL[1], rel_err(lg, olg)
        check_codes_teacher_forced(m, h, codes, 3, 1)
    finally:
        m.close()


def _guided(lg, p, cfg):
    # the kernel's guided logits, in the same fp32 operations
    if cfg > 0:
        return lg[2 * p + 1] + np.float32(cfg) * (lg[2 * p] - lg[2 * p + 1])
    return lg[p]


def _check_topk_codes(ora, codes, lg, k, seed, frame, cfg, slice_start):
    # decision-level parity: the oracle's top-k draw on the GPU's own logits
    npick = lg.shape[0] // 2 if cfg > 0 else lg.shape[0]
    for p in range(npick):
        want = ora.topk_draw(_guided(lg, p, cfg), k, 1.0, seed, frame, p, slice_start)
        rows = (2 * p, 2 * p + 1) if cfg > 0 else (p,)
        for r in rows:
            assert codes[r] == want, (p, k, codes, want)


@pytest.mark.parametrize("rows,cfg,k", [(2, 1.5, 50), (1, 0.0, 7), (2, 1.5, 1), (4, 1.5, 50),
                                        (3, 0.0, 511)])
def test_tiny_topk_draw(ora, rows, cfg, k):
    s = synth.TINY
    m = Model(s, seed=14, max_rows=4, oracle=False)
    try:
        m.m3.m3_set_top_k(m.ctx, k)
        m.kv_setup(rows=rows, n_prefill=30, max_pos=100)
        x = synth.frame_input(s, rows, 14, 0)
        for f in range(6):
            pos = [30 + f] * rows
            codes, h, lg = m.decode(pos, seed=3, frame=f, x_in=x, cfg_scale=cfg)
            _check_topk_codes(ora, codes, lg, k, 3, f, cfg, s.slice_start)
        # back to the plain draw: some code outside the top-k shows up over frames
        m.m3.m3_set_top_k(m.ctx, 0)
        codes, h, lg = m.decode([40] * rows, seed=3, frame=9, x_in=x, cfg_scale=cfg)
        _check_topk_codes(ora, codes, lg, 0, 3, 9, cfg, s.slice_start)
    finally:
        m.close()


def test_topk_rejects_negative(ora):
    from autoregressive_audio_token_b200 import m3
    m = Model(synth.TINY, seed=15, oracle=False)
    try:
        with pytest.raises(m3.M3Error) as e:
            m3.m3_set_top_k(m.ctx, -1)
        assert e.value.code == m3.M3_EINVAL
    finally:
        m.close()


def test_tiny_ragged_vocab_slice(ora):
    # a sampled slice of 500 rows: the last 8-row weight unit is partly padding
    import dataclasses
    s = dataclasses.replace(synth.TINY, slice_len=500)
    m = Model(s, seed=13, max_rows=2)
    try:
        kc, vc = m.kv_setup(rows=2, n_prefill=20, max_pos=64)
        x = synth.frame_input(s, 2, 13, 0)
        codes, h, lg = m.decode([20, 20], seed=4, frame=1, x_in=x, cfg_scale=1.5)
        oc, oh, olg = m.ora.decode_frame(kc, vc, [20, 20], 4, 1, bits(x), cfg_scale=1.5)
        assert lg.shape[-1] == 500
        assert rel_err(lg, olg) <= TOL[0], rel_err(lg, olg)
        check_codes_teacher_forced(m, h, codes, 4, 1, cfg_scale=1.5)
    finally:
        m.close()


@pytest.mark.parametrize("kv_f16", [False, True])
def test_tiny_long_context_many_tiles(ora, kv_f16):
    # positions up to 700 with bucket 256: several 32-position tiles per warp,
    # splits crossing page boundaries, partial last tiles
    s = synth.TINY
    m = Model(s, seed=8, kv_f16=kv_f16, max_rows=2)
    try:
        kc, vc = m.kv_setup(rows=2, n_prefill=650, max_pos=768)
        x = synth.frame_input(s, 2, 8, 0)
        for f, pos in enumerate([[650, 651], [700, 37], [767, 255]]):
            codes, h, lg = m.decode(pos, 3, f, x)
            oc, oh, olg = m.ora.decode_frame(kc, vc, pos, 3, f, bits(x))
            assert rel_err(lg, olg) <= TOL[0], (pos, rel_err(lg, olg))
            check_codes_teacher_forced(m, h, codes, 3, f)
    finally:
        m.close()


def test_kv_written_matches_oracle(ora):
    s = synth.TINY
    m = Model(s, seed=2, kv_f16=False)
    try:
        kc, vc = m.kv_setup(rows=1, n_prefill=10, max_pos=64)
        x = synth.frame_input(s, 1, 2, 0)
        m.decode([10], 1, 0, x)
        m.ora.decode_frame(kc, vc, [10], 1, 0, bits(x))
        k, v = m.m3.m3_kv_get(m.ctx, 0, s.n_layers, 11, s.n_kv_heads, s.head_dim)
        k = k.numpy().view(np.uint16)
        v = v.numpy().view(np.uint16)
        assert np.array_equal(k[:, :10], kc[0, :, :10]) and np.array_equal(v[:, :10], vc[0, :, :10])
        assert rel_err(f32(k[:, 10]), f32(kc[0, :, 10])) < 2e-2
        assert rel_err(f32(v[:, 10]), f32(vc[0, :, 10])) < 2e-2
    finally:
        m.close()


def test_bucket_growth_across_pages(ora):
    # positions cross the 32-position bucket boundary; new buckets are zeroed
    s = synth.TINY
    m = Model(s, seed=3)
    try:
        kc, vc = m.kv_setup(rows=1, n_prefill=30, max_pos=200, bucket=32)
        x = synth.frame_input(s, 1, 3, 0)
        for f, pos in enumerate([30, 31, 32, 33, 70, 130]):
            codes, h, lg = m.decode([pos], 2, f, x)
            oc, oh, olg = m.ora.decode_frame(kc, vc, [pos], 2, f, bits(x))
            assert rel_err(lg, olg) <= TOL[0], (pos, rel_err(lg, olg))
    finally:
        m.close()


def test_determinism_and_graph_equivalence(ora, monkeypatch):
    s = synth.TINY
    outs = []
    for no_graph in ("0", "0", "1"):
        monkeypatch.setenv("M3_NO_GRAPH", no_graph)
        m = Model(s, seed=4, oracle=False)
        try:
            m.kv_setup(rows=2, n_prefill=50, max_pos=100)
            x = synth.frame_input(s, 2, 4, 0)
            res = [m.decode([50 + f, 50 + f], 9, f, x, cfg_scale=1.5) for f in range(3)]
            outs.append(res)
        finally:
            m.close()
    for a, b in zip(outs[0], outs[1]):
        for u, v in zip(a, b):
            assert np.array_equal(u, v)
    for a, b in zip(outs[0], outs[2]):
        for u, v in zip(a, b):
            assert np.array_equal(u, v)


def test_errors_are_status_codes(ora):
    from autoregressive_audio_token_b200 import m3
    s = synth.TINY
    m = Model(s, seed=5, oracle=False)
    try:
        x = synth.frame_input(s, 1, 5, 0).cuda()
        codes = torch.empty(1, dtype=torch.int32, device="cuda")
        with pytest.raises(m3.M3Error) as e:
            m3.m3_decode_frame(m.ctx, [0], 1, 0, x, 0.0, 1.0, codes)
        assert e.value.code == m3.M3_ESTATE
        m.kv_setup(rows=2, n_prefill=0, max_pos=64)
        with pytest.raises(m3.M3Error) as e:
            m3.m3_decode_frame(m.ctx, [64], 1, 0, x, 0.0, 1.0, codes)
        assert e.value.code == m3.M3_ECAPACITY
        with pytest.raises(m3.M3Error) as e:
            m3.m3_decode_frame(m.ctx, [3], 1, 0, x, 1.5, 1.0, codes)  # odd rows with CFG
        assert e.value.code == m3.M3_EINVAL
        # the context is still usable
        m3.m3_decode_frame(m.ctx, [0], 1, 0, x, 0.0, 1.0, codes)
        m3.m3_sync_status(m.ctx)
        # launch accounting: parameter block, RoPE table, 5 per layer, sampler
        assert m3.m3_frame_kernels(m.ctx, 1) == 2 + 5 * s.n_layers + 1
        with pytest.raises(m3.M3Error) as e:
            m3.m3_frame_kernels(m.ctx, 0)
        assert e.value.code == m3.M3_EINVAL
        with pytest.raises(m3.M3Error) as e:  # no depth decoder in this config
            m3.m3_depth_kernels(m.ctx, 1)
        assert e.value.code == m3.M3_ESTATE
    finally:
        m.close()


# -------------------------------------------------- one 8B decoder layer ----

@pytest.mark.parametrize("ring", ["64x3", "64x2", "8x4"])
@pytest.mark.parametrize("wdtype,rows,kv_f16", [(0, 1, False), (0, 2, False), (1, 1, False),
                                                (1, 2, True)])
def test_layer8b_vs_oracle(ora, wdtype, rows, kv_f16, ring, monkeypatch):
    # 64 KB x 3 is the default ring (the down projection, whose activations
    # leave no room for it, takes the cluster-split kernel); with 64 KB x 2 a
    # 16-row unit of K = 4096 is two bf16 stages or one int8 stage and the
    # down projection streams each unit in six or three parts; with 8 KB
    # stages every GEMV splits its units into many parts
    kb, ns = ring.split("x")
    monkeypatch.setenv("M3_GEMV_STAGE_KB", kb)
    monkeypatch.setenv("M3_GEMV_STAGES", ns)
    s = synth.LAYER8B
    m = Model(s, seed=11, device="cuda", wdtype=wdtype, max_rows=2, kv_f16=kv_f16)
    try:
        kc, vc = m.kv_setup(rows=rows, n_prefill=1024, max_pos=1100)
        x = synth.frame_input(s, rows, 11, 0)
        pos = [1024] * rows
        codes, h, lg = m.decode(pos, 77, 0, x)
        oc, oh, olg = m.ora.decode_frame(kc, vc, pos, 77, 0, bits(x))
        assert rel_err(lg, olg) <= TOL[wdtype], rel_err(lg, olg)
        check_codes_teacher_forced(m, h, codes, 77, 0)
        if ring == "64x3":
            # the top-k 50 draw over the 16384-row slice, on the GPU's own logits
            m.m3.m3_set_top_k(m.ctx, 50)
            codes, h, lg = m.decode([p + 1 for p in pos], 77, 1, x)
            _check_topk_codes(ora, codes, lg, 50, 77, 1, 0.0, s.slice_start)
            m.m3.m3_set_top_k(m.ctx, 0)
        if wdtype == 1:
            # the GPU's quantised weights are the oracle's, bit for bit
            L0 = m.layers[0]
            for which, name in enumerate(["wq", "wk", "wv", "wo", "wg", "wu", "wd"]):
                W = L0[name]
                q, sc = m.m3.m3_export_weight(m.ctx, which, 0, W.shape[0], W.shape[1], True)
                qo, so = ora.quantize(bits(W), None)
                assert np.array_equal(q.numpy(), qo), name
                assert np.array_equal(sc.numpy()[:, 0], so), name
    finally:
        m.close()


@pytest.mark.parametrize("rows,wdtype", [(8, 0), (16, 0), (8, 1), (12, 0), (16, 1)])
def test_layer8b_many_rows(ora, rows, wdtype):
    # the 8B layer at 8 and 16 rows: the down projection's activations
    # (K = 12288) leave no room for the default ring, so the launch plans
    # fall back to two stages or dynamic claiming
    s = synth.LAYER8B
    m = Model(s, seed=17, device="cuda", wdtype=wdtype, max_rows=16)
    try:
        kc, vc = m.kv_setup(rows=rows, n_prefill=64, max_pos=80)
        x = synth.frame_input(s, rows, 17, 0)
        pos = [64] * rows
        cfg = 1.5 if rows % 2 == 0 else 0.0
        codes, h, lg = m.decode(pos, 5, 0, x, cfg_scale=cfg)
        oc, oh, olg = m.ora.decode_frame(kc, vc, pos, 5, 0, bits(x), cfg_scale=cfg)
        assert rel_err(lg, olg) <= TOL[wdtype], rel_err(lg, olg)
        check_codes_teacher_forced(m, h, codes, 5, 0, cfg_scale=cfg)
    finally:
        m.close()


@pytest.mark.parametrize("n_ctx", [4500, 9000])
def test_layer8b_16rows_long_context(ora, n_ctx):
    # the batched-variations workload's widest point: 8 CFG pairs (16 rows,
    # per-row KV seeds) at a song context of 4500 or 9000 frames (the
    # DiffSynth-Studio article's 9000-frame cap): 18 / 36 KV pages per row,
    # 4.5-9 k positions per split-K attention
    s = synth.LAYER8B
    rows = 16
    m = Model(s, seed=23, device="cuda", max_rows=rows)
    try:
        kc, vc = m.kv_setup(rows=rows, n_prefill=n_ctx - 1, max_pos=n_ctx, seed=23)
        x = synth.frame_input(s, rows, 23, 0)
        pos = [n_ctx - 1] * rows
        codes, h, lg = m.decode(pos, 5, 0, x, cfg_scale=1.5)
        oc, oh, olg = m.ora.decode_frame(kc, vc, pos, 5, 0, bits(x), cfg_scale=1.5)
        err = rel_err(lg, olg)
        assert err <= TOL[0], err
        assert rel_err(f32(h), f32(oh)) <= TOL[0]
        check_codes_teacher_forced(m, h, codes, 5, 0, cfg_scale=1.5)
        # the new token's K/V of two rows at the last position
        for r in (0, rows - 1):
            k, v = m.m3.m3_kv_get(m.ctx, r, s.n_layers, n_ctx, s.n_kv_heads, s.head_dim)
            assert rel_err(f32(k.numpy().view(np.uint16)[0, n_ctx - 1]),
                           f32(kc[r, 0, n_ctx - 1])) <= TOL[0]
            assert rel_err(f32(v.numpy().view(np.uint16)[0, n_ctx - 1]),
                           f32(vc[r, 0, n_ctx - 1])) <= TOL[0]
    finally:
        m.close()


# -------------------------------------------------------- depth decoder ----

@pytest.mark.parametrize("rows", [2, 16])
def test_depth_decoder_full_size(ora, rows):
    # the 8B model's depth decoder (16 heads of 64, hidden 1024, 4 layers,
    # SwiGLU 2816, 7 codebooks of 1024, input 4096): one CFG pair (the
    # attention inside the O projection's step) and 8 pairs (the attention
    # as its own step, two 8-row MMA blocks, the input projection's rows in
    # two passes): logits against the oracle, every draw by the draw rule
    s, D, cfg = synth.LAYER8B, synth.DEPTH, 1.5
    m = Model(s, seed=9, depth=D, max_rows=rows)
    try:
        assert m.m3.m3_depth_kernels(m.ctx, rows) == 1  # the persistent kernel
        h = synth.normal((rows, s.hidden), 9, "hframe", std=1.0).cuda()
        code0 = torch.tensor(([11, 16383] + [(977 * r) % 16384 for r in range(2, rows)])[:rows],
                             dtype=torch.int32, device="cuda")
        codes = torch.empty((rows, D.codebooks), dtype=torch.int32, device="cuda")
        lg = torch.empty((rows, D.codebooks, D.vocab), dtype=torch.float32, device="cuda")
        m.m3.m3_depth_decode(m.ctx, h, code0, 5, 2, cfg, 1.0, codes, logits=lg)
        torch.cuda.synchronize()
        m.m3.m3_sync_status(m.ctx)
        gc = codes.cpu().numpy()
        oc, olg = m.ora_depth.decode(bits(h), code0.cpu().numpy(), 5, 2, cfg_scale=cfg,
                                     forced=gc)
        glg = lg.cpu().numpy()
        for j in range(D.codebooks):
            assert rel_err(glg[:, j], olg[:, j]) <= TOL[1], (j, rel_err(glg[:, j], olg[:, j]))
        check_depth_draws(glg, gc, 5, 2, cfg_scale=cfg)
    finally:
        m.close()


def test_depth_decoder_row_counts_interleaved(ora):
    # one context, calls of 16, 2 and again 16 rows (the persistent kernel's
    # two attention modes): the repeated call is bit-identical to the first
    s = synth.TINY
    D = synth.DepthShape(hidden=256, n_layers=2, n_heads=4, head_dim=64, ffn=384, codebooks=7,
                         vocab=128, sem_vocab=s.slice_len, in_hidden=s.hidden)
    m = Model(s, seed=7, depth=D, max_rows=16, oracle=False)
    try:
        def call(rows, seed):
            h = synth.normal((rows, s.hidden), seed, "hframe").cuda()
            code0 = torch.tensor([(53 * r + seed) % s.slice_len for r in range(rows)],
                                 dtype=torch.int32, device="cuda")
            codes = torch.empty((rows, D.codebooks), dtype=torch.int32, device="cuda")
            lg = torch.empty((rows, D.codebooks, D.vocab), dtype=torch.float32, device="cuda")
            m.m3.m3_depth_decode(m.ctx, h, code0, 3, seed, 1.5, 1.0, codes, logits=lg)
            torch.cuda.synchronize()
            m.m3.m3_sync_status(m.ctx)
            return codes.cpu().numpy(), lg.cpu().numpy()
        c1, l1 = call(16, 1)
        for i in range(3):
            call(2, 2 + i)
        c2, l2 = call(16, 1)
        assert np.array_equal(c1, c2) and np.array_equal(l1, l2)
    finally:
        m.close()


def test_depth_decoder_separate_launches(ora):
    # codebooks of 120 entries (not whole 16-row tiles): the persistent kernel
    # does not take the shape and the decoder runs as separate launches
    s = synth.TINY
    D = synth.DepthShape(hidden=256, n_layers=2, n_heads=4, head_dim=64, ffn=384, codebooks=7,
                         vocab=120, sem_vocab=s.slice_len, in_hidden=s.hidden)
    rows, cfg = 2, 1.5
    m = Model(s, seed=6, depth=D, max_rows=rows)
    try:
        assert m.m3.m3_depth_kernels(m.ctx, rows) > 1
        h = synth.normal((rows, s.hidden), 6, "hframe").cuda()
        code0 = torch.tensor([3, 77], dtype=torch.int32, device="cuda")
        codes = torch.empty((rows, D.codebooks), dtype=torch.int32, device="cuda")
        lg = torch.empty((rows, D.codebooks, D.vocab), dtype=torch.float32, device="cuda")
        m.m3.m3_depth_decode(m.ctx, h, code0, 31, 4, cfg, 1.0, codes, logits=lg)
        torch.cuda.synchronize()
        m.m3.m3_sync_status(m.ctx)
        gc = codes.cpu().numpy()
        oc, olg = m.ora_depth.decode(bits(h), code0.cpu().numpy(), 31, 4, cfg_scale=cfg,
                                     forced=gc)
        glg = lg.cpu().numpy()
        for j in range(D.codebooks):
            assert rel_err(glg[:, j], olg[:, j]) <= TOL[1], (j, rel_err(glg[:, j], olg[:, j]))
        check_depth_draws(glg, gc, 31, 4, cfg_scale=cfg)
    finally:
        m.close()


@pytest.mark.parametrize("rows,cfg", [(1, 0.0), (2, 1.5), (4, 1.5), (12, 1.5), (16, 0.0)])
def test_depth_decoder_teacher_forced(ora, rows, cfg):
    # 1..8 rows of 4 heads: the attention inside the O projection's step;
    # 12 and 16 rows: as its own step, two 8-row MMA blocks
    s = synth.TINY
    D = synth.DepthShape(hidden=256, n_layers=2, n_heads=4, head_dim=64, ffn=384, codebooks=7,
                         vocab=128, sem_vocab=s.slice_len, in_hidden=s.hidden)
    m = Model(s, seed=6, depth=D, max_rows=max(2, rows))
    try:
        assert m.m3.m3_depth_kernels(m.ctx, rows) == 1  # the persistent kernel
        h = synth.normal((rows, s.hidden), 6, "hframe").cuda()
        code0 = torch.tensor(([3, 77, 5, 400] + [(37 * r) % s.slice_len for r in range(4, rows)])[:rows],
                             dtype=torch.int32, device="cuda")
        codes = torch.empty((rows, D.codebooks), dtype=torch.int32, device="cuda")
        lg = torch.empty((rows, D.codebooks, D.vocab), dtype=torch.float32, device="cuda")
        m.m3.m3_depth_decode(m.ctx, h, code0, 31, 4, cfg, 1.0, codes, logits=lg)
        torch.cuda.synchronize()
        m.m3.m3_sync_status(m.ctx)
        gc = codes.cpu().numpy()
        oc, olg = m.ora_depth.decode(bits(h), code0.cpu().numpy(), 31, 4, cfg_scale=cfg,
                                     forced=gc)
        glg = lg.cpu().numpy()
        for j in range(D.codebooks):
            assert rel_err(glg[:, j], olg[:, j]) <= TOL[1], (j, rel_err(glg[:, j], olg[:, j]))
        # every drawn code against the oracle's draw on the GPU's own logits
        check_depth_draws(glg, gc, 31, 4, cfg_scale=cfg)
        # quantised depth weights are bit-exact
        W = m.dw["heads"][2]
        q, sc = m.m3.m3_export_weight(m.ctx, 17 + 2, 0, W.shape[0], W.shape[1], True, W.shape[1] // 128)
        qo, so = ora.quantize(bits(W), 128)
        assert np.array_equal(q.numpy(), qo) and np.array_equal(sc.numpy(), so)
    finally:
        m.close()
