"""GPU checks of the pieces the frame parity tests reach only through their
decisions, through the C ABI:
  * the Gumbel noise of the draws, bit for bit against the oracle's
    generator (the diffusers issue "MiniMax Music 3 modular pipeline",
    finding 3: Gumbel-argmax on counter-based noise), over the code block's
    vocab rows, the end token's row and the depth decoder's (j << 32) | i
    indices;
  * failure detection without a GPU fault: host-injected allocation, copy and
    graph-capture failures return their status and leave the context usable;
    a bounded device-side wait that is never satisfied gives up and is
    reported as M3_ETIMEOUT;
  * resume: frames 16..31 decoded after the KV cache of frames 0..15 was read
    back (m3_kv_get) and written into a new context (m3_kv_set) give the same
    codes and bits as decoding 0..31 straight.
"""
import numpy as np
import pytest
import torch

import synth
from gpu_util import Model, bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


# ------------------------------------------------------------------ noise ----

def test_gumbel_noise_bit_exact(ora):
    from autoregressive_audio_token_b200 import m3
    cases = [(0, 0, 0, 151675, 16384), (1000, 7, 1, 151675, 16384), (99, 123456, 3, 151675, 16384),
             (2 ** 63 + 5, 2 ** 40, 7, 0, 16384), (17, 4, 0, 151670, 1)]
    cases += [(31, 4, 1, j << 32, 1024) for j in range(1, 8)]
    cases += [(5, 1499, 0, 1024, 30000)]
    total = 0
    for seed, frame, row, base, n in cases:
        g = m3.m3_gumbel_fill(seed, frame, row, base, n)
        torch.cuda.synchronize()
        got = g.cpu().numpy().view(np.uint32)
        ref = ora.gumbel_fill(seed, frame, row, base, n).view(np.uint32)
        bad = np.nonzero(got != ref)[0]
        assert bad.size == 0, (seed, frame, row, base, bad[:5], got[bad[:5]], ref[bad[:5]])
        total += n
    assert total >= 100000


# -------------------------------------------------------- failure paths ----

def _frame(m, pos, frame, x):
    return m.decode([pos] * x.shape[0], 5, frame, x)


def test_injected_failures_leave_context_usable(ora):
    s = synth.TINY
    m = Model(s, seed=2, max_rows=2, oracle=False)
    ref = Model(s, seed=2, max_rows=2, oracle=False)
    M3 = m.m3
    try:
        for mm in (m, ref):
            M3.m3_kv_alloc(mm.ctx, 2, 600, 0, 256)
        K, V = synth.kv_prefill(s, 2, 100, 2)
        # a host-to-device copy of a host source fails, then succeeds
        M3.m3_inject_fault(m.ctx, M3.M3_FAULT_H2D, 1)
        with pytest.raises(M3.M3Error) as e:
            M3.m3_kv_set(m.ctx, 0, K[0], V[0])
        assert e.value.code == M3.M3_ECUDA and "injected" in str(e.value)
        for mm in (m, ref):
            for r in range(2):
                M3.m3_kv_set(mm.ctx, r, K[r], V[r])
        x = synth.frame_input(s, 2, 2, 0)
        # the first frame's graph capture fails, then the frame runs
        M3.m3_inject_fault(m.ctx, M3.M3_FAULT_GRAPH, 1)
        with pytest.raises(M3.M3Error) as e:
            _frame(m, 100, 0, x)
        assert e.value.code == M3.M3_ECUDA
        a = _frame(m, 100, 0, x)
        b = _frame(ref, 100, 0, x)
        assert all(np.array_equal(u, v) for u, v in zip(a, b))
        # the KV bucket of position 300 cannot be allocated, then can
        M3.m3_inject_fault(m.ctx, M3.M3_FAULT_ALLOC, 1)
        with pytest.raises(M3.M3Error) as e:
            _frame(m, 300, 1, x)
        assert e.value.code == M3.M3_ENOMEM
        a = _frame(m, 300, 1, x)
        b = _frame(ref, 300, 1, x)
        assert all(np.array_equal(u, v) for u, v in zip(a, b))
        # a scheduled fault that never comes due can be cancelled
        M3.m3_inject_fault(m.ctx, M3.M3_FAULT_ALLOC, 1000)
        M3.m3_inject_fault(m.ctx, M3.M3_FAULT_NONE, 0)
        with pytest.raises(M3.M3Error) as e:
            M3.m3_inject_fault(m.ctx, 9, 1)
        assert e.value.code == M3.M3_EINVAL
    finally:
        m.close()
        ref.close()


def test_fault_environment_variable(ora, monkeypatch):
    from autoregressive_audio_token_b200 import m3
    s = synth.TINY
    monkeypatch.setenv("M3_FAULT", "alloc:3")
    with pytest.raises(m3.M3Error) as e:
        m3.m3_create(m3.config_from_shapes(s))
    assert e.value.code == m3.M3_ENOMEM
    monkeypatch.setenv("M3_FAULT", "bogus")
    with pytest.raises(m3.M3Error) as e:
        m3.m3_create(m3.config_from_shapes(s))
    assert e.value.code == m3.M3_EINVAL
    monkeypatch.delenv("M3_FAULT")
    m3.m3_destroy(m3.m3_create(m3.config_from_shapes(s)))


def test_bounded_wait_gives_up(ora):
    s = synth.TINY
    m = Model(s, seed=2, max_rows=2, oracle=False)
    M3 = m.m3
    try:
        M3.m3_kv_alloc(m.ctx, 2, 128)
        x = synth.frame_input(s, 2, 2, 0)
        before = _frame(m, 10, 0, x)
        M3.m3_stalled_wait(m.ctx, 2000)
        with pytest.raises(M3.M3Error) as e:
            M3.m3_sync_status(m.ctx)
        assert e.value.code == M3.M3_ETIMEOUT
        M3.m3_sync_status(m.ctx)  # cleared
        after = _frame(m, 10, 0, x)  # the context still decodes, identically
        assert all(np.array_equal(u, v) for u, v in zip(before, after))
        with pytest.raises(M3.M3Error):
            M3.m3_stalled_wait(m.ctx, 0)
    finally:
        m.close()


# ----------------------------------------------------------------- resume ----

def test_resume_from_kv_roundtrip(ora):
    """32 frames with each frame's code fed back as the next input, straight,
    against 16 frames, the cache read back and written into a new context,
    and 16 more: identical codes, hidden states and logits."""
    from autoregressive_audio_token_b200 import m3 as M3
    s = synth.TINY
    rows, p0, F = 2, 40, 32
    table = synth.embedding(s, 4).cuda()

    def run(m, frames, x, pos0, f0):
        out = []
        codes = torch.empty(rows, dtype=torch.int32, device="cuda")
        h = torch.empty((rows, s.hidden), dtype=torch.bfloat16, device="cuda")
        lg = torch.empty((rows, s.slice_len), dtype=torch.float32, device="cuda")
        for f in range(frames):
            M3.m3_decode_frame(m.ctx, [pos0 + f] * rows, 8, f0 + f, x, 1.5, 1.0, codes, h, lg)
            out.append((codes.cpu().numpy().copy(), bits(h), lg.cpu().numpy().copy()))
            M3.m3_embed(m.ctx, codes, table, s.slice_start, x)
        torch.cuda.synchronize()
        M3.m3_sync_status(m.ctx)
        return out

    K, V = synth.kv_prefill(s, rows, p0, 4)
    x0 = synth.frame_input(s, rows, 4, 0).cuda()
    a = Model(s, seed=4, max_rows=rows, oracle=False)
    b = Model(s, seed=4, max_rows=rows, oracle=False)
    c = Model(s, seed=4, max_rows=rows, oracle=False)
    try:
        for mm in (a, b):
            M3.m3_kv_alloc(mm.ctx, rows, 128)
            for r in range(rows):
                M3.m3_kv_set(mm.ctx, r, K[r].cuda(), V[r].cuda())
        straight = run(a, F, x0.clone(), p0, 0)
        xb = x0.clone()
        first = run(b, F // 2, xb, p0, 0)
        # checkpoint: positions 0 .. p0 + F/2 - 1 of every row, into a fresh context
        n = p0 + F // 2
        M3.m3_kv_alloc(c.ctx, rows, 128)
        for r in range(rows):
            k, v = M3.m3_kv_get(b.ctx, r, s.n_layers, n, s.n_kv_heads, s.head_dim)
            M3.m3_kv_set(c.ctx, r, k.view(torch.bfloat16), v.view(torch.bfloat16))
        b.close()
        second = run(c, F - F // 2, xb, p0 + F // 2, F // 2)
        for f, (u, v) in enumerate(zip(straight, first + second)):
            for i in range(3):
                assert np.array_equal(u[i], v[i]), (f, i)
    finally:
        a.close()
        b.close()
        c.close()
