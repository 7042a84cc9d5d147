"""The allocation-free draw (m3_sample_noalloc) against m3_decode_frame and
against the oracle's sampler.

Some callers cannot allocate GPU memory on the thread that draws a frame: a
real-time audio callback that must not block on the allocator, a host
thread that runs while another thread captures a CUDA graph (an allocation
there would break the capture), or an embedder whose device memory is
budgeted up front.  For them m3_sample_noalloc runs the frame's lm_head +
CFG + Gumbel-argmax draw with its scratch in a static device array of the
library.  This test runs it on m3_decode_frame's own final hidden state,
twice in a row (two frames), and requires
  * the same codes and logits as m3_decode_frame (the same kernel: identical,
    checked within the parity tolerance, max relative error 2e-2 bf16 /
    5e-2 int8);
  * logits within that tolerance of the oracle's sampler on the same hidden
    state, and codes equal to the oracle's draw except where the oracle's
    top-2 margin is below 1e-3;
  * no device allocation: free device memory is unchanged around a call
    after the first;
for bf16 weights, bf16 with the end token as an extra candidate, and int8
weights with one scale per row.  Collected last so that a failure here does
not stop the rest of the GPU suite.
"""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _rel(a, b):
    return float(np.max(np.abs(a.astype(np.float64) - b.astype(np.float64))) /
                 max(np.max(np.abs(b.astype(np.float64))), 1e-30))


@pytest.mark.parametrize("variant", ["bf16", "bf16_end", "int8"])
def test_sample_noalloc_matches_decode_frame_and_oracle(variant):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from autoregressive_audio_token_b200 import m3
    from oracle import oracle as O
    s = synth.TINY_END if variant == "bf16_end" else synth.TINY
    wdtype = m3.M3_W_INT8 if variant == "int8" else m3.M3_W_BF16
    tol = 5e-2 if variant == "int8" else 2e-2
    has_end = s.end_token >= 0
    n_cand = s.slice_len + (1 if has_end else 0)
    rows = 2
    ctx = m3.m3_create(m3.config_from_shapes(s, None, max_rows=rows))
    try:
        layers = [synth.layer_weights(s, 3, l) for l in range(s.n_layers)]
        fn, lm = synth.final_norm(s, 3), synth.lm_head_slice(s, 3)
        end_row = synth.lm_head_end_row(s, 3) if has_end else None
        m3.m3_load_weights(ctx, [{k: v.cuda() for k, v in L.items()} for L in layers], 0,
                           fn.cuda(), lm.cuda(), wdtype=wdtype,
                           lm_end_row=end_row.cuda() if has_end else None)
        body = O.Body(s, layers, fn, lm, wfmt=1 if variant == "int8" else 0,
                      lm_end_row=end_row)
        m3.m3_kv_alloc(ctx, rows, 128)
        K, V = synth.kv_prefill(s, rows, 32, 3)
        for r in range(rows):
            m3.m3_kv_set(ctx, r, K[r].cuda(), V[r].cuda())
        x = synth.frame_input(s, rows, 3, 0).cuda()
        codes = torch.empty(rows, dtype=torch.int32, device="cuda")
        h = torch.empty((rows, s.hidden), dtype=torch.bfloat16, device="cuda")
        lg = torch.empty((rows, n_cand), dtype=torch.float32, device="cuda")
        codes2 = torch.empty(rows, dtype=torch.int32, device="cuda")
        lg2 = torch.empty_like(lg)
        for frame in range(2):  # two calls in a row
            m3.m3_decode_frame(ctx, [32 + frame] * rows, 17, frame, x, 1.5, 1.0, codes, h, lg)
            codes2.fill_(-1)
            torch.cuda.synchronize()
            free0 = torch.cuda.mem_get_info()[0]
            m3.m3_sample_noalloc(ctx, h, 17, frame, 1.5, 1.0, codes2, lg2)
            torch.cuda.synchronize()
            free1 = torch.cuda.mem_get_info()[0]
            m3.m3_sync_status(ctx)
            if frame == 1:  # (the first call may still load kernel code lazily)
                assert free1 == free0, (free0, free1)
            g, gd = lg2.cpu().numpy(), lg.cpu().numpy()
            assert _rel(g, gd) <= tol
            assert np.array_equal(codes2.cpu().numpy(), codes.cpu().numpy())
            # the oracle's sampler on the same final hidden state
            hb = O.bits(h)
            oc, olg, margin = body.sample(hb, 17, frame, cfg_scale=1.5, with_margin=True)
            assert olg.shape == g.shape
            assert _rel(g, olg) <= tol, _rel(g, olg)
            gc = codes2.cpu().numpy()
            mism = oc != gc
            assert np.all(margin[mism] < 1e-3), (oc, gc, margin)
        with pytest.raises(m3.M3Error) as e:
            m3.m3_sample_noalloc(ctx, torch.zeros((17, s.hidden), dtype=torch.bfloat16,
                                                  device="cuda"), 1, 0, 0.0, 1.0,
                                 torch.empty(17, dtype=torch.int32, device="cuda"))
        assert e.value.code == m3.M3_EINVAL
    finally:
        m3.m3_destroy(ctx)
