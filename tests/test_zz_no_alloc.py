"""The allocation-free draw (m3_sample_noalloc) against m3_decode_frame.

Callers that cannot allocate GPU memory on their decode thread use
m3_sample_noalloc with scratch that lives in a static device array.  This
test runs it on m3_decode_frame's own final hidden state, twice in a row
(two frames), and requires the same codes and the same logits (within the
parity tolerance, max relative error 2e-2; the kernel is the same, so they
are expected to be identical).  Collected last so that a failure here does
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


def test_sample_noalloc_matches_decode_frame():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from autoregressive_audio_token_b200 import m3
    s = synth.TINY
    rows = 2
    ctx = m3.m3_create(m3.config_from_shapes(s, None, max_rows=rows))
    try:
        layers = [{k: v.cuda() for k, v in synth.layer_weights(s, 3, l).items()}
                  for l in range(s.n_layers)]
        m3.m3_load_weights(ctx, layers, 0, synth.final_norm(s, 3).cuda(),
                           synth.lm_head_slice(s, 3).cuda())
        m3.m3_kv_alloc(ctx, rows, 128)
        K, V = synth.kv_prefill(s, rows, 32, 3)
        for r in range(rows):
            m3.m3_kv_set(ctx, r, K[r].cuda(), V[r].cuda())
        x = synth.frame_input(s, rows, 3, 0).cuda()
        for frame in range(2):  # two calls in a row
            codes = torch.empty(rows, dtype=torch.int32, device="cuda")
            h = torch.empty((rows, s.hidden), dtype=torch.bfloat16, device="cuda")
            lg = torch.empty((rows, s.slice_len), dtype=torch.float32, device="cuda")
            m3.m3_decode_frame(ctx, [32 + frame] * rows, 17, frame, x, 1.5, 1.0, codes, h, lg)
            codes2 = torch.full((rows,), -1, dtype=torch.int32, device="cuda")
            lg2 = torch.empty_like(lg)
            m3.m3_sample_noalloc(ctx, h, 17, frame, 1.5, 1.0, codes2, lg2)
            torch.cuda.synchronize()
            m3.m3_sync_status(ctx)
            assert _rel(lg2.cpu().numpy(), lg.cpu().numpy()) <= 2e-2
            assert np.array_equal(codes2.cpu().numpy(), codes.cpu().numpy())
        with pytest.raises(m3.M3Error) as e:
            m3.m3_sample_noalloc(ctx, torch.zeros((17, s.hidden), dtype=torch.bfloat16,
                                                  device="cuda"), 1, 0, 0.0, 1.0,
                                 torch.empty(17, dtype=torch.int32, device="cuda"))
        assert e.value.code == m3.M3_EINVAL
    finally:
        m3.m3_destroy(ctx)
