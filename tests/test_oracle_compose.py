"""Pins of the oracle's layer stack (the composition over n_layers).

The single-layer step is pinned by the unit pins (norms, RoPE, attention,
MLP wiring, the KV write); these pin how the stack composes it, which the
36-layer body relies on:
  * an L-layer body equals L one-layer bodies run in sequence, bit for bit,
    each with its own weights and its own cache slot, the output of layer l
    the input of layer l + 1 (a swapped weight or cache index, or a layer
    fed the stack's input instead of the previous output, fails);
  * a 36-layer stack whose output projections (W_o, W_d) are zero leaves the
    residual stream unchanged, and with all layers identical but one, only
    that layer's cache slot differs.
"""
import dataclasses

import numpy as np
import pytest
import torch

import synth
from oracle import oracle as O


def _cache_prefill(shape, rows, max_pos, n_prefill, seed):
    g = np.random.default_rng(seed)
    shp = (rows, shape.n_layers, max_pos, shape.n_kv_heads, shape.head_dim)
    kc, vc = np.zeros(shp, np.uint16), np.zeros(shp, np.uint16)
    for c in (kc, vc):
        v = g.standard_normal((rows, shape.n_layers, n_prefill, shape.n_kv_heads,
                               shape.head_dim)).astype(np.float32)
        c[:, :, :n_prefill] = O.bits(torch.from_numpy(v).to(torch.bfloat16))
    return kc, vc


@pytest.mark.parametrize("wfmt", [0, 1])
def test_stack_equals_chained_single_layers(wfmt):
    s3 = dataclasses.replace(synth.TINY, n_layers=3)
    s1 = dataclasses.replace(synth.TINY, n_layers=1)
    layers = [synth.layer_weights(s3, 31, l) for l in range(3)]
    body3 = O.Body(s3, layers, None, None, wfmt=wfmt)
    ones = [O.Body(s1, [layers[l]], None, None, wfmt=wfmt) for l in range(3)]
    rows, max_pos, n0 = 2, 24, 9
    kc3, vc3 = _cache_prefill(s3, rows, max_pos, n0, 5)
    kc1 = [np.ascontiguousarray(kc3[:, l:l + 1]) for l in range(3)]
    vc1 = [np.ascontiguousarray(vc3[:, l:l + 1]) for l in range(3)]
    for t in range(6):
        pos = [n0 + t, n0 + 2 * t]  # the rows at different positions
        x = O.bits(synth.frame_input(s3, rows, 7, t))
        y3 = body3.body(kc3, vc3, pos, x.copy())
        y = x.copy()
        for l in range(3):
            y = ones[l].body(kc1[l], vc1[l], pos, y)
        assert np.array_equal(y3, y), t
        for l in range(3):
            assert np.array_equal(kc3[:, l], kc1[l][:, 0]), (t, l)
            assert np.array_equal(vc3[:, l], vc1[l][:, 0]), (t, l)
    # the layers are distinct: the same chain in another order differs
    kr = [np.ascontiguousarray(kc3[:, l:l + 1]) for l in range(3)]
    vr = [np.ascontiguousarray(vc3[:, l:l + 1]) for l in range(3)]
    yr = x.copy()
    for l in (2, 1, 0):
        yr = ones[l].body(kr[l], vr[l], pos, yr)
    assert not np.array_equal(yr, y3)


def test_zero_projection_stack_36_layers():
    s = dataclasses.replace(synth.TINY, n_layers=36)
    base = synth.layer_weights(s, 3, 0)
    base["wo"] = torch.zeros_like(base["wo"])
    base["wd"] = torch.zeros_like(base["wd"])
    odd = dict(base)
    odd["k_norm"] = (base["k_norm"].float() * 1.5).to(torch.bfloat16)  # changes K only
    layers = [odd if l == 17 else base for l in range(36)]
    body = O.Body(s, layers, None, None)
    rows, max_pos, n0 = 2, 16, 5
    kc, vc = _cache_prefill(s, rows, max_pos, n0, 8)
    x = O.bits(synth.frame_input(s, rows, 4, 0))
    pos = [n0, n0 + 3]
    y = body.body(kc, vc, pos, x.copy())
    assert np.array_equal(y, x)  # zero output projections: the residual passes through
    for r, p in enumerate(pos):
        for l in range(36):
            same_k = np.array_equal(kc[r, l, p], kc[r, 0, p])
            assert same_k == (l != 17), (r, l)
            assert np.array_equal(vc[r, l, p], vc[r, 0, p]), (r, l)  # V has no norm
        assert np.any(kc[r, 0, p] != 0)
