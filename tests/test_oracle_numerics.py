"""Pins for the oracle's building blocks: int8 quantiser, GEMV, RMSNorm, RoPE,
attention.  Each check comes from mathematics or from a closed form, not
from re-running the oracle's own formula.

Precision follows "MiniMax Music 3 on Metal" (section "Precision is the
reference's"): fp32 norms, rope and attention sums with bf16 roundings, int8
weight-only with a scale per row or per group of 128.
"""
import math

import numpy as np
import pytest


def _bf16_bits_from_f32(x):
    """Exact bf16 bit patterns of values already representable in bf16."""
    x = np.asarray(x, np.float32)
    b = x.view(np.uint32)
    assert ((b & 0xFFFF) == 0).all(), "value not representable in bf16"
    return (b >> 16).astype(np.uint16)


def _rand_bf16(rng, shape, std=1.0):
    x = (rng.standard_normal(shape) * std).astype(np.float32)
    b = x.view(np.uint32) & 0xFFFF0000  # truncate to bf16
    return (b >> 16).astype(np.uint16)


def _f(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


# ------------------------------------------------------------ quantiser -----

@pytest.mark.parametrize("group", [None, 128])
def test_quantize_roundtrip_bound_and_absmax(ora, group):
    rng = np.random.default_rng(1)
    w = _rand_bf16(rng, (64, 512), std=0.02)
    w[3] = 0  # a zero row
    q, s = ora.quantize(w, group)
    wf = _f(w)
    g = 512 if group is None else group
    s2 = s.reshape(64, -1)
    for r in range(64):
        for j in range(512 // g):
            blk = wf[r, j * g:(j + 1) * g].astype(np.float64)
            qb = q[r, j * g:(j + 1) * g].astype(np.int64)
            sc = float(s2[r, j])
            amax = np.abs(blk).max()
            if amax == 0:
                assert sc == 0 and (qb == 0).all()
                continue
            # the absmax element maps to +-127
            assert abs(qb[np.argmax(np.abs(blk))]) == 127
            # round trip within half a step; fl(w/s) may be off by |w/s| * 2^-24 <= 127 * 2^-24
            assert np.all(np.abs(blk - sc * qb) <= sc * (0.5 + 127 * 2.0 ** -24) * (1 + 1e-12))
            assert np.all(np.abs(qb) <= 127)


def test_quantize_idempotent(ora):
    # re-quantising a dequantised row returns the same codes when the
    # dequantised values are representable (scale a power of two)
    rng = np.random.default_rng(2)
    q0 = rng.integers(-127, 128, size=(16, 256)).astype(np.int8)
    q0[:, 0] = 127
    q0[:, 128] = -127
    w = _bf16_bits_from_f32(q0.astype(np.float32) * np.float32(2.0 ** -7))
    q, s = ora.quantize(w, None)
    assert (s == np.float32(2.0 ** -7)).all()
    assert (q == q0).all()
    q, s = ora.quantize(w, 128)
    assert (q == q0).all()


def test_int8_gemv_equals_bf16_on_exact_multiples(ora):
    # y = s * sum(q x) and sum((s q) x) agree bit for bit when s is a power of two
    rng = np.random.default_rng(3)
    q0 = rng.integers(-127, 128, size=(40, 384)).astype(np.int8)
    q0[:, 5] = -127
    q0[:, 133] = 127
    q0[:, 300] = -127
    w = _bf16_bits_from_f32(q0.astype(np.float32) * np.float32(2.0 ** -9))
    x = rng.standard_normal(384).astype(np.float32)
    y_bf = ora.gemv(w=w, wfmt=0, x=x)
    q, s = ora.quantize(w, None)
    y_q = ora.gemv(q=q, s=s, wfmt=1, x=x)
    assert np.array_equal(y_bf, y_q)
    qg, sg = ora.quantize(w, 128)
    y_g = ora.gemv(q=qg, s=sg, wfmt=2, x=x)
    ref = (w.astype(np.uint32) << 16).view(np.float32).astype(np.float64) @ x.astype(np.float64)
    assert np.allclose(y_g, ref, rtol=0, atol=1e-4 * np.abs(ref).max())


def test_gemv_vs_fp64(ora):
    rng = np.random.default_rng(4)
    for rows, cols in [(1, 1), (3, 7), (17, 256), (9, 4096)]:
        w = _rand_bf16(rng, (rows, cols), 0.02)
        x = rng.standard_normal(cols).astype(np.float32)
        y = ora.gemv(w=w, wfmt=0, x=x)
        ref = _f(w).astype(np.float64) @ x.astype(np.float64)
        bound = cols * 2.0 ** -24 * (np.abs(_f(w)).astype(np.float64) @ np.abs(x)) + 1e-30
        assert np.all(np.abs(y - ref) <= bound)


def test_gemv_rows_are_not_transposed(ora):
    # a single 1 at (r, c) picks x[c] into y[r]
    w = np.zeros((5, 7), np.float32)
    w[3, 6] = 1.0
    x = np.arange(7, dtype=np.float32) + 1
    y = ora.gemv(w=_bf16_bits_from_f32(w), wfmt=0, x=x)
    assert y.tolist() == [0, 0, 0, 7, 0]


# --------------------------------------------------------------- RMSNorm ----

@pytest.mark.parametrize("rows", [2, 4, 600])
def test_rmsnorm_vs_fp64(ora, rows):
    # the contract check of "MiniMax Music 3 on Metal" (Receipts, kernel
    # contract): rms norm against float64 at 2, 4 and 600 rows of 4096
    rng = np.random.default_rng(rows)
    H = 4096
    eps = 1e-6
    g = _rand_bf16(rng, (H,), 0.01)
    g = ((np.float32(1.0) + _f(g)).view(np.uint32) >> 16).astype(np.uint16)  # 1 + small, truncated
    x = _f(_rand_bf16(rng, (rows, H), 1.0))
    gf = _f(g).astype(np.float64)
    for r in range(rows):
        out = ora.rmsnorm(x[r], g, eps)
        xr = x[r].astype(np.float64)
        ref = gf * xr / np.sqrt(np.mean(xr * xr) + eps)
        # two bf16 roundings (2 * 2^-8 relative) plus the fp32 sum (k * 2^-24)
        tol = np.abs(ref) * (2 * 2.0 ** -8 + H * 2.0 ** -24) + 1e-30
        assert np.all(np.abs(out - ref) <= tol)


def test_rmsnorm_scale_invariant(ora):
    rng = np.random.default_rng(5)
    H = 1024
    g = _bf16_bits_from_f32(np.ones(H, np.float32))
    x = _f(_rand_bf16(rng, (H,)))
    base = ora.rmsnorm(x, g, 0.0)
    for k in (-8, -3, 1, 6):
        assert np.array_equal(ora.rmsnorm(x * np.float32(2.0 ** k), g, 0.0), base)
    # output has unit RMS up to the bf16 rounding
    assert abs(math.sqrt(np.mean(base.astype(np.float64) ** 2)) - 1.0) < 2 ** -8


def test_rmsnorm_gain_is_elementwise(ora):
    H = 64
    x = np.ones(H, np.float32)
    g = np.zeros(H, np.float32)
    g[10] = 2.0
    out = ora.rmsnorm(x, _bf16_bits_from_f32(g), 0.0)
    assert out[10] == 2.0 and np.count_nonzero(out) == 1


# ------------------------------------------------------------------ RoPE ----

def test_rope_closed_form_basis_vectors(ora):
    theta = 1e6
    d = 8
    for pos in (0, 1, 5, 1499, 8999):
        for i in range(d // 2):
            v = np.zeros(d, np.float32)
            v[i] = 1.0
            out = ora.rope(v, pos, theta)
            ang = pos * theta ** (-2.0 * i / d)
            # (e_i) -> cos * e_i + sin * e_{i+d/2}
            assert abs(out[i] - math.cos(ang)) < 1e-6
            assert abs(out[i + d // 2] - math.sin(ang)) < 1e-6
            assert np.count_nonzero(np.abs(out) > 1e-7) <= 2


def test_rope_identity_at_zero_and_norm_preserving(ora):
    rng = np.random.default_rng(6)
    v = rng.standard_normal(128).astype(np.float32)
    assert np.array_equal(ora.rope(v, 0, 1e6), v)
    for pos in (1, 77, 1500, 9000):
        out = ora.rope(v, pos, 1e6)
        assert abs(np.linalg.norm(out.astype(np.float64)) - np.linalg.norm(v.astype(np.float64))) \
            < 1e-5 * np.linalg.norm(v)


def test_rope_relative_position(ora):
    rng = np.random.default_rng(7)
    q = rng.standard_normal(128).astype(np.float32)
    k = rng.standard_normal(128).astype(np.float32)
    def dot(m, n):
        return float(np.dot(ora.rope(q, m, 1e6).astype(np.float64), ora.rope(k, n, 1e6).astype(np.float64)))
    for m, n, t in [(10, 3, 100), (500, 499, 1000), (7, 7, 300)]:
        assert abs(dot(m, n) - dot(m + t, n + t)) < 1e-3


# ------------------------------------------------------------- attention ----

def test_attention_vs_fp64_softmax(ora):
    rng = np.random.default_rng(8)
    for n, d in [(1, 64), (2, 64), (37, 64), (300, 64), (129, 128)]:
        q = rng.standard_normal(d).astype(np.float32)
        k = rng.standard_normal((n, d)).astype(np.float32)
        v = rng.standard_normal((n, d)).astype(np.float32)
        out = ora.attention(q, k, v)
        s = (k.astype(np.float64) @ q.astype(np.float64)) / math.sqrt(d)
        p = np.exp(s - s.max())
        p /= p.sum()
        ref = p @ v.astype(np.float64)
        assert np.allclose(out, ref, rtol=0, atol=1e-5 * max(1.0, np.abs(ref).max()))


def test_attention_special_cases(ora):
    rng = np.random.default_rng(9)
    d = 64
    q = rng.standard_normal(d).astype(np.float32)
    v = rng.standard_normal((5, d)).astype(np.float32)
    k = rng.standard_normal((1, d)).astype(np.float32)
    assert np.array_equal(ora.attention(q, k, v[:1]), v[0])  # one position -> v_0
    kk = np.repeat(k, 5, 0)  # equal keys -> mean of V
    assert np.allclose(ora.attention(q, kk, v), v.astype(np.float64).mean(0), atol=1e-6)


def test_gemv_fp64_comparator(ora):
    """The summation-order comparator of the oracle's GEMV: with fp64 sums the
    result is the fp64 dot product rounded once to fp32 (numpy's fp64 matmul,
    within one fp32 step), in every weight format; outside the block the
    sequential fp32 definition is back."""
    rng = np.random.default_rng(5)
    rows, cols = 64, 4096
    w = (rng.standard_normal((rows, cols)).astype(np.float32) * 0.02)
    wb = (w.view(np.uint32) >> 16).astype(np.uint16)
    wf = (wb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    x = rng.standard_normal(cols).astype(np.float32)
    y32 = ora.gemv(w=wb, wfmt=0, x=x)
    with ora.accum64():
        y64 = ora.gemv(w=wb, wfmt=0, x=x)
        q, s = ora.quantize(wb, None)
        yq = ora.gemv(q=q, s=s, wfmt=1, x=x)
        qg, sg = ora.quantize(wb, 128)
        yg = ora.gemv(q=qg, s=sg, wfmt=2, x=x)
    ref = (wf @ x.astype(np.float64)).astype(np.float32)
    step = np.spacing(np.abs(ref))
    assert np.all(np.abs(y64 - ref) <= step)
    refq = (q.astype(np.float64) @ x.astype(np.float64) * s.astype(np.float64)).astype(np.float32)
    assert np.all(np.abs(yq - refq) <= np.spacing(np.abs(refq)))
    refg = sum((qg[:, g * 128:(g + 1) * 128].astype(np.float64) @ x[g * 128:(g + 1) * 128]
                .astype(np.float64)) * sg[:, g] for g in range(cols // 128)).astype(np.float32)
    assert np.all(np.abs(yg - refg) <= 2 * np.spacing(np.abs(refg)))
    assert np.array_equal(ora.gemv(w=wb, wfmt=0, x=x), y32)
    assert not np.array_equal(y32, y64)  # the two orders do differ
