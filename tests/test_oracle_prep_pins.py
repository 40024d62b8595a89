"""Pins of the feature-preparation oracle (Video DeltaNet, Section 2.3: a
depthwise 5 x 5 spatial and five-tap temporal short convolution on K and V,
then SiLU; L2 normalisation of Q and K).  Each test checks the oracle against
something other than its own formula: brute force, impulse responses,
identity filters, textbook values, or a symmetry."""

import numpy as np
import pytest

import oracle as ref
from frame_wise_delta_vda_b200 import inputs as gen


def _brute_conv(X, ws, wt):
    """Direct 3-D cross-correlation with the outer-product kernel
    wt[c, s] * ws[c, i, j] and explicit bounds checks (zero outside)."""
    T, Hl, Wl, d = X.shape
    out = np.zeros_like(X)
    for t in range(T):
        for y in range(Hl):
            for x in range(Wl):
                for c in range(d):
                    acc = 0.0
                    for s in range(5):
                        tt = t + s - 2
                        if not 0 <= tt < T:
                            continue
                        for i in range(5):
                            yy = y + i - 2
                            if not 0 <= yy < Hl:
                                continue
                            for j in range(5):
                                xx = x + j - 2
                                if 0 <= xx < Wl:
                                    acc += wt[c, s] * ws[c, i, j] * X[tt, yy, xx, c]
                    out[t, y, x, c] = acc
    return out


def test_short_conv_equals_brute_force_3d():
    rng = np.random.default_rng(500)
    T, Hl, Wl, d = 4, 3, 6, 2
    X = rng.standard_normal((T, Hl * Wl, d))
    ws = rng.standard_normal((d, 5, 5))
    wt = rng.standard_normal((d, 5))
    got = ref.short_conv(X, ws, wt, Hl, Wl)
    want = _brute_conv(X.reshape(T, Hl, Wl, d), ws, wt).reshape(T, Hl * Wl, d)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_spatial_and_temporal_filters_commute():
    rng = np.random.default_rng(501)
    X = rng.standard_normal((5, 4, 7, 3))
    ws = rng.standard_normal((3, 5, 5))
    wt = rng.standard_normal((3, 5))
    a = ref.conv_temporal(ref.conv_spatial(X, ws), wt)
    b = ref.conv_spatial(ref.conv_temporal(X, wt), ws)
    np.testing.assert_allclose(a, b, atol=1e-12)


def test_impulse_response_is_the_flipped_filter():
    """A unit impulse at (t0, y0, x0) in channel c comes out as the filter
    mirrored about the impulse (cross-correlation), clipped by the zero
    padding; other channels stay zero."""
    rng = np.random.default_rng(502)
    T, Hl, Wl, d = 7, 6, 6, 2
    ws = rng.standard_normal((d, 5, 5))
    wt = rng.standard_normal((d, 5))
    X = np.zeros((T, Hl, Wl, d))
    t0, y0, x0, c = 3, 1, 4, 1
    X[t0, y0, x0, c] = 1.0
    out = ref.conv_temporal(ref.conv_spatial(X, ws), wt)
    want = np.zeros_like(X)
    for s in range(5):
        for i in range(5):
            for j in range(5):
                t, y, x = t0 - (s - 2), y0 - (i - 2), x0 - (j - 2)
                if 0 <= t < T and 0 <= y < Hl and 0 <= x < Wl:
                    want[t, y, x, c] = wt[c, s] * ws[c, i, j]
    np.testing.assert_array_equal(out, want)


def test_constant_input_sums_in_bounds_taps():
    """On a constant input every output is the sum of the filter taps that land
    inside the clip: all 125 in the interior, fewer at edges and corners."""
    d = 1
    ws = np.arange(25, dtype=np.float64).reshape(1, 5, 5) / 10
    wt = np.array([[1.0, 2.0, 3.0, 4.0, 5.0]])
    X = np.ones((6, 5, 5, d))
    out = ref.conv_temporal(ref.conv_spatial(X, ws), wt)
    assert out[2, 2, 2, 0] == pytest.approx(ws.sum() * wt.sum())
    # frame 0, corner (0, 0): taps s >= 2, i >= 2, j >= 2 only
    assert out[0, 0, 0, 0] == pytest.approx(ws[0, 2:, 2:].sum() * wt[0, 2:].sum())


def test_silu_and_l2_textbook_values():
    assert ref.silu(0.0) == 0.0
    assert ref.silu(40.0) == pytest.approx(40.0)
    assert abs(ref.silu(-40.0)) < 1e-15
    assert ref.silu(1.0) == pytest.approx(1.0 / (1.0 + np.exp(-1.0)))
    x = np.array([[3.0, 4.0]])
    np.testing.assert_allclose(ref.l2_normalize(x), x / np.sqrt(25.0 + ref.L2_EPS))
    np.testing.assert_array_equal(ref.l2_normalize(np.zeros((1, 4))), np.zeros((1, 4)))


def test_identity_filters_leave_only_the_pointwise_maps():
    """Centre-tap filters make the convolution the identity, so the prepared
    features are L2(q), L2(SiLU(k)), SiLU(v) in the [B, H, T, U, d] layout."""
    pw = gen.PrepWorkload("id", 2, 3, 4, 3, 5, 8, 7)
    x = gen.make_prep_inputs(pw)
    ident_s = np.zeros((pw.H, pw.d, 5, 5))
    ident_s[:, :, 2, 2] = 1.0
    ident_t = np.zeros((pw.H, pw.d, 5))
    ident_t[:, :, 2] = 1.0
    q, k, v = (gen.as_f64(x[n]) for n in ("q", "k", "v"))
    qo, ko, vo = ref.prep(q, k, v, ident_s, ident_t, ident_s, ident_t, pw.Hl, pw.Wl)
    for b in range(pw.B):
        for h in range(pw.H):
            kk = k[b, :, :, h]
            np.testing.assert_allclose(qo[b, h], q[b, :, :, h] / np.sqrt((q[b, :, :, h] ** 2).sum(-1, keepdims=True)
                                                                         + ref.L2_EPS), atol=1e-14)
            sk = kk / (1 + np.exp(-kk))
            np.testing.assert_allclose(ko[b, h], sk / np.sqrt((sk ** 2).sum(-1, keepdims=True) + ref.L2_EPS),
                                       atol=1e-14)
            np.testing.assert_allclose(vo[b, h], v[b, :, :, h] / (1 + np.exp(-v[b, :, :, h])), atol=1e-14)


def test_grid_transpose_symmetry():
    """Transposing the latent grid (Hl <-> Wl) together with the spatial
    filters transposes the output: the filter is applied in grid coordinates."""
    rng = np.random.default_rng(503)
    T, Hl, Wl, d = 3, 4, 6, 2
    X = rng.standard_normal((T, Hl, Wl, d))
    ws = rng.standard_normal((d, 5, 5))
    wt = rng.standard_normal((d, 5))
    a = ref.short_conv(X.reshape(T, Hl * Wl, d), ws, wt, Hl, Wl).reshape(T, Hl, Wl, d)
    Xt = X.transpose(0, 2, 1, 3).copy()
    b = ref.short_conv(Xt.reshape(T, Wl * Hl, d), ws.transpose(0, 2, 1), wt, Wl, Hl).reshape(T, Wl, Hl, d)
    np.testing.assert_allclose(b.transpose(0, 2, 1, 3), a, atol=1e-12)


def test_scaled_centre_taps_apply_silu_after_the_filter():
    """Centre taps a (spatial) and b (temporal) scale the input by a*b, so the
    features are L2(SiLU(a b k)) and SiLU(a b v): the nonlinearity follows the
    convolution (SiLU(3x) differs from 3 SiLU(x))."""
    pw = gen.PrepWorkload("scaled", 1, 2, 3, 2, 3, 4, 8)
    x = gen.make_prep_inputs(pw)
    s = np.zeros((pw.H, pw.d, 5, 5))
    s[:, :, 2, 2] = 1.5
    t = np.zeros((pw.H, pw.d, 5))
    t[:, :, 2] = 2.0
    q, k, v = (gen.as_f64(x[n]) for n in ("q", "k", "v"))
    _, ko, vo = ref.prep(q, k, v, s, t, s, t, pw.Hl, pw.Wl)
    for h in range(pw.H):
        k3 = 3.0 * k[0, :, :, h]
        sk = k3 / (1 + np.exp(-k3))
        np.testing.assert_allclose(ko[0, h], sk / np.sqrt((sk ** 2).sum(-1, keepdims=True) + ref.L2_EPS), atol=1e-13)
        v3 = 3.0 * v[0, :, :, h]
        np.testing.assert_allclose(vo[0, h], v3 / (1 + np.exp(-v3)), atol=1e-13)
