"""Plain float64 CPU oracle for the linear branch's feature preparation (VDA-Prep).

TEST INFRASTRUCTURE ONLY: used by the test-suite and the benchmark's CPU
baseline, never by the product path.

Source: "Video DeltaNet: A Video-Native Hybrid Attention for Livestream Video
Generation", Section 2.3 (the linear branch's feature map) and Section 5
(the fused VDA-Prep step).  The linear branch applies a separable short
convolution to K and V, a depthwise 5 x 5 spatial filter and a five-tap
temporal filter, then SiLU; Q and K are L2-normalised; the result is laid
out frame-major per head.

Readings of what the pages leave open:
  * inputs are the projections of the interior video tokens, [B, T, U, H, d]
    (frame-major tokens, heads inner), token u = y * Wl + x on the Hl x Wl
    latent grid; outputs are [B, H, T, U, d];
  * the filters are per head and channel (depthwise over the H * d channels),
    cross-correlations as in common deep-learning convolution layers, with
    zero padding of 2 on every side (same-size outputs, spatially within the
    frame and temporally over the interior frames), no bias;
  * order: spatial filter, temporal filter, SiLU; K is then L2-normalised;
    Q is only L2-normalised; V gets no normalisation;
  * L2 normalisation x / sqrt(sum(x^2) + 1e-6) over the head dimension.
"""

from __future__ import annotations

import numpy as np

L2_EPS = 1e-6


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def silu(x):
    """SiLU(x) = x * sigmoid(x)."""
    x = _f64(x)
    return x / (1.0 + np.exp(-x))


def l2_normalize(x, eps=L2_EPS):
    """x / sqrt(sum(x^2) + eps) over the last axis."""
    x = _f64(x)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def conv_spatial(X, w):
    """Depthwise 5 x 5 cross-correlation over the latent grid, zero padding 2.
    X: [T, Hl, Wl, d]; w: [d, 5, 5].  out[t, y, x, c] =
    sum_{i, j} w[c, i, j] * X[t, y + i - 2, x + j - 2, c]."""
    X = _f64(X)
    w = _f64(w)
    T, Hl, Wl, d = X.shape
    P = np.zeros((T, Hl + 4, Wl + 4, d))
    P[:, 2:Hl + 2, 2:Wl + 2, :] = X
    out = np.zeros_like(X)
    for i in range(5):
        for j in range(5):
            out += w[:, i, j] * P[:, i:i + Hl, j:j + Wl, :]
    return out


def conv_temporal(X, w):
    """Depthwise five-tap cross-correlation over frames, zero padding 2.
    X: [T, Hl, Wl, d]; w: [d, 5].  out[t, ..., c] = sum_s w[c, s] * X[t + s - 2, ..., c]."""
    X = _f64(X)
    w = _f64(w)
    T = X.shape[0]
    P = np.zeros((T + 4,) + X.shape[1:])
    P[2:T + 2] = X
    out = np.zeros_like(X)
    for s in range(5):
        out += w[:, s] * P[s:s + T]
    return out


def short_conv(X, w_spatial, w_temporal, Hl, Wl):
    """The separable short convolution of one head: X [T, U, d] -> [T, U, d]."""
    T, U, d = X.shape
    G = _f64(X).reshape(T, Hl, Wl, d)
    return conv_temporal(conv_spatial(G, w_spatial), w_temporal).reshape(T, U, d)


def prep_head(q, k, v, wk_s, wk_t, wv_s, wv_t, Hl, Wl, eps=L2_EPS):
    """Prepared features of one (batch, head): q, k, v [T, U, d] (U = Hl * Wl)
    -> (q', k', v') with q' = L2(q), k' = L2(SiLU(conv(k))), v' = SiLU(conv(v))."""
    qn = l2_normalize(q, eps)
    kn = l2_normalize(silu(short_conv(k, wk_s, wk_t, Hl, Wl)), eps)
    vn = silu(short_conv(v, wv_s, wv_t, Hl, Wl))
    return qn, kn, vn


def prep(q, k, v, wk_s, wk_t, wv_s, wv_t, Hl, Wl, eps=L2_EPS, heads=None):
    """Whole-tensor form: q, k, v [B, T, U, H, d]; wk_s, wv_s [H, d, 5, 5];
    wk_t, wv_t [H, d, 5].  Returns q', k', v' [B, H, T, U, d] (or, with
    `heads` = list of (b, h), stacked [len(heads), T, U, d])."""
    Bn, T, U, Hn, d = q.shape
    pairs = heads if heads is not None else [(b, h) for b in range(Bn) for h in range(Hn)]
    outs = ([], [], [])
    for (b, h) in pairs:
        r = prep_head(q[b, :, :, h], k[b, :, :, h], v[b, :, :, h], wk_s[h], wk_t[h], wv_s[h], wv_t[h],
                      Hl, Wl, eps)
        for o, x in zip(outs, r):
            o.append(x)
    res = tuple(np.stack(o) for o in outs)
    if heads is None:
        res = tuple(x.reshape((Bn, Hn) + x.shape[1:]) for x in res)
    return res
