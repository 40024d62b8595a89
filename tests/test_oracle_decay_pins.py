"""Pins of the oracle's decay path: the channel-wise decay gate of Eq. 2 in
both scans and the decay bridge of Eq. A.4 (Video DeltaNet, Section 3.1 and
Appendix A.3).  Each test checks the oracle against something other than its
own formula: the no-decay path, a closed form, a second route that applies the
bridge frame by frame, a symmetry, or Proposition 1."""

import numpy as np
import pytest

import oracle as ref


def _case(rng, T, U=5, d_k=4, d_v=3, s0=True, a_lo=0.3):
    q = rng.standard_normal((T, U, d_k))
    k = rng.standard_normal((T, U, d_k))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, U, d_v))
    beta = 1 / (1 + np.exp(-rng.standard_normal((T, U))))
    g = rng.standard_normal((T, U, d_v))
    w = 1 + 0.1 * rng.standard_normal(d_v)
    S0f = rng.standard_normal((d_v, d_k)) if s0 else None
    S0r = rng.standard_normal((d_v, d_k)) if s0 else None
    alpha = rng.uniform(a_lo, 1.0, size=(T, d_k))
    return q, k, v, beta, g, w, S0f, S0r, alpha


def test_decay_of_one_is_the_plain_path():
    rng = np.random.default_rng(200)
    T, C, w = 12, 3, 1
    q, k, v, beta, g, wt, S0f, S0r, _ = _case(rng, T)
    y0 = ref.vda_forward_head(q, k, v, beta, g, wt, S0f, S0r, C, w)
    y1 = ref.vda_forward_head(q, k, v, beta, g, wt, S0f, S0r, C, w, alpha=np.ones((T, 4)))
    np.testing.assert_array_equal(y1, y0)


def test_decay_of_zero_reads_nothing():
    """alpha = 0 empties every bridged state (the bridge includes the query
    frame's own gate), so the output is exactly zero."""
    rng = np.random.default_rng(201)
    T, C, w = 10, 5, 0
    q, k, v, beta, g, wt, S0f, S0r, _ = _case(rng, T)
    y = ref.vda_forward_head(q, k, v, beta, g, wt, S0f, S0r, C, w, alpha=np.zeros((T, 4)))
    assert np.all(y == 0.0)


@pytest.mark.parametrize("T,C,w", [(10, 5, 1), (12, 5, 1), (7, 3, 0), (9, 2, 2),
                                   (6, 1, 1), (5, 5, 1), (11, 4, 3), (13, 3, 1), (1, 5, 0)])
def test_decay_naive_bridge_equals_chunked(T, C, w):
    """Second route: every query frame reruns both scans from the initial
    states and applies the bridge frame by frame (decay without writes), as
    Appendix A.3 describes it; the oracle uses products of gates instead."""
    rng = np.random.default_rng(300 + 7 * T + C + w)
    q, k, v, beta, g, wt, S0f, S0r, alpha = _case(rng, T)
    y = ref.vda_forward_head(q, k, v, beta, g, wt, S0f, S0r, C, w, alpha=alpha)
    y_naive = ref.vda_forward_head_naive(q, k, v, beta, g, wt, S0f, S0r, C, w, alpha=alpha)
    np.testing.assert_allclose(y, y_naive, rtol=0, atol=1e-12)


def test_decay_without_writes_is_a_product_of_gates():
    """With beta = 0 there are no writes: A = B = 0, every state only decays,
    and the state read at frame t is
      S0_fwd Diag(prod_{r<=t} alpha_r) + S0_rev Diag(prod_{r>=t} alpha_r)
    whatever the window (closed form of Eq. 2 + Eq. A.4)."""
    rng = np.random.default_rng(202)
    T = 9
    q, k, v, beta, g, wt, S0f, S0r, alpha = _case(rng, T)
    for C, w in [(3, 0), (3, 1), (2, 1), (9, 0)]:
        y = ref.vda_forward_head(q, k, v, np.zeros_like(beta), g, wt, S0f, S0r, C, w, alpha=alpha)
        for t in range(T):
            S = S0f * np.prod(alpha[:t + 1], axis=0) + S0r * np.prod(alpha[t:], axis=0)
            o = q[t] @ S.T
            ms = (o ** 2).mean(axis=-1, keepdims=True)
            want = wt * o / np.sqrt(ms + ref.RMS_EPS) / (1 + np.exp(-g[t]))
            np.testing.assert_allclose(y[t], want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("seed", range(5))
def test_decayed_transition_non_expansive(seed):
    """Proposition 1 (Appendix A.1): ||Diag(alpha)(I + A)^{-1}||_2 <= 1 for
    alpha in [0, 1] and beta >= 0."""
    rng = np.random.default_rng(400 + seed)
    d, U = 6, 20
    K = rng.standard_normal((U, d))
    beta = rng.uniform(0, 3, size=U)
    A, _ = ref.frame_stats(K, rng.standard_normal((U, d)), beta)
    alpha = rng.uniform(0, 1, size=d)
    M = np.diag(alpha) @ np.linalg.inv(np.eye(d) + A)
    assert np.linalg.norm(M, 2) <= 1 + 1e-12
    # the scan's decayed update applies exactly this map to the entering state
    S = rng.standard_normal((4, d))
    np.testing.assert_allclose(ref.frame_update(ref.decayed(S, alpha), A, np.zeros((4, d))),
                               S @ M, atol=1e-12)


def test_decay_time_reversal_symmetry():
    rng = np.random.default_rng(203)
    T, C, w = 12, 3, 1
    q, k, v, beta, g, wt, S0f, S0r, alpha = _case(rng, T)
    y = ref.vda_forward_head(q, k, v, beta, g, wt, S0f, S0r, C, w, alpha=alpha)
    flip = lambda a: a[::-1].copy()
    y_rev = ref.vda_forward_head(flip(q), flip(k), flip(v), flip(beta), flip(g), wt, S0r, S0f, C, w,
                                 alpha=flip(alpha))
    np.testing.assert_allclose(y_rev[::-1], y, atol=1e-12)


def test_decay_acts_on_key_channels():
    """Permuting the key channels of q, k, the initial states' columns and the
    gates together leaves the output unchanged: the decay scales the state's
    key columns (S Diag(alpha)), not its value rows."""
    rng = np.random.default_rng(204)
    T, C, w = 10, 2, 1
    d = 4
    q, k, v, beta, g, wt, S0f, S0r, alpha = _case(rng, T, d_k=d, d_v=d)
    perm = rng.permutation(d)
    y = ref.vda_forward_head(q, k, v, beta, g, wt, S0f, S0r, C, w, alpha=alpha)
    y_p = ref.vda_forward_head(q[..., perm], k[..., perm], v, beta, g, wt, S0f[:, perm], S0r[:, perm], C, w,
                               alpha=alpha[:, perm])
    np.testing.assert_allclose(y_p, y, atol=1e-12)


def test_scalar_decay_keeps_rotation_invariance():
    """A gate equal on every channel commutes with rotations of the key space,
    so rotating keys, queries and initial states leaves the output unchanged."""
    rng = np.random.default_rng(205)
    T, C, w = 9, 3, 1
    q, k, v, beta, g, wt, S0f, S0r, _ = _case(rng, T)
    alpha = np.repeat(rng.uniform(0.3, 1.0, size=(T, 1)), 4, axis=1)
    Rm, _ = np.linalg.qr(rng.standard_normal((4, 4)))
    y = ref.vda_forward_head(q, k, v, beta, g, wt, S0f, S0r, C, w, alpha=alpha)
    y_rot = ref.vda_forward_head(q @ Rm.T, k @ Rm.T, v, beta, g, wt, S0f @ Rm.T, S0r @ Rm.T, C, w,
                                 alpha=alpha)
    np.testing.assert_allclose(y_rot, y, atol=1e-12)


@pytest.mark.parametrize("T,C,decay", [(10, 5, False), (11, 4, True), (7, 3, True), (6, 1, False), (5, 5, True)])
def test_chunk_composed_maps_give_the_boundary_states(T, C, decay):
    """Eq. A.1's affine form composed chunk by chunk (the chunk-wise scan of
    Section 5) reaches the same boundary states as the frame-by-frame scans,
    in both directions, with and without decay."""
    rng = np.random.default_rng(600 + 10 * T + C)
    q, k, v, beta, g, wt, S0f, S0r, alpha = _case(rng, T)
    a = alpha if decay else None
    _, inter = ref.vda_forward_head(q, k, v, beta, g, wt, S0f, S0r, C, 1, keep=True, alpha=a)
    want = ref.boundary_states(inter["P"], inter["R"], S0f, S0r, T, C)
    got = ref.boundary_states_by_chunk_maps(inter["A"], inter["B"], S0f, S0r, T, C, alpha=a)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-11)
