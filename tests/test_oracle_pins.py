"""Pins for the float64 oracle: closed forms, invariants and brute force that
fix what the paper's equations compute, so that a plausible slip in the oracle
(a transposed operand, a dropped beta, a left- instead of right-multiply, an
off-by-one gather index, a wrong RMSNorm) fails at least one test here.

Paper: "Video DeltaNet: A Video-Native Hybrid Attention for Livestream Video
Generation" (arXiv 2609.20744).
"""

import json
import os

import numpy as np
import pytest

import oracle as ref
from frame_wise_delta_vda_b200 import inputs as gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_frame(rng, U, d_k, d_v, unit_keys=True, beta_scale=1.0):
    K = rng.standard_normal((U, d_k))
    if unit_keys:
        K /= np.linalg.norm(K, axis=1, keepdims=True)
    V = rng.standard_normal((U, d_v))
    beta = beta_scale / (1.0 + np.exp(-rng.standard_normal(U)))
    return K, V, beta


# --- Eq. (3b): matrix form == per-token summation form ----------------------
def test_stats_equal_token_sums():
    rng = np.random.default_rng(10)
    K, V, beta = _rand_frame(rng, U=7, d_k=5, d_v=3)
    A, B = ref.frame_stats(K, V, beta)
    A_sum = sum(beta[u] * np.outer(K[u], K[u]) for u in range(7))
    B_sum = sum(beta[u] * np.outer(V[u], K[u]) for u in range(7))
    assert A.shape == (5, 5) and B.shape == (3, 5)
    np.testing.assert_allclose(A, A_sum, rtol=0, atol=1e-13)
    np.testing.assert_allclose(B, B_sum, rtol=0, atol=1e-13)


# --- Eq. (5): the normal equation S (I + A) = S_bar + B ---------------------
@pytest.mark.parametrize("wl_name", ["tiny", "small"])
def test_normal_equation_residual(wl_name):
    wl = gen.WORKLOADS[wl_name]
    x = gen.head_inputs(wl, 0, 0)
    k, v, beta = gen.as_f64(x["k"]), gen.as_f64(x["v"]), x["beta"]
    rng = np.random.default_rng(11)
    S = rng.standard_normal((wl.d, wl.d))
    for t in range(wl.T):
        A, B = ref.frame_stats(k[t], v[t], beta[t])
        S_new = ref.frame_update(S, A, B)
        rhs = S + B
        res = np.linalg.norm(S_new @ (np.eye(wl.d) + A) - rhs) / np.linalg.norm(rhs)
        assert res <= 1e-10
        S = S_new


def test_normal_equation_rectangular_state():
    """d_v != d_k: the update right-multiplies by the d_k x d_k inverse."""
    rng = np.random.default_rng(12)
    K, V, beta = _rand_frame(rng, U=9, d_k=6, d_v=4)
    S_bar = rng.standard_normal((4, 6))
    A, B = ref.frame_stats(K, V, beta)
    S = ref.frame_update(S_bar, A, B)
    assert S.shape == (4, 6)
    np.testing.assert_allclose(S @ (np.eye(6) + A), S_bar + B, atol=1e-12)


# --- U = 1: Sherman-Morrison -------------------------------------------------
@pytest.mark.parametrize("unit", [True, False])
def test_single_token_sherman_morrison(unit):
    rng = np.random.default_rng(13)
    d_k, d_v = 6, 5
    k = rng.standard_normal(d_k)
    if unit:
        k /= np.linalg.norm(k)
    v = rng.standard_normal(d_v)
    b = 0.7
    S_bar = rng.standard_normal((d_v, d_k))
    A, B = ref.frame_stats(k[None], v[None], np.array([b]))
    S = ref.frame_update(S_bar, A, B)
    inv = np.eye(d_k) - (b / (1.0 + b * (k @ k))) * np.outer(k, k)
    expected = (S_bar + b * np.outer(v, k)) @ inv
    np.testing.assert_allclose(S, expected, rtol=0, atol=1e-14)
    # read-back along the written key: (S_bar k + b |k|^2 v) / (1 + b |k|^2)
    kk = k @ k
    np.testing.assert_allclose(S @ k, (S_bar @ k + b * kk * v) / (1 + b * kk), atol=1e-13)


# --- Eq. (4): the update minimises the joint frame objective ----------------
@pytest.mark.parametrize("U", [3, 9])
def test_update_minimises_objective_by_gradient_descent(U):
    rng = np.random.default_rng(14 + U)
    d_k, d_v = 6, 4
    K, V, beta = _rand_frame(rng, U=U, d_k=d_k, d_v=d_v)
    S_bar = rng.standard_normal((d_v, d_k))

    def objective(S):
        fit = sum(beta[u] * np.sum((S @ K[u] - V[u]) ** 2) for u in range(U))
        return 0.5 * np.sum((S - S_bar) ** 2) + 0.5 * fit

    def gradient(S):
        g = S - S_bar
        for u in range(U):
            g = g + beta[u] * np.outer(S @ K[u] - V[u], K[u])
        return g

    # Lipschitz constant of the gradient <= 1 + sum_u beta_u |k_u|^2
    L = 1.0 + sum(beta[u] * (K[u] @ K[u]) for u in range(U))
    S = S_bar.copy()
    for _ in range(4000):
        S = S - gradient(S) / L
    S_closed = ref.frame_update(S_bar, *ref.frame_stats(K, V, beta))
    np.testing.assert_allclose(S_closed, S, rtol=0, atol=1e-10)
    assert np.linalg.norm(gradient(S_closed)) < 1e-12
    for _ in range(5):
        P = 1e-3 * rng.standard_normal(S.shape)
        assert objective(S_closed + P) > objective(S_closed)


# --- Proposition 1: non-expansive inherited-state transition ----------------
@pytest.mark.parametrize("wl_name", ["tiny", "small", "corr"])
def test_transition_non_expansive(wl_name):
    wl = gen.WORKLOADS[wl_name]
    x = gen.head_inputs(wl, 0, wl.H - 1)
    k, v, beta = gen.as_f64(x["k"]), gen.as_f64(x["v"]), x["beta"]
    rng = np.random.default_rng(15)
    zero = np.zeros((wl.d, wl.d))
    for t in range(0, wl.T, max(1, wl.T // 6)):
        A, B = ref.frame_stats(k[t], v[t], beta[t])
        M = ref.frame_update(np.eye(wl.d), A, zero)      # = (I + A)^{-1}
        sv = np.linalg.svd(M, compute_uv=False)
        assert sv.max() <= 1.0 + 1e-12
        assert sv.min() > 0.0
        S1 = rng.standard_normal((wl.d, wl.d))
        S2 = rng.standard_normal((wl.d, wl.d))
        d_out = np.linalg.norm(ref.frame_update(S1, A, B) - ref.frame_update(S2, A, B))
        assert d_out <= np.linalg.norm(S1 - S2) * (1 + 1e-12)


# --- Eq. (A.3): repeated-key saturation --------------------------------------
@pytest.mark.parametrize("U,b", [(9, 0.3), (1008, 0.5), (4, 2.0)])
def test_repeated_key_saturation(U, b):
    rng = np.random.default_rng(16)
    d_k, d_v = 6, 5
    k = rng.standard_normal(d_k)
    k /= np.linalg.norm(k)
    K = np.tile(k, (U, 1))
    V = rng.standard_normal((U, d_v))
    S_bar = rng.standard_normal((d_v, d_k))
    A, B = ref.frame_stats(K, V, np.full(U, b))
    S = ref.frame_update(S_bar, A, B)
    s = S_bar @ k
    v_bar = V.mean(axis=0)
    expected = s / (1 + U * b) + (U * b / (1 + U * b)) * v_bar
    np.testing.assert_allclose(S @ k, expected, rtol=0, atol=1e-12)
    # the transition's eigenvalue along k is 1 / (1 + U b): evidence weight
    # 1 - 1/(1 + U b) = U b / (1 + U b) < 1
    M = ref.frame_update(np.eye(d_k), A, np.zeros((d_k, d_k)))
    np.testing.assert_allclose(M @ k, k / (1 + U * b), atol=1e-13)
    assert 1 - 1 / (1 + U * b) < 1
    # directions orthogonal to k are untouched
    w = rng.standard_normal(d_k)
    w -= (w @ k) * k
    np.testing.assert_allclose(S @ w, S_bar @ w, atol=1e-12)


# --- Appendix A.2: orthonormal keys each get beta / (1 + beta) --------------
def test_orthonormal_keys_write_weight():
    rng = np.random.default_rng(17)
    d_k, d_v, b = 7, 4, 0.8
    Qm, _ = np.linalg.qr(rng.standard_normal((d_k, d_k)))
    K = Qm.T                                    # rows are orthonormal keys
    V = rng.standard_normal((d_k, d_v))
    S_bar = rng.standard_normal((d_v, d_k))
    S = ref.frame_update(S_bar, *ref.frame_stats(K, V, np.full(d_k, b)))
    for u in range(d_k):
        np.testing.assert_allclose(S @ K[u], (S_bar @ K[u] + b * V[u]) / (1 + b), atol=1e-13)


# --- Eq. (3c) vs Eq. (5): agree to first order in beta ----------------------
def test_batch_rule_is_first_order_limit():
    rng = np.random.default_rng(18)
    K, V, beta = _rand_frame(rng, U=12, d_k=6, d_v=5)
    S_bar = rng.standard_normal((5, 6))
    ratios = []
    for eps in (1e-2, 1e-3, 1e-4):
        A, B = ref.frame_stats(K, V, eps * beta)
        diff = np.linalg.norm(ref.frame_update(S_bar, A, B) - ref.batch_rule_update(S_bar, A, B))
        ratios.append(diff / eps ** 2)
    assert ratios[0] > 0
    # O(beta^2): diff / eps^2 converges to a nonzero constant
    assert abs(ratios[1] - ratios[2]) / ratios[2] < 2e-3
    assert abs(ratios[0] - ratios[2]) / ratios[2] < 5e-2


# --- Appendix A.3 gather: windows and boundary states ------------------------
def test_window_bounds_hand_table():
    # T = 12 interior frames, C = 5 (ragged last chunk of 2), w = 1
    assert [ref.window_bounds(c, 12, 5, 1) for c in range(3)] == [(0, 9), (0, 11), (5, 11)]
    # T = 30, C = 5, w = 1: interior chunks see frames [5(c-1), 5(c+2) - 1]
    assert ref.window_bounds(0, 30, 5, 1) == (0, 9)
    assert ref.window_bounds(2, 30, 5, 1) == (5, 19)
    assert ref.window_bounds(5, 30, 5, 1) == (20, 29)
    # w = 0: the window is the chunk itself
    assert ref.window_bounds(3, 30, 5, 0) == (15, 19)


def _small_case(rng, T, U=3, d_k=4, d_v=3, s0=True):
    q = rng.standard_normal((T, U, d_k))
    k = rng.standard_normal((T, U, d_k))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, U, d_v))
    beta = 1 / (1 + np.exp(-rng.standard_normal((T, U))))
    g = rng.standard_normal((T, U, d_v))
    w = 1 + 0.1 * rng.standard_normal(d_v)
    S0f = rng.standard_normal((d_v, d_k)) if s0 else None
    S0r = rng.standard_normal((d_v, d_k)) if s0 else None
    return q, k, v, beta, g, w, S0f, S0r


@pytest.mark.parametrize("T,C,w", [(10, 5, 1), (12, 5, 1), (7, 3, 0), (9, 2, 2),
                                   (6, 1, 1), (5, 5, 1), (11, 4, 3), (13, 3, 1), (1, 5, 0)])
def test_naive_rescan_equals_chunked_oracle(T, C, w):
    rng = np.random.default_rng(100 + 7 * T + C + w)
    args = _small_case(rng, T)
    y = ref.vda_forward_head(*args, C, w)
    y_naive = ref.vda_forward_head_naive(*args, C, w)
    np.testing.assert_allclose(y, y_naive, rtol=0, atol=1e-12)


def test_time_reversal_symmetry():
    rng = np.random.default_rng(19)
    T, C, w = 12, 3, 1
    q, k, v, beta, g, wt, S0f, S0r = _small_case(rng, T)
    y = ref.vda_forward_head(q, k, v, beta, g, wt, S0f, S0r, C, w)
    flip = lambda a: a[::-1].copy()
    y_rev = ref.vda_forward_head(flip(q), flip(k), flip(v), flip(beta), flip(g), wt, S0r, S0f, C, w)
    np.testing.assert_allclose(y_rev[::-1], y, atol=1e-12)


def test_boundary_states_match_direct_scans():
    rng = np.random.default_rng(20)
    T, C = 11, 4
    q, k, v, beta, g, wt, S0f, S0r = _small_case(rng, T)
    _, inter = ref.vda_forward_head(q, k, v, beta, g, wt, S0f, S0r, C, 1, keep=True)
    st = ref.boundary_states(inter["P"], inter["R"], S0f, S0r, T, C)
    nc = ref.num_chunks(T, C)
    assert st.shape == (2, nc + 1, 3, 4)
    for j in range(nc + 1):
        P = S0f.copy()
        for r in range(0, min(j * C, T)):
            P = ref.frame_update(P, *ref.frame_stats(k[r], v[r], beta[r]))
        np.testing.assert_allclose(st[0, j], P, atol=1e-12)
        R = S0r.copy()
        for r in range(T - 1, min(j * C, T) - 1, -1):
            R = ref.frame_update(R, *ref.frame_stats(k[r], v[r], beta[r]))
        np.testing.assert_allclose(st[1, j], R, atol=1e-12)


# --- Eq. (1b): the prompt is counted once ------------------------------------
def test_text_state_counted_once():
    rng = np.random.default_rng(21)
    T, C, w = 10, 5, 0
    q, k, v, beta, g, wt, _, _ = _small_case(rng, T)
    S_text = rng.standard_normal((3, 4))
    y = ref.vda_forward_head(q, k, v, np.zeros_like(beta), g, wt, S_text / 2, S_text / 2, C, w)
    for t in range(T):
        o = q[t] @ S_text.T
        ms = (o ** 2).mean(axis=-1, keepdims=True)
        np.testing.assert_allclose(y[t], wt * o / np.sqrt(ms + ref.RMS_EPS) / (1 + np.exp(-g[t])),
                                   atol=1e-12)


def test_text_state_orthonormal_prompt():
    """A prompt of orthonormal unit keys with gate b writes b/(1+b) of each
    value into the empty state (Appendix A.2 with S_bar = 0)."""
    rng = np.random.default_rng(22)
    d, b = 5, 0.25
    Qm, _ = np.linalg.qr(rng.standard_normal((d, d)))
    V = rng.standard_normal((d, d))
    S = ref.text_state(Qm.T, V, np.full(d, b))
    for u in range(d):
        np.testing.assert_allclose(S @ Qm[:, u], b * V[u] / (1 + b), atol=1e-13)


# --- invariance under a rotation of the key/query channel space --------------
def test_key_rotation_invariance():
    rng = np.random.default_rng(23)
    T, C, w = 9, 3, 1
    q, k, v, beta, g, wt, S0f, S0r = _small_case(rng, T)
    Rm, _ = np.linalg.qr(rng.standard_normal((4, 4)))
    y = ref.vda_forward_head(q, k, v, beta, g, wt, S0f, S0r, C, w)
    y_rot = ref.vda_forward_head(q @ Rm.T, k @ Rm.T, v, beta, g, wt, S0f @ Rm.T, S0r @ Rm.T, C, w)
    np.testing.assert_allclose(y_rot, y, atol=1e-12)


# --- Eq. (1c) readout on a hand-built example --------------------------------
def test_readout_hand_example():
    with open(os.path.join(GOLDEN, "readout_hand_example.json")) as f:
        case = json.load(f)
    d = len(case["q"])
    q = np.array(case["q"], dtype=np.float64).reshape(1, 1, d)
    k = np.ones((1, 1, d)) / np.sqrt(d)
    v = np.zeros((1, 1, d))
    beta = np.zeros((1, 1))
    g = np.array(case["gate_logits"], dtype=np.float64).reshape(1, 1, d)
    w = np.array(case["rms_weight"], dtype=np.float64)
    S0 = np.array(case["S0_fwd"], dtype=np.float64)
    y = ref.vda_forward_head(q, k, v, beta, g, w, S0, S0, 1, 0)
    expected = np.array([eval(s, {}) for s in case["expected_y"]], dtype=np.float64)
    np.testing.assert_allclose(y[0, 0], expected, rtol=case["rtol"], atol=0)


# --- reading 5: a window covering the clip returns the S0 readout (0 here) ---
def test_tiny_workload_output_is_exactly_zero():
    wl = gen.WORKLOADS["tiny"]
    x = gen.make_inputs(wl)
    y = ref.vda_forward(gen.as_f64(x["q"]), gen.as_f64(x["k"]), gen.as_f64(x["v"]), x["beta"],
                        gen.as_f64(x["gate"]), x["rms_weight"], None, None, wl.chunk, wl.window_chunks)
    assert y.shape == (1, 2, 10, 16, 16)
    assert np.all(y == 0.0)


def test_generator_is_deterministic_and_head_local():
    wl = gen.WORKLOADS["small"]
    a = gen.make_inputs(wl)
    b = gen.head_inputs(wl, 0, 5)
    for key in ("q", "k", "v", "gate", "beta"):
        np.testing.assert_array_equal(a[key][0, 5], b[key])
    kf = gen.as_f64(a["k"])
    np.testing.assert_allclose(np.linalg.norm(kf, axis=-1), 1.0, atol=1e-2)
    assert a["q"].dtype == np.uint16 and a["beta"].dtype == np.float32


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.00390625, 1.01171875, -2.5, 3.0e-3, 65504.0], dtype=np.float32)
    bits = gen.f32_to_bf16_bits(x)
    back = gen.bf16_bits_to_f32(bits)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: rounds to the even one (1.0)
    assert back[1] == 1.0
    # 1 + 3 * 2^-8 is a tie between 1 + 2^-7 and 1 + 2^-6: rounds to even (1 + 2^-6)
    assert back[2] == np.float32(1.015625)
    assert back[0] == 1.0 and back[3] == -2.5
    assert np.all(np.abs(back - x) <= np.abs(x) * 2.0 ** -8)
