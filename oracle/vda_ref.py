"""Plain float64 CPU oracle for the bidirectional Video Delta Attention (VDA) branch.

TEST INFRASTRUCTURE ONLY.  This module exists to check the CUDA library against
the paper's definitions.  Only the test-suite, the smoke check and the CPU
baseline leg of the benchmark may import it; the product path never does.

Source: "Video DeltaNet: A Video-Native Hybrid Attention for Livestream Video
Generation" (arXiv 2609.20744, HTML version).  Every function names the
section / equation it writes out.  Nothing here is blocked, fused or reordered
beyond what those equations state; the only library primitives used are a
matrix product and a dense linear solve (LAPACK, via numpy).

Notation (per batch b, head h, interior latent frame t):
  K_t in R^{U x d_k}, V_t in R^{U x d_v}, beta_t in R^U, Q_t in R^{U x d_k},
  G_t in R^{U x d_v} (gate logits), state S in R^{d_v x d_k}, read as o = S q.

Readings of points the paper leaves open:
  * decay: without `alpha` the gate is 1, so S_bar_t = S_{t-1} and there is no
    decay bridge; with `alpha` [T, d_k] in [0, 1] (Eq. 2) both scans use
    S_bar_t = S_{t+-1} Diag(alpha_t) with the frame's own alpha_t, and query
    frame t reads the bridged states of Eq. A.4; a side without distant frames
    bridges its initial state over the same frames;
  * chunks tile the interior frame index from 0: chunk c = [cC, cC + C);
    a ragged last chunk is allowed;
  * the window of chunk c is chunks [c - w, c + w], clipped to interior
    frames; a side with no distant frames reads its initial state;
  * a window that covers the whole clip still returns the formula's value
    RMSNorm((S0_fwd + S0_rev) q) * sigmoid(g) (zero when both S0 are zero);
  * RMSNorm(o) = w * o / sqrt(mean(o^2) + eps) over d_v, eps = 1e-6, with one
    weight vector w in R^{d_v} shared by all heads; gate = sigmoid(logit),
    applied after the weight.

Parity pins: every function here is pinned by tests in
tests/test_oracle_pins.py against closed forms, invariants and brute force.
"""

from __future__ import annotations

import numpy as np

RMS_EPS = 1e-6


def _f64(x):
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# Section 3.1, Eq. (3b): frame statistics.
# ---------------------------------------------------------------------------
def frame_stats(K, V, beta):
    """A_t = K_t^T Diag(beta_t) K_t  and  B_t = V_t^T Diag(beta_t) K_t  (Eq. 3b).

    K: [U, d_k], V: [U, d_v], beta: [U].  Returns (A [d_k, d_k], B [d_v, d_k]).
    """
    K = _f64(K)
    V = _f64(V)
    beta = _f64(beta)
    beta_K = K * beta[:, None]          # Diag(beta) K
    A = K.T @ beta_K
    B = V.T @ beta_K
    return A, B


# ---------------------------------------------------------------------------
# Section 3.2, Eq. (5): the joint frame-wise update.
# ---------------------------------------------------------------------------
def frame_update(S_bar, A, B):
    """S_t = (S_bar_t + B_t)(I + A_t)^{-1}  (Eq. 5), solved from the normal
    equation S_t (I + A_t) = S_bar_t + B_t rather than by forming the inverse.

    S_bar: [d_v, d_k]; A: [d_k, d_k]; B: [d_v, d_k].
    """
    S_bar = _f64(S_bar)
    A = _f64(A)
    B = _f64(B)
    d_k = A.shape[0]
    rhs = S_bar + B
    # S (I + A) = rhs   <=>   (I + A)^T S^T = rhs^T
    return np.linalg.solve((np.eye(d_k) + A).T, rhs.T).T


def batch_rule_update(S_bar, A, B):
    """The frozen-state batched rule S^batch = S_bar (I - A) + B  (Eq. 3c).

    Not part of the VDA path: used only as the first-order-in-beta contrast.
    """
    S_bar = _f64(S_bar)
    d_k = A.shape[0]
    return S_bar @ (np.eye(d_k) - _f64(A)) + _f64(B)


def text_state(K_text, V_text, beta_text):
    """One frame-wise update of the zero state from L prompt tokens treated as a
    single frame: S = B'(I + A')^{-1} with (A', B') from Eq. (3b) over the text
    tokens (Eq. 5 with S_bar = 0).  The paper starts both scans from a text
    state (Eq. 1b); the benchmark workloads draw the text gates already halved.
    """
    A, B = frame_stats(K_text, V_text, beta_text)
    d_v, d_k = B.shape
    return frame_update(np.zeros((d_v, d_k)), A, B)


# ---------------------------------------------------------------------------
# Section 2.2 / Appendix A.3: bidirectional scans, boundary gather, readout.
# ---------------------------------------------------------------------------
def num_chunks(T, chunk):
    return (T + chunk - 1) // chunk


def window_bounds(c, T, chunk, window_chunks):
    """Local window [l, h] of query chunk c clipped to interior frames 0..T-1
    (Appendix A.3): chunks c - w .. c + w, i.e. frames (c-w)C .. (c+w+1)C - 1."""
    lo = max(0, (c - window_chunks) * chunk)
    hi = min(T - 1, (c + window_chunks + 1) * chunk - 1)
    return lo, hi


def decayed(S, alpha_t):
    """S_bar = S Diag(alpha_t)  (Eq. 2): channel-wise decay of the key columns."""
    return _f64(S) * _f64(alpha_t)[None, :]


def forward_scan(S0, A_all, B_all, alpha=None):
    """Forward states P_t = (P_{t-1} Diag(alpha_t) + B_t)(I + A_t)^{-1},
    P_{-1} = S0 (Section 2.2; Eq. 2 and Eq. 5; alpha None means 1).
    Returns the list [P_0, ..., P_{T-1}]."""
    P = _f64(S0)
    out = []
    for t in range(len(A_all)):
        S_bar = P if alpha is None else decayed(P, alpha[t])
        P = frame_update(S_bar, A_all[t], B_all[t])
        out.append(P)
    return out


def reverse_scan(S0, A_all, B_all, alpha=None):
    """Reverse states R_t = (R_{t+1} Diag(alpha_t) + B_t)(I + A_t)^{-1},
    R_T = S0: the same frame update, run backwards from frame T-1 to frame 0.
    Returns the list [R_0, ..., R_{T-1}] indexed by frame."""
    T = len(A_all)
    R = _f64(S0)
    out = [None] * T
    for t in range(T - 1, -1, -1):
        S_bar = R if alpha is None else decayed(R, alpha[t])
        R = frame_update(S_bar, A_all[t], B_all[t])
        out[t] = R
    return out


def gathered_state(c, T, chunk, window_chunks, P, R, S0_fwd, S0_rev):
    """S~ for query chunk c (Eq. A.4 with alpha = 1): the forward state just
    before the window plus the reverse state just after it; a side without
    distant frames contributes its initial state."""
    lo, hi = window_bounds(c, T, chunk, window_chunks)
    left = P[lo - 1] if lo > 0 else _f64(S0_fwd)
    right = R[hi + 1] if hi < T - 1 else _f64(S0_rev)
    return left + right


def gathered_state_frame(t, T, chunk, window_chunks, P, R, S0_fwd, S0_rev, alpha):
    """S~_t for query frame t with the decay bridge (Eq. A.4):
      S~_t = P_{l-1} Diag(prod_{r=l}^{t} alpha_r) + R_{h+1} Diag(prod_{r=t}^{h} alpha_r)
    with [l, h] the window of t's chunk; a side without distant frames starts
    from its initial state.  The products are channel-wise."""
    c = t // chunk
    lo, hi = window_bounds(c, T, chunk, window_chunks)
    alpha = _f64(alpha)
    left = P[lo - 1] if lo > 0 else _f64(S0_fwd)
    right = R[hi + 1] if hi < T - 1 else _f64(S0_rev)
    a_left = np.prod(alpha[lo:t + 1], axis=0)
    a_right = np.prod(alpha[t:hi + 1], axis=0)
    return left * a_left[None, :] + right * a_right[None, :]


def rms_gate(o, g, w, eps=RMS_EPS):
    """Linear-branch epilogue of Eq. (1c): sigmoid(g) * RMSNorm(o), where
    RMSNorm(o) = w * o / sqrt(mean(o^2) + eps) over the last axis (d_v)."""
    o = _f64(o)
    g = _f64(g)
    w = _f64(w)
    ms = np.mean(o * o, axis=-1, keepdims=True)
    return (w * o / np.sqrt(ms + eps)) * (1.0 / (1.0 + np.exp(-g)))


def vda_forward_head(q, k, v, beta, gate, rms_weight, S0_fwd, S0_rev,
                     chunk, window_chunks, eps=RMS_EPS, keep=False, alpha=None):
    """Bidirectional VDA for one (batch, head).

    q, k: [T, U, d_k]; v, gate: [T, U, d_v]; beta: [T, U]; rms_weight: [d_v];
    S0_fwd, S0_rev: [d_v, d_k] or None (zero state); alpha: [T, d_k] decay
    gates in [0, 1] or None (no decay).
    Returns y [T, U, d_v] (float64) and, if keep, a dict with A, B, M and the
    per-frame states P, R.

    Steps (Algorithm 1 of the paper, steps 3-7):
      stats (Eq. 3b) -> forward and reverse scans of Eq. 5 (with the decay of
      Eq. 2 when alpha is given) -> gather of the out-of-window states (Eq. A.4,
      with its decay bridge when alpha is given) -> o = S~ q (Eq. 1a) ->
      RMSNorm and gate (Eq. 1c).
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    beta = _f64(beta)
    gate = _f64(gate)
    T, U, d_k = k.shape
    d_v = v.shape[2]
    S0_fwd = np.zeros((d_v, d_k)) if S0_fwd is None else _f64(S0_fwd)
    S0_rev = np.zeros((d_v, d_k)) if S0_rev is None else _f64(S0_rev)

    A_all, B_all = [], []
    for t in range(T):
        A_t, B_t = frame_stats(k[t], v[t], beta[t])
        A_all.append(A_t)
        B_all.append(B_t)
    P = forward_scan(S0_fwd, A_all, B_all, alpha)
    R = reverse_scan(S0_rev, A_all, B_all, alpha)

    y = np.empty((T, U, d_v))
    if alpha is None:
        for c in range(num_chunks(T, chunk)):
            S_tilde = gathered_state(c, T, chunk, window_chunks, P, R, S0_fwd, S0_rev)
            for t in range(c * chunk, min(T, (c + 1) * chunk)):
                o = q[t] @ S_tilde.T              # o_u = S~ q_u for every token u
                y[t] = rms_gate(o, gate[t], rms_weight, eps)
    else:
        for t in range(T):
            S_tilde = gathered_state_frame(t, T, chunk, window_chunks, P, R, S0_fwd, S0_rev, alpha)
            y[t] = rms_gate(q[t] @ S_tilde.T, gate[t], rms_weight, eps)
    if not keep:
        return y
    M_all = [np.linalg.inv(np.eye(d_k) + A_t) for A_t in A_all]
    return y, dict(A=np.stack(A_all), B=np.stack(B_all), M=np.stack(M_all),
                   P=np.stack(P), R=np.stack(R))


def boundary_states(P, R, S0_fwd, S0_rev, T, chunk):
    """The chunk-boundary states a readout can need, per direction:
      fwd[j] = state after frames [0, jC)   (fwd[0] = S0_fwd), j = 0..NC
      rev[j] = state after frames [jC, T)   (rev[NC] = S0_rev), j = 0..NC
    where NC = ceil(T / C); fwd[NC] is the final forward state P_{T-1} and
    rev[0] the final reverse state R_0.  Returns an array [2, NC+1, d_v, d_k]."""
    nc = num_chunks(T, chunk)
    S0_fwd = _f64(S0_fwd)
    S0_rev = _f64(S0_rev)
    fwd = [S0_fwd] + [P[min(j * chunk, T) - 1] for j in range(1, nc + 1)]
    rev = [R[j * chunk] for j in range(nc)] + [S0_rev]
    return np.stack([np.stack(fwd), np.stack(rev)])


def frame_map(A, B, alpha_t=None):
    """The frame update as an affine map of the entering state (Appendix A.1,
    Eq. A.1): S_t = S_{t-1} M_t + J_t with M_t = Diag(alpha_t)(I + A_t)^{-1}
    and J_t = B_t (I + A_t)^{-1}.  Returns (M_t, J_t)."""
    A = _f64(A)
    d_k = A.shape[0]
    inv = np.linalg.inv(np.eye(d_k) + A)
    M = inv if alpha_t is None else _f64(alpha_t)[:, None] * inv
    return M, _f64(B) @ inv


def compose_maps(first, second):
    """Apply `first` then `second`: S -> (S M1 + J1) M2 + J2 = S (M1 M2) + (J1 M2 + J2)."""
    (M1, J1), (M2, J2) = first, second
    return M1 @ M2, J1 @ M2 + J2


def boundary_states_by_chunk_maps(A_all, B_all, S0_fwd, S0_rev, T, chunk, alpha=None):
    """A second route to the boundary states (the chunk-wise scan of Section 5):
    each chunk's frames are composed into one affine map (Eq. A.1), in frame
    order for the forward scan and in reverse frame order for the reverse scan,
    and the short chunk sequence is scanned in both directions.  Returns the
    same [2, NC+1, d_v, d_k] array as boundary_states."""
    nc = num_chunks(T, chunk)
    maps = [frame_map(A_all[t], B_all[t], None if alpha is None else alpha[t]) for t in range(T)]
    fwd = [_f64(S0_fwd)]
    for j in range(nc):
        frames = range(j * chunk, min(T, (j + 1) * chunk))
        m = None
        for t in frames:
            m = maps[t] if m is None else compose_maps(m, maps[t])
        fwd.append(fwd[-1] @ m[0] + m[1])
    rev = [None] * (nc + 1)
    rev[nc] = _f64(S0_rev)
    for j in range(nc - 1, -1, -1):
        frames = range(min(T, (j + 1) * chunk) - 1, j * chunk - 1, -1)
        m = None
        for t in frames:
            m = maps[t] if m is None else compose_maps(m, maps[t])
        rev[j] = rev[j + 1] @ m[0] + m[1]
    return np.stack([np.stack(fwd), np.stack(rev)])


def vda_forward(q, k, v, beta, gate, rms_weight, S0_fwd, S0_rev,
                chunk, window_chunks, eps=RMS_EPS, heads=None, alpha=None):
    """Whole-tensor wrapper: q, k: [B, H, T, U, d_k]; v, gate: [B, H, T, U, d_v];
    beta: [B, H, T, U]; S0_*: [B, H, d_v, d_k] or None; alpha: [B, H, T, d_k]
    or None.

    Streams one (b, h) at a time.  `heads` optionally restricts the work to a
    list of (b, h) pairs; the result then holds only those heads, in order,
    as an array [len(heads), T, U, d_v]."""
    Bn, Hn = k.shape[0], k.shape[1]
    pairs = heads if heads is not None else [(b, h) for b in range(Bn) for h in range(Hn)]
    out = []
    for (b, h) in pairs:
        s0f = None if S0_fwd is None else S0_fwd[b, h]
        s0r = None if S0_rev is None else S0_rev[b, h]
        a = None if alpha is None else alpha[b, h]
        out.append(vda_forward_head(q[b, h], k[b, h], v[b, h], beta[b, h], gate[b, h],
                                    rms_weight, s0f, s0r, chunk, window_chunks, eps, alpha=a))
    out = np.stack(out)
    if heads is None:
        out = out.reshape((Bn, Hn) + out.shape[1:])
    return out


# ---------------------------------------------------------------------------
# A second, independent route: rescan from scratch for every query frame.
# ---------------------------------------------------------------------------
def vda_forward_head_naive(q, k, v, beta, gate, rms_weight, S0_fwd, S0_rev,
                           chunk, window_chunks, eps=RMS_EPS, alpha=None):
    """O(T^2) restatement of Appendix A.3 for small cases: for each query frame
    t, rebuild P_{l_t - 1} by running the forward update over frames
    0..l_t - 1 from S0_fwd, and R_{h_t + 1} by running the reverse update over
    frames T-1..h_t + 1 from S0_rev; statistics are recomputed per token with
    the summation form of Eq. (3b); no state is reused between queries.
    With alpha, each update first decays its entering state (Eq. 2), and the
    bridge is taken as the paper describes it, frame by frame: decay without
    writes over frames l_t..t (forward) and h_t..t (reverse)."""
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    beta = _f64(beta)
    gate = _f64(gate)
    T, U, d_k = k.shape
    d_v = v.shape[2]
    S0_fwd = np.zeros((d_v, d_k)) if S0_fwd is None else _f64(S0_fwd)
    S0_rev = np.zeros((d_v, d_k)) if S0_rev is None else _f64(S0_rev)

    def stats_by_token(r):
        A = np.zeros((d_k, d_k))
        B = np.zeros((d_v, d_k))
        for u in range(U):
            A += beta[r, u] * np.outer(k[r, u], k[r, u])
            B += beta[r, u] * np.outer(v[r, u], k[r, u])
        return A, B

    y = np.empty((T, U, d_v))
    for t in range(T):
        c = t // chunk
        lo = max(0, (c - window_chunks) * chunk)
        hi = min(T - 1, (c + window_chunks + 1) * chunk - 1)
        left = S0_fwd.copy()
        for r in range(0, lo):
            enter = left if alpha is None else decayed(left, alpha[r])
            left = frame_update(enter, *stats_by_token(r))
        right = S0_rev.copy()
        for r in range(T - 1, hi, -1):
            enter = right if alpha is None else decayed(right, alpha[r])
            right = frame_update(enter, *stats_by_token(r))
        if alpha is not None:
            for r in range(lo, t + 1):
                left = decayed(left, alpha[r])
            for r in range(hi, t - 1, -1):
                right = decayed(right, alpha[r])
        S_t = left + right
        for u in range(U):
            o = S_t @ q[t, u]
            ms = np.sum(o * o) / d_v
            sig = 1.0 / (1.0 + np.exp(-gate[t, u]))
            y[t, u] = rms_weight * o / np.sqrt(ms + eps) * sig
    return y
