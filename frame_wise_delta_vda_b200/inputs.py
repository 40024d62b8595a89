"""Seeded synthetic inputs for the bidirectional VDA branch.

This module draws random inputs and nothing else: it holds none of the
method's arithmetic (no frame statistics, no solve, no scan, no readout) and
imports nothing from the rest of the package, so both the CUDA path and the
float64 oracle can consume the same inputs without sharing any code.

The five workloads follow the paper's 14.3 s, 768p setting in shape
(latent video (24, 102, 48, 84) -> 100 interior frames, 24 x 42 = 1008 tokens
per frame after 2 x 2 patchify, chunk = 5 latent frames, window = own chunk
+-1) at reduced and full scale; each workload's shapes, distributions and
seed are stated in its `Workload` entry below.

Every (tensor, batch, head) stream has its own numpy SeedSequence
(entropy = [seed, tensor id, b, h]), so any head can be regenerated alone
(the oracle checks sampled heads of the full-size workloads) and the result
does not depend on generation order.  bfloat16 values are produced by
round-to-nearest-even of the float32 draw and are returned as uint16 bit
patterns; `bf16_bits_to_f32` widens them exactly.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

# Stream ids: fixed draw identities (q, k, v, beta, gate, rms weight, text,
# key basis, decay).
_Q, _K, _V, _BETA, _GATE, _W, _KT, _VT, _BT, _KBASIS, _ALPHA = range(11)


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int           # interior latent frames
    U: int           # tokens per frame
    d: int           # d_k = d_v
    chunk: int
    window_chunks: int
    dtype: str       # "bf16" or "f32" for q/k/v/gate/out
    seed: int
    key_mode: str = "gaussian"      # "gaussian" | "subspace8"
    beta_mean: float = 0.0          # beta = sigmoid(N(beta_mean, 1))
    rms_weight: str = "ones"        # "ones" | "jitter" (1 + 0.1 N(0,1))
    text_tokens: int = 0            # > 0: S0 from a text frame
    alpha_mean: float | None = None  # decay gates alpha = sigmoid(N(alpha_mean, 1)); None: no decay
    notes: str = field(default="", compare=False)

    @property
    def frame_heads(self):
        return self.B * self.H * self.T

    @property
    def tokens(self):
        """Frame-tokens B*T*U: the unit of the throughput metric."""
        return self.B * self.T * self.U


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 10, 16, 16, 5, 1, "f32", 0),
    "small": Workload("small", 1, 8, 20, 240, 64, 5, 1, "bf16", 1, rms_weight="jitter"),
    "corr": Workload("corr", 1, 16, 30, 1024, 128, 5, 1, "bf16", 2,
                     key_mode="subspace8", beta_mean=2.0),
    "full": Workload("full", 1, 48, 60, 1008, 128, 5, 1, "bf16", 3, text_tokens=256),
    "long": Workload("long", 2, 48, 120, 1008, 128, 5, 1, "bf16", 4, text_tokens=256),
    # the same shapes with the channel-wise decay gate of Eq. 2 and its bridge
    "small_decay": Workload("small_decay", 1, 8, 20, 240, 64, 5, 1, "bf16", 11, rms_weight="jitter",
                            alpha_mean=2.5),
    "corr_decay": Workload("corr_decay", 1, 16, 30, 1024, 128, 5, 1, "bf16", 12,
                           key_mode="subspace8", beta_mean=2.0, alpha_mean=2.5),
    "full_decay": Workload("full_decay", 1, 48, 60, 1008, 128, 5, 1, "bf16", 13, text_tokens=256,
                           alpha_mean=2.5),
}


def custom(name="custom", **kw):
    """A workload with explicit fields (tests use it for edge cases)."""
    base = dict(B=1, H=1, T=10, U=16, d=16, chunk=5, window_chunks=1, dtype="f32", seed=0)
    base.update(kw)
    return Workload(name, **base)


# ---------------------------------------------------------------------------
def _rng(seed, sid, b, h):
    return np.random.default_rng(np.random.SeedSequence([int(seed), sid, b, h]))


def f32_to_bf16_bits(x):
    """Round float32 values to bfloat16 (round to nearest, ties to even);
    returns the 16-bit patterns as uint16."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32)
    rounded = bits + np.uint32(0x7FFF) + ((bits >> np.uint32(16)) & np.uint32(1))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits):
    """Exact widening of bfloat16 bit patterns (uint16) to float32."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _unit_rows(x):
    n = np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=-1, keepdims=True))
    return (x / np.maximum(n, 1e-30)).astype(np.float32)


def _sigmoid32(x):
    return (1.0 / (1.0 + np.exp(-x.astype(np.float64)))).astype(np.float32)


def _store(x, dtype):
    return f32_to_bf16_bits(x) if dtype == "bf16" else np.ascontiguousarray(x, np.float32)


def head_inputs(wl: Workload, b: int, h: int):
    """Inputs of one (batch, head): dict of q, k, v, gate ([T, U, d], bf16 bits
    or float32), beta ([T, U] float32), alpha ([T, d] float32) if the workload
    has a decay gate and, if it has a text prompt, k_text, v_text ([L, d]) and
    beta_text ([L] float32)."""
    T, U, d = wl.T, wl.U, wl.d
    out = {}
    q = _rng(wl.seed, _Q, b, h).standard_normal((T, U, d), dtype=np.float32)
    out["q"] = _store(_unit_rows(q), wl.dtype)
    if wl.key_mode == "subspace8":
        # keys = L2-normalise(rank-8 subspace projection of N(0,1) + 0.05 N(0,1))
        basis_src = _rng(wl.seed, _KBASIS, b, h).standard_normal((d, 8))
        Qb, _ = np.linalg.qr(basis_src)                # orthonormal d x 8 basis
        rk = _rng(wl.seed, _K, b, h)
        z = rk.standard_normal((T, U, d), dtype=np.float32).astype(np.float64)
        n = rk.standard_normal((T, U, d), dtype=np.float32).astype(np.float64)
        k = (z @ Qb) @ Qb.T + 0.05 * n
        out["k"] = _store(_unit_rows(k), wl.dtype)
    else:
        k = _rng(wl.seed, _K, b, h).standard_normal((T, U, d), dtype=np.float32)
        out["k"] = _store(_unit_rows(k), wl.dtype)
    out["v"] = _store(_rng(wl.seed, _V, b, h).standard_normal((T, U, d), dtype=np.float32), wl.dtype)
    beta_logit = _rng(wl.seed, _BETA, b, h).standard_normal((T, U), dtype=np.float32) + np.float32(wl.beta_mean)
    out["beta"] = _sigmoid32(beta_logit)
    out["gate"] = _store(_rng(wl.seed, _GATE, b, h).standard_normal((T, U, d), dtype=np.float32), wl.dtype)
    if wl.alpha_mean is not None:
        # channel-wise decay gates alpha_t in (0, 1), one per frame and key channel
        a_logit = _rng(wl.seed, _ALPHA, b, h).standard_normal((T, d), dtype=np.float32) + np.float32(wl.alpha_mean)
        out["alpha"] = _sigmoid32(a_logit)
    if wl.text_tokens > 0:
        L = wl.text_tokens
        kt = _rng(wl.seed, _KT, b, h).standard_normal((L, d), dtype=np.float32)
        out["k_text"] = _store(_unit_rows(kt), wl.dtype)
        out["v_text"] = _store(_rng(wl.seed, _VT, b, h).standard_normal((L, d), dtype=np.float32), wl.dtype)
        # text write gates sigmoid(N(0,1)), halved so that both scans together
        # carry the prompt once
        out["beta_text"] = (_sigmoid32(_rng(wl.seed, _BT, b, h).standard_normal(L, dtype=np.float32))
                            * np.float32(0.5))
    return out


def rms_weight(wl: Workload):
    """The RMSNorm weight vector [d_v] (float32), shared by all heads."""
    if wl.rms_weight == "jitter":
        g = _rng(wl.seed, _W, 0, 0).standard_normal(wl.d, dtype=np.float32)
        return (np.float32(1.0) + np.float32(0.1) * g).astype(np.float32)
    return np.ones(wl.d, dtype=np.float32)


def make_inputs(wl: Workload, heads=None):
    """All inputs as contiguous arrays [B, H, ...] (or, with `heads` = list of
    (b, h), stacked [len(heads), ...]).  Keys: q, k, v, gate, beta, rms_weight
    and, when the workload has a prompt, k_text, v_text, beta_text."""
    pairs = heads if heads is not None else [(b, h) for b in range(wl.B) for h in range(wl.H)]
    per = [head_inputs(wl, b, h) for (b, h) in pairs]
    out = {}
    for key in per[0]:
        arr = np.stack([p[key] for p in per])
        if heads is None:
            arr = arr.reshape((wl.B, wl.H) + arr.shape[1:])
        out[key] = np.ascontiguousarray(arr)
    out["rms_weight"] = rms_weight(wl)
    return out


def as_f64(x):
    """float64 view of a generated array (bf16 bits are widened exactly)."""
    if x.dtype == np.uint16:
        return bf16_bits_to_f32(x).astype(np.float64)
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# Feature preparation (VDA-Prep) inputs: the QKV projections of the interior
# video tokens, before the linear branch's feature map, and its filters.
# ---------------------------------------------------------------------------
_PQ, _PK, _PV, _PWKS, _PWKT, _PWVS, _PWVT = range(20, 27)


@dataclass(frozen=True)
class PrepWorkload:
    name: str
    B: int
    H: int
    T: int           # interior latent frames
    Hl: int          # latent grid rows
    Wl: int          # latent grid columns (tokens per frame U = Hl * Wl)
    d: int
    seed: int

    @property
    def U(self):
        return self.Hl * self.Wl

    @property
    def tokens(self):
        return self.B * self.T * self.U


PREP_WORKLOADS = {
    "prep_small": PrepWorkload("prep_small", 1, 4, 6, 6, 8, 64, 21),
    "prep_odd": PrepWorkload("prep_odd", 2, 3, 5, 3, 7, 128, 22),
    # the full-size grid with 16 heads and 20 frames (0.25 GB per direction): profiling size
    "prep_mid": PrepWorkload("prep_mid", 1, 16, 20, 24, 42, 128, 24),
    # the full-size shapes: 60 interior frames of a 24 x 42 latent grid
    "prep_full": PrepWorkload("prep_full", 1, 48, 60, 24, 42, 128, 23),
}


def prep_head_inputs(pw: PrepWorkload, b: int, h: int):
    """Raw q, k, v of one (batch, head) as [T, U, d] bf16 bits (N(0,1) draws),
    and the head's filters: wk_s, wv_s [d, 5, 5] ~ N(0, 0.2^2) and wk_t, wv_t
    [d, 5] ~ N(0, 0.45^2) (float32)."""
    T, U, d = pw.T, pw.U, pw.d
    out = {}
    for key, sid in (("q", _PQ), ("k", _PK), ("v", _PV)):
        out[key] = f32_to_bf16_bits(_rng(pw.seed, sid, b, h).standard_normal((T, U, d), dtype=np.float32))
    for key, sid in (("wk_s", _PWKS), ("wv_s", _PWVS)):
        out[key] = (np.float32(0.2) * _rng(pw.seed, sid, 0, h).standard_normal((d, 5, 5), dtype=np.float32))
    for key, sid in (("wk_t", _PWKT), ("wv_t", _PWVT)):
        out[key] = (np.float32(0.45) * _rng(pw.seed, sid, 0, h).standard_normal((d, 5), dtype=np.float32))
    return out


def make_prep_inputs(pw: PrepWorkload):
    """All prep inputs: q, k, v [B, T, U, H, d] (bf16 bits, heads inner, as a
    projection lays them out) and the filters wk_s, wv_s [H, d, 5, 5],
    wk_t, wv_t [H, d, 5] (float32; filters are per head, shared by batches)."""
    per = {(b, h): prep_head_inputs(pw, b, h) for b in range(pw.B) for h in range(pw.H)}
    out = {}
    for key in ("q", "k", "v"):
        arr = np.empty((pw.B, pw.T, pw.U, pw.H, pw.d), dtype=np.uint16)
        for (b, h), x in per.items():
            arr[b, :, :, h, :] = x[key]
        out[key] = arr
    for key in ("wk_s", "wk_t", "wv_s", "wv_t"):
        out[key] = np.ascontiguousarray(np.stack([per[(0, h)][key] for h in range(pw.H)]))
    return out
