"""Torch-facing binding of libvda.so, with the C ABI's names.

Argument marshalling only: shape/dtype/device checks, pointer extraction and
the current CUDA stream.  Every step of the computation runs in the library's
CUDA kernels; there is no PyTorch or CPU implementation here.
"""

from __future__ import annotations

import ctypes

import torch

from ._lib import (VDA_BF16, VDA_F32, VDA_SCAN_AUTO, VDA_SCAN_CHUNKS, VDA_SCAN_FRAMES, VdaArgs,  # noqa: F401
                   VdaError, VdaPrepArgs, check, lib)

_SCAN_FORMS = {"auto": VDA_SCAN_AUTO, "frames": VDA_SCAN_FRAMES, "chunks": VDA_SCAN_CHUNKS}

_DTYPES = {torch.bfloat16: VDA_BF16, torch.float32: VDA_F32}


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check_tensor(name, t, dtype=None, shape=None, device=None, allow_none=False, on_host=False):
    if t is None:
        if allow_none:
            return
        raise ValueError(f"{name} is required")
    if on_host:
        if t.is_cuda:
            raise ValueError(f"{name} must be a host tensor")
    elif not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def make_args(q, k, v, beta, gate, rms_weight, S0_fwd, S0_rev, out, chunk, window_chunks,
              eps=1e-6, stream=None, check_device=True, alpha=None, scan_form="auto"):
    """Build the C `vda_args` block from tensors (device or host)."""
    if q.dim() != 5:
        raise ValueError("q must be [B, H, T, U, d_k]")
    Bn, Hn, T, U, d_k = q.shape
    d_v = v.shape[-1]
    dt = _DTYPES.get(q.dtype)
    if dt is None:
        raise ValueError(f"unsupported dtype {q.dtype} (bf16 or float32)")
    dev = q.device
    # host tensors (vda_forward_host) get the same shape and dtype checks
    chk = _check_tensor if check_device else (lambda *a, **k: _check_tensor(*a[:4], None, **k, on_host=True))
    chk("q", q, q.dtype, (Bn, Hn, T, U, d_k), dev)
    chk("k", k, q.dtype, (Bn, Hn, T, U, d_k), dev)
    chk("v", v, q.dtype, (Bn, Hn, T, U, d_v), dev)
    chk("gate", gate, q.dtype, (Bn, Hn, T, U, d_v), dev)
    chk("out", out, q.dtype, (Bn, Hn, T, U, d_v), dev)
    chk("beta", beta, torch.float32, (Bn, Hn, T, U), dev)
    chk("rms_weight", rms_weight, torch.float32, (d_v,), dev)
    chk("S0_fwd", S0_fwd, torch.float32, (Bn, Hn, d_v, d_k), dev, allow_none=True)
    chk("S0_rev", S0_rev, torch.float32, (Bn, Hn, d_v, d_k), dev, allow_none=True)
    chk("alpha", alpha, torch.float32, (Bn, Hn, T, d_k), dev, allow_none=True)
    a = VdaArgs()
    a.dtype = dt
    a.q, a.k, a.v, a.beta, a.gate = (t.data_ptr() for t in (q, k, v, beta, gate))
    a.rms_weight = rms_weight.data_ptr()
    a.S0_fwd = S0_fwd.data_ptr() if S0_fwd is not None else None
    a.S0_rev = S0_rev.data_ptr() if S0_rev is not None else None
    a.out = out.data_ptr()
    a.B, a.H, a.T, a.U, a.d_k, a.d_v = Bn, Hn, T, U, d_k, d_v
    a.chunk, a.window_chunks = int(chunk), int(window_chunks)
    a.eps = float(eps)
    a.stream = _stream(stream).value if check_device else None
    a.alpha = alpha.data_ptr() if alpha is not None else None
    if scan_form not in _SCAN_FORMS:
        raise ValueError(f"scan_form must be one of {sorted(_SCAN_FORMS)}")
    a.scan_form = _SCAN_FORMS[scan_form]
    return a


def vda_workspace_bytes(B, H, T, U, d_k, d_v, chunk, dtype=torch.bfloat16):
    return int(lib().vda_workspace_bytes(B, H, T, U, d_k, d_v, chunk, _DTYPES[dtype]))


def workspace_for(q, v, chunk):
    """A device workspace tensor sized for these inputs (uint8, 256-aligned)."""
    Bn, Hn, T, U, d_k = q.shape
    n = vda_workspace_bytes(Bn, Hn, T, U, d_k, v.shape[-1], chunk, q.dtype)
    return torch.empty(n, dtype=torch.uint8, device=q.device)


def vda_forward(q, k, v, beta, gate, rms_weight, S0_fwd=None, S0_rev=None, chunk=5,
                window_chunks=1, out=None, workspace=None, states_out=None, stats_out=None,
                eps=1e-6, stream=None, alpha=None, scan_form="auto"):
    """Bidirectional VDA forward (see include/vda.h).  Returns `out`.

    Without `workspace`, `states_out`, `stats_out`, `alpha` or a `scan_form`
    other than "auto" this calls `vda_forward` / `vda_forward_f32`
    (stream-ordered workspace); otherwise `vda_forward_ex`.  `alpha`
    [B, H, T, d_k] float32 adds the decay gate; `scan_form` ("auto", "frames",
    "chunks") selects the scan form of the tensor-core path.
    """
    if out is None:
        out = torch.empty(q.shape[:-1] + (v.shape[-1],), dtype=q.dtype, device=q.device)
    a = make_args(q, k, v, beta, gate, rms_weight, S0_fwd, S0_rev, out, chunk, window_chunks, eps, stream,
                  alpha=alpha, scan_form=scan_form)
    L = lib()
    if (workspace is None and states_out is None and stats_out is None and eps == 1e-6 and alpha is None
            and scan_form == "auto"):
        fn = L.vda_forward if a.dtype == VDA_BF16 else L.vda_forward_f32
        rc = fn(a.q, a.k, a.v, a.beta, a.gate, a.rms_weight, a.S0_fwd, a.S0_rev,
                a.B, a.H, a.T, a.U, a.d_k, a.d_v, a.chunk, a.window_chunks, a.out, a.stream)
        check(rc, "vda_forward")
        return out
    if workspace is None:
        workspace = workspace_for(q, v, chunk)
    for name, t in (("states_out", states_out), ("stats_out", stats_out)):
        if t is not None:
            _check_tensor(name, t, torch.float32, None, q.device)
    rc = L.vda_forward_ex(ctypes.byref(a), _ptr(workspace), workspace.numel(),
                          _ptr(states_out), _ptr(stats_out))
    check(rc, "vda_forward_ex")
    return out


def vda_prep(q_in, k_in, v_in, wk_s, wk_t, wv_s, wv_t, Hl, Wl, q_out=None, k_out=None, v_out=None,
             eps=1e-6, stream=None):
    """Feature preparation of the linear branch (see include/vda.h):
    q_in, k_in, v_in [B, T, U, H, d] bf16 (U = Hl * Wl) -> q', k', v'
    [B, H, T, U, d] bf16 with q' = L2(q), k' = L2(SiLU(conv(k))),
    v' = SiLU(conv(v)); filters wk_s, wv_s [H, d, 5, 5], wk_t, wv_t [H, d, 5]
    float32.  Returns (q_out, k_out, v_out)."""
    if q_in.dim() != 5:
        raise ValueError("q_in must be [B, T, U, H, d]")
    Bn, T, U, Hn, d = q_in.shape
    if U != Hl * Wl:
        raise ValueError(f"U = {U} is not Hl * Wl = {Hl} * {Wl}")
    dev = q_in.device
    for name, t in (("q_in", q_in), ("k_in", k_in), ("v_in", v_in)):
        _check_tensor(name, t, torch.bfloat16, (Bn, T, U, Hn, d), dev)
    for name, t in (("wk_s", wk_s), ("wv_s", wv_s)):
        _check_tensor(name, t, torch.float32, (Hn, d, 5, 5), dev)
    for name, t in (("wk_t", wk_t), ("wv_t", wv_t)):
        _check_tensor(name, t, torch.float32, (Hn, d, 5), dev)
    outs = []
    for name, t in (("q_out", q_out), ("k_out", k_out), ("v_out", v_out)):
        if t is None:
            t = torch.empty((Bn, Hn, T, U, d), dtype=torch.bfloat16, device=dev)
        _check_tensor(name, t, torch.bfloat16, (Bn, Hn, T, U, d), dev)
        outs.append(t)
    a = VdaPrepArgs()
    a.q_in, a.k_in, a.v_in = q_in.data_ptr(), k_in.data_ptr(), v_in.data_ptr()
    a.wk_s, a.wk_t, a.wv_s, a.wv_t = wk_s.data_ptr(), wk_t.data_ptr(), wv_s.data_ptr(), wv_t.data_ptr()
    a.q_out, a.k_out, a.v_out = (t.data_ptr() for t in outs)
    a.B, a.H, a.T, a.Hl, a.Wl, a.d = Bn, Hn, T, int(Hl), int(Wl), d
    a.eps = float(eps)
    a.stream = _stream(stream).value
    check(lib().vda_prep(ctypes.byref(a)), "vda_prep")
    return tuple(outs)


def vda_text_state(k_text, v_text, beta_text, S_out=None, workspace=None, stream=None):
    """S = B'(I + A')^{-1} per (b, h) from L prompt tokens (one frame-wise
    update of the zero state).  k_text [B,H,L,d_k], v_text [B,H,L,d_v],
    beta_text [B,H,L] float32.  Returns S [B,H,d_v,d_k] float32."""
    Bn, Hn, Lt, d_k = k_text.shape
    d_v = v_text.shape[-1]
    dt = _DTYPES[k_text.dtype]
    _check_tensor("k_text", k_text, k_text.dtype, (Bn, Hn, Lt, d_k))
    _check_tensor("v_text", v_text, k_text.dtype, (Bn, Hn, Lt, d_v), k_text.device)
    _check_tensor("beta_text", beta_text, torch.float32, (Bn, Hn, Lt), k_text.device)
    if S_out is None:
        S_out = torch.empty((Bn, Hn, d_v, d_k), dtype=torch.float32, device=k_text.device)
    _check_tensor("S_out", S_out, torch.float32, (Bn, Hn, d_v, d_k), k_text.device)
    L = lib()
    n = int(L.vda_text_state_workspace_bytes(Bn, Hn, Lt, d_k, d_v, dt))
    if workspace is None:
        workspace = torch.empty(max(n, 1), dtype=torch.uint8, device=k_text.device)
    rc = L.vda_text_state(dt, _ptr(k_text), _ptr(v_text), _ptr(beta_text), Bn, Hn, Lt, d_k, d_v,
                          _ptr(S_out), _ptr(workspace), workspace.numel(), _stream(stream))
    check(rc, "vda_text_state")
    return S_out


def vda_forward_host_bytes(q, v, chunk):
    Bn, Hn, T, U, d_k = q.shape
    return int(lib().vda_forward_host_bytes(Bn, Hn, T, U, d_k, v.shape[-1], chunk, _DTYPES[q.dtype]))


def vda_forward_host(q, k, v, beta, gate, rms_weight, S0_fwd, S0_rev, out, chunk, window_chunks,
                     device_buffer, eps=1e-6, alpha=None):
    """End-to-end forward from host (CPU, ideally pinned) tensors; copies in,
    computes on the current CUDA device and copies `out` back (synchronous)."""
    for name, t in (("q", q), ("k", k), ("v", v), ("beta", beta), ("gate", gate),
                    ("rms_weight", rms_weight), ("out", out), ("S0_fwd", S0_fwd), ("S0_rev", S0_rev),
                    ("alpha", alpha)):
        if t is not None and (t.is_cuda or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous host tensor")
    a = make_args(q, k, v, beta, gate, rms_weight, S0_fwd, S0_rev, out, chunk, window_chunks, eps,
                  check_device=False, alpha=alpha)
    if not device_buffer.is_cuda:
        raise ValueError("device_buffer must be a CUDA tensor")
    rc = lib().vda_forward_host(ctypes.byref(a), _ptr(device_buffer), device_buffer.numel())
    check(rc, "vda_forward_host")
    return out


def vda_forward_noalloc(q, k, v, beta, gate, rms_weight, S0_fwd=None, S0_rev=None, chunk=5,
                        window_chunks=1, out=None, eps=1e-6, stream=None, alpha=None):
    """Forward through `vda_forward_noalloc`: the library uses its fixed
    internal scratch array instead of any allocation (sizes must fit in
    NOALLOC_SCRATCH_BYTES of workspace).  The caller passes a preallocated
    `out`: this route exists for callers that cannot allocate, so it never
    creates a tensor itself."""
    if out is None:
        raise ValueError("vda_forward_noalloc needs a preallocated `out` (this route allocates nothing)")
    a = make_args(q, k, v, beta, gate, rms_weight, S0_fwd, S0_rev, out, chunk, window_chunks, eps, stream,
                  alpha=alpha)
    check(lib().vda_forward_noalloc(ctypes.byref(a)), "vda_forward_noalloc")
    return out


def vda_device_status(stream=None):
    """Synchronise and return the library's device error status (0 = OK)."""
    return int(lib().vda_device_status(_stream(stream)))


def vda_launches_per_forward(B, H, T, U, d_k, d_v, chunk, dtype=torch.bfloat16):
    return int(lib().vda_launches_per_forward(B, H, T, U, d_k, d_v, chunk, _DTYPES[dtype]))


class StageTimer:
    """Per-stage device time (stats, inverse, scan, readout) of the next
    `max_calls` forward calls, from CUDA events the library records on the
    launching stream."""

    NAMES = ("stats", "inverse", "scan", "readout")

    def __init__(self, max_calls):
        check(lib().vda_timing_enable(int(max_calls)), "vda_timing_enable")

    def read(self):
        ms = (ctypes.c_float * 4)()
        calls = ctypes.c_int(0)
        check(lib().vda_timing_read(ms, 4, ctypes.byref(calls)), "vda_timing_read")
        return {n: float(ms[i]) for i, n in enumerate(self.NAMES)}, int(calls.value)
