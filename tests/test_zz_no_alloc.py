"""The allocation-free entry point `vda_forward_noalloc`.

Some callers cannot allocate device memory at the point where they run this
op (a host framework that owns every device allocation, a plugin inside such
a host, a fixed-footprint serving loop that forbids allocator calls), so the
library offers one forward that takes its scratch from a fixed array inside
the library instead of cudaMalloc or a caller workspace.  These tests call it
through the C ABI several times in a row, on different inputs, head dims and
options, and check each result against the existing workspace entry point
(`vda_forward_ex`): the same kernels run in the same launch configuration, so
the outputs must agree bit for bit.  One head of each case is also checked
against the float64 oracle at the suite's tolerance.  The last case (decay
gates, no initial states) runs after a larger call has left non-zero data in
the shared array, so a scratch word read before it is written would show.
Sizes beyond the fixed scratch are refused before anything is launched.

This file is named to be collected last, so a run that stops at the first
failure has already run every other test.
"""

import ctypes

import numpy as np
import pytest

from frame_wise_delta_vda_b200 import _lib, inputs as gen
from _helpers import TOL, oracle_head, rel_err, to_numpy_f64, to_torch


def _dummy_args(**kw):
    a = _lib.VdaArgs()
    a.dtype = 0
    for f in ("q", "k", "v", "beta", "gate", "rms_weight", "out"):
        setattr(a, f, 0x10000)          # aligned placeholders, never dereferenced
    a.B, a.H, a.T, a.U, a.d_k, a.d_v, a.chunk, a.window_chunks = 1, 48, 60, 1008, 128, 128, 5, 1
    a.eps = 1e-6
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def test_noalloc_refuses_sizes_beyond_its_scratch():
    L = _lib.lib()
    a = _dummy_args()
    # the full-scale workload needs about 650 MB of scratch (A, B, the M operand
    # images, boundary states and bridge products), far beyond the fixed array
    need = L.vda_workspace_bytes(1, 48, 60, 1008, 128, 128, 5, 0)
    assert 600e6 < need < 700e6 and need > _lib.NOALLOC_SCRATCH_BYTES
    assert L.vda_forward_noalloc(ctypes.byref(a)) == _lib.VDA_ERR_WORKSPACE
    assert L.vda_forward_noalloc(ctypes.byref(_dummy_args(B=0))) == _lib.VDA_ERR_INVALID_ARGUMENT
    assert L.vda_forward_noalloc(None) == _lib.VDA_ERR_INVALID_ARGUMENT


def test_noalloc_binding_never_allocates_the_output():
    torch = pytest.importorskip("torch")
    from frame_wise_delta_vda_b200 import api
    z = torch.zeros((1, 1, 1, 1, 16))
    with pytest.raises(ValueError):
        api.vda_forward_noalloc(z, z, z, z[..., 0], z, z[0, 0, 0, 0], out=None)


CASES = [
    # name, workload fields, initial states, decay gates
    ("simt_d64", dict(H=8, T=20, U=240, d=64, chunk=5, window_chunks=1, dtype="bf16", seed=31), True, False),
    ("tc_d128", dict(H=2, T=11, U=200, d=128, chunk=5, window_chunks=1, dtype="bf16", seed=32), True, False),
    ("tc_d128_decay_noS0", dict(H=2, T=9, U=130, d=128, chunk=2, window_chunks=1, dtype="bf16", seed=33,
                                alpha_mean=1.5), False, True),
]


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_on_calls_in_a_row():
    import torch
    from frame_wise_delta_vda_b200 import api

    L = _lib.lib()
    wls = [(gen.custom(name, **f), s0, dec) for name, f, s0, dec in CASES]
    for wl, _, _ in wls:
        assert L.vda_workspace_bytes(wl.B, wl.H, wl.T, wl.U, wl.d, wl.d, wl.chunk, 0) \
            <= _lib.NOALLOC_SCRATCH_BYTES
    # the cases run in a row and share the scratch array; the second leaves
    # more scratch in use than the third needs
    for wl, with_s0, with_alpha in wls:
        x = gen.make_inputs(wl)
        t = {k: to_torch(v, "cuda") for k, v in x.items()}
        S0 = None
        if with_s0:
            rng = np.random.default_rng(wl.seed)
            S0 = to_torch((0.2 * rng.standard_normal((wl.B, wl.H, wl.d, wl.d))).astype(np.float32), "cuda")
        alpha = t["alpha"] if with_alpha else None
        want = api.vda_forward(t["q"], t["k"], t["v"], t["beta"], t["gate"], t["rms_weight"], S0, S0,
                               chunk=wl.chunk, window_chunks=wl.window_chunks,
                               workspace=api.workspace_for(t["q"], t["v"], wl.chunk), alpha=alpha)
        got = torch.full_like(want, float("nan"))
        a = api.make_args(t["q"], t["k"], t["v"], t["beta"], t["gate"], t["rms_weight"], S0, S0, got,
                          wl.chunk, wl.window_chunks, alpha=alpha)
        assert L.vda_forward_noalloc(ctypes.byref(a)) == _lib.VDA_OK
        torch.cuda.synchronize()
        assert api.vda_device_status() == 0
        # same kernels, same launches: bit for bit
        assert torch.equal(got.view(torch.int16), want.view(torch.int16)), wl.name
        # and one head against the float64 oracle
        xh = {k: (v[0, 1] if k != "rms_weight" else v) for k, v in x.items()}
        s0h = None if S0 is None else S0[0, 1].double().cpu().numpy()
        y_ref = oracle_head(xh, wl, s0h, s0h)
        assert rel_err(to_numpy_f64(got[0, 1]), y_ref) <= TOL[wl.dtype], wl.name
