"""The allocation-free entry point `vda_forward_noalloc`.

Some callers cannot allocate device memory at the point where they run this
op (a host framework that owns every device allocation, a plugin inside such
a host, a fixed-footprint serving loop that forbids allocator calls), so the
library offers one forward that takes its scratch from a fixed array inside
the library instead of cudaMalloc or a caller workspace.  These tests call it
through the C ABI twice in a row, on different inputs and head dims, and
check each result against the existing workspace entry point
(`vda_forward_ex`) with the suite's tolerance; they also check that sizes
beyond the fixed scratch are refused before anything is launched.

This file is named to be collected last, so a run that stops at the first
failure has already run every other test.
"""

import ctypes

import numpy as np
import pytest

from frame_wise_delta_vda_b200 import _lib, inputs as gen
from _helpers import TOL, rel_err, to_numpy_f64, to_torch


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
    a = _dummy_args()                    # the full-scale workload needs ~460 MB of scratch
    assert L.vda_workspace_bytes(1, 48, 60, 1008, 128, 128, 5, 0) > _lib.NOALLOC_SCRATCH_BYTES
    assert L.vda_forward_noalloc(ctypes.byref(a)) == _lib.VDA_ERR_WORKSPACE
    assert L.vda_forward_noalloc(ctypes.byref(_dummy_args(B=0))) == _lib.VDA_ERR_INVALID_ARGUMENT
    assert L.vda_forward_noalloc(None) == _lib.VDA_ERR_INVALID_ARGUMENT


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row():
    import torch
    from frame_wise_delta_vda_b200 import api

    L = _lib.lib()
    cases = [
        gen.custom("noalloc_a", H=8, T=20, U=240, d=64, chunk=5, window_chunks=1, dtype="bf16", seed=31),
        gen.custom("noalloc_b", H=2, T=11, U=200, d=128, chunk=5, window_chunks=1, dtype="bf16", seed=32),
    ]
    for wl in cases:
        assert L.vda_workspace_bytes(wl.B, wl.H, wl.T, wl.U, wl.d, wl.d, wl.chunk, 0) \
            <= _lib.NOALLOC_SCRATCH_BYTES
    for wl in cases:                      # two calls in a row, sharing the scratch array
        x = gen.make_inputs(wl)
        t = {k: to_torch(v, "cuda") for k, v in x.items()}
        rng = np.random.default_rng(wl.seed)
        S0 = to_torch((0.2 * rng.standard_normal((wl.B, wl.H, wl.d, wl.d))).astype(np.float32), "cuda")
        want = api.vda_forward(t["q"], t["k"], t["v"], t["beta"], t["gate"], t["rms_weight"], S0, S0,
                               chunk=wl.chunk, window_chunks=wl.window_chunks,
                               workspace=api.workspace_for(t["q"], t["v"], wl.chunk))
        got = torch.full_like(want, float("nan"))
        a = api.make_args(t["q"], t["k"], t["v"], t["beta"], t["gate"], t["rms_weight"], S0, S0, got,
                          wl.chunk, wl.window_chunks)
        assert L.vda_forward_noalloc(ctypes.byref(a)) == _lib.VDA_OK
        torch.cuda.synchronize()
        assert api.vda_device_status() == 0
        g, w = to_numpy_f64(got), to_numpy_f64(want)
        for h in range(wl.H):
            assert rel_err(g[0, h], w[0, h]) <= TOL[wl.dtype], (wl.name, h)
