"""Failure detection without a GPU fault: a kernel's bounded wait on a flag
that nothing sets runs out, the library records a wait time-out, the host
reads it through vda_device_status, and the context stays usable."""

import pytest

from frame_wise_delta_vda_b200 import inputs as gen

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def test_bounded_wait_reports_timeout_and_context_survives():
    from frame_wise_delta_vda_b200 import api
    from frame_wise_delta_vda_b200._lib import check, lib
    L = lib()
    assert api.vda_device_status() == 0
    check(L.vda_selftest_wait_timeout(1000, None), "vda_selftest_wait_timeout")
    assert api.vda_device_status() == 5        # VDA_ERR_TIMEOUT, read once ...
    assert api.vda_device_status() == 0        # ... and cleared
    # the context still runs the op
    wl = gen.custom("after_timeout", H=1, T=4, U=8, d=16, chunk=2, window_chunks=0, dtype="f32", seed=3)
    x = gen.make_inputs(wl)
    t = {k: torch.from_numpy(v).cuda() for k, v in x.items()}
    out = api.vda_forward(t["q"], t["k"], t["v"], t["beta"], t["gate"], t["rms_weight"], chunk=2, window_chunks=0)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
    assert api.vda_device_status() == 0


def test_selftest_rejects_bad_limits():
    from frame_wise_delta_vda_b200._lib import lib
    L = lib()
    assert L.vda_selftest_wait_timeout(0, None) == 1
    assert L.vda_selftest_wait_timeout(2000000, None) == 1
