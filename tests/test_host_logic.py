"""Host-side logic that needs no GPU: the benchmark's byte and roofline
bookkeeping, the recorded-traffic guard, the input generator's decay and
feature-preparation draws, and the binding's argument checks."""

import importlib.util
import os

import numpy as np
import pytest

from frame_wise_delta_vda_b200 import inputs as gen

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_algorithmic_bytes_of_the_full_workload():
    b = _bench()
    wl = gen.WORKLOADS["full"]
    alg = b.algorithmic(wl)
    FH, U, d = 2880, 1008, 128
    assert alg["op"]["bytes"] == FH * (5 * U * d * 2 + 4 * U)
    assert alg["op"]["flops"] == FH * (6 * U * d * d + 5 * d ** 3)
    # HBM-bound: the byte time exceeds the flop time at the measured peaks
    t_bytes = alg["op"]["bytes"] / 6451.8e9
    t_flops = alg["op"]["flops"] / 1655.5e12
    assert t_bytes > t_flops and 570e-6 < t_bytes < 590e-6
    # the decay gates add their own bytes
    dec = b.algorithmic(gen.WORKLOADS["full_decay"])
    assert dec["op"]["bytes"] - alg["op"]["bytes"] == FH * d * 4


def test_stage_kernels_follow_the_path():
    b = _bench()
    tc = b.stage_kernels(gen.WORKLOADS["full"])
    assert tc["readout"][1] == "k_readout_tc" and tc["inverse"][1] == "k_inverse_tc"
    # the streaming kernels are HBM-limited; the inverse and the scan are dependent chains
    assert tc["stats"][0] == tc["readout"][0] == "hbm"
    assert tc["inverse"][0] == tc["scan"][0] == "latency"
    simt = b.stage_kernels(gen.WORKLOADS["tiny"])
    assert simt["readout"][1] == "k_readout_simt" and simt["inverse"] == ("alu", "k_gj_inverse", ["kernels_simt.cuh"])


def test_recorded_traffic_turns_null_when_the_kernel_changes(monkeypatch):
    b = _bench()
    if not os.path.exists(os.path.join(ROOT, "profiles", "dram_traffic.json")):
        pytest.skip("no recorded traffic")
    monkeypatch.setattr(b, "source_hash", lambda *names: "0000000000000000")
    assert b.recorded_traffic("k_readout_tc") is None
    assert b.recorded_traffic("not_a_kernel") is None


def test_decay_draws():
    wl = gen.WORKLOADS["small_decay"]
    x = gen.head_inputs(wl, 0, 3)
    a = x["alpha"]
    assert a.shape == (wl.T, wl.d) and a.dtype == np.float32
    assert np.all(a > 0) and np.all(a < 1) and 0.8 < a.mean() < 0.95
    np.testing.assert_array_equal(a, gen.head_inputs(wl, 0, 3)["alpha"])
    # the decay stream does not disturb the other draws of the base workload
    base = gen.head_inputs(gen.Workload(**{**wl.__dict__, "alpha_mean": None}), 0, 3)
    for k in ("q", "k", "v", "beta", "gate"):
        np.testing.assert_array_equal(base[k], x[k])


def test_prep_draws_and_layout():
    pw = gen.PREP_WORKLOADS["prep_odd"]
    x = gen.make_prep_inputs(pw)
    assert x["q"].shape == (pw.B, pw.T, pw.U, pw.H, pw.d) and x["q"].dtype == np.uint16
    assert x["wk_s"].shape == (pw.H, pw.d, 5, 5) and x["wv_t"].shape == (pw.H, pw.d, 5)
    for (b, h) in [(0, 0), (1, 2)]:
        one = gen.prep_head_inputs(pw, b, h)
        for k in ("q", "k", "v"):
            np.testing.assert_array_equal(x[k][b, :, :, h, :], one[k])
        np.testing.assert_array_equal(x["wk_s"][h], one["wk_s"])


def test_binding_checks_shapes_before_the_library():
    torch = pytest.importorskip("torch")
    from frame_wise_delta_vda_b200 import api
    B, H, T, U, d = 1, 2, 3, 4, 16
    z = lambda *s, dt=torch.float32: torch.zeros(s, dtype=dt)
    q = z(B, H, T, U, d)
    args = (q, q, q, z(B, H, T, U), q, z(d), None, None, z(B, H, T, U, d), 5, 1)
    api.make_args(*args, check_device=False)
    with pytest.raises(ValueError):
        api.make_args(*args, check_device=False, alpha=z(B, H, T, d + 1))
    with pytest.raises(ValueError):
        api.make_args(q, q, q, z(B, H, T, U + 1), q, z(d), None, None, z(B, H, T, U, d), 5, 1,
                      check_device=False)
    a = api.make_args(*args, check_device=False, alpha=z(B, H, T, d))
    assert a.alpha is not None


def test_bench_line_carries_the_contract_keys(capsys):
    """emit() with made-up timings prints one JSON line with the keys the
    benchmark contract names (no GPU involved)."""
    import json
    import types
    b = _bench()
    wl = gen.WORKLOADS["full"]
    args = types.SimpleNamespace(steps=7, warmup=3, no_cpu_baseline=True)
    stage = {"stats": 0.35 * 7, "inverse": 0.32 * 7, "scan": 0.19 * 7, "readout": 0.40 * 7}
    clocks = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 9}
    e2e = {"e2e_s": 0.058, "h2d": 123, "d2h": 45}
    b.emit(args, wl, 1, 1.3, stage, 7, clocks, e2e, 28)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "clocks", "e2e", "gpu_launches",
              "head_tokens_per_s"):
        assert k in line, k
    assert line["value"] == pytest.approx(wl.tokens / 1.3e-3)
    assert line["roofline"]["stage"] == "readout" and line["roofline"]["kernel"] == "k_readout_tc"
    assert line["roofline"]["frac"] == pytest.approx(line["roofline"]["achieved"] / line["roofline"]["peak"])
    assert line["e2e"]["h2d_bytes_per_step"] == 123 and line["e2e"]["d2h_bytes_per_step"] == 45
    assert "workload" in line["config"] and line["scaling"] == "weak"
