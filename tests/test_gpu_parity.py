"""Parity of the CUDA path (through the C ABI) with the float64 oracle.

Bar: relative Frobenius error per (b, h) <= 1e-2 for bf16 I/O and <= 1e-4 for
float32 I/O; intermediates (A, B, M, boundary states) are diagnostic, with
the bounds of TOL_INTER (10x tighter than the output bound).  Full-size workloads run in the launch configuration the
benchmark times and are compared on sampled heads.
"""

import numpy as np
import pytest

import oracle as ref
from frame_wise_delta_vda_b200 import inputs as gen
from _helpers import TOL, TOL_INTER, oracle_head, oracle_text_state, rel_err, to_numpy_f64, to_torch

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _api():
    from frame_wise_delta_vda_b200 import api
    return api


def _device_inputs(wl, x):
    dev = torch.device("cuda:0")
    t = {k: to_torch(v, dev) for k, v in x.items()}
    return t


def _run(wl, t, S0f=None, S0r=None, keep=False, window=None, chunk=None):
    api = _api()
    chunk = wl.chunk if chunk is None else chunk
    window = wl.window_chunks if window is None else window
    Bn, Hn, T, U, d = t["q"].shape
    states = stats = None
    if keep:
        nc = (T + chunk - 1) // chunk
        states = torch.empty((2, Bn, Hn, nc + 1, d, d), dtype=torch.float32, device="cuda")
        stats = torch.empty((3, Bn, Hn, T, d, d), dtype=torch.float32, device="cuda")
    out = api.vda_forward(t["q"], t["k"], t["v"], t["beta"], t["gate"], t["rms_weight"], S0f, S0r,
                          chunk=chunk, window_chunks=window, states_out=states, stats_out=stats,
                          workspace=api.workspace_for(t["q"], t["v"], chunk) if keep else None)
    torch.cuda.synchronize()
    assert api.vda_device_status() == 0
    return out, states, stats


def _head_x(x, b, h):
    return {k: (v[b, h] if k != "rms_weight" else v) for k, v in x.items()}


# --- the three small workloads: every head, plus intermediates --------------
@pytest.mark.parametrize("name", ["tiny", "small", "corr"])
def test_workload_parity_all_heads(name):
    wl = gen.WORKLOADS[name]
    x = gen.make_inputs(wl)
    t = _device_inputs(wl, x)
    out, states, stats = _run(wl, t, keep=True)
    y = to_numpy_f64(out)
    st = states.cpu().double().numpy()
    sa = stats.cpu().double().numpy()
    worst = {"out": 0.0, "states": 0.0, "A": 0.0, "B": 0.0, "M": 0.0}
    for b in range(wl.B):
        for h in range(wl.H):
            xh = _head_x(x, b, h)
            y_ref, inter = oracle_head(xh, wl, keep=True)
            e = rel_err(y[b, h], y_ref)
            worst["out"] = max(worst["out"], e)
            assert e <= TOL[wl.dtype], (name, b, h, e)
            bs = ref.boundary_states(inter["P"], inter["R"], np.zeros((wl.d, wl.d)),
                                     np.zeros((wl.d, wl.d)), wl.T, wl.chunk)
            errs = {"states": rel_err(st[:, b, h], bs), "A": rel_err(sa[0, b, h], inter["A"]),
                    "B": rel_err(sa[1, b, h], inter["B"]), "M": rel_err(sa[2, b, h], inter["M"])}
            for key, e in errs.items():
                worst[key] = max(worst[key], e)
                assert e <= TOL_INTER[wl.dtype], (key, b, h, e)
    print(f"{name}: worst per-head rel err " + ", ".join(f"{k} {v:.3e}" for k, v in worst.items()))


def test_tiny_output_is_exactly_zero():
    wl = gen.WORKLOADS["tiny"]
    t = _device_inputs(wl, gen.make_inputs(wl))
    out, _, _ = _run(wl, t)
    assert torch.count_nonzero(out).item() == 0


# --- full-size workloads: sampled heads, text initial state ------------------
@pytest.mark.parametrize("name,heads", [("full", [(0, 0), (0, 23), (0, 47)]),
                                        ("long", [(0, 0), (1, 30), (1, 47)])])
def test_full_size_parity_sampled_heads(name, heads):
    api = _api()
    wl = gen.WORKLOADS[name]
    x = gen.make_inputs(wl)
    t = _device_inputs(wl, x)
    S0 = api.vda_text_state(t["k_text"], t["v_text"], t["beta_text"])
    # the benchmark's launch: bf16, d = 128, preallocated workspace
    ws = api.workspace_for(t["q"], t["v"], wl.chunk)
    out = api.vda_forward(t["q"], t["k"], t["v"], t["beta"], t["gate"], t["rms_weight"], S0, S0,
                          chunk=wl.chunk, window_chunks=wl.window_chunks, workspace=ws)
    torch.cuda.synchronize()
    assert api.vda_device_status() == 0
    S0_np = S0.cpu().double().numpy()
    for (b, h) in heads:
        xh = _head_x(x, b, h)
        S_text = oracle_text_state(xh)
        assert rel_err(S0_np[b, h], S_text) <= TOL_INTER[wl.dtype]
        y_ref = oracle_head(xh, wl, S_text, S_text)
        e = rel_err(to_numpy_f64(out[b, h]), y_ref)
        assert e <= TOL[wl.dtype], (name, b, h, e)


# --- edge cases --------------------------------------------------------------
EDGE = [
    # name, fields
    ("ragged_T", dict(T=12, U=16, d=16, chunk=5, window_chunks=1, dtype="f32")),
    ("odd_U", dict(T=10, U=17, d=32, chunk=5, window_chunks=1, dtype="f32")),
    ("T1", dict(T=1, U=8, d=16, chunk=5, window_chunks=0, dtype="f32")),
    ("w0", dict(T=9, U=8, d=16, chunk=3, window_chunks=0, dtype="f32")),
    ("covering", dict(T=7, U=8, d=16, chunk=2, window_chunks=5, dtype="f32")),
    ("chunk1", dict(T=6, U=5, d=16, chunk=1, window_chunks=1, dtype="f32")),
    ("B2_d64", dict(B=2, H=3, T=10, U=33, d=64, chunk=5, window_chunks=1, dtype="f32")),
    ("d128_f32", dict(H=2, T=10, U=70, d=128, chunk=5, window_chunks=1, dtype="f32")),
    ("bf16_d64_ragged", dict(H=2, T=13, U=40, d=64, chunk=5, window_chunks=1, dtype="bf16")),
    ("bf16_d64_B2", dict(B=2, H=3, T=9, U=70, d=64, chunk=4, window_chunks=1, dtype="bf16")),
    ("bf16_d128_oddU", dict(H=2, T=11, U=129, d=128, chunk=5, window_chunks=1, dtype="bf16")),
    ("bf16_d128_U1", dict(H=1, T=6, U=1, d=128, chunk=2, window_chunks=0, dtype="bf16")),
    ("bf16_d128_long_chunk", dict(H=1, T=4, U=300, d=128, chunk=3, window_chunks=0, dtype="bf16")),
]


@pytest.mark.parametrize("name,fields", EDGE, ids=[e[0] for e in EDGE])
@pytest.mark.parametrize("with_s0", [False, True])
def test_edge_case_parity(name, fields, with_s0):
    wl = gen.custom(name, seed=11, **fields)
    x = gen.make_inputs(wl)
    t = _device_inputs(wl, x)
    S0f = S0r = None
    s0f_np = s0r_np = None
    if with_s0:
        rng = np.random.default_rng(5)
        s0f_np = (0.3 * rng.standard_normal((wl.B, wl.H, wl.d, wl.d))).astype(np.float32)
        s0r_np = (0.3 * rng.standard_normal((wl.B, wl.H, wl.d, wl.d))).astype(np.float32)
        S0f, S0r = to_torch(s0f_np, "cuda"), to_torch(s0r_np, "cuda")
    out, states, _ = _run(wl, t, S0f, S0r, keep=True)
    y = to_numpy_f64(out)
    st = states.cpu().double().numpy()
    for b in range(wl.B):
        for h in range(wl.H):
            xh = _head_x(x, b, h)
            f = None if s0f_np is None else s0f_np[b, h].astype(np.float64)
            r = None if s0r_np is None else s0r_np[b, h].astype(np.float64)
            y_ref, inter = oracle_head(xh, wl, f, r, keep=True)
            e = rel_err(y[b, h], y_ref)
            assert e <= TOL[wl.dtype], (name, b, h, e)
            zero = np.zeros((wl.d, wl.d))
            bs = ref.boundary_states(inter["P"], inter["R"], zero if f is None else f,
                                     zero if r is None else r, wl.T, wl.chunk)
            assert rel_err(st[:, b, h], bs) <= TOL_INTER[wl.dtype]


# --- resuming the forward scan across calls ----------------------------------
def test_forward_scan_resumes_across_calls():
    api = _api()
    wl = gen.custom("resume", H=2, T=20, U=24, d=32, chunk=5, window_chunks=1, dtype="f32", seed=3)
    t = _device_inputs(wl, gen.make_inputs(wl))
    _, st_all, _ = _run(wl, t, keep=True)
    first = {k: (v[:, :, :10].contiguous() if v.dim() >= 3 and k not in ("rms_weight",) else v)
             for k, v in t.items()}
    second = {k: (v[:, :, 10:].contiguous() if v.dim() >= 3 and k not in ("rms_weight",) else v)
              for k, v in t.items()}
    wl10 = gen.custom("resume10", H=2, T=10, U=24, d=32, chunk=5, window_chunks=1, dtype="f32", seed=3)
    _, st1, _ = _run(wl10, first, keep=True)
    carry = st1[0, :, :, 2].contiguous()                 # state after frames [0, 10)
    _, st2, _ = _run(wl10, second, S0f=carry, keep=True)
    # forward boundaries of the whole clip at frames 10, 15, 20 == second call's 0, 1, 2
    a = st_all[0, :, :, 2:].cpu().double().numpy()
    b = st2[0].cpu().double().numpy()
    assert rel_err(b, a) <= 1e-5


# --- Proposition 1 on the device: the scan never amplifies a state change -----
def test_scan_is_non_expansive_on_device():
    wl = gen.WORKLOADS["corr"]
    x = gen.make_inputs(wl, heads=[(0, 0), (0, 1)])
    t = {k: to_torch(v, "cuda") for k, v in x.items()}
    t = {k: (v.unsqueeze(0) if k != "rms_weight" else v) for k, v in t.items()}
    rng = np.random.default_rng(9)
    S0 = to_torch(rng.standard_normal((1, 2, 128, 128)).astype(np.float32), "cuda")
    dS = to_torch((1e-2 * rng.standard_normal((1, 2, 128, 128))).astype(np.float32), "cuda")
    _, s1, _ = _run(wl, t, S0f=S0, keep=True)
    _, s2, _ = _run(wl, t, S0f=S0 + dS, keep=True)
    d_in = torch.linalg.vector_norm(dS.double(), dim=(-2, -1))          # [1, 2]
    d_out = torch.linalg.vector_norm((s2[0] - s1[0]).double(), dim=(-2, -1))  # [1, 2, NC+1]
    assert torch.all(d_out <= d_in[..., None] * (1 + 1e-3) + 1e-6)
    assert torch.all(d_out[..., 1:] <= d_out[..., :-1] * (1 + 1e-3) + 1e-6)


# --- the host-buffer entry point and determinism ------------------------------
@pytest.mark.parametrize("name", ["small", "corr"])
def test_forward_host_matches_device_path_bitwise(name):
    """The host-buffer entry runs the heads in groups; each group takes the
    scan form the whole problem takes (at 16 heads the per-frame scans, while
    a group of 2 heads alone would take the chunk-wise ones), so the result
    is the device entry's bit for bit."""
    api = _api()
    wl = gen.WORKLOADS[name]
    x = gen.make_inputs(wl)
    t = _device_inputs(wl, x)
    out_dev, _, _ = _run(wl, t)
    host = {k: to_torch(v, "cpu").pin_memory() for k, v in x.items()}
    out_host = torch.empty_like(host["q"]).pin_memory()
    buf = torch.empty(api.vda_forward_host_bytes(host["q"], host["v"], wl.chunk), dtype=torch.uint8,
                      device="cuda")
    api.vda_forward_host(host["q"], host["k"], host["v"], host["beta"], host["gate"], host["rms_weight"],
                         None, None, out_host, wl.chunk, wl.window_chunks, buf)
    assert torch.equal(out_host.view(torch.int16), out_dev.cpu().view(torch.int16))


def test_repeated_runs_are_bitwise_identical():
    wl = gen.WORKLOADS["corr"]
    t = _device_inputs(wl, gen.make_inputs(wl))
    a, _, _ = _run(wl, t)
    b, _, _ = _run(wl, t)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_stage_timer_reports_every_stage():
    api = _api()
    wl = gen.WORKLOADS["small"]
    t = _device_inputs(wl, gen.make_inputs(wl))
    timer = api.StageTimer(3)
    for _ in range(3):
        _run(wl, t)
    ms, calls = timer.read()
    assert calls == 3
    assert all(v > 0 for v in ms.values()), ms


def test_text_state_parity_f32():
    api = _api()
    rng = np.random.default_rng(4)
    kt = rng.standard_normal((2, 3, 40, 32)).astype(np.float32)
    kt /= np.linalg.norm(kt, axis=-1, keepdims=True)
    vt = rng.standard_normal((2, 3, 40, 32)).astype(np.float32)
    bt = (0.5 / (1 + np.exp(-rng.standard_normal((2, 3, 40))))).astype(np.float32)
    S = api.vda_text_state(to_torch(kt, "cuda"), to_torch(vt, "cuda"), to_torch(bt, "cuda"))
    S = S.cpu().double().numpy()
    for b in range(2):
        for h in range(3):
            want = ref.text_state(kt[b, h], vt[b, h], bt[b, h])
            assert rel_err(S[b, h], want) <= 1e-5
