"""Parity of the decay path (channel-wise gate of Eq. 2 in both scans and the
decay bridge of Eq. A.4) with the float64 oracle, through the C ABI.

Same bars as the plain path: relative Frobenius error per (b, h) <= 1e-2 for
bf16 I/O and <= 1e-4 for float32 I/O; boundary states within TOL_INTER.
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


def _dev(x):
    return {k: to_torch(v, "cuda") for k, v in x.items()}


def _head_x(x, b, h):
    return {k: (v[b, h] if k != "rms_weight" else v) for k, v in x.items()}


def _run(wl, t, S0f=None, S0r=None, alpha="from_inputs", keep=True):
    api = _api()
    Bn, Hn, T, U, d = t["q"].shape
    a = t["alpha"] if isinstance(alpha, str) else alpha
    states = None
    if keep:
        nc = (T + wl.chunk - 1) // wl.chunk
        states = torch.empty((2, Bn, Hn, nc + 1, d, d), dtype=torch.float32, device="cuda")
    out = api.vda_forward(t["q"], t["k"], t["v"], t["beta"], t["gate"], t["rms_weight"], S0f, S0r,
                          chunk=wl.chunk, window_chunks=wl.window_chunks, states_out=states,
                          workspace=api.workspace_for(t["q"], t["v"], wl.chunk), alpha=a)
    torch.cuda.synchronize()
    assert api.vda_device_status() == 0
    return out, states


def _check_heads(wl, x, out, states, s0f=None, s0r=None, heads=None):
    y = to_numpy_f64(out)
    st = None if states is None else states.cpu().double().numpy()
    pairs = heads or [(b, h) for b in range(wl.B) for h in range(wl.H)]
    worst = {"out": 0.0, "states": 0.0}
    for (b, h) in pairs:
        xh = _head_x(x, b, h)
        f = None if s0f is None else s0f[b, h].astype(np.float64)
        r = None if s0r is None else s0r[b, h].astype(np.float64)
        y_ref, inter = oracle_head(xh, wl, f, r, keep=True)
        e = rel_err(y[b, h], y_ref)
        worst["out"] = max(worst["out"], e)
        assert e <= TOL[wl.dtype], (wl.name, b, h, e)
        if st is not None:
            zero = np.zeros((wl.d, wl.d))
            bs = ref.boundary_states(inter["P"], inter["R"], zero if f is None else f,
                                     zero if r is None else r, wl.T, wl.chunk)
            es = rel_err(st[:, b, h], bs)
            worst["states"] = max(worst["states"], es)
            assert es <= TOL_INTER[wl.dtype], ("states", wl.name, b, h, es)
    return worst


@pytest.mark.parametrize("name", ["small_decay", "corr_decay"])
def test_decay_workload_parity_all_heads(name):
    wl = gen.WORKLOADS[name]
    x = gen.make_inputs(wl)
    out, states = _run(wl, _dev(x))
    worst = _check_heads(wl, x, out, states)
    print(f"{name}: worst per-head rel err out {worst['out']:.3e}, states {worst['states']:.3e}")


def test_decay_full_size_sampled_heads():
    """The full-size shapes with decay, in the benchmark's launch (bf16, d = 128,
    preallocated workspace), text initial state, sampled heads."""
    api = _api()
    wl = gen.WORKLOADS["full_decay"]
    x = gen.make_inputs(wl)
    t = _dev(x)
    S0 = api.vda_text_state(t["k_text"], t["v_text"], t["beta_text"])
    out, _ = _run(wl, t, S0, S0, keep=False)
    S0_np = S0.cpu().double().numpy()
    for (b, h) in [(0, 0), (0, 29), (0, 47)]:
        xh = _head_x(x, b, h)
        S_text = oracle_text_state(xh)
        y_ref = oracle_head(xh, wl, S0_np[b, h], S0_np[b, h])
        e = rel_err(to_numpy_f64(out[b, h]), y_ref)
        assert e <= TOL[wl.dtype], ("full_decay", b, h, e)
        assert rel_err(S0_np[b, h], S_text) <= TOL_INTER[wl.dtype]


EDGE = [
    # name, fields (every case has decay gates)
    ("f32_ragged_w0", dict(T=7, U=40, d=16, chunk=3, window_chunks=0, dtype="f32")),
    ("f32_chunk1", dict(T=5, U=9, d=32, chunk=1, window_chunks=1, dtype="f32")),
    ("f32_covering", dict(T=6, U=8, d=16, chunk=2, window_chunks=4, dtype="f32")),
    ("bf16_d64", dict(H=2, T=11, U=33, d=64, chunk=4, window_chunks=1, dtype="bf16")),
    ("bf16_d128_ragged_tiles", dict(H=2, T=9, U=130, d=128, chunk=2, window_chunks=1, dtype="bf16")),
    ("bf16_d128_covering", dict(H=1, T=6, U=200, d=128, chunk=3, window_chunks=1, dtype="bf16")),
    ("bf16_d128_T1", dict(H=1, T=1, U=64, d=128, chunk=5, window_chunks=0, dtype="bf16")),
]


@pytest.mark.parametrize("name,fields", EDGE, ids=[e[0] for e in EDGE])
@pytest.mark.parametrize("with_s0", [False, True])
def test_decay_edge_case_parity(name, fields, with_s0):
    wl = gen.custom(name, seed=17, alpha_mean=1.5, **fields)
    x = gen.make_inputs(wl)
    t = _dev(x)
    s0f = s0r = None
    S0f = S0r = None
    if with_s0:
        rng = np.random.default_rng(6)
        s0f = (0.3 * rng.standard_normal((wl.B, wl.H, wl.d, wl.d))).astype(np.float32)
        s0r = (0.3 * rng.standard_normal((wl.B, wl.H, wl.d, wl.d))).astype(np.float32)
        S0f, S0r = to_torch(s0f, "cuda"), to_torch(s0r, "cuda")
    out, states = _run(wl, t, S0f, S0r)
    _check_heads(wl, x, out, states, s0f, s0r)


@pytest.mark.parametrize("fields", [dict(H=2, T=10, U=40, d=32, dtype="f32"),
                                    dict(H=2, T=10, U=150, d=128, dtype="bf16")],
                         ids=["simt_f32", "tc_bf16"])
def test_decay_of_one_matches_plain_path(fields):
    """alpha = 1 takes the decay kernels (per-frame readout units, bridge
    products) and must give the plain path's result."""
    wl = gen.custom("ones", seed=18, chunk=5, window_chunks=1, **fields)
    x = gen.make_inputs(wl)
    t = _dev(x)
    ones = torch.ones(t["q"].shape[:3] + (wl.d,), dtype=torch.float32, device="cuda")
    out_plain, st_plain = _run(wl, t, alpha=None)
    out_one, st_one = _run(wl, t, alpha=ones)
    assert rel_err(to_numpy_f64(out_one), to_numpy_f64(out_plain)) <= 1e-6
    assert rel_err(st_one.cpu().double().numpy(), st_plain.cpu().double().numpy()) <= 1e-6


def test_decay_host_entry_matches_device_path_bitwise():
    api = _api()
    wl = gen.custom("host_decay", H=3, T=10, U=100, d=128, chunk=5, window_chunks=1, dtype="bf16", seed=19,
                    alpha_mean=2.0)
    x = gen.make_inputs(wl)
    t = _dev(x)
    out_dev, _ = _run(wl, t, keep=False)
    host = {k: to_torch(v, "cpu").pin_memory() for k, v in x.items()}
    out_host = torch.empty_like(host["q"]).pin_memory()
    buf = torch.empty(api.vda_forward_host_bytes(host["q"], host["v"], wl.chunk), dtype=torch.uint8,
                      device="cuda")
    api.vda_forward_host(host["q"], host["k"], host["v"], host["beta"], host["gate"], host["rms_weight"],
                         None, None, out_host, wl.chunk, wl.window_chunks, buf, alpha=host["alpha"])
    assert torch.equal(out_host.view(torch.int16), out_dev.cpu().view(torch.int16))
