"""Parity of the chunk-wise scans (Video DeltaNet, Section 5 "Chunk-wise scans",
Appendix A.1: every chunk's frames composed into S -> S P_c + J_c, then the
chunk maps scanned per chain) with the float64 oracle, through the C ABI.

The boundary states of `scan_form="chunks"` are compared with the oracle's
frame-by-frame boundary states (TOL_INTER) and with the per-frame kernels'
states; outputs with the oracle (TOL).  Cases cover the correlated-key stress
workload with and without decay gates, ragged last chunks, one-frame chunks,
a clip shorter than a chunk, and initial states.
"""

import numpy as np
import pytest

import oracle as ref
from frame_wise_delta_vda_b200 import inputs as gen
from _helpers import TOL, TOL_INTER, oracle_head, rel_err, to_numpy_f64, to_torch

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _api():
    from frame_wise_delta_vda_b200 import api
    return api


def _head_x(x, b, h):
    return {k: (v[b, h] if k != "rms_weight" else v) for k, v in x.items()}


def _run(wl, t, form, S0f=None, S0r=None):
    api = _api()
    Bn, Hn, T, U, d = t["q"].shape
    nc = (T + wl.chunk - 1) // wl.chunk
    states = torch.empty((2, Bn, Hn, nc + 1, d, d), dtype=torch.float32, device="cuda")
    out = api.vda_forward(t["q"], t["k"], t["v"], t["beta"], t["gate"], t["rms_weight"], S0f, S0r,
                          chunk=wl.chunk, window_chunks=wl.window_chunks, states_out=states,
                          workspace=api.workspace_for(t["q"], t["v"], wl.chunk), alpha=t.get("alpha"),
                          scan_form=form)
    torch.cuda.synchronize()
    assert api.vda_device_status() == 0
    return out, states


def _check(wl, x, out, states, s0f=None, s0r=None):
    y = to_numpy_f64(out)
    st = states.cpu().double().numpy()
    worst = {"out": 0.0, "states": 0.0}
    for b in range(wl.B):
        for h in range(wl.H):
            xh = _head_x(x, b, h)
            f = None if s0f is None else s0f[b, h].astype(np.float64)
            r = None if s0r is None else s0r[b, h].astype(np.float64)
            y_ref, inter = oracle_head(xh, wl, f, r, keep=True)
            e = rel_err(y[b, h], y_ref)
            worst["out"] = max(worst["out"], e)
            assert e <= TOL[wl.dtype], (wl.name, b, h, e)
            zero = np.zeros((wl.d, wl.d))
            bs = ref.boundary_states(inter["P"], inter["R"], zero if f is None else f,
                                     zero if r is None else r, wl.T, wl.chunk)
            es = rel_err(st[:, b, h], bs)
            worst["states"] = max(worst["states"], es)
            assert es <= TOL_INTER[wl.dtype], ("states", wl.name, b, h, es)
    return worst


@pytest.mark.parametrize("name", ["corr", "corr_decay"])
def test_chunk_scan_parity_all_heads(name):
    wl = gen.WORKLOADS[name]
    x = gen.make_inputs(wl)
    t = {k: to_torch(v, "cuda") for k, v in x.items()}
    out_c, st_c = _run(wl, t, "chunks")
    worst = _check(wl, x, out_c, st_c)
    # the two scan forms agree to the hi/lo operand rounding
    out_f, st_f = _run(wl, t, "frames")
    d_st = rel_err(st_c.cpu().double().numpy(), st_f.cpu().double().numpy())
    d_out = rel_err(to_numpy_f64(out_c), to_numpy_f64(out_f))
    print(f"{name} chunk-wise scans: worst per-head rel err out {worst['out']:.3e}, "
          f"states {worst['states']:.3e}; vs per-frame scans: states {d_st:.3e}, out {d_out:.3e}")
    assert d_st <= TOL_INTER[wl.dtype]


EDGE = [
    # name, fields (d = 128, bf16: the tensor-core path)
    ("ragged", dict(H=2, T=13, U=70, chunk=5, window_chunks=1)),
    ("chunk1", dict(H=1, T=6, U=40, chunk=1, window_chunks=1)),
    ("T_below_chunk", dict(H=2, T=3, U=50, chunk=5, window_chunks=0)),
    ("chunk3_w0", dict(H=3, T=10, U=33, chunk=3, window_chunks=0)),
    ("decay_ragged", dict(H=2, T=11, U=64, chunk=4, window_chunks=1, alpha_mean=1.5)),
    ("decay_T1", dict(H=1, T=1, U=64, chunk=5, window_chunks=0, alpha_mean=1.5)),
    ("B2", dict(B=2, H=2, T=12, U=48, chunk=4, window_chunks=1)),
]


@pytest.mark.parametrize("name,fields", EDGE, ids=[e[0] for e in EDGE])
@pytest.mark.parametrize("with_s0", [False, True])
def test_chunk_scan_edge_cases(name, fields, with_s0):
    wl = gen.custom(name, seed=23, d=128, dtype="bf16", **fields)
    x = gen.make_inputs(wl)
    t = {k: to_torch(v, "cuda") for k, v in x.items()}
    s0f = s0r = None
    S0f = S0r = None
    if with_s0:
        rng = np.random.default_rng(8)
        s0f = (0.3 * rng.standard_normal((wl.B, wl.H, wl.d, wl.d))).astype(np.float32)
        s0r = (0.3 * rng.standard_normal((wl.B, wl.H, wl.d, wl.d))).astype(np.float32)
        S0f, S0r = to_torch(s0f, "cuda"), to_torch(s0r, "cuda")
    out, states = _run(wl, t, "chunks", S0f, S0r)
    _check(wl, x, out, states, s0f, s0r)


def test_chunk_scan_six_heads_full_length_sampled():
    """Six heads of the full-size shapes (the per-rank load of an 8-way head
    split of 48 heads), where the automatic choice takes the chunk-wise
    scans: the automatic run equals the forced chunk-wise run bitwise, and
    sampled heads match the oracle."""
    api = _api()
    wl = gen.custom("six_heads", seed=29, H=6, T=60, U=1008, d=128, chunk=5, window_chunks=1, dtype="bf16")
    assert api.vda_launches_per_forward(wl.B, wl.H, wl.T, wl.U, wl.d, wl.d, wl.chunk) == 5
    x = gen.make_inputs(wl)
    t = {k: to_torch(v, "cuda") for k, v in x.items()}
    out_c, st_c = _run(wl, t, "chunks")
    out_a, st_a = _run(wl, t, "auto")
    assert torch.equal(out_a.view(torch.int16), out_c.view(torch.int16))
    assert torch.equal(st_a, st_c)
    y = to_numpy_f64(out_c)
    for h in (0, 5):
        y_ref = oracle_head(_head_x(x, 0, h), wl)
        assert rel_err(y[0, h], y_ref) <= TOL[wl.dtype]
