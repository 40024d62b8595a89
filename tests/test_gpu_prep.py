"""Parity of the feature-preparation kernels (vda_prep, through the C ABI)
with the float64 oracle: q' = L2(q), k' = L2(SiLU(conv(k))), v' = SiLU(conv(v))
in the [B, H, T, U, d] layout.  Bar: relative Frobenius error per (b, h) and
tensor <= 1e-2 (bf16 outputs)."""

import numpy as np
import pytest

import oracle as ref
from frame_wise_delta_vda_b200 import inputs as gen
from _helpers import TOL, rel_err, to_numpy_f64, to_torch

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _api():
    from frame_wise_delta_vda_b200 import api
    return api


def _run(pw, x):
    api = _api()
    t = {k: to_torch(v, "cuda") for k, v in x.items()}
    outs = api.vda_prep(t["q"], t["k"], t["v"], t["wk_s"], t["wk_t"], t["wv_s"], t["wv_t"], pw.Hl, pw.Wl)
    torch.cuda.synchronize()
    return [to_numpy_f64(o) for o in outs]


def _check(pw, x, got, heads=None):
    pairs = heads or [(b, h) for b in range(pw.B) for h in range(pw.H)]
    want = ref.prep(gen.as_f64(x["q"]), gen.as_f64(x["k"]), gen.as_f64(x["v"]), x["wk_s"], x["wk_t"],
                    x["wv_s"], x["wv_t"], pw.Hl, pw.Wl, heads=pairs)
    worst = 0.0
    for i, (b, h) in enumerate(pairs):
        for name, g, w in zip("qkv", got, want):
            e = rel_err(g[b, h], w[i])
            worst = max(worst, e)
            assert e <= TOL["bf16"], (pw.name, name, b, h, e)
    return worst


@pytest.mark.parametrize("name", ["prep_small", "prep_odd"])
def test_prep_parity_all_heads(name):
    pw = gen.PREP_WORKLOADS[name]
    x = gen.make_prep_inputs(pw)
    worst = _check(pw, x, _run(pw, x))
    print(f"{name}: worst rel err {worst:.3e}")


def test_prep_full_size_sampled_heads():
    pw = gen.PREP_WORKLOADS["prep_full"]
    x = gen.make_prep_inputs(pw)
    got = _run(pw, x)
    _check(pw, x, got, heads=[(0, 0), (0, 21), (0, 47)])


EDGE = [
    ("d16", dict(B=1, H=2, T=4, Hl=5, Wl=6, d=16)),
    ("d32_T1", dict(B=1, H=2, T=1, Hl=4, Wl=4, d=32)),
    ("row_grid", dict(B=1, H=1, T=3, Hl=1, Wl=9, d=64)),
    ("column_grid", dict(B=2, H=1, T=3, Hl=7, Wl=1, d=128)),
    ("T2_wide", dict(B=1, H=2, T=2, Hl=3, Wl=53, d=128)),
]


@pytest.mark.parametrize("name,fields", EDGE, ids=[e[0] for e in EDGE])
def test_prep_edge_cases(name, fields):
    pw = gen.PrepWorkload(name, seed=31, **fields)
    x = gen.make_prep_inputs(pw)
    _check(pw, x, _run(pw, x))


def test_prep_rejects_a_grid_row_too_wide_for_shared_memory():
    api = _api()
    pw = gen.PrepWorkload("too_wide", 1, 1, 2, 2, 80, 128, 32)
    x = gen.make_prep_inputs(pw)
    t = {k: to_torch(v, "cuda") for k, v in x.items()}
    with pytest.raises(api.VdaError) as e:
        api.vda_prep(t["q"], t["k"], t["v"], t["wk_s"], t["wk_t"], t["wv_s"], t["wv_t"], pw.Hl, pw.Wl)
    assert e.value.status == 2   # VDA_ERR_UNSUPPORTED
