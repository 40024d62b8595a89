"""Host-only checks of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments before touching the GPU."""

import ctypes
import re

import pytest

from frame_wise_delta_vda_b200 import _lib
from frame_wise_delta_vda_b200._lib import VdaArgs


@pytest.fixture(scope="module")
def L():
    return _lib.lib()


def test_library_exports_every_header_symbol(L):
    names = _lib.header_symbols()
    assert len(names) >= 13
    for n in names:
        assert hasattr(L, n), n
    # and the binding declares every one of them
    assert set(names) == set(_lib._SIGNATURES)


def test_status_strings(L):
    assert L.vda_status_string(0) == b"VDA_OK"
    assert L.vda_status_string(1) == b"VDA_ERR_INVALID_ARGUMENT"
    assert L.vda_status_string(5) == b"VDA_ERR_TIMEOUT"
    assert L.vda_status_string(99) == b"VDA_ERR_UNKNOWN"


def test_status_enum_matches_header():
    text = open(_lib.HEADER).read()
    for name in ("VDA_OK", "VDA_ERR_INVALID_ARGUMENT", "VDA_ERR_UNSUPPORTED", "VDA_ERR_WORKSPACE",
                 "VDA_ERR_CUDA", "VDA_ERR_TIMEOUT", "VDA_BF16", "VDA_F32", "VDA_SCAN_AUTO", "VDA_SCAN_FRAMES",
                 "VDA_SCAN_CHUNKS"):
        m = re.search(rf"\b{name}\s*=\s*(\d+)", text)
        assert m and int(m.group(1)) == getattr(_lib, name), name


@pytest.mark.parametrize("struct,mirror", [("vda_args", VdaArgs), ("vda_prep_args", _lib.VdaPrepArgs)])
def test_argument_structs_mirror_the_header(struct, mirror):
    """The ctypes mirrors list the C structs' fields in the header's order."""
    text = open(_lib.HEADER).read()
    body = re.search(r"typedef struct " + struct + r" \{(.*?)\} " + struct + ";", text, re.S).group(1)
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    fields = []
    for decl in body.split(";"):
        decl = decl.strip()
        if decl:
            fields += [n.strip().lstrip("*") for n in re.sub(r"^(const\s+)?\w+\s*\**", "", decl).split(",")]
    assert fields == [f[0] for f in mirror._fields_]


def test_workspace_bytes(L):
    # full-scale workload: A/M and B per frame-head plus chunk-boundary states
    n = L.vda_workspace_bytes(1, 48, 60, 1008, 128, 128, 5, 0)
    fh, dd = 48 * 60, 128 * 128 * 4
    assert n >= 2 * fh * dd + 2 * 48 * 13 * dd
    assert n % 256 == 0 or n > 0
    assert L.vda_workspace_bytes(0, 48, 60, 1008, 128, 128, 5, 0) == 0
    assert L.vda_workspace_bytes(1, 1, 1, 1, 128, 64, 5, 0) == 0      # d_k != d_v
    assert L.vda_workspace_bytes(1, 1, 1, 1, 96, 96, 5, 0) == 0       # unsupported d
    assert L.vda_workspace_bytes(1, 1, 1, 1, 16, 16, 5, 7) == 0       # bad dtype


def _args(**kw):
    a = VdaArgs()
    a.dtype = 0
    for f in ("q", "k", "v", "beta", "gate", "rms_weight", "out"):
        setattr(a, f, 0x10000)          # aligned dummy addresses, never dereferenced
    a.S0_fwd = None
    a.S0_rev = None
    a.B, a.H, a.T, a.U, a.d_k, a.d_v, a.chunk, a.window_chunks = 1, 2, 10, 16, 16, 16, 5, 1
    a.eps = 1e-6
    a.stream = None
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,status", [
    (dict(B=0), 1), (dict(T=-1), 1), (dict(U=0), 1), (dict(chunk=0), 1), (dict(window_chunks=-1), 1),
    (dict(q=None), 1), (dict(out=None), 1), (dict(beta=None), 1), (dict(rms_weight=None), 1),
    (dict(k=0x10004), 1),                  # misaligned
    (dict(S0_fwd=0x10008), 1),             # misaligned optional pointer
    (dict(dtype=3), 1),
    (dict(d_k=16, d_v=32), 2),             # d_k != d_v
    (dict(d_k=48, d_v=48), 2),             # unsupported head dim
    (dict(scan_form=3), 1), (dict(scan_form=-1), 1),
    (dict(scan_form=2, H=800000, T=1500, chunk=2), 2),   # 4 x 800000 x 750 composition CTAs
])
def test_forward_ex_rejects_bad_arguments(L, kw, status):
    a = _args(**kw)
    rc = L.vda_forward_ex(ctypes.byref(a), ctypes.c_void_p(0x100000), 1 << 30, None, None)
    assert rc == status


def test_forward_ex_rejects_small_or_misaligned_workspace(L):
    a = _args()
    need = L.vda_workspace_bytes(1, 2, 10, 16, 16, 16, 5, 0)
    assert L.vda_forward_ex(ctypes.byref(a), None, need, None, None) == 3
    assert L.vda_forward_ex(ctypes.byref(a), ctypes.c_void_p(0x100000), need - 1, None, None) == 3
    assert L.vda_forward_ex(ctypes.byref(a), ctypes.c_void_p(0x100010), need, None, None) == 3
    assert L.vda_forward_ex(None, ctypes.c_void_p(0x100000), need, None, None) == 1


def test_text_state_and_host_entry_validation(L):
    assert L.vda_text_state(0, None, None, None, 1, 1, 4, 16, 16, None, None, 0, None) == 1
    assert L.vda_text_state(0, 0x100, 0x100, 0x100, 1, 1, 4, 16, 32, 0x100, None, 0, None) == 2
    assert L.vda_text_state_workspace_bytes(1, 1, 4, 16, 16, 0) > 0
    a = _args(q=None)
    assert L.vda_forward_host(ctypes.byref(a), ctypes.c_void_p(0x100000), 1 << 30) == 1
    a = _args()
    assert L.vda_forward_host(ctypes.byref(a), ctypes.c_void_p(0x100000), 16) == 3
    assert L.vda_forward_host_bytes(1, 48, 60, 1008, 128, 128, 5, 0) > 0


def test_launch_count(L):
    assert L.vda_launches_per_forward(1, 2, 10, 16, 16, 16, 5, 1) >= 4
    assert L.vda_launches_per_forward(1, 2, 10, 16, 16, 24, 5, 1) == 0
    # tensor-core path: per-frame scans at 48 heads (4 launches), chunk-wise
    # scans (compose + chunk chains: 5 launches) at 6 heads of the same shapes;
    # without a GPU the library assumes 148 SMs
    assert L.vda_launches_per_forward(1, 48, 60, 1008, 128, 128, 5, 0) == 4
    assert L.vda_launches_per_forward(1, 6, 60, 1008, 128, 128, 5, 0) == 5
    assert L.vda_launches_per_forward(1, 6, 60, 1008, 128, 128, 1, 0) == 4   # one-frame chunks


@pytest.mark.parametrize("H,chunk,T,launches", [
    (6, 5, 60, 5),    # six heads: 288 composition CTAs, two waves
    (7, 5, 60, 4), (12, 5, 60, 4), (24, 5, 60, 4), (48, 5, 60, 4),
    (16, 5, 30, 4),   # the correlated-key shapes: 384 CTAs
    (2, 5, 30, 5),
    (6, 5, 5, 4),     # a single chunk: nothing to shorten
    (2, 1, 60, 4),    # one-frame chunks: nothing to compose
])
def test_automatic_scan_form(L, H, chunk, T, launches):
    # the chunk-wise scans (two launches) when their 4 B H NC composition CTAs
    # fit in two waves of 148 SMs, with more than one frame per chunk and more
    # than one chunk; otherwise the per-frame scans (one launch)
    nc = (T + chunk - 1) // chunk
    rule = 5 if (chunk > 1 and T > chunk and 4 * H * nc <= 2 * 148) else 4
    assert launches == rule
    assert L.vda_launches_per_forward(1, H, T, 256, 128, 128, chunk, 0) == launches


def test_d64_tensor_core_workspace(L):
    # d = 64, bf16: the tensor-core path adds the scan's operand images
    # (16 KB per frame-head) to A/M, B and the boundary states; fp32 I/O at
    # d = 64 runs the SIMT path without them
    fh, dd = 8 * 20, 64 * 64 * 4
    bf16 = L.vda_workspace_bytes(1, 8, 20, 240, 64, 64, 5, 0)
    f32 = L.vda_workspace_bytes(1, 8, 20, 240, 64, 64, 5, 1)
    assert bf16 - f32 == fh * 16384
    assert f32 >= 2 * fh * dd + 2 * 8 * 5 * dd
    assert L.vda_launches_per_forward(1, 8, 20, 240, 64, 64, 5, 0) == 4


def test_chunk_maps_fit_the_workspace(L):
    # the chunk maps (J_c fp32 + P_c image, 128 KB per direction and chunk)
    # live in A's region when 4 NC <= T, else in a region of their own
    fh_dd = 128 * 128 * 4
    base = L.vda_workspace_bytes(1, 6, 60, 1008, 128, 128, 5, 0)
    one = L.vda_workspace_bytes(1, 6, 60, 1008, 128, 128, 1, 0)
    assert one - base >= 2 * 6 * (60 - 12) * fh_dd       # more boundary states and the maps
    assert one >= 6 * 60 * fh_dd + 4 * 6 * 60 * fh_dd


def test_timing_read_without_calls(L):
    ms = (ctypes.c_float * 4)()
    calls = ctypes.c_int(-1)
    assert L.vda_timing_read(ms, 4, ctypes.byref(calls)) == 0
    assert calls.value == 0 and list(ms) == [0.0] * 4


def test_prep_argument_checks_without_a_gpu(L):
    """vda_prep validates its arguments before touching the device."""
    from frame_wise_delta_vda_b200._lib import VdaPrepArgs
    assert L.vda_prep(None) == 1
    a = VdaPrepArgs()
    for f in ("q_in", "k_in", "v_in", "wk_s", "wk_t", "wv_s", "wv_t", "q_out", "k_out", "v_out"):
        setattr(a, f, 4096)            # aligned placeholders, never dereferenced
    a.B, a.H, a.T, a.Hl, a.Wl, a.d = 1, 2, 3, 4, 5, 48
    assert L.vda_prep(ctypes.byref(a)) == 2          # d not supported
    a.d = 64
    a.k_in = 4100                                     # misaligned
    assert L.vda_prep(ctypes.byref(a)) == 1
    a.k_in = 4096
    a.T = 0
    assert L.vda_prep(ctypes.byref(a)) == 1
