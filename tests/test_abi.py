"""The C-ABI library on the host: it loads, exports every declared entry point
and rejects bad arguments before touching a GPU (CPU only)."""
import ctypes

import pytest

from sparse_long_sequence_lf_b200 import _lib, build


@pytest.fixture(scope="module")
def L():
    build.build()
    return _lib.lib()


def test_exports_every_declared_symbol(L):
    names = _lib.header_symbols()
    assert len(names) >= 10
    for name in names:
        assert hasattr(L, name), f"{name} declared in include/lf_attention.h but not exported"


def test_version_and_status_strings(L):
    assert L.lf_version() >= 10000
    for code in _lib.STATUS:
        s = L.lf_status_string(code)
        assert s and s != b"unknown status"
    assert L.lf_status_string(12345) == b"unknown status"


def test_workspace_size(L):
    a = L.lf_workspace_size(1, 12, 4096, 64, 1)
    b = L.lf_workspace_size(1, 12, 4096, 64, 64)
    assert a > 0 and b > a and a % 256 == 0
    assert L.lf_workspace_size(1, 12, 4096, 128, 1) == 0     # head size other than 64
    assert L.lf_workspace_size(0, 12, 4096, 64, 1) == 0
    assert L.lf_workspace_size(1, 12, 4096, 64, 5000) == 0   # max_global > n
    assert L.lf_workspace_size(1, 257, 16, 64, 0) == 0       # too many heads
    assert L.lf_host_staging_size(2, 1, 12, 4096, 64) >= 7 * 12 * 4096 * 64 * 2


def _run(L, **over):
    # Fake, 256-byte aligned addresses: every call below fails a host-side
    # check or finds no device before anything is dereferenced.
    a = dict(dtype=2, B=1, H=2, n=64, d=64, q=256, k=256, v=256, qg=256, kg=256, vg=256,
             max_global=0, window=8, dil=None, causal=0, out=512, ws=256, wsb=1 << 20)
    a.update(over)
    P = ctypes.c_void_p
    return L.lf_attention_run(a["dtype"], a["B"], a["H"], a["n"], a["d"], P(a["q"]), P(a["k"]),
                              P(a["v"]), P(a["qg"]), P(a["kg"]), P(a["vg"]), a["max_global"],
                              a["window"], a["dil"], a["causal"], P(a["out"]), P(a["ws"]),
                              a["wsb"], None)


def test_argument_checks_before_any_launch(L):
    assert _run(L, d=128) == -2
    assert _run(L, dtype=7) == -1
    assert _run(L, window=3) == -1
    assert _run(L, window=0) == -1
    assert _run(L, causal=1, window=0) == -1
    assert _run(L, causal=1, max_global=2) == -2
    assert _run(L, q=0) == -1
    assert _run(L, q=264) == -1                       # not 16-byte aligned
    assert _run(L, out=520) == -1
    assert _run(L, n=0) == -1
    assert _run(L, ws=0) == -3
    assert _run(L, ws=255) == -3                      # misaligned workspace
    assert _run(L, wsb=16) == -3                      # too small
    dil = (ctypes.c_int32 * 2)(1, 0)
    assert _run(L, dil=dil) == -1


def test_valid_call_without_gpu_reports_no_device(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _run(L) == -7
    assert L.lf_global_index(ctypes.c_void_p(1), 1, 8, ctypes.c_void_p(1), ctypes.c_void_p(1),
                             None) == -7


def test_backward_argument_checks(L):
    import torch
    P = ctypes.c_void_p

    def bwd(**over):
        a = dict(dtype=2, B=1, H=2, n=64, d=64, t=256, out=512, dout=512, g=768,
                 max_global=0, window=8, causal=0, ws=256, wsb=1 << 20, sc=256, scb=1 << 20)
        a.update(over)
        t = P(a["t"])
        return L.lf_attention_backward(
            a["dtype"], a["B"], a["H"], a["n"], a["d"], t, t, t, t, t, t, P(a["out"]),
            P(a["dout"]), a["max_global"], a["window"], None, a["causal"], P(a["g"]), P(a["g"]),
            P(a["g"]), P(a["g"]), P(a["g"]), P(a["g"]), P(a["ws"]), a["wsb"], P(a["sc"]),
            a["scb"], None)

    assert L.lf_backward_scratch_size(1, 2, 64, 64, 0) >= 2 * 4 * 2 * 64
    assert L.lf_backward_scratch_size(1, 2, 64, 32, 0) == 0
    assert bwd(d=32) == -2
    assert bwd(window=3) == -1
    assert bwd(dout=0) == -1
    assert bwd(g=520) == -1                             # misaligned gradient
    assert bwd(ws=0) == -3
    assert bwd(sc=0) == -3
    assert bwd(sc=264) == -3                            # misaligned scratch
    assert bwd(scb=8) == -3                             # scratch too small
    if not torch.cuda.is_available():
        assert bwd() == -7
