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


def test_ffn_and_encoder_argument_checks(L):
    import torch
    P = ctypes.c_void_p
    assert L.lf_ffn_workspace_size(1, 64, 128, 512) >= 64 * 512 * 2 + 64 * 128 * 4
    assert L.lf_ffn_workspace_size(1, 64, 100, 512) == 0        # hidden not a multiple of 64
    assert L.lf_ffn_workspace_size(1, 64, 128, 0) == 0

    def ffn(**over):
        a = dict(dtype=2, B=1, n=64, hid=128, inter=256, h=256, w=512, out=768, eps=1e-5,
                 ws=1024, wsb=1 << 20)
        a.update(over)
        return L.lf_ffn_block(a["dtype"], a["B"], a["n"], a["hid"], a["inter"], P(a["h"]),
                              P(a["w"]), None, P(a["w"]), None, P(a["w"]), P(a["w"]),
                              ctypes.c_float(a["eps"]), P(a["out"]), P(a["ws"]), a["wsb"],
                              None, None)

    assert ffn(dtype=0) == -2                                    # fp32: unsupported
    assert ffn(dtype=9) == -1
    assert ffn(hid=96) == -2                                     # not a multiple of 64
    assert ffn(h=0) == -1
    assert ffn(out=520) == -1                                    # misaligned
    assert ffn(eps=-1.0) == -1
    assert ffn(ws=0) == -3
    assert ffn(wsb=16) == -3
    if not torch.cuda.is_available():
        assert ffn() == -7

    from sparse_long_sequence_lf_b200._lib import LAYER_FIELDS, LayerWeights
    assert L.lf_encoder_workspace_size(1, 64, 2, 64, 256, 0) > 0
    assert L.lf_encoder_workspace_size(1, 64, 2, 32, 256, 0) == 0   # head size other than 64
    assert L.lf_encoder_workspace_size(1, 64, 2, 64, 100, 0) == 0   # inter not a multiple of 64

    def enc(layers=2, windows=(8, 16), **over):
        a = dict(dtype=2, B=1, n=64, H=2, d=64, inter=256, x=256, out=512, mg=0, eps=1e-5,
                 ws=1024, wsb=1 << 24, skip=None, misalign=None)
        a.update(over)
        arr = (LayerWeights * layers)()
        for i in range(layers):
            for f in LAYER_FIELDS:
                setattr(arr[i], f, 4096)
        if a["skip"]:
            setattr(arr[layers - 1], a["skip"], None)
        if a["misalign"]:
            setattr(arr[layers - 1], a["misalign"], 4104)
        win = (ctypes.c_int32 * layers)(*windows)
        return L.lf_encoder_forward(a["dtype"], a["B"], a["n"], a["H"], a["d"], a["inter"], layers,
                                    arr, win, None, P(a["x"]), None, None, a["mg"],
                                    ctypes.c_float(a["eps"]), P(a["out"]), P(a["ws"]), a["wsb"],
                                    None)

    assert enc(d=32) == -2
    assert enc(dtype=0) == -2
    assert enc(inter=100) == -2
    assert enc(layers=2, windows=(8, 7)) == -1                   # odd window in the last layer
    assert enc(skip="w_2") == -1                                 # missing weight
    assert enc(misalign="b_1") == -1                             # misaligned bias
    assert enc(mg=2, skip="w_qg") == -1                          # global queries need w_qg
    assert enc(ws=0) == -3
    assert enc(wsb=16) == -3
    if not torch.cuda.is_available():
        assert enc() == -7


def test_host_copy_bytes_counts_only_what_the_kernels_read():
    # Q, K, V always; Qg, Kg, Vg only when the global mask has a global token.
    import torch
    from sparse_long_sequence_lf_b200 import host_copy_bytes
    B, H, n = 2, 3, 500
    tb = B * H * n * 64 * 2
    assert host_copy_bytes(torch.bfloat16, B, H, n) == 3 * tb
    lm = torch.ones(B, n, dtype=torch.uint8)
    gm = torch.zeros(B, n, dtype=torch.uint8)
    assert host_copy_bytes(torch.bfloat16, B, H, n, lm, gm) == 3 * tb + 2 * B * n
    gm[1, 499] = 1
    assert host_copy_bytes(torch.bfloat16, B, H, n, lm, gm) == 6 * tb + 2 * B * n
    assert host_copy_bytes(torch.float32, B, H, n, None, gm) == 12 * tb + B * n
