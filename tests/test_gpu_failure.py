"""Failure detection of the tensor-core forward and the exponential it uses.

The bounded-wait test plants a stall on the host side of the kernel (CTA 0
never loads, and never signals, the query tile of its first item), makes the
wait limit short, and checks that the call returns, that the device status
word says LF_ERR_DEVICE_TIMEOUT, and that the next normal call on the same
stream and workspace is correct.  Nothing faults, traps or spins forever: the
kernel gives up after the limit, drains its own copies and products, frees
its tensor memory and returns.
"""
import numpy as np
import pytest
import torch

import sparse_long_sequence_lf_b200 as lf
from sparse_long_sequence_lf_b200 import _lib
from sparse_long_sequence_lf_b200.workloads import Workload, make_inputs
from gpu_helpers import TOL, assert_close, oracle_forward, to_dev

pytestmark = pytest.mark.gpu

DEFAULT_WAIT_NS = 1_000_000_000


def _forward(g, wl, ws, mg):
    return lf.attention_forward(g["q"], g["k"], g["v"], g["qg"], g["kg"], g["vg"],
                                g["local_mask"], g["global_mask"], window=wl.window,
                                dilation=g["dilation"], max_global=mg, workspace=ws)


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_bounded_wait_runs_out_and_reports_timeout(dtype):
    wl = Workload("stall-" + dtype, dtype, 1, 3, 3000, 256, globals_kind="first:2", seed=31)
    x = make_inputs(wl)
    g = to_dev(x)
    ws = lf.new_workspace(wl.B, wl.H, wl.n, 2)
    lib = _lib.lib()
    try:
        assert lib.lf_test_forward_hooks(2_000_000, 1) == 0      # 2 ms, planted stall
        _forward(g, wl, ws, 2)
        assert lf.workspace_status(ws) == -5                      # LF_ERR_DEVICE_TIMEOUT
    finally:
        assert lib.lf_test_forward_hooks(DEFAULT_WAIT_NS, 0) == 0
    # The context is usable and the same stream and workspace give the right
    # answer again (the forward prepares the workspace anew).
    out = _forward(g, wl, ws, 2)
    assert lf.workspace_status(ws) == 0
    assert_close(out, oracle_forward(x), TOL[dtype], "after timeout")


def test_wait_limit_zero_is_refused():
    assert _lib.lib().lf_test_forward_hooks(0, 0) == -1


def test_exp2_polynomial_relative_error():
    # The cubic 2^x of the kernel against 2^x in double precision over
    # [-125, 8] (the kernel's arguments are at most 8): relative error below
    # 7.5e-5, its stated bound, on a fine grid, at the integers and at the
    # half-integers (the ends of the fitted interval).  Below -125 the result
    # only has to be tiny and not negative: at most 2^-124.
    x = torch.cat([torch.linspace(-125.0, 8.0, 1_000_001, dtype=torch.float64),
                   torch.arange(-125, 9, dtype=torch.float64),
                   torch.arange(-125, 8, dtype=torch.float64) + 0.5]).float().cuda()
    y = torch.empty_like(x)
    assert _lib.lib().lf_exp2_poly_eval(_lib_ptr(x), _lib_ptr(y), x.numel(), None) == 0
    torch.cuda.synchronize()
    want = torch.exp2(x.double())
    rel = ((y.double() - want).abs() / want).max().item()
    assert rel < 7.5e-5, rel
    low = torch.tensor([-125.3, -125.9, -126.0, -126.4, -127.0, -200.0, -1e30, float("-inf")],
                       device="cuda")
    ylow = torch.empty_like(low)
    assert _lib.lib().lf_exp2_poly_eval(_lib_ptr(low), _lib_ptr(ylow), low.numel(), None) == 0
    torch.cuda.synchronize()
    assert torch.all(ylow >= 0) and torch.all(ylow <= 2.0 ** -124)
    # An odd count: the last element is computed alone.
    z = torch.tensor([0.25, -3.75, 1.0], device="cuda")
    yz = torch.empty_like(z)
    assert _lib.lib().lf_exp2_poly_eval(_lib_ptr(z), _lib_ptr(yz), 3, None) == 0
    torch.cuda.synchronize()
    np.testing.assert_allclose(yz.cpu().numpy(), np.exp2(z.cpu().numpy()), rtol=7.5e-5)


def _lib_ptr(t):
    import ctypes
    return ctypes.c_void_p(t.data_ptr())
