"""Pins of the backward oracle (oracle/backward.py): its forward agrees with
the independent C oracle, and its gradients agree with central finite
differences of that C oracle's forward."""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward as bwd
from sparse_long_sequence_lf_b200.workloads import Workload, make_inputs


def _case(**kw):
    wl = Workload("bwd", "f32", **kw)
    x = make_inputs(wl)
    return wl, x


@pytest.mark.parametrize("kw", [
    dict(B=1, H=2, n=40, window=8, dilation=(1, 2), globals_kind="list:3,31", pad_tail=(5,),
         seed=41),
    dict(B=2, H=1, n=33, window=5, causal=True, seed=42),
    # two batches with their own padding and global tokens, heads with their
    # own dilations
    dict(B=2, H=2, n=36, window=6, dilation=(1, 3), globals_kind="list:2,30;7",
         pad_tail=(0, 9), seed=49),
])
def test_forward_agrees_with_the_c_oracle(kw):
    wl, x = _case(**kw)
    f = lambda a: a.double()
    o = bwd.forward(*(f(x[k]) for k in ("q", "k", "v", "qg", "kg", "vg")), x["local_mask"],
                    x["global_mask"], window=wl.window, dilation=x["dilation"],
                    causal=wl.causal)
    ref = oracle.forward(x["q"], x["k"], x["v"], x["qg"], x["kg"], x["vg"], x["local_mask"],
                         x["global_mask"], window=wl.window, dilation=x["dilation"],
                         causal=wl.causal)
    np.testing.assert_allclose(o.numpy(), ref, atol=1e-12)


def test_gradients_agree_with_finite_differences_of_the_c_oracle():
    wl, x = _case(B=1, H=1, n=14, window=4, dilation=(2,), globals_kind="list:2,9",
                  pad_tail=(2,), seed=43)
    rng = np.random.default_rng(44)
    dout = rng.standard_normal((1, 1, 14, 64))
    names = ("q", "k", "v", "qg", "kg", "vg")
    base = {k: x[k].double().numpy().copy() for k in names}
    grads = bwd.backward(*(base[k] for k in names), x["local_mask"], x["global_mask"], dout,
                         window=wl.window, dilation=x["dilation"])

    def loss(arrs):
        o = oracle.forward(*(arrs[k] for k in names), x["local_mask"], x["global_mask"],
                           window=wl.window, dilation=x["dilation"])
        return float((o * dout).sum())

    eps = 1e-6
    for name in names:
        for (i, e) in [(0, 0), (2, 5), (9, 63), (11, 17), (13, 1)]:
            a = {k: v.copy() for k, v in base.items()}
            a[name][0, 0, i, e] += eps
            up = loss(a)
            a[name][0, 0, i, e] -= 2 * eps
            dn = loss(a)
            fd = (up - dn) / (2 * eps)
            assert abs(fd - grads[name][0, 0, i, e]) < 1e-6, (name, i, e, fd,
                                                               grads[name][0, 0, i, e])


def test_padded_rows_and_unused_projections_get_no_gradient():
    wl, x = _case(B=1, H=1, n=20, window=4, globals_kind="list:5", pad_tail=(4,), seed=45)
    dout = np.ones((1, 1, 20, 64))
    g = bwd.backward(*(x[k] for k in ("q", "k", "v", "qg", "kg", "vg")), x["local_mask"],
                     x["global_mask"], dout, window=wl.window)
    # padded rows (16..19) are neither queries nor keys
    for k in ("q", "k", "v", "qg", "kg", "vg"):
        assert np.all(g[k][0, 0, 16:] == 0)
    # Qg is used only at the global row, Q only at the others
    assert np.all(g["qg"][0, 0, [i for i in range(20) if i != 5]] == 0)
    assert np.all(g["q"][0, 0, 5] == 0)


def test_full_window_gradients_equal_sdpa_autograd():
    # With the window covering the sequence, no global token and no padding,
    # the attention is textbook full attention: its gradients are those of
    # torch's scaled_dot_product_attention (fp64, CPU autograd).
    wl, x = _case(B=1, H=2, n=24, window=64, seed=45)
    rng = np.random.default_rng(46)
    dout = rng.standard_normal((1, 2, 24, 64))
    names = ("q", "k", "v", "qg", "kg", "vg")
    arrs = {k: x[k].double().numpy() for k in names}
    got = bwd.backward(*(arrs[k] for k in names), None, None, dout, window=wl.window)
    q, k, v = (torch.from_numpy(arrs[n].copy()).requires_grad_(True) for n in ("q", "k", "v"))
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v)
    (o * torch.from_numpy(dout)).sum().backward()
    for name, t in (("q", q), ("k", k), ("v", v)):
        np.testing.assert_allclose(got[name], t.grad.numpy(), atol=1e-10)
    for name in ("qg", "kg", "vg"):                       # no global rows
        assert not np.any(got[name])


def test_all_global_gradients_equal_sdpa_autograd_on_global_projections():
    # Every token global: every row attends to all tokens through Qg, Kg, Vg.
    wl, x = _case(B=1, H=1, n=20, window=4, globals_kind="first:20", seed=47)
    rng = np.random.default_rng(48)
    dout = rng.standard_normal((1, 1, 20, 64))
    names = ("q", "k", "v", "qg", "kg", "vg")
    arrs = {k: x[k].double().numpy() for k in names}
    got = bwd.backward(*(arrs[k] for k in names), None, x["global_mask"], dout,
                       window=wl.window)
    qg, kg, vg = (torch.from_numpy(arrs[n].copy()).requires_grad_(True)
                  for n in ("qg", "kg", "vg"))
    o = torch.nn.functional.scaled_dot_product_attention(qg, kg, vg)
    (o * torch.from_numpy(dout)).sum().backward()
    for name, t in (("qg", qg), ("kg", kg), ("vg", vg)):
        np.testing.assert_allclose(got[name], t.grad.numpy(), atol=1e-10)
    for name in ("q", "k", "v"):                          # no local rows
        assert not np.any(got[name])
