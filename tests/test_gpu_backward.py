"""Parity of the attention backward (CUDA, through the C ABI) with the fp64
oracle of oracle/backward.py: all six gradients, element by element.

Tolerance: |got - want| <= atol + rtol * |want| per element, with
atol = rtol = 1e-4 for fp32 and 2e-2 for fp16 / bf16.  The inputs are exact
in both; the kernels sum in fp32 and round each gradient once to the dtype
(2^-9 relative for bf16), and D_i = <dO_i, O_i> is formed from the forward
output as the library returned it (rounded to the dtype), whose error enters
every dS of the row; the relative term covers the keys of global tokens,
whose gradients sum over every row of the head.
"""
import numpy as np
import pytest
import torch

import sparse_long_sequence_lf_b200 as lf
from gpu_helpers import max_global_of, to_dev
from oracle import backward as obw
from sparse_long_sequence_lf_b200.workloads import Workload, make_inputs, make_output_grad

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "f16": 2e-2, "bf16": 2e-2}
NAMES = ("q", "k", "v", "qg", "kg", "vg")

CASES = [
    Workload("n1", "bf16", 1, 1, 1, 2),
    Workload("n130-ragged", "bf16", 1, 2, 130, 16, seed=1),
    Workload("band-only", "bf16", 1, 2, 300, 32, seed=2),
    Workload("padded-global", "bf16", 2, 2, 500, 32, globals_kind="list:3,480;7,499",
             pad_tail=(30, 1), seed=3),
    Workload("dilated-globals", "f16", 1, 4, 900, 40, dilation=(1, 2, 3, 5),
             globals_kind="random:20", pad_tail=(77,), seed=4),
    Workload("all-global", "bf16", 1, 1, 96, 8, globals_kind="first:96", seed=5),
    Workload("global-last", "bf16", 1, 2, 600, 64, globals_kind="list:599", seed=6),
    Workload("all-padded-batch", "bf16", 2, 1, 300, 16, globals_kind="first:2",
             pad_tail=(300, 0), seed=7),
    Workload("causal-w1", "bf16", 1, 1, 200, 1, causal=True, seed=8),
    Workload("causal-w7-dil2", "f16", 1, 2, 333, 7, dilation=(2, 1), causal=True, seed=9),
    Workload("fp32-mixed", "f32", 2, 3, 600, 50, dilation=(1, 2, 4), globals_kind="random:9",
             pad_tail=(0, 41), seed=10),
    Workload("fp32-causal", "f32", 1, 2, 513, 33, dilation=(1, 3), causal=True, seed=11),
    Workload("g40-n1500", "bf16", 1, 2, 1500, 64, globals_kind="random:40", pad_tail=(5,),
             seed=12),
    # 7 + 8 + 9 + 10 residue classes exceed the tensor-core path's 24 tensor
    # maps: the whole call takes the CUDA-core kernels
    Workload("residue-budget", "bf16", 1, 4, 300, 8, dilation=(7, 8, 9, 10),
             globals_kind="random:3", seed=14),
    # At most 8 global tokens: the streamed global-column sums (8 exactly,
    # dilations, padding; and the fp32 path with 3)
    Workload("g8-dilated", "f16", 1, 3, 777, 40, dilation=(1, 2, 3), globals_kind="random:8",
             pad_tail=(33,), seed=21),
    Workload("fp32-g3", "f32", 1, 2, 400, 24, dilation=(1, 2), globals_kind="random:3",
             seed=22),
]


def run_case(wl, *, extra_global=0):
    x = make_inputs(wl)
    dout = make_output_grad(wl)
    g = to_dev(x)
    mg = max_global_of(x) + extra_global
    ws = lf.new_workspace(wl.B, wl.H, wl.n, mg, "cuda")
    kw = dict(window=wl.window, dilation=x["dilation"], causal=wl.causal, max_global=mg)
    out = lf.attention_forward(g["q"], g["k"], g["v"], g["qg"], g["kg"], g["vg"],
                               g["local_mask"], g["global_mask"], workspace=ws, **kw)
    grads = lf.attention_backward(g["q"], g["k"], g["v"], g["qg"], g["kg"], g["vg"], out,
                                  dout.cuda(), workspace=ws, **kw)
    torch.cuda.synchronize()
    assert lf.workspace_status(ws) == 0
    ref = obw.backward(x["q"], x["k"], x["v"], x["qg"], x["kg"], x["vg"], x["local_mask"],
                       x["global_mask"], dout, window=wl.window, dilation=x["dilation"],
                       causal=wl.causal)
    tol = TOL[wl.dtype]
    for nm in NAMES:
        got = grads[nm].float().cpu().numpy().astype(np.float64)
        want = ref[nm]
        assert np.all(np.isfinite(got)), f"{wl.name} d{nm}: non-finite"
        err = np.abs(got - want) - tol * np.abs(want)
        worst = np.unravel_index(int(np.argmax(err)), err.shape)
        assert err.max() <= tol, (f"{wl.name} d{nm}: err {abs(got[worst] - want[worst]):.3e} at "
                                  f"{worst}: got {got[worst]:.5f} want {want[worst]:.5f}")
    return grads, ref


@pytest.mark.parametrize("wl", CASES, ids=[w.name for w in CASES])
def test_backward_all_gradients(wl):
    run_case(wl)


def test_backward_spare_global_slots():
    # max_global above the actual count: the spare slots contribute nothing.
    run_case(Workload("spare-slots", "bf16", 1, 2, 400, 32, globals_kind="random:5", seed=13),
             extra_global=7)


def test_backward_zero_rows_are_zero():
    wl = Workload("zeros", "bf16", 2, 2, 500, 32, globals_kind="list:3,480;7,499",
                  pad_tail=(30, 1), seed=3)
    grads, _ = run_case(wl)
    gm = make_inputs(wl)["global_mask"].bool()
    lm = torch.ones((2, 500), dtype=torch.bool)
    lm[0, 470:] = False
    lm[1, 499:] = False
    for b in range(2):
        pad = ~lm[b]
        nonglobal = ~gm[b].bool()
        for nm in NAMES:
            assert torch.count_nonzero(grads[nm][b][:, pad.cuda()]) == 0, nm
        assert torch.count_nonzero(grads["qg"][b][:, nonglobal.cuda()]) == 0
        assert torch.count_nonzero(grads["q"][b][:, (gm[b] & lm[b]).cuda()]) == 0


def test_backward_rejects_bad_scratch():
    wl = Workload("bad", "bf16", 1, 1, 64, 8)
    x = to_dev(make_inputs(wl))
    ws = lf.new_workspace(1, 1, 64, 0, "cuda")
    out = lf.attention_forward(x["q"], x["k"], x["v"], x["qg"], x["kg"], x["vg"], window=8,
                               max_global=0, workspace=ws)
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(lf.LfError):
        lf.attention_backward(x["q"], x["k"], x["v"], x["qg"], x["kg"], x["vg"], out, out,
                              window=8, max_global=0, workspace=ws, scratch=small)


@pytest.mark.parametrize("use_lse", [False, True], ids=["recomputed-lse", "forward-lse"])
@pytest.mark.parametrize("name", ["bf16-b1h12-n4096-w512-g1", "fp16-b2h16-n4096-w512-g64-pad300"])
def test_backward_full_size_sampled_heads(name, use_lse):
    # The benchmark's workloads at full size through the same calls (with the
    # forward's log-sum-exp, as the benchmark times it, and without); heads
    # are independent, so the oracle checks heads 0 and H-1 of every batch
    # element by element (a few seconds of fp64 each).
    from sparse_long_sequence_lf_b200.workloads import WORKLOADS
    wl = WORKLOADS[name]
    x = make_inputs(wl)
    dout = make_output_grad(wl)
    g = to_dev(x)
    mg = max_global_of(x)
    ws = lf.new_workspace(wl.B, wl.H, wl.n, mg, "cuda")
    kw = dict(window=wl.window, dilation=x["dilation"], causal=wl.causal, max_global=mg)
    lse = (torch.empty((wl.B, wl.H, wl.n), dtype=torch.float32, device="cuda") if use_lse
           else None)
    out = lf.attention_forward(g["q"], g["k"], g["v"], g["qg"], g["kg"], g["vg"],
                               g["local_mask"], g["global_mask"], workspace=ws, lse=lse, **kw)
    grads = lf.attention_backward(g["q"], g["k"], g["v"], g["qg"], g["kg"], g["vg"], out,
                                  dout.cuda(), workspace=ws, lse=lse, **kw)
    torch.cuda.synchronize()
    assert lf.workspace_status(ws) == 0
    tol = TOL[wl.dtype]
    for h in (0, wl.H - 1):
        sl = lambda t: t[:, h:h + 1].contiguous()
        ref = obw.backward(*(sl(x[k]) for k in NAMES), x["local_mask"], x["global_mask"],
                           sl(dout), window=wl.window, dilation=[x["dilation"][h]],
                           causal=wl.causal)
        for nm in NAMES:
            got = grads[nm][:, h:h + 1].float().cpu().numpy().astype(np.float64)
            want = ref[nm]
            assert np.all(np.isfinite(got)), f"{name} head {h} d{nm}: non-finite"
            excess = np.abs(got - want) - tol * np.abs(want)
            worst = np.unravel_index(int(np.argmax(excess)), excess.shape)
            assert excess.max() <= tol, (f"{name} head {h} d{nm}: err "
                                         f"{abs(got[worst] - want[worst]):.3e} at {worst}")


# ------------------------------------------------- log-sum-exp from the forward
LSE_CASES = [c for c in CASES if c.dtype != "f32" and c.name != "n1"] + [
    Workload("lse-dil-causal", "bf16", 1, 3, 700, 48, dilation=(1, 2, 3), causal=True, seed=15),
]


def _lse_want(x, wl):
    """log2 of each valid row's softmax denominator, from the oracle's key
    sets (fp64): log2 sum_j exp(<q_i, k_j> / 8) for a non-global row and
    log2 sum_j exp(<qg_i, kg_j> / 8) for a global row."""
    local, glob = obw.key_masks(x["local_mask"], x["global_mask"], B=wl.B, H=wl.H, n=wl.n,
                                window=wl.window, dilation=x["dilation"], causal=wl.causal)
    out, rows = [], []
    for qn, kn, mk in (("q", "k", local), ("qg", "kg", glob)):
        s = torch.einsum("bhid,bhjd->bhij", x[qn].double(), x[kn].double()) / 8.0
        m = torch.from_numpy(mk)
        out.append((torch.logsumexp(s.masked_fill(~m, float("-inf")), dim=-1)
                    / np.log(2.0)).numpy())
        rows.append(m.any(dim=-1).numpy())
    return out, rows


@pytest.mark.parametrize("wl", LSE_CASES, ids=[w.name for w in LSE_CASES])
def test_backward_with_forward_lse(wl):
    # The forward writes each valid row's log-sum-exp (log2 units); the
    # backward given it skips its first passes.  Both against fp64.
    x = make_inputs(wl)
    dout = make_output_grad(wl)
    g = to_dev(x)
    mg = max_global_of(x)
    ws = lf.new_workspace(wl.B, wl.H, wl.n, mg, "cuda")
    kw = dict(window=wl.window, dilation=x["dilation"], causal=wl.causal, max_global=mg)
    lse = torch.full((wl.B, wl.H, wl.n), float("nan"), dtype=torch.float32, device="cuda")
    out = lf.attention_forward(g["q"], g["k"], g["v"], g["qg"], g["kg"], g["vg"],
                               g["local_mask"], g["global_mask"], workspace=ws, lse=lse, **kw)
    grads = lf.attention_backward(g["q"], g["k"], g["v"], g["qg"], g["kg"], g["vg"], out,
                                  dout.cuda(), workspace=ws, lse=lse, **kw)
    torch.cuda.synchronize()
    assert lf.workspace_status(ws) == 0
    (want_b, want_g), (rows_b, rows_g) = _lse_want(x, wl)
    got = lse.cpu().numpy().astype(np.float64)
    isg = (np.zeros((wl.B, wl.n), bool) if x["global_mask"] is None
           else x["global_mask"].numpy().astype(bool))
    band = rows_b & ~isg[:, None, :]
    glob = rows_g & isg[:, None, :]
    # The forward's sums use its 2^x (relative error below 7.5e-5).
    assert np.all(np.abs(got[band] - want_b[band]) <= 1e-3), wl.name
    assert np.all(np.abs(got[glob] - want_g[glob]) <= 1e-3), wl.name + " (global rows)"
    ref = obw.backward(x["q"], x["k"], x["v"], x["qg"], x["kg"], x["vg"], x["local_mask"],
                       x["global_mask"], dout, window=wl.window, dilation=x["dilation"],
                       causal=wl.causal)
    tol = TOL[wl.dtype]
    for nm in NAMES:
        got_g = grads[nm].float().cpu().numpy().astype(np.float64)
        err = np.abs(got_g - ref[nm]) - tol * np.abs(ref[nm])
        assert err.max() <= tol, f"{wl.name} d{nm}: {err.max():.3e}"


def test_lse_entry_points_refuse_fp32_and_null():
    from sparse_long_sequence_lf_b200 import _lib
    L = _lib.lib()
    rc = L.lf_attention_forward_lse(_lib.LF_F32, 1, 1, 64, 64, *([None] * 8), 0, 8, None, 0,
                                    None, None, None, 0, None)
    assert rc in (-1, -2)
    rc = L.lf_attention_backward_lse(_lib.LF_BF16, 1, 1, 64, 64, *([None] * 9), 0, 8, None, 0,
                                     *([None] * 6), None, 0, None, 0, None)
    assert rc == -1
