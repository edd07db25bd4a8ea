"""Parity of the output layer (lf_output_layer: heads concatenated, output
projection, bias, residual, LayerNorm) with the fp64 oracle, element by
element on the same rounded inputs."""
import numpy as np
import pytest
import torch

from oracle.projection import output_layer as oracle_output_layer
import sparse_long_sequence_lf_b200 as lf
from sparse_long_sequence_lf_b200.workloads import Workload, make_output_inputs

pytestmark = pytest.mark.gpu

# LayerNorm outputs are unit scale (times gamma ~ 1): the 16-bit rounding of
# the result dominates (relative 2^-9 bf16, 2^-12 fp16).
TOL = {"bf16": 2e-2, "f16": 4e-3}

CASES = [
    Workload("out-b2-n300-h2", "bf16", 2, 2, 300, 16, seed=31),     # ragged rows, 2 batches
    Workload("out-b1-n1000-h3", "f16", 1, 3, 1000, 16, seed=32),    # odd head count
    Workload("out-b1-n128-h16", "bf16", 1, 16, 128, 16, seed=33),   # one row tile, hidden 1024
    Workload("out-b1-n4096-h12", "bf16", 1, 12, 4096, 512, seed=34),  # Longformer-base shape
    Workload("out-b1-n70-h20", "f16", 1, 20, 70, 16, seed=35),      # rows longer than 1024
]


@pytest.mark.parametrize("wl", CASES, ids=[w.name for w in CASES])
def test_output_layer_matches_oracle(wl):
    x = make_output_inputs(wl)
    d = {k: v.cuda() for k, v in x.items()}
    out = lf.output_layer(d["attn"], d["wo"], d["bo"], d["residual"], d["gamma"], d["beta"],
                          eps=1e-5)
    torch.cuda.synchronize()
    f64 = lambda t: t.double().numpy()
    ref = oracle_output_layer(f64(x["attn"]), f64(x["wo"]), f64(x["bo"]), f64(x["residual"]),
                              f64(x["gamma"]), f64(x["beta"]), eps=1e-5)
    err = np.abs(out.double().cpu().numpy() - ref)
    worst = np.unravel_index(int(np.argmax(err)), err.shape)
    assert err.max() <= TOL[wl.dtype], (err.max(), worst)


def test_output_layer_argument_checks():
    from sparse_long_sequence_lf_b200 import _lib
    import ctypes
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    a = torch.zeros((1, 1, 8, 64), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda")
    r = torch.zeros((1, 8, 64), dtype=torch.bfloat16, device="cuda")
    v = torch.zeros((64,), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(lf.output_workspace_size(1, 8, 1), dtype=torch.uint8, device="cuda")
    L = _lib.lib()
    args = lambda **kw: dict(dict(dt=_lib.LF_BF16, eps=1e-5, wsb=ws.numel()), **kw)
    def call(**kw):
        c = args(**kw)
        return L.lf_output_layer(c["dt"], 1, 8, 1, 64, P(a), P(w), None, P(r), P(v), P(v),
                                 c["eps"], P(r), P(ws), c["wsb"], None, None)
    assert call() == 0
    torch.cuda.synchronize()
    assert call(dt=_lib.LF_F32) == -2
    assert call(eps=-1.0) == -1
    assert call(wsb=16) == -3
