"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
and compare it element by element with the fp64 oracle on the same inputs."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import sparse_long_sequence_lf_b200 as lf
from sparse_long_sequence_lf_b200.workloads import make_inputs

# Tolerances (max abs error against the fp64 oracle; unit-scale inputs).
TOL = {"f32": 1e-4, "f16": 2e-2, "bf16": 2e-2}


def to_dev(x: dict, dev="cuda") -> dict:
    return {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in x.items()}


def max_global_of(x) -> int:
    gm = x["global_mask"]
    return 0 if gm is None else int((gm != 0).sum(dim=1).max().item())


def gpu_forward(x: dict, *, max_global=None, out=None, workspace=None):
    g = to_dev(x)
    mg = max_global_of(x) if max_global is None else max_global
    res = lf.attention_forward(g["q"], g["k"], g["v"], g["qg"], g["kg"], g["vg"],
                               g["local_mask"], g["global_mask"], window=x["window"],
                               dilation=x["dilation"], causal=x["causal"], max_global=mg,
                               out=out, workspace=workspace)
    torch.cuda.synchronize()
    return res


def oracle_forward(x: dict, **kw):
    return oracle.forward(x["q"], x["k"], x["v"], x["qg"], x["kg"], x["vg"], x["local_mask"],
                          x["global_mask"], window=x["window"], dilation=x["dilation"],
                          causal=x["causal"], **kw)


def assert_close(gpu_out, ref, tol, what):
    got = gpu_out.float().cpu().numpy() if torch.is_tensor(gpu_out) else gpu_out
    assert got.shape == ref.shape, f"{what}: shape {got.shape} vs {ref.shape}"
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    worst = np.unravel_index(int(np.argmax(err)), err.shape)
    assert err.max() <= tol, (f"{what}: max abs err {err.max():.3e} > {tol:.1e} at {worst}: "
                              f"got {got[worst]:.5f} want {ref[worst]:.5f}")
    return float(err.max())


def check_workload(wl, *, max_global=None):
    x = make_inputs(wl)
    out = gpu_forward(x, max_global=max_global)
    ref = oracle_forward(x)
    return assert_close(out, ref, TOL[wl.dtype], wl.name)
