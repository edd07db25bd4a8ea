"""Parity of the projection prologue (lf_qkv_projection) with the fp64 oracle
(oracle/projection.py) on the same rounded inputs, element by element."""
import numpy as np
import pytest
import torch

import oracle
from oracle.projection import projection_forward
import sparse_long_sequence_lf_b200 as lf
from sparse_long_sequence_lf_b200.workloads import Workload, make_layer_inputs

pytestmark = pytest.mark.gpu

# Outputs are unit scale; the GPU rounds each to the 16-bit type (relative
# 2^-9 for bf16, 2^-12 for fp16) after an fp32 sum over H*64 products.
TOL = {"bf16": 2e-2, "f16": 4e-3}

CASES = [
    # ragged token count, two k-slices, five column tiles, globals in both batches
    Workload("proj-b2-n300-h2", "bf16", 2, 2, 300, 16, globals_kind="random:5", seed=21),
    # odd head count: the last column tile is half outside
    Workload("proj-b1-n1000-h3-noglobal", "f16", 1, 3, 1000, 16, seed=22),
    # Longformer-base width (12 k-slices), 130 global rows: two gathered tiles
    Workload("proj-b1-n200-h12-g130", "bf16", 1, 12, 200, 16, globals_kind="random:130", seed=23),
    # globals at the front (question tokens), padded tail
    Workload("proj-b2-n513-h4-g64", "f16", 2, 4, 513, 16, globals_kind="first:64",
             pad_tail=(0, 40), seed=24),
    # the headline shape
    Workload("proj-b1-n4096-h12-g1", "bf16", 1, 12, 4096, 512, globals_kind="first:1", seed=25),
]


def _run(wl):
    x = make_layer_inputs(wl)
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
    gm = d["global_mask"]
    if gm is None:
        gm = torch.zeros((wl.B, wl.n), dtype=torch.uint8, device="cuda")
    gidx, counts = lf.global_index(gm)
    # The oracle takes its global index from the CPU oracle's compaction of
    # the host mask, never from the CUDA path; the GPU compaction must agree.
    ref_gidx, ref_counts = oracle.global_index(gm.cpu().numpy())
    assert np.array_equal(gidx.cpu().numpy(), ref_gidx)
    assert np.array_equal(counts.cpu().numpy(), ref_counts)
    mg = int(ref_counts.max())
    sentinel = torch.full((wl.B, wl.H, wl.n, 64), 3.0, dtype=x["x"].dtype, device="cuda")
    out = lf.qkv_projection(d["x"], d["w"], d["bias"], d["wqg"], d["bqg"], gidx, counts,
                            H=wl.H, max_global=mg, out={"qg": sentinel.clone()})
    torch.cuda.synchronize()
    f64 = lambda t: t.double().cpu().numpy()
    ref = projection_forward(f64(x["x"]), f64(x["w"]), f64(x["bias"]), f64(x["wqg"]),
                             f64(x["bqg"]), ref_gidx, ref_counts, H=wl.H,
                             qg_init=f64(sentinel))
    return out, ref, ref_gidx, ref_counts


@pytest.mark.parametrize("wl", CASES, ids=[w.name for w in CASES])
def test_projection_matches_oracle(wl):
    out, ref, gidx, counts = _run(wl)
    for name in ("q", "k", "v", "kg", "vg", "qg"):
        got = out[name].double().cpu().numpy()
        err = np.abs(got - ref[name])
        worst = np.unravel_index(int(np.argmax(err)), err.shape)
        assert err.max() <= TOL[wl.dtype], (name, err.max(), worst)
    # Qg rows away from the global positions are untouched (sentinel 3.0).
    got = out["qg"].float().cpu().numpy()
    for b in range(wl.B):
        glob = set(gidx[b, :counts[b]].tolist())
        others = [i for i in range(wl.n) if i not in glob]
        assert np.all(got[b][:, others] == 3.0)


def test_projection_feeds_the_attention():
    # The projection's outputs go straight into the attention forward; the
    # oracle attention runs on the same tensors.
    wl = CASES[0]
    out, ref, gidx, counts = _run(wl)
    x = make_layer_inputs(wl)
    lm = x["local_mask"]
    att = lf.attention_forward(out["q"], out["k"], out["v"], out["qg"], out["kg"], out["vg"],
                               lm.cuda() if lm is not None else None, x["global_mask"].cuda(),
                               window=wl.window, max_global=int(counts.max()))
    torch.cuda.synchronize()
    c = {k: t.cpu() for k, t in out.items()}
    want = oracle.forward(c["q"], c["k"], c["v"], c["qg"], c["kg"], c["vg"], lm,
                          x["global_mask"], window=wl.window, dilation=[1] * wl.H, causal=False)
    assert np.abs(att.double().cpu().numpy() - want).max() <= 2e-2


def test_projection_rejects_fp32_and_misalignment():
    x = torch.zeros((1, 8, 64), dtype=torch.float32, device="cuda")
    w = torch.zeros((320, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(ValueError):
        lf.qkv_projection(x, w, H=1)
    from sparse_long_sequence_lf_b200 import _lib
    import ctypes
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    buf = torch.zeros(8 * 64 * 6 + 8, dtype=torch.bfloat16, device="cuda")
    xb = torch.zeros((1, 8, 64), dtype=torch.bfloat16, device="cuda")
    wb = torch.zeros((320, 64), dtype=torch.bfloat16, device="cuda")
    o = [buf[j * 512:(j + 1) * 512] for j in range(6)]
    rc = _lib.lib().lf_qkv_projection(_lib.LF_F32, 1, 8, 1, 64, P(xb), P(wb), None, None, None,
                                      None, None, 0, *[P(t) for t in o], None, None)
    assert rc == -2
    mis = buf[1:513]
    rc = _lib.lib().lf_qkv_projection(_lib.LF_BF16, 1, 8, 1, 64, P(xb), P(wb), None, None, None,
                                      None, None, 0, P(mis), *[P(t) for t in o[1:]], None, None)
    assert rc == -1
