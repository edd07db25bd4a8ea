"""Parity of the CUDA path (through the C ABI) with the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import sparse_long_sequence_lf_b200 as lf
from gpu_helpers import TOL, assert_close, check_workload, gpu_forward, max_global_of, \
    oracle_forward, to_dev
from sparse_long_sequence_lf_b200.workloads import WORKLOADS, Workload, make_inputs, \
    random_workload

pytestmark = pytest.mark.gpu


# --------------------------------------------------------------- compaction
@pytest.mark.parametrize("B,n,dens", [(1, 1, 1.0), (3, 31, 0.3), (2, 1000, 0.02),
                                      (2, 1025, 0.0), (1, 4096, 1.0), (4, 16384, 0.002),
                                      (2, 3333, 0.5)])
def test_global_index_bit_exact(B, n, dens):
    rng = np.random.default_rng(B * 100000 + n)
    gm = (rng.random((B, n)) < dens).astype(np.uint8)
    gm[gm > 0] = rng.integers(1, 256, size=int(gm.sum()), dtype=np.uint8)
    gidx, counts = lf.global_index(torch.from_numpy(gm).cuda())
    torch.cuda.synchronize()
    ref_idx, ref_counts = oracle.global_index(gm)
    assert np.array_equal(counts.cpu().numpy(), ref_counts)
    assert np.array_equal(gidx.cpu().numpy(), ref_idx)


# ------------------------------------------------------- small exact cases
EDGE = [
    Workload("n1", "bf16", 1, 1, 1, 2),
    Workload("n5-w4", "bf16", 1, 2, 5, 4),
    Workload("n130-ragged", "bf16", 1, 2, 130, 16),
    Workload("n300-full-window", "bf16", 1, 1, 300, 1024),
    Workload("n257-w512-g1", "bf16", 1, 3, 257, 512, globals_kind="first:1"),
    Workload("dil3-n10", "bf16", 1, 1, 10, 4, dilation=(3,)),
    Workload("dil-gt-n", "bf16", 1, 2, 5, 2, dilation=(7, 1)),
    Workload("causal-w1", "bf16", 1, 1, 200, 1, causal=True),
    Workload("causal-w7-dil2", "bf16", 1, 2, 333, 7, dilation=(2, 1), causal=True),
    Workload("causal-w300-dil3", "bf16", 1, 1, 1000, 300, dilation=(3,), causal=True),
    Workload("global-last", "bf16", 1, 2, 600, 64, globals_kind="list:599"),
    Workload("g150-two-tiles", "bf16", 1, 2, 700, 32, globals_kind="random:150", seed=5),
    Workload("g300-three-tiles", "f16", 1, 1, 1300, 16, globals_kind="random:300", seed=6),
    Workload("all-global", "bf16", 1, 1, 96, 8, globals_kind="first:96"),
    Workload("padded-global", "bf16", 2, 2, 500, 32, globals_kind="list:3,480;7,499",
             pad_tail=(30, 1)),
    Workload("all-padded-batch", "bf16", 2, 1, 300, 16, globals_kind="first:2",
             pad_tail=(300, 0)),
    Workload("dilated-globals", "f16", 1, 4, 900, 40, dilation=(1, 2, 3, 5),
             globals_kind="random:20", pad_tail=(77,), seed=9),
    # (dilation, residue) classes 7 + 8 + 9 + 10 = 34: the last head does not
    # fit the residue tensor maps and loads its rows one by one
    Workload("residue-budget", "bf16", 2, 4, 1200, 48, dilation=(7, 8, 9, 10),
             globals_kind="random:11", pad_tail=(0, 90), seed=15),
    Workload("residue-budget-causal", "f16", 1, 3, 1500, 100, dilation=(11, 12, 13),
             causal=True, seed=16),
    Workload("fp32-mixed", "f32", 2, 3, 600, 50, dilation=(1, 2, 4), globals_kind="random:9",
             pad_tail=(0, 41), seed=10),
    Workload("fp32-causal", "f32", 1, 2, 513, 33, dilation=(1, 3), causal=True, seed=11),
    Workload("fp16-w2", "f16", 1, 2, 257, 2, globals_kind="first:3", seed=12),
    # Global tokens in the free columns of the last window tile: from column 32
    # (window 80: the last tile holds 16 keys), 60 tokens over two chunks,
    # with dilations and padding; the edge items keep tiles of their own.
    Workload("globals-share-last-tile", "bf16", 1, 3, 1000, 80, dilation=(1, 2, 3),
             globals_kind="random:60", pad_tail=(50,), seed=17),
    # global rows merged by the last chunk (8 chunks of 512 keys) ...
    Workload("merge-8-chunks", "bf16", 1, 2, 4096, 16, globals_kind="random:40",
             pad_tail=(5,), seed=13),
    # ... and by the separate merge kernel (9 chunks)
    Workload("merge-9-chunks", "f16", 1, 2, 4097, 16, globals_kind="random:40",
             pad_tail=(5,), seed=14),
    # More band items than a full grid holds at once (296 item slots on a
    # B200), so slots take second items from the counter: dilations, global
    # tokens and padding ...
    Workload("items-beyond-grid", "bf16", 1, 8, 6000, 512, dilation=(1, 1, 1, 1, 2, 2, 3, 3),
             globals_kind="random:3", pad_tail=(40,), seed=15),
    # ... and 384 items of a single key tile each over three batches.
    Workload("single-tile-items", "f16", 3, 64, 192, 8, dilation=(2,) * 64, seed=16),
]


@pytest.mark.parametrize("wl", EDGE, ids=[w.name for w in EDGE])
def test_edge_cases_all_elements(wl):
    check_workload(wl)


def test_padding_in_the_middle():
    wl = Workload("mid-pad", "bf16", 1, 2, 800, 64, dilation=(1, 2), globals_kind="list:10,400")
    x = make_inputs(wl)
    lm = torch.ones((1, 800), dtype=torch.uint8)
    lm[0, 100:180] = 0
    lm[0, 401:407] = 0
    lm[0, 10] = 0                         # a global position that is padding
    x["local_mask"] = lm
    out = gpu_forward(x)
    ref = oracle_forward(x)
    assert_close(out, ref, TOL["bf16"], "mid-pad")
    assert torch.all(out[0, :, 100:180] == 0)


@pytest.mark.parametrize("seed", range(16))
def test_random_sweep(seed):
    rng = np.random.default_rng(4242 + seed)
    dtype = ["bf16", "f16", "f32"][seed % 3]
    wl = random_workload(rng, dtype=dtype, max_n=1100, name=f"random{seed}")
    check_workload(wl)


# ------------------------------------------------------- full-size workloads
def _sample_rows(wl, x):
    """Row blocks checked against the oracle: both ends, the middle, and every
    global row."""
    n = wl.n
    blocks = [(0, min(n, 256)), (max(0, n // 2 - 128), min(n, n // 2 + 128)),
              (max(0, n - 256), n)]
    if x["global_mask"] is not None:
        pos = sorted(set(np.flatnonzero(x["global_mask"].numpy().any(axis=0)).tolist()))
        blocks += [(p, p + 1) for p in pos]
    return blocks


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_full_size_workload(name):
    wl = WORKLOADS[name]
    x = make_inputs(wl)
    out = gpu_forward(x).float().cpu().numpy()
    # Heads 0, H/2, H-1 and the first head of every distinct dilation.
    dil = list(x["dilation"])
    heads = sorted({0, wl.H // 2, wl.H - 1} | {dil.index(d) for d in set(dil)})
    tol = TOL[wl.dtype]
    for h in heads:
        xs = dict(x)
        for key in ("q", "k", "v", "qg", "kg", "vg"):
            xs[key] = x[key][:, h:h + 1].contiguous()
        xs["dilation"] = [x["dilation"][h]]
        for (r0, r1) in _sample_rows(wl, x):
            ref = oracle_forward(xs, row_range=(r0, r1))
            assert_close(out[:, h:h + 1, r0:r1], ref[:, :, r0:r1], tol,
                         f"{name} head {h} rows {r0}:{r1}")
    # Properties at every row: finite, padded rows zero, convex combination.
    assert np.all(np.isfinite(out))
    if x["local_mask"] is not None:
        pad = x["local_mask"].numpy() == 0
        for b in range(wl.B):
            assert np.all(out[b][:, pad[b]] == 0.0)
    bound = max(float(x["v"].float().abs().max()), float(x["vg"].float().abs().max()))
    assert np.abs(out).max() <= bound * (1 + 1e-2)


# --------------------------------------------------------------- API paths
def test_prepare_once_run_twice():
    wl = WORKLOADS["fp16-b2h16-n4096-w512-g64-pad300"].with_(H=2)
    x1, x2 = make_inputs(wl), make_inputs(wl, seed=99)
    g1, g2 = to_dev(x1), to_dev(x2)
    B, H, n = wl.B, wl.H, wl.n
    ws = lf.new_workspace(B, H, n, 64)
    lf.attention_prepare(g1["local_mask"], g1["global_mask"], B=B, H=H, n=n, max_global=64,
                         workspace=ws)
    outs = []
    for g in (g1, g2):
        outs.append(lf.attention_run(g["q"], g["k"], g["v"], g["qg"], g["kg"], g["vg"],
                                     window=wl.window, dilation=g["dilation"], max_global=64,
                                     workspace=ws))
    torch.cuda.synchronize()
    assert lf.workspace_status(ws) == 0
    for x, o in zip((x1, x2), outs):
        assert_close(o, oracle_forward(x), TOL["f16"], "prepare/run")


def test_repeat_calls_are_identical():
    wl = Workload("repeat", "bf16", 1, 3, 2000, 128, globals_kind="random:40", seed=3)
    x = make_inputs(wl)
    a = gpu_forward(x)
    b = gpu_forward(x)
    assert torch.equal(a, b)


def test_every_row_written_and_no_overrun():
    wl = Workload("guard", "bf16", 2, 3, 1111, 64, dilation=(1, 2, 3),
                  globals_kind="random:13", pad_tail=(0, 100), seed=21)
    x = make_inputs(wl)
    numel = wl.B * wl.H * wl.n * 64
    guard = 4096
    buf = torch.full((numel + 2 * guard,), float("nan"), dtype=torch.bfloat16, device="cuda")
    out = buf[guard:guard + numel].view(wl.B, wl.H, wl.n, 64)
    gpu_forward(x, out=out)
    assert torch.isnan(buf[:guard]).all() and torch.isnan(buf[-guard:]).all()
    assert torch.isfinite(out).all()
    assert_close(out, oracle_forward(x), TOL["bf16"], "guard")


def test_global_overflow_is_reported():
    wl = Workload("overflow", "bf16", 1, 1, 512, 32, globals_kind="first:20")
    x = make_inputs(wl)
    g = to_dev(x)
    ws = lf.new_workspace(1, 1, 512, 8)
    lf.attention_forward(g["q"], g["k"], g["v"], g["qg"], g["kg"], g["vg"], g["local_mask"],
                         g["global_mask"], window=32, max_global=8, workspace=ws)
    assert lf.workspace_status(ws) == lf.LfError(-6).code
    # The next correct call clears the status word.
    lf.attention_forward(g["q"], g["k"], g["v"], g["qg"], g["kg"], g["vg"], g["local_mask"],
                         g["global_mask"], window=32, max_global=20,
                         workspace=lf.new_workspace(1, 1, 512, 20))
    torch.cuda.synchronize()


@pytest.mark.parametrize("globals_kind", ["first:3", "random:20", "random:150", "none"])
def test_host_entry_matches_device_entry(globals_kind):
    # The host path copies Qg, Kg, Vg only with global tokens; the staging
    # buffer starts as 0xFF bytes (NaN for bf16), so a read of anything not
    # copied shows in the output.
    wl = Workload("host", "bf16", 2, 2, 1500, 256, globals_kind=globals_kind, pad_tail=(10, 0),
                  seed=8)
    x = make_inputs(wl)
    dev_out = gpu_forward(x).cpu()
    mg = max_global_of(x)
    pin = {k: (v.pin_memory() if torch.is_tensor(v) else v) for k, v in x.items()}
    host_out = torch.empty_like(pin["q"]).pin_memory()
    staging = torch.full((lf.host_staging_size(torch.bfloat16, 2, 2, 1500),), 0xFF,
                         dtype=torch.uint8, device="cuda")
    ws = lf.new_workspace(2, 2, 1500, mg)
    lf.attention_forward_host(pin["q"], pin["k"], pin["v"], pin["qg"], pin["kg"], pin["vg"],
                              pin["local_mask"], pin["global_mask"], window=256, max_global=mg,
                              out=host_out, staging=staging, workspace=ws)
    assert torch.equal(host_out, dev_out)


def test_aliased_global_projections():
    wl = Workload("alias", "f16", 1, 2, 700, 100, globals_kind="list:0,350")
    x = make_inputs(wl)
    x["qg"], x["kg"], x["vg"] = x["q"], x["k"], x["v"]
    g = to_dev(x)
    out = lf.attention_forward(g["q"], g["k"], g["v"], g["q"], g["k"], g["v"],
                               g["local_mask"], g["global_mask"], window=100, max_global=2)
    torch.cuda.synchronize()
    assert_close(out, oracle_forward(x), TOL["f16"], "alias")


@pytest.mark.parametrize("kw,code", [
    (dict(window=3), -1), (dict(window=0), -1), (dict(dilation=[0, 1]), -1),
    (dict(causal=True, max_global=1), -2),
])
def test_invalid_arguments(kw, code):
    wl = Workload("bad", "bf16", 1, 2, 256, 16, globals_kind="first:1")
    g = to_dev(make_inputs(wl))
    args = dict(window=16, max_global=1)
    args.update(kw)
    with pytest.raises(lf.LfError) as e:
        lf.attention_forward(g["q"], g["k"], g["v"], g["qg"], g["kg"], g["vg"], None,
                             g["global_mask"], **args)
    assert e.value.code == code


def test_misaligned_tensor_rejected():
    # A tensor that starts 4 bytes past a 16-byte boundary is refused before
    # any launch.
    wl = Workload("misaligned", "bf16", 1, 2, 256, 16, globals_kind="first:1")
    g = to_dev(make_inputs(wl))
    q = g["q"]
    buf = torch.zeros(q.numel() + 8, dtype=q.dtype, device=q.device)
    q_off = buf[2:2 + q.numel()].view(q.shape)
    q_off.copy_(q)
    with pytest.raises(lf.LfError) as e:
        lf.attention_forward(q_off, g["k"], g["v"], g["qg"], g["kg"], g["vg"], None,
                             g["global_mask"], window=16, max_global=1)
    assert e.value.code == -1
