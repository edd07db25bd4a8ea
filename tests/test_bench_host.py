"""Host logic of bench.py on CPU: max-over-ranks timing with two gloo ranks,
whole-job throughput, and the oracle reference arm."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    dist = bench.init_dist(world, "gloo")
    local_ms = [12.5, 40.0][rank]
    mx = bench.reduce_max(local_ms, "cpu")
    rate = bench.whole_job_rate(6.277e9, 100, world, mx)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, mx, rate))


def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, mx, rate in res:
        assert mx == 40.0
        assert rate == pytest.approx(6.277e9 * 100 * 2 / 0.040)


def test_single_process_reduce_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(3.5, "cpu") == 3.5
    assert bench.whole_job_rate(10, 4, 1, 2.0) == pytest.approx(20000.0)


def _run_bench(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                          capture_output=True, text=True, env=env, timeout=600)


def test_reference_arm_prints_one_json_line():
    r = _run_bench(["--impl", "reference", "--steps", "3", "--warmup", "3",
                    "--workload", "fp32-b1h2-n512-w64-g1", "--reference-seconds", "3"])
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "TFLOP/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


def test_reference_arm_other_ranks_do_no_work():
    r = _run_bench(["--impl", "reference", "--gpus", "2", "--steps", "3", "--warmup", "3"],
                   {"WORLD_SIZE": "2", "RANK": "1", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_warmup_below_three_is_rejected():
    r = _run_bench(["--warmup", "2"])
    assert r.returncode != 0


def test_projection_cpu_baseline_line_is_well_formed():
    import numpy as np
    import bench
    from sparse_long_sequence_lf_b200.workloads import Workload
    wl = Workload("proj-host", "bf16", 1, 2, 40, 8, globals_kind="list:3,17", seed=5)
    gidx = -np.ones((1, 40), dtype=np.int32)
    gidx[0, :2] = [3, 17]
    cpu = bench.run_projection_cpu_baseline(wl, np.array([2]), gidx, 2, budget_s=0.05)
    assert cpu["kind"] == "oracle" and cpu["unit"] == "TFLOP/s" and cpu["value"] > 0
    assert bench.projection_flops(wl, [2], 2) == 2.0 * 40 * 128 * 640 + 2.0 * 2 * 128 * 128


def _shard_rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch
    import bench
    import oracle
    from sparse_long_sequence_lf_b200.sharding import gather_heads, head_ranges, shard_inputs
    from sparse_long_sequence_lf_b200.workloads import Workload, make_inputs
    dist = bench.init_dist(world, "gloo")
    wl = Workload("shard", "f32", 2, 5, 96, 16, dilation=(1, 2, 1, 3, 2),
                  globals_kind="list:0,40;7", pad_tail=(0, 9), seed=21)
    x = make_inputs(wl)
    ranges = head_ranges(wl.H, world)
    xs = shard_inputs(x, *ranges[rank])
    mine = oracle.forward(xs["q"], xs["k"], xs["v"], xs["qg"], xs["kg"], xs["vg"],
                          xs["local_mask"], xs["global_mask"], window=wl.window,
                          dilation=xs["dilation"], causal=wl.causal)
    full = gather_heads(torch.from_numpy(np.ascontiguousarray(mine)), ranges).numpy()
    dist.barrier()
    dist.destroy_process_group()
    if rank == 0:
        ref = oracle.forward(x["q"], x["k"], x["v"], x["qg"], x["kg"], x["vg"],
                             x["local_mask"], x["global_mask"], window=wl.window,
                             dilation=x["dilation"], causal=wl.causal)
        q.put(bool(np.array_equal(full, ref)))


def test_head_ranges_cover_the_heads_once():
    from sparse_long_sequence_lf_b200.sharding import head_ranges
    for H in (1, 5, 12, 16):
        for world in range(1, H + 1):
            r = head_ranges(H, world)
            assert r[0][0] == 0 and r[-1][1] == H
            assert all(a[1] == b[0] for a, b in zip(r, r[1:]))
            sizes = [h1 - h0 for h0, h1 in r]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1


def test_two_gloo_ranks_split_one_problem_by_heads():
    # Each rank computes its heads (uneven split: 3 and 2) with the oracle;
    # the gathered heads equal the whole problem exactly.
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    assert q.get(timeout=10) is True


def test_head_split_applies_to_the_attention_op_only(monkeypatch):
    import bench
    monkeypatch.setenv("WORLD_SIZE", "1")
    with pytest.raises(SystemExit):
        bench.main(["--shard", "heads", "--op", "backward"])
