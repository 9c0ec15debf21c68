"""The benchmark's multi-rank path on CPU: two gloo ranks (one process each,
127.0.0.1 rendezvous) take the max of their times and report the whole-job
throughput, as bench.py does with NCCL on GPUs."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [10.0 + rank, 20.0 - rank]          # rank 1 is slower on the first value
        got = bench.max_over_ranks(mine, dist, torch.device("cpu"))
        value = bench.whole_job_tflops(world, 1e12, got[0])
        dist.barrier()
        q.put((rank, got, value))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_whole_job_value():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    out = sorted(q.get(timeout=10) for _ in range(world))
    for rank, got, value in out:
        assert got == [11.0, 20.0]                 # max over ranks, element by element
        assert value == pytest.approx(2 * 1e12 / 11e-3 / 1e12)


def test_single_rank_is_identity():
    assert bench.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
    assert bench.whole_job_tflops(1, 2e12, 1000.0) == pytest.approx(2.0)


def _run_reference(extra_env, workload="two_batch_bf16_n1024_d64"):
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, **extra_env)
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                        "--steps", "3", "--warmup", "3", "--cpu-seconds", "0.3",
                        "--workload", workload], capture_output=True, text=True, env=env,
                       timeout=300, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    return [json.loads(ln) for ln in lines]


def test_reference_arm_line():
    """The oracle arm prints one line with the base contract's keys, its own
    workload's metric, and an e2e block with no host transfers."""
    import attn_inputs
    (out,) = _run_reference({"RANK": "0", "WORLD_SIZE": "1"})
    w = attn_inputs.BY_NAME["two_batch_bf16_n1024_d64"]
    assert out["impl"] == "reference" and out["metric"] == bench.metric_for(w)
    assert out["value"] > 0 and out["unit"] == "TFLOP/s" and out["steps"] == 3
    assert out["cpu_baseline"]["kind"] == "oracle" and out["cpu_baseline"]["value"] == out["value"]
    assert out["e2e"] == {"value": out["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                          "d2h_bytes_per_step": 0}
    assert out["config"]["workload"] == "two_batch_bf16_n1024_d64"
    # the same configuration dict as the GPU arm prints for this workload
    assert out["config"] == bench.config_dict(w, 1)
    # the step time is extrapolated from the units the oracle did run, and says so
    assert out["extrapolated"] is True
    m = out["measured"]
    assert m["units_timed"] >= 1 and m["seconds"] > 0 and m["units_per_step"] == w.B * w.Hq
    assert abs(out["ms_per_step"] - m["ms_per_unit"] * m["units_per_step"]) <= \
        0.5 * out["ms_per_step"] + 1.0


def test_reference_arm_other_ranks_are_silent():
    assert _run_reference({"RANK": "1", "WORLD_SIZE": "2"}) == []
