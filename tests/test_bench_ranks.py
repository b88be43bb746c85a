"""The benchmark on CPU, no GPU.  Two gloo ranks on 127.0.0.1 run the same
cross-rank reduction the GPU ranks run over NCCL (max of per-rank device
timings) and the whole-job throughput formula (weak scaling: one replica per
rank, the slowest rank's time); the oracle arm prints the one JSON line the
benchmark contract asks for."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        # rank r measured (10 + r) ms for the step and (7 - r) ms for the attention
        mx = bench.max_over_ranks([10.0 + rank, 7.0 - rank], torch.device("cpu"))
        dist.barrier()
        q.put((rank, mx, bench.job_tflops(world, 3.5e12, mx[1])))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_count_every_replica():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, mx, tf in got:
        assert mx == [11.0, 7.0]                      # the slowest rank sets each timing
        assert tf == pytest.approx(2 * 3.5e12 / 7e-3 / 1e12)


def test_single_process_is_the_identity():
    import bench
    assert bench.max_over_ranks([1.5, 2.5], torch.device("cpu")) == [1.5, 2.5]
    assert bench.job_tflops(1, 1e12, 1.0) == pytest.approx(1000.0)


def test_reference_arm_prints_the_contract_line():
    # the oracle arm on the tiny grid, as the driver launches it (one JSON line on stdout)
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--config", "tiny",
                          "--steps", "2", "--warmup", "1", "--cpu-seconds", "2"],
                         capture_output=True, text=True, timeout=600, cwd=root,
                         env={**os.environ, "CUDA_VISIBLE_DEVICES": ""})
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    r = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert k in r, k
    assert r["impl"] == "reference" and r["steps"] == 2 and r["warmup"] == 1 and r["value"] > 0
    assert r["higher_is_better"] is True and r["unit"] == r["e2e"]["unit"] == "TFLOP/s"
    assert r["e2e"]["h2d_bytes_per_step"] == 0 and r["e2e"]["d2h_bytes_per_step"] == 0
    assert r["cpu_baseline"]["kind"] == "oracle" and r["cpu_baseline"]["cores"] >= 1
    assert "tiny grid 8x16x16" in r["metric"] and "workload" in r["config"]
