"""Host side of the multi-GPU bench path, on CPU with two gloo ranks.

Several GPUs run independent replicas of the step (the step has no exchange),
so the only collective steps are the bench's own: a barrier around the timed
region and the maximum of the step time over ranks; the whole-job value is the
work of all ranks over that maximum.  These tests run those helpers in two
spawned processes, and launch the oracle arm of the bench under torchrun with
two ranks (rank 0 alone prints its line, the other exits 0 without work)."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    try:
        import torch

        import bench
        barrier, max_over_ranks, finish = bench.init_ranks(world, torch.device("cpu"), "gloo",
                                                           timeout_s=60)
        barrier()
        ms = max_over_ranks(1.5 + rank)      # each rank its own step time
        value = bench.whole_job_tflops(world, bench.FLOPS_PER_STEP, ms)
        line = bench.bench_line(world, 5, 1, ms, value, {"sm_mhz": None}, None, None,
                                {"kernels": {}})
        barrier()
        finish()
        q.put((rank, ms, value, line, None))
    except Exception as e:  # reported to the parent, which fails the test
        q.put((rank, None, None, None, repr(e)))


def test_two_gloo_ranks_barrier_max_and_line():
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = {}
    try:
        for _ in range(2):
            rank, ms, value, line, err = q.get(timeout=120)
            assert err is None, err
            got[rank] = (ms, value, line)
    finally:
        for p in procs:
            p.join(timeout=30)
            if p.is_alive():
                p.kill()
    import bench
    for rank in (0, 1):
        ms, value, line = got[rank]
        assert ms == 2.5                          # the slower rank decides
        assert value == pytest.approx(2 * bench.FLOPS_PER_STEP / 2.5e-3 / 1e12)
        assert line["n_gpus"] == 2 and line["scaling"] == "weak"
        assert line["config"]["global_batch_tokens"] == 2 * bench.M
        assert line["config"]["parallelism"] == "replicas"
        assert line["value"] == round(value, 2) and line["warmup"] == 3
        assert line["gpu_launches"] == bench.KERNELS_PER_STEP * 5
    assert all(p.exitcode == 0 for p in procs)


def test_whole_job_value_single_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.whole_job_tflops(1, 2e12, 1000.0) == pytest.approx(2.0)
    assert bench.whole_job_tflops(4, 2e12, 1000.0) == pytest.approx(8.0)


def test_reference_arm_under_torchrun_two_ranks(ora):
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1                      # rank 0 alone prints
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
