"""The multi-rank path of bench.py on CPU: two gloo ranks, no GPU.

With N GPUs the bench runs N replicas of the workload, one process per GPU, with no
collective on the data path. What N > 1 adds is host logic: the process group, the
barriers around the timed region, the slowest rank's time (max over ranks), the whole-job
throughput, and one JSON line from rank 0. These tests run that logic as two gloo
processes on 127.0.0.1.
"""

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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup(backend="gloo")
    bench.barrier(w)
    slowest = bench.max_over_ranks(1.5 + r, w)       # rank r "took" 1.5 + r ms
    value = bench.job_throughput(1000, w, slowest)
    bench.barrier(w)
    dist.destroy_process_group()
    q.put((r, w, slowest, value))


def test_two_gloo_ranks_agree_on_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for r, (rank, world, slowest, value) in enumerate(got):
        assert (rank, world) == (r, 2)
        assert slowest == 2.5                       # the max over ranks, on every rank
        assert value == pytest.approx(2 * 1000 / 2.5e-3)


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_prints_on_rank_zero_only(rank):
    env = dict(os.environ, WORLD_SIZE="2", RANK=str(rank), LOCAL_RANK=str(rank), CUDA_VISIBLE_DEVICES="")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "3", "--ref-sample", "64"], env=env, capture_output=True, text=True,
                         timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    if rank:
        assert lines == []
    else:
        line = json.loads(lines[-1])
        assert line["impl"] == "reference" and line["n_gpus"] == 2
        assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
