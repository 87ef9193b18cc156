"""The N > 1 logic of bench.py on CPU: world-size-2 gloo ranks.

bench.py runs replicas (every rank the same round on its own GPU, no data-path
collective); the only collectives are the timing barrier and the max over ranks.  These
tests run that logic as two gloo processes, and the reference arm's rank split.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, local = bench.dist_setup()
    bench.barrier(w)
    t_max = bench.dist_max(times[r], w)
    bench.barrier(w)
    value = bench.job_throughput(10.0, 4, w, t_max)
    out_q.put((r, w, local, dist.get_backend(), t_max, value))
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_max_over_ranks_and_job_throughput_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    times = [0.75, 1.25]
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, times, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=90) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    for r, (rank, world, local, backend, t_max, value) in enumerate(got):
        assert (rank, world, local, backend) == (r, 2, r, "gloo")
        # both ranks see the slowest rank's time, and the job rate counts both replicas
        assert t_max == 1.25
        assert value == pytest.approx(2 * 4 * 10.0 / 1.25)


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1",
               MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "2", "--warmup", "3"],
                       env=env, capture_output=True, text=True, timeout=120, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_line_on_a_small_case(capsys):
    sys.path.insert(0, ROOT)
    import argparse

    import bench
    from synth import gen
    case = gen.attn_case(1)
    args = argparse.Namespace(gpus=1, steps=2, warmup=3)
    assert bench.run_reference(args, 1, 0, case=case) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["value"] > 0 and line["unit"] == "GB/s" and line["higher_is_better"]
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
