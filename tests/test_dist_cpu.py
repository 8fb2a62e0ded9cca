"""The N > 1 path of bench.py on CPU: world_size-2 gloo process groups.

The decode step shards by replica (every rank runs its own workload, no data-path
collective), so what crosses ranks is host plumbing only: the process group, the
barrier around the timed region, the max over ranks of the step time, and rank 0
printing the one JSON line.  These run here with gloo instead of NCCL."""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from synth import Workload, spec_by_name  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE="2", RANK=str(rank),
                      LOCAL_RANK=str(rank))
    import torch.distributed as dist
    ws, r, local = bench.dist_setup()
    try:
        assert dist.get_backend() == "gloo"
        bench.barrier(ws)
        mx = bench.reduce_max(1.5 + rank, ws)  # rank 1 is the slower one
        q.put((r, ws, mx, bench.whole_job_rate(4, ws, mx)))
        bench.barrier(ws)
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_max_time_and_aggregate_units():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for r, (rank, ws, mx, rate) in enumerate(got):
        assert (rank, ws) == (r, 2)
        assert mx == 2.5  # both ranks see the slowest rank's time
        assert rate == pytest.approx(2 * 4 / 2.5e-3)  # 4 query tokens per rank, 2 ranks


def test_whole_job_rate_single_rank():
    assert bench.whole_job_rate(1, 1, 0.05) == pytest.approx(20000.0)


def test_ranks_get_distinct_replicas():
    # weak scaling: rank r draws its workload from seed + r
    s = spec_by_name("tiny")
    a = Workload(s.replace(seed=s.seed + 0)).numpy("q_c")
    b = Workload(s.replace(seed=s.seed + 1)).numpy("q_c")
    assert a.shape == b.shape and not (a == b).all()


@pytest.mark.slow
def test_reference_arm_under_torchrun_prints_one_line_from_rank_zero():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2", "--master-addr",
           "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"), "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "3", "--workload", "tiny", "--ref-budget", "1"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"


def test_combined_rate_sums_bytes_and_times():
    bulk = {"csa_bytes": 2.0e9, "csa_us": 400.0, "hca_bytes": 1.0e9, "hca_us": 200.0}
    c = bench.combined_rate(bulk, 23.0e6, 0.05, 6538.3)
    assert c["bytes"] == pytest.approx(3.023e9)
    assert c["us"] == pytest.approx(650.0)
    assert c["gbs"] == pytest.approx(3.023e9 / 650e-6 / 1e9)
    assert c["frac_of_measured_hbm"] == pytest.approx(c["gbs"] / 6538.3)
