"""The multi-process plumbing of bench.py, on CPU: two gloo ranks (the path is replicas
only -- every rank runs its own problem and no data-path collective exists -- so what
needs checking is the launch contract: rendezvous, barriers, the max-over-ranks timing
and the whole-job aggregate)."""
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    r, w, local = bench.dist_init(world)
    assert (r, w, local) == (rank, world, rank) and dist.get_backend() == "gloo"
    bench.barrier(w)
    t = bench.max_over_ranks(1.0 + rank, w)           # rank-local "ms per step"
    v = bench.job_throughput(2.0e9, t, w)              # whole-job ops/s in TOPS
    bench.barrier(w)
    dist.destroy_process_group()
    q.put((rank, t, v))


def test_two_gloo_ranks_rendezvous_and_take_the_max():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=5) for _ in procs)
    for rank, t, v in got:
        assert t == 2.0                                  # the slowest rank's time
        assert v == pytest.approx(2 * 2.0e9 / 2.0e-3 / 1e12)   # both ranks' work / max time


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_throughput(1.0e12, 1.0, 1) == pytest.approx(1000.0)


def test_reference_arm_prints_the_contract_line():
    """bench.py --impl reference times the oracle on the host cores (no GPU) and prints one
    JSON line with the contract's keys, the reference arm's marker and its CPU baseline."""
    import json
    import subprocess
    import sys
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "3", "--warmup", "3", "--workload", "tiny_m16_n256_k512"],
                         cwd=ROOT, capture_output=True, text=True, timeout=300, check=True)
    line = json.loads(out.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["steps"] == 3 and line["warmup"] == 3
    assert line["value"] > 0 and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["config"]["workload"] == "tiny_m16_n256_k512"


def test_reference_arm_under_torchrun_prints_once():
    """Launched as the multi-GPU bench is (torchrun, 2 ranks; gloo here), rank 0 alone runs
    the oracle and prints one line, and every rank exits 0."""
    import json
    import subprocess
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "3",
           "--warmup", "3", "--workload", "tiny_m16_n256_k512"]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300, check=True)
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
