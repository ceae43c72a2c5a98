"""Multi-rank plumbing of bench.py on CPU with the gloo backend, world size 2:
the max/sum-over-ranks timing reductions, the barrier, and the reference arm
launched through torch.distributed.run as a multi-GPU run is launched
(rank 0 alone prints one JSON line, the other rank exits 0)."""
import json
import os
import socket
import subprocess
import sys
from pathlib import Path

import torch
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parents[1]


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, str(ROOT))
    import bench
    bench.init_dist(world, "gloo")
    mx = bench.max_over_ranks(1.5 + rank, world, "cpu")
    sm = bench.sum_over_ranks(10.0 * (rank + 1), world, "cpu")
    bench.barrier(world)
    q.put((rank, mx, sm))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_timing_reductions_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, mx, sm in got:
        assert mx == 2.5 and sm == 30.0


def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), str(ROOT / "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "2", "--warmup", "3",
           "--config", "tiny", "--cpu-budget", "1"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    proc = subprocess.run(cmd, capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert proc.returncode == 0, proc.stderr[-2000:]
    lines = [ln for ln in proc.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, proc.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0


def test_parse_cpulist():
    """The sysfs CPU lists bench.py binds each rank to."""
    import bench
    assert bench.parse_cpulist("0-15\n") == set(range(16))
    assert bench.parse_cpulist("0-3,8,10-11") == {0, 1, 2, 3, 8, 10, 11}
    assert bench.parse_cpulist("") == set()


def test_timing_statistics_and_host_description():
    """The region / launch statistics the JSON line reports: nearest-rank
    p10 / p90, median and mean of a known list; the CPU-baseline host record."""
    sys.path.insert(0, str(ROOT))
    import bench
    st = bench.stats_ms([float(x) for x in range(1, 101)])   # 1 .. 100 ms
    assert st["n"] == 100 and st["mean"] == 50.5 and st["median"] == 50.5
    assert st["p10"] == 11.0 and st["p90"] == 90.0            # ranks round(0.1 * 99), round(0.9 * 99)
    one = bench.stats_ms([3.0])
    assert one["p10"] == one["p90"] == one["median"] == 3.0
    host = bench.host_description()
    assert host["os_cpu_count"] == os.cpu_count() and host["cores_used"] == 1
