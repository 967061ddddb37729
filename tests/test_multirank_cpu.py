"""The N > 1 launch path on CPU (two gloo ranks; no GPU).

The forward path shards into independent replicas (no exchange between heads
or batches), so the only multi-rank logic is the benchmark's: every timed
figure is the slowest rank's (an all-reduce MAX after a barrier), and under
torchrun the reference arm runs on rank 0 alone while the other ranks exit 0.
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
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_max_worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench.sync_ranks(dist, device_sync=False)
        # rank r "measured" 1.5 (r + 1) seconds; all must report the slowest
        out.put((rank, bench.rank_max(1.5 * (rank + 1), dist, device="cpu")))
        bench.sync_ranks(dist, device_sync=False)
    finally:
        dist.destroy_process_group()


def test_rank_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_max_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    got = sorted(out.get(timeout=10) for _ in range(2))
    assert got == [(0, 3.0), (1, 3.0)]


def test_rank_max_without_process_group_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.rank_max(2.25, None) == 2.25


@pytest.mark.timeout(600)
def test_reference_arm_under_torchrun_two_ranks():
    """bench.py --impl reference --gpus 2 launched as two ranks: exit 0 and one
    JSON line (rank 0's) with impl "reference" and n_gpus 2."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--impl", "reference",
           "--gpus", "2", "--workload", "tiny", "--steps", "1", "--warmup", "3", "--ref-rows", "32"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"


def test_gpus_flag_must_match_world_size():
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--gpus", "2", "--workload", "tiny"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=120)
    assert r.returncode != 0 and "WORLD_SIZE" in (r.stderr + r.stdout)
