"""The multi-GPU host logic of bench.py, exercised with two gloo ranks on the CPU:
barriers, the max-over-ranks timing reduction, the weak-scaling whole-job rate,
and the reference arm printing its line from rank 0 only."""
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.rank_barrier(world)
        ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        slowest = bench.max_over_ranks_value(ms, world, "cpu")
        rate = bench.whole_job_rate(world, 31744, slowest)
        bench.rank_barrier(world)
        out[rank] = (slowest, rate)
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_rate():
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    assert out[0] == out[1]
    slowest, rate = out[0]
    assert slowest == 15.0
    assert abs(rate - 2 * 31744 / 15e-3) < 1e-6 * rate


def test_reference_arm_prints_from_rank_zero_only():
    """`bench.py --impl reference` launched as two ranks: one JSON line, from rank 0."""
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE="2",
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen(
            [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
             "--steps", "1", "--warmup", "0"], env=env, stdout=subprocess.PIPE,
            stderr=subprocess.DEVNULL, text=True))
    outs = [p.communicate(timeout=600)[0] for p in procs]
    assert all(p.returncode == 0 for p in procs)
    lines = [ln for o in outs for ln in o.splitlines() if ln.startswith("{")]
    assert len(lines) == 1 and '"impl": "reference"' in lines[0]
    assert outs[1].strip() == ""
