"""The bench's multi-rank path on CPU with the gloo backend (world size 2):
max-over-ranks timing, sum of the units all ranks processed, independent
per-rank inputs, and the reference arm running on rank 0 only.  Each rank owns
its own sequences, so nothing else crosses ranks."""
import datetime
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from quantized_kv_cache_18_b200 import workloads as W
        w = W.with_sizes(W.WORKLOADS["tiny"], seq_len=64)
        ms, units = bench.combine_ranks(1.0 + rank, 100.0 * (rank + 1), world, "cpu")
        K, V, q, kn, vn = bench.device_inputs(w, "cpu", 2, rank)
        out_q.put((rank, ms, units, float(K.float().sum()), float(q.float().sum()), tuple(K.shape)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_combine_and_draw_independent_batches():
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for rank, ms, units, _, _, shape in res:
        assert ms == 2.0           # the slower rank's time
        assert units == 300.0      # every rank's bytes
        assert shape == (1, 2, 64, 64)
    assert res[0][3] != res[1][3] and res[0][4] != res[1][4]   # different sequences per rank


def test_single_rank_combine_is_identity():
    import bench
    assert bench.combine_ranks(3.5, 7.0, 1, "cpu") == (3.5, 7.0)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "3", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""
