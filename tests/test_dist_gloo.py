"""The bench's multi-rank host logic with two gloo ranks on the CPU: per-rank
seeds, max-over-ranks timing, and the reference arm printing one line on rank 0
only.  No GPU and no data-path collective are involved (the path shards into
independent replicas)."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank, world, port):
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)


def _worker_reduce(rank, world, port, out):
    _env(rank, world, port)
    import datetime
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    w, r, lr = bench.dist_env()
    bench.barrier()
    m = bench.reduce_max(10.0 + 5.0 * rank)
    out[rank] = (w, r, lr, m, bench.rank_seed(0, rank))
    dist.destroy_process_group()


def _worker_reference(rank, world, port, out):
    _env(rank, world, port)
    import bench
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.main(["--impl", "reference", "--gpus", str(world), "--steps", "1", "--warmup", "0",
                    "--ref-seconds", "0.2", "--workload", "llama3-8b-s512-b1"])
    out[rank] = buf.getvalue()


def _run(fn, world=2):
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=fn, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0, "rank exited with %s" % p.exitcode
    return dict(out)


def test_max_over_ranks_and_seeds():
    out = _run(_worker_reduce)
    assert sorted(out) == [0, 1]
    for rank, (w, r, lr, m, seed) in out.items():
        assert (w, r, lr) == (2, rank, rank)
        assert m == 15.0  # the slowest rank's time
    assert out[0][4] != out[1][4]  # each rank draws its own batch


def test_reference_arm_prints_once():
    out = _run(_worker_reference)
    lines0 = [l for l in out[0].splitlines() if l.strip()]
    assert len(lines0) == 1 and out[1].strip() == ""
    rec = json.loads(lines0[0])
    assert rec["impl"] == "reference" and rec["unit"] == "TFLOP/s" and rec["value"] > 0
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["e2e"]["h2d_bytes_per_step"] == 0
