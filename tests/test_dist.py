"""bench.py's multi-process plumbing on CPU with the gloo backend, world size 2:
max-over-ranks timing, the barrier, and the reference (oracle) arm, which only
rank 0 runs and prints (the other ranks exit 0 without work).  Multi-GPU runs
are independent replicas (one video per GPU), so this host-side logic is the
whole of the N > 1 path apart from the kernels themselves."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch

    import bench
    try:
        bench.dist_init(world, "gloo")
        cpu = torch.device("cpu")
        m = bench.max_over_ranks(float(rank * 10 + 1), cpu)
        bench.barrier(cpu)
        buf = io.StringIO()
        with redirect_stdout(buf):
            rc = bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "0",
                             "--gpus", str(world)])
        q.put((rank, m, rc, buf.getvalue()))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_rank_gloo_plumbing():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, m, rc, out in res:
        assert m == 11.0          # max over ranks of (1, 11)
        assert rc == 0
        if rank == 0:
            line = json.loads(out.strip().splitlines()[-1])
            assert line["impl"] == "reference" and line["n_gpus"] == world
            assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
            assert line["e2e"]["h2d_bytes_per_step"] == 0
        else:
            assert out.strip() == ""  # only rank 0 runs and prints the reference arm
