"""The bench's multi-rank host logic on the CPU (world size 2, gloo).

bench.py runs one replica per GPU; the process group carries only a barrier and
the max over ranks of each timed region.  Here two host processes run the same
functions with the gloo backend."""
import io
import os
import socket
import sys
from contextlib import redirect_stdout
from pathlib import Path

import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parents[1]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, str(ROOT))
    import torch.distributed as dist
    import bench
    ws, r, local = bench.dist_setup(backend="gloo")
    bench.barrier(ws)
    m = bench.max_over_ranks(1.5 * (r + 1), ws, device="cpu")
    bench.barrier(ws)
    q.put((r, ws, local, m))
    dist.destroy_process_group()


def test_two_ranks_time_by_the_slowest():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_rank, args=(r, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    out = sorted(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out == [(0, 2, 0, 3.0), (1, 2, 1, 3.0)]


def test_reference_arm_other_ranks_do_no_work():
    sys.path.insert(0, str(ROOT))
    import bench

    class Args:
        steps, warmup = 1, 3

    buf = io.StringIO()
    with redirect_stdout(buf):
        assert bench.run_reference(Args, 2, 1) is None
    assert buf.getvalue() == ""
