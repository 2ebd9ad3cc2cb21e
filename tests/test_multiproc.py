"""Multi-rank host logic of bench.py on CPU with the gloo backend, world
size 2: timings are reduced with a max over ranks, the whole-job value sums
every rank's elements over the slowest rank's time, and the reference arm
runs on rank 0 only (the other ranks exit 0 without work or output)."""
import os
import socket
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import io
    import contextlib
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    mine = [10.0 + rank, 5.0 - rank, 1.0 * rank]
    got = bench.max_over_ranks(mine)
    value = bench.aggregate(1000, world, got[0] / 4)
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        rc = bench.main(["--impl", "reference", "--gpus", str(world), "--steps", "1", "--warmup", "3",
                         "--workload", "tiny_f32", "--ref-lanes", "1"])
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, got, value, rc, buf.getvalue()))


def test_bench_rank_logic_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(2):
        r, got, value, rc, text = q.get(timeout=240)
        out[r] = (got, value, rc, text)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in (0, 1):
        got, value, rc, _ = out[r]
        assert got == [11.0, 5.0, 1.0]              # element-wise max over the two ranks
        assert abs(value - 2 * 1000 / (11.0 / 4 / 1e3)) < 1e-6
        assert rc == 0
    assert '"impl": "reference"' in out[0][3]
    assert out[1][3] == ""                         # rank 1 prints nothing
