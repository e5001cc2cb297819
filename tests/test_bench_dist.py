"""The multi-rank host logic of bench.py on CPU: two `gloo` ranks.

Checks what the GPU run relies on: every rank joins, the barriers pass,
the elapsed time reported is the max over ranks on every rank, each rank
draws a different token batch, the whole-job value counts the work of all
ranks, and the reference arm runs on rank 0 alone.
"""

import contextlib
import io
import os
import socket
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    try:
        w, r, local = bench.dist_setup("gloo")
        bench.barrier(w)
        elapsed = bench.max_over_ranks(10.0 + 5.0 * r, w)
        seeds = [None] * w
        dist.all_gather_object(seeds, bench.rank_seed("qkv_m4352_k3840_n11520", r))
        value = bench.job_value(2.0e12, 4, w, elapsed)
        # the reference arm prints on rank 0 only; other ranks return at once
        out = io.StringIO()
        if r != 0:
            args = bench.parse_args(["--impl", "reference", "--steps", "1", "--warmup", "0"])
            with contextlib.redirect_stdout(out):
                bench.bench_reference(args, w, r)
        bench.barrier(w)
        q.put((r, w, local, elapsed, seeds, value, out.getvalue()))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=5) for _ in range(world))
    for r, (rank, w, local, elapsed, seeds, value, printed) in enumerate(res):
        assert rank == r and w == world and local == r
        assert elapsed == 15.0                     # max over ranks, on every rank
        assert len(set(seeds)) == world            # independent batches
        assert abs(value - 2.0e12 * 4 * world / 15e-3 / 1e12) < 1e-9
        assert printed == ""


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    env = {k: os.environ.pop(k) for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK") if k in os.environ}
    try:
        w, r, local = bench.dist_setup("gloo")
        assert (w, r, local) == (1, 0, 0)
        assert bench.max_over_ranks(3.5, w) == 3.5
        bench.barrier(w)
    finally:
        os.environ.update(env)
