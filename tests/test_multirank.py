"""The multi-rank path of bench.py on CPU: two gloo ranks on 127.0.0.1.

bench.py runs one process per GPU; ranks share nothing on the data path (each
quantizes its own replica of the step) and meet only to reduce timings.  This
checks, without a GPU, that every rank gets the slowest rank's time, that
the reference arm runs on rank 0 alone while the other ranks exit quietly,
and that a rank which leaves between steps (exits, or stays alive without
joining) ends the others' next reduction with an error instead of a hang."""
import contextlib
import datetime
import io
import json
import os
import socket
import sys
import types

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, queue):
    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        slowest = bench.max_over_ranks(10.0 + 5.0 * rank, dist, torch.device("cpu"))
        out = io.StringIO()
        with contextlib.redirect_stdout(out):
            bench.run_reference(types.SimpleNamespace(steps=1, warmup=0), rank, world)
        dist.barrier()
        queue.put((rank, slowest, out.getvalue()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_timings_and_print_once():
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        results = sorted(queue.get(timeout=180) for _ in range(2))
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert [p.exitcode for p in procs] == [0, 0]
    (r0, slow0, out0), (r1, slow1, out1) = results
    assert (r0, r1) == (0, 1)
    assert slow0 == slow1 == 15.0
    assert out1 == ""
    line = json.loads(out0.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0


def test_single_process_timing_is_unchanged():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.25, None, None) == 3.25


def _dropout_worker(rank, world, port, queue, mode="exits"):
    """Rank 1 leaves between steps, before the timing reduction: it exits
    ("exits") or stays alive without joining ("stalls").  Rank 0 must learn
    of it from the collective -- an error from the closed peer, or the
    process group's 5 s timeout -- and not wait for ever."""
    import time
    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    dist.barrier()                      # both ranks joined
    if rank == 1:
        queue.put((1, "left", 0.0))
        queue.close()
        queue.join_thread()              # the message is sent before the process ends
        if mode == "stalls":
            time.sleep(20)               # alive, but never joins the reduction
        os._exit(0)                      # no collective in flight, no further steps
    t0 = time.time()
    try:
        bench.max_over_ranks(1.0, dist, torch.device("cpu"))
        queue.put((0, "no error", time.time() - t0))
    except Exception as e:               # gloo: peer closed, or the timeout
        queue.put((0, type(e).__name__, time.time() - t0))
    queue.close()
    queue.join_thread()
    os._exit(0)


@pytest.mark.parametrize("mode", ["exits", "stalls"])
def test_a_rank_that_leaves_ends_the_others_reduction_with_an_error(mode):
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dropout_worker, args=(r, 2, port, queue, mode)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        results = dict((r, (what, dt)) for r, what, dt in (queue.get(timeout=120) for _ in range(2)))
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert results[1][0] == "left"
    what, dt = results[0]
    assert what != "no error", "the reduction completed without the departed rank"
    assert dt < 19.0                     # before the stalled rank would have ended
