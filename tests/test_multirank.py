"""Multi-rank host logic of bench.py on CPU: two gloo ranks (127.0.0.1).

Decoding shards by tensor with no collective on the data path; the only
cross-rank steps are the barrier and the max-over-ranks of the step time,
checked here, plus the rule that only rank 0 runs the CPU reference arm."""
import contextlib
import io
import multiprocessing as mp
import os
import socket

import pytest


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def worker(rank, world, port, q):
    try:
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                          WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
        import datetime

        import torch.distributed as dist

        import bench
        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
        layer = bench.rank_layer(rank, None)
        ms = 10.0 + 5.0 * rank
        dist.barrier()
        slowest = bench.max_over_ranks(ms, dist)
        gbs = bench.whole_job_gbs(world, 2 * 218_103_808, slowest)
        dist.barrier()
        dist.destroy_process_group()
        # the reference arm: every rank but 0 exits at once without output
        out = io.StringIO()
        rc = None
        if rank != 0:
            with contextlib.redirect_stdout(out):
                rc = bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"])
        q.put((rank, layer, slowest, gbs, rc, out.getvalue()))
    except Exception as e:  # pragma: no cover - reported to the parent
        q.put((rank, "error", repr(e), None, None, None))


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(r[1] != "error" for r in results), results
    (r0, l0, s0, g0, _, _), (r1, l1, s1, g1, rc1, out1) = results
    assert (l0, l1) == (0, 1)                       # each rank decodes its own layer
    assert s0 == s1 == 15.0                         # both see the slowest rank's time
    assert g0 == g1 == pytest.approx(2 * 2 * 218_103_808 / 15e-3 / 1e9)
    assert rc1 == 0 and out1 == ""                  # reference arm: rank 1 does nothing
