"""The benchmark's multi-rank host logic on CPU: two gloo ranks.

bench.py shards by sequence: each rank decodes its own batch (distinct seeds), there is no
data-path collective, and the step time is the max over ranks, which every rank receives.
These checks run the same helpers bench.py uses, as two processes on 127.0.0.1.
"""

import contextlib
import io
import multiprocessing as mp
import os
import socket
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    try:
        import torch.distributed as dist

        import bench

        r, w, local = bench.dist_setup(world, backend="gloo")
        bench.barrier(w)
        step_ms = 0.25 + 0.1 * r          # rank 1 is the slower one
        ms = bench.max_over_ranks(step_ms, w)
        value = bench.job_tokens_per_s(w, ms)
        bench.barrier(w)
        # the reference arm: only rank 0 works and prints; the others return at once
        out = io.StringIO()
        with contextlib.redirect_stdout(out):
            if r != 0:
                bench.run_reference(type("Args", (), dict(gpus=w, steps=1, warmup=0))())
        dist.destroy_process_group()
        q.put((r, w, local, ms, value, bench.shard_seed(r), out.getvalue()))
    except Exception as e:  # noqa: BLE001
        q.put((rank, "error", repr(e)))


def test_two_gloo_ranks_share_the_max_step_time_and_own_disjoint_batches():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
    assert all(p.exitcode == 0 for p in procs)
    by_rank = {}
    for res in results:
        assert res[1] != "error", res
        by_rank[res[0]] = res
    import bench

    assert set(by_rank) == {0, 1}
    for r, (rank, world, local, ms, value, seed, printed) in by_rank.items():
        assert world == 2 and local == r
        assert abs(ms - 0.35) < 1e-12                   # the slower rank's time, on both ranks
        assert abs(value - 2 * bench.B_PER_GPU / 0.35e-3) < 1e-6
        assert printed == ""                             # rank 1 of the reference arm stays silent
    assert by_rank[0][5] != by_rank[1][5]                # each rank draws its own sequences
