"""The N > 1 bench path on CPU: two gloo ranks run the host-side logic that
`bench.py --gpus 2` runs under torchrun (independent replicas, no data-path
collective): the process-group setup, the max-over-ranks of the timed region,
disjoint per-rank token streams and the whole-job throughput."""

import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import bench
    dist, r, w, local = bench.dist_setup(world, backend="gloo")
    # each rank a different time: the job takes the slowest
    ms = bench.barrier_max(dist, 10.0 + 5.0 * r, device="cpu")
    ids = bench.rank_token_ids(r, 4)
    dist.barrier()
    out.put((r, w, local, ms, ids, bench.job_tokens_per_s(8, w, 1, ms)))
    dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, w0, l0, ms0, ids0, tps0), (r1, w1, l1, ms1, ids1, tps1) = res
    assert (r0, r1) == (0, 1) and w0 == w1 == 2 and (l0, l1) == (0, 1)
    assert ms0 == ms1 == 15.0                      # max over ranks
    assert not set(ids0) & set(ids1)               # independent token streams
    assert tps0 == tps1 == pytest.approx(8 * 2 * 1 / 0.015)  # all ranks' tokens / slowest time


def test_single_process_defaults():
    sys.path.insert(0, ROOT)
    import bench
    os.environ.pop("WORLD_SIZE", None)
    assert bench.dist_setup(1, backend="gloo") == (None, 0, 1, 0)
    assert bench.barrier_max(None, 3.0) == 3.0
    assert bench.rank_token_ids(0, 3) == [0, 1, 2]
