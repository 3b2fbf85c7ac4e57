"""Multi-process (world_size 2, gloo, CPU) tests of the batch sharding used
across GPUs: the shares cover the batch exactly once, the all-gather puts
every share back in place, and the timing reduction takes the slowest rank.
The per-rank compute is the fp64 oracle here (no GPU needed)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from deformable_convolution_sparse_b200.sharding import batch_shard, forward_sharded, max_over_ranks
from deformable_convolution_sparse_b200.workloads import make_inputs


def test_batch_shard_partitions_every_batch():
    for N in range(0, 40):
        for W in range(1, 9):
            spans = [batch_shard(N, W, r) for r in range(W)]
            assert spans[0][0] == 0 and spans[-1][1] == N
            for (a, b), (c, d) in zip(spans, spans[1:]):
                assert b == c
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        batch_shard(4, 2, 2)


def _oracle_compute(calls):
    import oracle

    def compute(x, om, **kw):
        calls.append(x.shape[0])
        out = oracle.dcnv4_forward(x.double().numpy(), om.double().numpy(), **kw)
        return torch.from_numpy(out)
    return compute


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, N, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x, om = make_inputs(N, 9, 10, 16, 2, 3, 9, 10, "f32", ("normal", 0, 1.5), seed=21)
        calls = []
        full = forward_sharded(x, om, G=2, K=3, pad=1, compute=_oracle_compute(calls))
        own = forward_sharded(x, om, G=2, K=3, pad=1, gather=False, compute=_oracle_compute([]))
        slowest = max_over_ranks(1.0 + rank)
        q.put((rank, calls, full.numpy(), own.shape[0], slowest))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("N", [5, 2, 1])
def test_gloo_world2_shard_and_gather(N):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, N, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    import oracle
    x, om = make_inputs(N, 9, 10, 16, 2, 3, 9, 10, "f32", ("normal", 0, 1.5), seed=21)
    ref = oracle.dcnv4_forward(x.double().numpy(), om.double().numpy(), G=2, K=3, pad=1)
    for rank, calls, full, own_n, slowest in results:
        lo, hi = batch_shard(N, world, rank)
        assert calls == [hi - lo]          # each rank computed only its own share
        assert own_n == hi - lo
        np.testing.assert_array_equal(full, ref)
        assert slowest == 2.0


def _failing_worker(rank, world, port, q):
    """Rank 1's compute raises before the all-gather; rank 0 must get an error, not wait for good."""
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=20))
    x, om = make_inputs(4, 9, 10, 16, 2, 3, 9, 10, "f32", ("normal", 0, 1.5), seed=22)

    def compute(xs, oms, **kw):
        if rank == 1:
            raise RuntimeError("injected failure")
        return _oracle_compute([])(xs, oms, **kw)

    try:
        forward_sharded(x, om, G=2, K=3, pad=1, compute=compute)
        q.put((rank, "finished"))
    except RuntimeError as e:
        q.put((rank, "injected" if "injected failure" in str(e) else "peer error"))
    # rank 1 leaves without taking part in the collective; rank 0 leaves after its error
    q.close()
    q.join_thread()
    os._exit(0)


def test_gloo_failed_rank_ends_the_collective_with_an_error():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_failing_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
    assert got == {0: "peer error", 1: "injected"}
