"""World-size-2 gloo tests (CPU) of the multi-rank host logic used by bench.py.

The path shards with no data-path collective: every rank runs independent layers
(weak scaling) or a contiguous head range of one layer; the only collectives are the
barrier and the max-over-ranks of the step time.
"""

import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from block_sparse_attention_ibcs_b200.inputs import WORKLOADS

        bench.barrier(world)
        m = bench.max_over_ranks(10.0 + rank, world)
        lo, hi = bench.shard_heads(40, world, rank)
        weak = bench.rank_heads(WORKLOADS["wan14b"], world, rank, "weak")
        strong = bench.rank_heads(WORKLOADS["wan14b"], world, rank, "strong")
        q.put((rank, m, weak, strong, lo, hi))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_sharding():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[1] for r in res] == [11.0, 11.0]  # max over ranks seen by both
    # weak: a layer of 80 heads, 40 per rank; strong: the 40-head layer split in two
    assert (res[0][2], res[1][2]) == ((0, 40, 80), (40, 80, 80))
    assert (res[0][3], res[1][3]) == ((0, 20, 40), (20, 40, 40))
    assert (res[0][4], res[0][5], res[1][4], res[1][5]) == (0, 20, 20, 40)


@pytest.mark.parametrize("H,world", [(40, 8), (24, 5), (12, 1), (3, 4)])
def test_shard_heads_partition(H, world):
    got = [bench.shard_heads(H, world, r) for r in range(world)]
    assert got[0][0] == 0 and got[-1][1] == H
    assert all(a[1] == b[0] for a, b in zip(got, got[1:]))
    sizes = [hi - lo for lo, hi in got]
    assert max(sizes) - min(sizes) <= 1
