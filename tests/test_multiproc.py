"""The multi-GPU host logic of bench.py on CPU: two gloo ranks.

Tokens are independent, so N GPUs each process their own contiguous block of
tokens with no collective on the data path; the only collectives are the
barriers around the timed region and the max-over-ranks of its duration.
This test runs those on CPU ranks (gloo) and checks that the token blocks of
all ranks tile the global batch exactly once.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, T_global, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import bench
    d = bench.Dist()
    assert (d.rank, d.world) == (rank, world)
    d.init("gloo")
    lo, hi = bench.shard_tokens(T_global, world, rank)
    d.barrier()
    slow = d.max(float(10 * rank + 1), "cpu")      # ranks report different times
    d.barrier()
    d.close()
    out.put((rank, lo, hi, slow))


@pytest.mark.parametrize("world,T", [(2, 8192), (2, 8193), (3, 10)])
def test_token_shards_and_max_over_ranks(world, T):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, T, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    covered = []
    for rank, lo, hi, slow in res:
        covered.extend(range(lo, hi))
        assert slow == float(10 * (world - 1) + 1)   # every rank sees the slowest rank's time
    assert covered == list(range(T))                 # each token exactly once, in order
    sizes = [hi - lo for _, lo, hi, _ in res]
    assert max(sizes) - min(sizes) <= 1


def test_shard_tokens_single_rank():
    import bench
    assert bench.shard_tokens(8192, 1, 0) == (0, 8192)
    assert bench.shard_tokens(0, 4, 3) == (0, 0)
