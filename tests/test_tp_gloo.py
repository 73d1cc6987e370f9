"""The tensor-parallel composition (qk_norm_attention_b200.tp) on CPU ranks.

Two and three gloo ranks run qknorm_tp_fwd on their column slices of the same
rows. The library's kernels need a GPU, so here the two kernel calls the
composition makes are replaced by float64 stand-ins written from the same
definitions (the oracle's shard sums; the apply step's sum over the gathered
blocks in rank order and its full-width divisor). What this checks is the
host side: each rank's slice, the one all-gather of Q's and K's sums, its
rank-major layout, and which block each apply reads. Joined, the ranks'
outputs must equal the oracle's normalisation of the whole rows.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _stand_in_stats(x, P, stats=None):
    import oracle
    S = oracle.get().partial_sumsq(x.numpy().astype(np.float32), P, "f32")
    out = torch.from_numpy(S.astype(np.float32))
    if stats is not None:
        stats.copy_(out)
        return stats
    return out


def _stand_in_apply(x, gamma, stats, eps, out=None):
    ranks, T, Pl = stats.shape
    S = stats.double().permute(1, 0, 2).reshape(T, ranks * Pl).sum(dim=1)   # global shard order
    r = 1.0 / torch.sqrt(S / (ranks * x.shape[1]) + eps)
    y = (x.double() * gamma.double()) * r[:, None]
    return y if out is None else out.copy_(y)


def _stand_in_stats_qk(q, k, P, stats=None):
    out = torch.stack((_stand_in_stats(q, P), _stand_in_stats(k, P)))
    return out if stats is None else stats.copy_(out)


def _stand_in_apply_qk(q, k, gq, gk, stats, eps, out_q=None, out_k=None):
    return (_stand_in_apply(q, gq, stats[:, 0], eps, out_q),
            _stand_in_apply(k, gk, stats[:, 1], eps, out_k))


def _rank_main(rank, world, port, T, Dq, Dk, P, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import qk_norm_attention_b200.tp as tp
    tp.qknorm_partial_sumsq_qk = _stand_in_stats_qk
    tp.qknorm_apply_tp_qk = _stand_in_apply_qk
    rng = np.random.default_rng(5)                    # every rank draws the same full rows
    q = torch.from_numpy(rng.standard_normal((T, Dq)).astype(np.float32))
    k = torch.from_numpy(rng.standard_normal((T, Dk)).astype(np.float32))
    gq = torch.from_numpy(rng.uniform(0.5, 1.5, Dq).astype(np.float32))
    gk = torch.from_numpy(rng.uniform(0.5, 1.5, Dk).astype(np.float32))
    dq, dk = Dq // world, Dk // world
    sl = lambda a, d: a[..., rank * d:(rank + 1) * d].contiguous()
    yq, yk = tp.qknorm_tp_fwd(sl(q, dq), sl(k, dk), sl(gq, dq), sl(gk, dk), P // world, 1e-6)
    dist.barrier()
    dist.destroy_process_group()
    out.put((rank, yq.numpy(), yk.numpy()))


@pytest.mark.parametrize("world,T,Dq,Dk,P", [(2, 9, 256, 64, 4), (3, 5, 384, 96, 3)])
def test_tp_composition_on_cpu_ranks(world, T, Dq, Dk, P):
    ctx = mp.get_context("spawn")
    qout = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, T, Dq, Dk, P, qout))
             for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((qout.get(timeout=120) for _ in procs), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    yq = np.concatenate([r[1] for r in res], axis=1)
    yk = np.concatenate([r[2] for r in res], axis=1)
    import oracle
    rng = np.random.default_rng(5)
    q = rng.standard_normal((T, Dq)).astype(np.float32)
    k = rng.standard_normal((T, Dk)).astype(np.float32)
    gq = rng.uniform(0.5, 1.5, Dq).astype(np.float32)
    gk = rng.uniform(0.5, 1.5, Dk).astype(np.float32)
    orc = oracle.get()
    eq, _ = orc.rmsnorm(q, gq, P, 1e-6, "f32")
    ek, _ = orc.rmsnorm(k, gk, P, 1e-6, "f32")
    np.testing.assert_allclose(yq, eq, rtol=1e-6)
    np.testing.assert_allclose(yk, ek, rtol=1e-6)
