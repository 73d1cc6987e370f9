"""Fault injection on the tensor-parallel step (qk_norm_attention_b200.tp),
on CPU ranks (gloo). No GPU is involved, and no device fault.

The SwiftQK review's Section 5c ("Failure and straggler handling") notes that
its SpinWait on a peer's flag has no timeout: one lost rank hangs the whole
group. Here three ranks run one step of qknorm_tp_fwd together (its outputs
must equal the oracle's), then the last rank leaves the group between steps:
it exits, or it stays alive and never joins step 2 (a straggler). The two
others call step 2 and must fail with TPExchangeError within the bound, not
wait forever. Both bounds are covered: the host-side ``timeout`` of the call,
and the process group's own timeout when the call is given none.

As in test_tp_gloo.py, the two kernel calls of the step are replaced by
float64 stand-ins, since the library's kernels need a GPU; what is under test
is the host side: the collective, its bound and the error it raises.
"""
import datetime
import os
import time

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from test_tp_gloo import _free_port, _stand_in_apply_qk, _stand_in_stats_qk

WORLD, T, DQ, DK, P = 3, 6, 192, 48, 3
STEP_TIMEOUT_S = 2.0       # the call's bound (host wait)
GROUP_TIMEOUT_S = 3.0      # the process group's bound, for calls without one
STALL_S = 30.0             # how long the straggler stays away (far beyond both bounds)


def _inputs():
    rng = np.random.default_rng(17)                 # every rank draws the same full rows
    q = rng.standard_normal((T, DQ)).astype(np.float32)
    k = rng.standard_normal((T, DK)).astype(np.float32)
    gq = rng.uniform(0.5, 1.5, DQ).astype(np.float32)
    gk = rng.uniform(0.5, 1.5, DK).astype(np.float32)
    return q, k, gq, gk


def _rank_main(rank, port, leave, bound, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(WORLD),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    group_timeout = GROUP_TIMEOUT_S if bound == "group" else 120.0
    dist.init_process_group("gloo", rank=rank, world_size=WORLD,
                            timeout=datetime.timedelta(seconds=group_timeout))
    import qk_norm_attention_b200.tp as tp
    tp.qknorm_partial_sumsq_qk = _stand_in_stats_qk
    tp.qknorm_apply_tp_qk = _stand_in_apply_qk
    q, k, gq, gk = (torch.from_numpy(a) for a in _inputs())
    dq, dk = DQ // WORLD, DK // WORLD
    sl = lambda a, d: a[..., rank * d:(rank + 1) * d].contiguous()
    args = (sl(q, dq), sl(k, dk), sl(gq, dq), sl(gk, dk), P // WORLD, 1e-6)
    call_timeout = STEP_TIMEOUT_S if bound == "call" else None
    # Step 1: every rank takes part.
    yq, yk = tp.qknorm_tp_fwd(*args, timeout=call_timeout)
    out.put(("step1", rank, yq.numpy(), yk.numpy()))
    if rank == WORLD - 1:
        # Leave between steps: nothing of this rank is in flight now.
        out.close()
        out.join_thread()
        if leave == "stall":
            time.sleep(STALL_S)                     # alive, but never joins step 2
        os._exit(0)
    # Step 2: the survivors call it; the last rank never does.
    t0 = time.monotonic()
    try:
        tp.qknorm_tp_fwd(*args, timeout=call_timeout)
        res = ("step2", rank, "completed", time.monotonic() - t0)
    except tp.TPExchangeError as e:
        res = ("step2", rank, str(e), time.monotonic() - t0)
    except Exception as e:                          # any other type is a failure of the test
        res = ("step2", rank, f"unexpected {type(e).__name__}: {e}", time.monotonic() - t0)
    out.put(res)
    out.close()
    out.join_thread()
    os._exit(0)                                     # the group is broken; skip its teardown


@pytest.mark.parametrize("leave", ["exit", "stall"])
@pytest.mark.parametrize("bound", ["call", "group"])
def test_survivors_fail_within_the_bound(leave, bound):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, port, leave, bound, out)) for r in range(WORLD)]
    for p in procs:
        p.start()
    try:
        got = [out.get(timeout=120) for _ in range(WORLD + WORLD - 1)]
    finally:
        for p in procs:
            p.join(timeout=5)
            if p.is_alive():                        # the straggler still sleeping
                p.terminate()
                p.join(timeout=10)
    step1 = sorted((g for g in got if g[0] == "step1"), key=lambda g: g[1])
    step2 = sorted((g for g in got if g[0] == "step2"), key=lambda g: g[1])
    assert [g[1] for g in step1] == list(range(WORLD))
    assert [g[1] for g in step2] == list(range(WORLD - 1))
    # Step 1's joined outputs equal the oracle's normalisation of the whole rows.
    import oracle
    q, k, gq, gk = _inputs()
    orc = oracle.get()
    np.testing.assert_allclose(np.concatenate([g[2] for g in step1], axis=1),
                               orc.rmsnorm(q, gq, P, 1e-6, "f32")[0], rtol=1e-6)
    np.testing.assert_allclose(np.concatenate([g[3] for g in step1], axis=1),
                               orc.rmsnorm(k, gk, P, 1e-6, "f32")[0], rtol=1e-6)
    # Step 2: each survivor raised TPExchangeError, and did so within its bound.
    limit = (STEP_TIMEOUT_S if bound == "call" else GROUP_TIMEOUT_S) + 15.0
    for _, rank, msg, elapsed in step2:
        assert msg != "completed", f"rank {rank}: step 2 completed without the third rank"
        assert not msg.startswith("unexpected"), f"rank {rank}: {msg}"
        assert f"rank {rank} of {WORLD}" in msg and "all-gather of the shard sums" in msg
        assert elapsed < limit, f"rank {rank} waited {elapsed:.1f} s (bound {limit} s)"
