"""Tensor-parallel QK-Norm: one rank's step.

SwiftQK technical review, Section 3, Algorithm 1 in its tensor-parallel
form. The hidden dimension of Q and K is split across the ranks of a group;
rank g holds columns [g * D_local, (g + 1) * D_local) of every row, i.e.
P_local of the P = ranks * P_local shards. Each rank

  Phase A  forms its shard sums of squares (qknorm_partial_sumsq_qk: Q's and
           K's [T, P_local] in one launch),
  exchange gathers every rank's sums (one all-gather over the group, Q and K
           together: [ranks, 2, T, P_local]),
  Phase B  adds the P sums of each row in order of the global shard index and
           forms r = rsqrt(S / (ranks * D_local) + eps),
  Phase C  writes (x * gamma) * r for its own slice
           (B and C: qknorm_apply_tp_qk, Q and K in one launch).

The result on rank g equals columns g of qknorm_fwd on the whole rows, bit for
bit: the same shard sums, added in the same order. The exchange is the
group's collective (NCCL on GPUs); everything else runs in the library's
kernels on the rank's own GPU.

A rank that fails or stops taking part (the review's Section 5c notes that
its SpinWait on a peer's flag has no timeout, so one lost rank hangs the
group) ends the others' exchange with an error, never an endless wait:
with ``timeout`` given, the host waits at most that long for the all-gather
and raises TPExchangeError; without it the wait stays asynchronous
(stream-ordered) and the process group's own timeout, set when the group was
created, bounds it.
"""
from __future__ import annotations

import datetime
from typing import Optional, Tuple

import torch
import torch.distributed as dist

from . import qknorm_apply_tp_qk, qknorm_partial_sumsq_qk


class TPExchangeError(RuntimeError):
    """The all-gather of the shard sums failed or did not complete in time on
    this rank (a peer left, failed or stalled). This rank's outputs for the
    step were not written."""


def gathered_stats_shape(ranks: int, T: int, P_local: int) -> Tuple[int, int, int, int]:
    """Shape of the exchanged sums: [ranks, 2 (Q, K), T, P_local]."""
    return (ranks, 2, T, P_local)


def qknorm_tp_fwd(q_local: torch.Tensor, k_local: torch.Tensor, gamma_q_local: torch.Tensor,
                  gamma_k_local: torch.Tensor, P_local: int, eps: float, group=None,
                  out_q: Optional[torch.Tensor] = None, out_k: Optional[torch.Tensor] = None,
                  gathered: Optional[torch.Tensor] = None,
                  timeout: Optional[float] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Layerwise QK-Norm of this rank's slices q_local [T, Dq_local] and
    k_local [T, Dk_local] (gamma slices to match), P_local shards each.
    Collective: every rank of `group` must call it with the same T and
    P_local. `gathered` may pass a preallocated [ranks, 2, T, P_local] fp32
    buffer.

    timeout: seconds the host waits for the exchange before raising
    TPExchangeError (the host then blocks until the all-gather has finished,
    which on GPUs costs the overlap of this step with the host). None: the
    wait is stream-ordered and bounded by the process group's timeout; an
    error the backend reports is raised as TPExchangeError too."""
    ranks = dist.get_world_size(group)
    T = q_local.shape[0]
    if k_local.shape[0] != T:
        raise ValueError("q_local and k_local must have the same number of rows")
    local = qknorm_partial_sumsq_qk(q_local, k_local, P_local)
    if gathered is None:
        gathered = torch.empty(gathered_stats_shape(ranks, T, P_local), dtype=torch.float32,
                               device=q_local.device)
    elif tuple(gathered.shape) != gathered_stats_shape(ranks, T, P_local):
        raise ValueError("gathered must be [ranks, 2, T, P_local]")
    rank = dist.get_rank(group)
    try:
        work = dist.all_gather_into_tensor(gathered.view(-1), local.view(-1), group=group,
                                           async_op=True)
        if timeout is None:
            work.wait()
        else:
            work.wait(timeout=datetime.timedelta(seconds=float(timeout)))
    except RuntimeError as e:
        bound = f"{timeout} s" if timeout is not None else "the process group's timeout"
        raise TPExchangeError(
            f"rank {rank} of {ranks}: the all-gather of the shard sums failed or did not finish "
            f"within {bound} (a peer left, failed or stalled): {e}") from e
    return qknorm_apply_tp_qk(q_local, k_local, gamma_q_local, gamma_k_local, gathered, eps,
                              out_q=out_q, out_k=out_k)
