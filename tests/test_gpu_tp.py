"""GPU: the tensor-parallel form of the path (Algorithm 1 with the hidden
dimension split across ranks), with the ranks emulated in one process on one
GPU: each rank's slice gets its shard sums from qknorm_partial_sumsq, the
sums are stacked as an all-gather would leave them, and each slice is
finished by qknorm_apply_tp. Joined, the slices must equal qknorm_fwd on the
whole rows bit for bit, and the oracle within tolerance."""
import numpy as np
import pytest
import torch

import oracle
import qknorm_workloads as W
from gpu_util import bits, check_outputs, to_device, to_host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def qk():
    import qk_norm_attention_b200 as qk
    qk.qknorm_force_variant(qk.VARIANT_AUTO, 0)
    return qk


def _emulated_tp(qk, q, k, gq, gk, P, ranks, eps):
    """Every rank's Phase A, the exchange as a stack, every rank's B and C."""
    T, Dq = q.shape
    Dk = k.shape[1]
    Pl = P // ranks
    dq, dk = Dq // ranks, Dk // ranks
    qs = [q[:, g * dq:(g + 1) * dq].contiguous() for g in range(ranks)]
    ks = [k[:, g * dk:(g + 1) * dk].contiguous() for g in range(ranks)]
    local = [torch.stack((qk.qknorm_partial_sumsq(a, Pl), qk.qknorm_partial_sumsq(b, Pl)))
             for a, b in zip(qs, ks)]
    gathered = torch.stack(local)                      # [ranks, 2, T, P_local]
    yq = [qk.qknorm_apply_tp(qs[g], gq[g * dq:(g + 1) * dq].contiguous(), gathered[:, 0], eps)
          for g in range(ranks)]
    yk = [qk.qknorm_apply_tp(ks[g], gk[g * dk:(g + 1) * dk].contiguous(), gathered[:, 1], eps)
          for g in range(ranks)]
    return torch.cat(yq, dim=1), torch.cat(yk, dim=1)


CASES = [
    # name, T, Dq, Dk, P, dtype, ranks
    ("13b", 2 * 148 + 3, 5120, 5120, 4, "bf16", 2),
    ("13b", 2 * 148 + 3, 5120, 5120, 4, "bf16", 4),
    ("gqa", 301, 5120, 1024, 8, "bf16", 2),
    ("gqa", 301, 5120, 1024, 8, "bf16", 8),
    ("tiny", 37, 256, 256, 2, "f32", 2),
    ("fp8", 150, 4096, 4096, 8, "e4m3", 4),
    ("one", 65, 4096, 1024, 4, "bf16", 1),
]


@pytest.mark.parametrize("name,T,Dq,Dk,P,dtype,ranks", CASES)
def test_tp_slices_equal_fused(qk, name, T, Dq, Dk, P, dtype, ranks):
    wl = W.custom(name, T, Dq, Dk, P, dtype=dtype, seed=61 + ranks)
    q, k = W.gen_rows(wl, "q", range(T)), W.gen_rows(wl, "k", range(T))
    gq, gk = W.gen_gamma(wl, "q"), W.gen_gamma(wl, "k")
    qd, kd, gqd, gkd = to_device(q), to_device(k), to_device(gq), to_device(gk)
    oq, ok = qk.qknorm_fwd(qd, kd, gqd, gkd, P, 1e-6)
    tq, tk = _emulated_tp(qk, qd, kd, gqd, gkd, P, ranks, 1e-6)
    torch.cuda.synchronize()
    assert torch.equal(bits(tq), bits(oq)), "TP Q slices differ from the fused Q"
    assert torch.equal(bits(tk), bits(ok)), "TP K slices differ from the fused K"
    if name in ("gqa", "tiny"):
        orc = oracle.get()
        eps = float(np.float32(1e-6))
        yq, _ = orc.rmsnorm(q, gq, P, eps, dtype, nthreads=8)
        check_outputs(to_host(tq), yq, dtype, f"tp {name} q")


def test_tp_rejects_bad_layouts(qk):
    x = torch.zeros(8, 1024, dtype=torch.bfloat16, device="cuda")
    g = torch.ones(1024, device="cuda")
    st = torch.zeros(2, 8, 4, device="cuda")
    L = qk.lib
    h = torch.cuda.current_stream().cuda_stream
    y = torch.empty_like(x)
    args = lambda stride, ranks: (x.data_ptr(), g.data_ptr(), st.data_ptr(), stride, y.data_ptr(),
                                  8, 1024, 4, ranks, 1e-6, 1, h)
    assert L.qknorm_apply_tp(*args(0, 2)) == 0
    assert L.qknorm_apply_tp(*args(31, 2)) == qk.QKNORM_ERR_INVALID_ARG   # blocks would overlap
    assert L.qknorm_apply_tp(*args(-1, 2)) == qk.QKNORM_ERR_INVALID_ARG
    assert L.qknorm_apply_tp(*args(0, 0)) == qk.QKNORM_ERR_INVALID_ARG
    bad = (x.data_ptr(), g.data_ptr(), st.data_ptr() + 2, 0, y.data_ptr(), 8, 1024, 4, 2, 1e-6, 1, h)
    assert L.qknorm_apply_tp(*bad) == qk.QKNORM_ERR_MISALIGNED             # stats not 4-byte aligned
    torch.cuda.synchronize()
