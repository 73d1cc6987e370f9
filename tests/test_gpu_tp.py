"""GPU: the tensor-parallel form of the path (Algorithm 1 with the hidden
dimension split across ranks), with the ranks emulated in one process on one
GPU: each rank's slice gets its shard sums from qknorm_partial_sumsq, the
sums are stacked as an all-gather would leave them, and each slice is
finished by qknorm_apply_tp (or both tensors at once: qknorm_partial_sumsq_qk
and qknorm_apply_tp_qk). Joined, the slices must equal qknorm_fwd on the
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


def _emulated_tp(qk, q, k, gq, gk, P, ranks, eps, two=False):
    """Every rank's Phase A, the exchange as a stack, every rank's B and C
    (two: Q and K of a rank in one launch per phase)."""
    T, Dq = q.shape
    Dk = k.shape[1]
    Pl = P // ranks
    dq, dk = Dq // ranks, Dk // ranks
    qs = [q[:, g * dq:(g + 1) * dq].contiguous() for g in range(ranks)]
    ks = [k[:, g * dk:(g + 1) * dk].contiguous() for g in range(ranks)]
    if two:
        local = [qk.qknorm_partial_sumsq_qk(a, b, Pl) for a, b in zip(qs, ks)]
    else:
        local = [torch.stack((qk.qknorm_partial_sumsq(a, Pl), qk.qknorm_partial_sumsq(b, Pl)))
                 for a, b in zip(qs, ks)]
    gathered = torch.stack(local)                      # [ranks, 2, T, P_local]
    if two:
        ys = [qk.qknorm_apply_tp_qk(qs[g], ks[g], gq[g * dq:(g + 1) * dq].contiguous(),
                                    gk[g * dk:(g + 1) * dk].contiguous(), gathered, eps)
              for g in range(ranks)]
        return torch.cat([y[0] for y in ys], dim=1), torch.cat([y[1] for y in ys], dim=1)
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
    ("wide_narrow", 333, 8192, 1024, 2, "bf16", 2),     # one side a CTA per row, one several rows
    ("fp8_narrow", 77, 2048, 1536, 8, "e4m3", 2),
    ("13b", 8 * 148 + 5, 5120, 5120, 8, "bf16", 8),
    ("fold64", 97, 4096, 4096, 64, "bf16", 8),         # 64 shard sums per row: two rounds of 32
    ("fold40", 51, 2560, 640, 40, "f32", 4),           # 40 sums: a round of 32 and one of 8
    ("v4", 333, 4096, 4096, 8, "bf16", 4),             # 128-vector slices: 4 vectors per lane
    ("fp8_v4", 150, 4096, 4096, 8, "e4m3", 2),
    ("13b_p8_r4", 2 * 148 + 3, 5120, 5120, 8, "bf16", 4),   # 160-vector slices, 4 blocks of 2 sums
]


@pytest.mark.parametrize("T,Dq,Dk,P,dtype", [(2 * 148 + 41, 5120, 1024, 8, "bf16"),
                                             (1000, 4096, 4096, 4, "bf16"),
                                             (301, 8192, 768, 4, "f32"),
                                             (77, 2048, 2048, 8, "e4m3"), (1, 256, 128, 2, "bf16")])
def test_two_tensor_calls_equal_one_tensor_calls(qk, T, Dq, Dk, P, dtype):
    """The one-launch statistics and apply of Q and K give the bits of the
    one-tensor calls, with the launch's blocks shared between the tensors."""
    wl = W.custom("two", T, Dq, Dk, P, dtype=dtype, seed=70 + P)
    q, k = to_device(W.gen_rows(wl, "q", range(T))), to_device(W.gen_rows(wl, "k", range(T)))
    gq, gk = to_device(W.gen_gamma(wl, "q")), to_device(W.gen_gamma(wl, "k"))
    st2 = qk.qknorm_partial_sumsq_qk(q, k, P)
    sq, sk = qk.qknorm_partial_sumsq(q, P), qk.qknorm_partial_sumsq(k, P)
    yq, yk = qk.qknorm_apply_tp_qk(q, k, gq, gk, st2[None], 1e-6)
    oq, ok = qk.qknorm_apply(q, gq, sq, 1e-6), qk.qknorm_apply(k, gk, sk, 1e-6)
    torch.cuda.synchronize()
    assert torch.equal(st2[0], sq) and torch.equal(st2[1], sk)
    assert torch.equal(bits(yq), bits(oq)) and torch.equal(bits(yk), bits(ok))
    assert qk.qknorm_device_errors() == 0


@pytest.mark.parametrize("two", [False, True])
@pytest.mark.parametrize("name,T,Dq,Dk,P,dtype,ranks", CASES)
def test_tp_slices_equal_fused(qk, name, T, Dq, Dk, P, dtype, ranks, two):
    wl = W.custom(name, T, Dq, Dk, P, dtype=dtype, seed=61 + ranks)
    q, k = W.gen_rows(wl, "q", range(T)), W.gen_rows(wl, "k", range(T))
    gq, gk = W.gen_gamma(wl, "q"), W.gen_gamma(wl, "k")
    qd, kd, gqd, gkd = to_device(q), to_device(k), to_device(gq), to_device(gk)
    oq, ok = qk.qknorm_fwd(qd, kd, gqd, gkd, P, 1e-6)
    tq, tk = _emulated_tp(qk, qd, kd, gqd, gkd, P, ranks, 1e-6, two)
    torch.cuda.synchronize()
    assert torch.equal(bits(tq), bits(oq)), "TP Q slices differ from the fused Q"
    assert torch.equal(bits(tk), bits(ok)), "TP K slices differ from the fused K"
    if name in ("gqa", "tiny", "fold64", "fold40"):
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


@pytest.mark.parametrize("dtype", ["bf16", "f32", "e4m3"])
@pytest.mark.parametrize("rowvec", [32, 33, 128, 129, 160, 161])
def test_narrow_apply_boundaries(qk, dtype, rowvec):
    """The split apply around the widths where the warp-per-row form changes
    its vectors per lane (32 x 1 .. 5) and where it hands over to the
    several-rows form (161 vectors): one tensor and two tensors per launch,
    bit-identical to the fused kernel. One shard (P = 1) so every width is a
    valid shape."""
    vec = {"bf16": 8, "f32": 4, "e4m3": 16}[dtype]
    D, Dk, T, P = rowvec * vec, 32 * vec, 2 * 148 + 3, 1
    wl = W.custom("narrow", T, D, Dk, P, dtype=dtype, seed=rowvec)
    q, k = to_device(W.gen_rows(wl, "q", range(T))), to_device(W.gen_rows(wl, "k", range(T)))
    gq, gk = to_device(W.gen_gamma(wl, "q")), to_device(W.gen_gamma(wl, "k"))
    oq, ok = qk.qknorm_fwd(q, k, gq, gk, P, 1e-6)
    sq = qk.qknorm_partial_sumsq(q, P)
    yq = qk.qknorm_apply(q, gq, sq, 1e-6)
    st2 = qk.qknorm_partial_sumsq_qk(q, k, P)
    tq, tk = qk.qknorm_apply_tp_qk(q, k, gq, gk, st2[None], 1e-6)
    torch.cuda.synchronize()
    assert torch.equal(bits(yq), bits(oq)), "one-tensor apply"
    assert torch.equal(bits(tq), bits(oq)) and torch.equal(bits(tk), bits(ok)), "two-tensor apply"
    assert qk.qknorm_device_errors() == 0
