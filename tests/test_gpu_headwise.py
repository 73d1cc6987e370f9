"""GPU parity of headwise QK-Norm (one factor per head) through the C ABI
against the float64 oracle, on head sizes that reach every segment width and
the multi-vector path, odd head counts, strides, and bit-identity with the
layerwise kernels when a tensor has one head."""
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
    return qk


@pytest.fixture(scope="module")
def orc():
    return oracle.get()


SHAPES = [
    # T, Hq, Hk, head_dim, dtype      (16-byte vectors per head)
    (37, 32, 8, 128, "bf16"),          # 16: two heads per warp
    (64, 40, 8, 128, "bf16"),          # 40 x 128 = the GQA Q width
    (19, 5, 3, 64, "bf16"),            # 8, odd head counts: partial units
    (11, 7, 7, 8, "bf16"),             # 1 vector per head: 32 heads per warp
    (13, 6, 2, 96, "bf16"),            # 12 vectors: 16-lane segments with idle lanes
    (9, 4, 2, 256, "bf16"),            # 32: one head per warp
    (7, 3, 1, 320, "bf16"),            # 40: two vectors per lane
    (5, 2, 2, 2048, "bf16"),           # 256: eight vectors per lane
    (17, 16, 4, 128, "f32"),           # 32 fp32 vectors
    (3 * 148 + 5, 32, 8, 128, "bf16"),  # many tokens per warp
]


@pytest.mark.parametrize("T,Hq,Hk,hd,dtype", SHAPES)
def test_headwise_against_oracle(qk, orc, T, Hq, Hk, hd, dtype):
    wl = W.custom(f"hw{hd}", T, Hq * hd, Hk * hd, 1, dtype=dtype, seed=hd + Hq)
    q = W.gen_rows(wl, "q", range(T))
    k = W.gen_rows(wl, "k", range(T))
    gq = W.gen_gamma(W.custom("gq", 1, hd, hd, 1, seed=hd + 1), "q")
    gk = W.gen_gamma(W.custom("gk", 1, hd, hd, 1, seed=hd + 2), "k")
    oq, ok = qk.qknorm_headwise_fwd(to_device(q), to_device(k), to_device(gq), to_device(gk), hd, 1e-6)
    torch.cuda.synchronize()
    eps = float(np.float32(1e-6))
    check_outputs(to_host(oq), orc.headwise(q, gq, hd, eps, dtype), dtype, "headwise q")
    check_outputs(to_host(ok), orc.headwise(k, gk, hd, eps, dtype), dtype, "headwise k")


@pytest.mark.parametrize("hd", [8, 64, 128, 320, 2048])
def test_one_head_equals_layerwise(qk, hd):
    """With one head per tensor, headwise QK-Norm is layerwise QK-Norm with
    P = 1: same reduction order, so the same bits."""
    T = 29
    wl = W.custom("one", T, hd, hd, 1, seed=60 + hd)
    q, k = to_device(W.gen_rows(wl, "q", range(T))), to_device(W.gen_rows(wl, "k", range(T)))
    gq, gk = to_device(W.gen_gamma(wl, "q")), to_device(W.gen_gamma(wl, "k"))
    hq, hk = qk.qknorm_headwise_fwd(q, k, gq, gk, hd, 1e-6)
    lq, lk = qk.qknorm_fwd(q, k, gq, gk, 1, 1e-6)
    torch.cuda.synchronize()
    assert torch.equal(bits(hq), bits(lq)) and torch.equal(bits(hk), bits(lk))


def test_headwise_strided_qkv_in_place(qk, orc):
    T, Hq, Hk, hd = 41, 16, 4, 128
    Dq, Dk = Hq * hd, Hk * hd
    wl = W.custom("hwqkv", T, Dq, Dk, 1, seed=61)
    q, k = W.gen_rows(wl, "q", range(T)), W.gen_rows(wl, "k", range(T))
    g = to_device(np.linspace(0.5, 1.5, hd).astype(np.float32))
    buf = torch.zeros((T, Dq + 2 * Dk), dtype=torch.bfloat16, device="cuda")
    buf[:, :Dq] = to_device(q)
    buf[:, Dq:Dq + Dk] = to_device(k)
    v = torch.randn((T, Dk), device="cuda").to(torch.bfloat16)
    buf[:, Dq + Dk:] = v
    qs, ks = buf[:, :Dq], buf[:, Dq:Dq + Dk]
    qk.qknorm_headwise_fwd(qs, ks, g, g, hd, 1e-6, out_q=qs, out_k=ks)
    torch.cuda.synchronize()
    gh = g.cpu().numpy()
    check_outputs(to_host(qs.contiguous()), orc.headwise(q, gh, hd, float(np.float32(1e-6)), "bf16"),
                  "bf16", "in-place q")
    check_outputs(to_host(ks.contiguous()), orc.headwise(k, gh, hd, float(np.float32(1e-6)), "bf16"),
                  "bf16", "in-place k")
    assert torch.equal(bits(buf[:, Dq + Dk:]), bits(v))
