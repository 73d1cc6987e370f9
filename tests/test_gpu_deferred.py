"""GPU parity of the deferred-normalisation steps: qknorm_xgamma (the weight
multiply alone) and qknorm_inv_rms (the per-token factor alone), through the
C ABI, against the float64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import qknorm_workloads as W
from gpu_util import bits, check_outputs, stats_depth, to_device, to_host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def qk():
    import qk_norm_attention_b200 as qk
    return qk


@pytest.fixture(scope="module")
def orc():
    return oracle.get()


CASES = [("tiny", None), ("decode", 64), ("prefill13b", 1031), ("gqa", 257), ("split_large", 777)]


def _rows(wl, T):
    return (W.gen_rows(wl, "q", range(T)), W.gen_rows(wl, "k", range(T)),
            W.gen_gamma(wl, "q"), W.gen_gamma(wl, "k"))


def inv_rms_tol(D, P, dtype):
    """Relative bound on r: half the relative error of S/D + eps (n roundings
    of non-negative terms, one division, one addition) plus rsqrtf's 2 ulp."""
    n = stats_depth(D, P, dtype) + 2
    return (0.5 * n + 4) * 2.0 ** -23


@pytest.mark.parametrize("name,T", CASES)
def test_xgamma_and_inv_rms_against_oracle(qk, orc, name, T):
    wl = W.WORKLOADS[name]
    T = T or wl.Ts[0]
    q, k, gq, gk = _rows(wl, T)
    for x, g in ((q, gq), (k, gk)):
        xd = to_device(x)
        u = qk.qknorm_xgamma(xd, to_device(g))
        r = qk.qknorm_inv_rms(xd, wl.P, wl.eps)
        torch.cuda.synchronize()
        check_outputs(to_host(u), orc.xgamma(x, g, wl.dtype), wl.dtype, f"{name} xgamma")
        r_or = orc.inv_rms(x, wl.P, float(np.float32(wl.eps)), wl.dtype)
        rel = np.abs(r.cpu().numpy().astype(np.float64) - r_or) / r_or
        assert rel.max() <= inv_rms_tol(x.shape[1], wl.P, wl.dtype), (name, rel.max())


@pytest.mark.parametrize("P", [1, 4, 16])
def test_inv_rms_is_the_fused_factor(qk, P):
    """fp32 data: x*gamma and *r are single fp32 roundings, so the fused output
    equals xgamma(x) * inv_rms computed separately, bit for bit."""
    wl = W.custom("factor", 301, 4096, 1024, P, dtype="f32", seed=51)
    q, k, gq, gk = _rows(wl, 301)
    qd, kd, gqd, gkd = to_device(q), to_device(k), to_device(gq), to_device(gk)
    oq, ok = qk.qknorm_fwd(qd, kd, gqd, gkd, P, wl.eps)
    for x, g, out in ((qd, gqd, oq), (kd, gkd, ok)):
        y = qk.qknorm_xgamma(x, g) * qk.qknorm_inv_rms(x, P, wl.eps)[:, None]
        torch.cuda.synchronize()
        assert torch.equal(bits(y), bits(out))


def test_xgamma_in_place_and_empty(qk):
    wl = W.custom("xg", 9, 2048, 2048, 1, seed=52)
    x = to_device(W.gen_rows(wl, "q", range(9)))
    g = to_device(W.gen_gamma(wl, "q"))
    ref = qk.qknorm_xgamma(x, g)
    qk.qknorm_xgamma(x, g, out=x)
    torch.cuda.synchronize()
    assert torch.equal(bits(x), bits(ref))
    e = torch.empty((0, 2048), dtype=torch.bfloat16, device="cuda")
    assert qk.qknorm_xgamma(e, g).shape == (0, 2048)
    assert qk.qknorm_inv_rms(e, 4, 1e-6).shape == (0,)


def test_deferred_prescale_cancels_on_gpu(qk, orc):
    """The deferred-norm identity through the kernels: normalising
    s_t * xgamma(x) gives the oracle's normalisation of xgamma(x) (eps = 0,
    s_t = 2^k so the scaled input is stored exactly)."""
    wl = W.custom("defer", 64, 4096, 4096, 4, seed=53)
    q, k, g1, g2 = _rows(wl, 64)
    z = qk.qknorm_xgamma(to_device(q), to_device(g1))
    s = torch.tensor([2.0 ** ((t % 9) - 4) for t in range(64)], device="cuda")[:, None]
    zs = (z.float() * s).to(torch.bfloat16)
    assert torch.equal(zs.float(), z.float() * s)
    y1, _ = qk.qknorm_fwd(z, z.clone(), to_device(g2), to_device(g2), 4, 0.0)
    y2, _ = qk.qknorm_fwd(zs, zs.clone(), to_device(g2), to_device(g2), 4, 0.0)
    torch.cuda.synchronize()
    ref, _ = orc.rmsnorm(to_host(z), g2, 4, 0.0, "bf16")
    check_outputs(to_host(y1), ref, "bf16", "z")
    check_outputs(to_host(y2), ref, "bf16", "s*z")
