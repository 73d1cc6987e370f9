"""GPU parity of the FP8 E4M3 path (E4M3 in and out, fp32 statistics): the
fused kernels (every variant), the split path, the deferred steps and the
headwise form, through the C ABI, against the float64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import qknorm_workloads as W
from gpu_util import bits, check_outputs, check_stats, to_device, to_host

pytestmark = pytest.mark.gpu

EPS = float(np.float32(1e-6))


@pytest.fixture(scope="module")
def qk():
    import qk_norm_attention_b200 as qk
    yield qk
    qk.qknorm_force_variant(qk.VARIANT_AUTO, 0)


@pytest.fixture(scope="module")
def orc():
    return oracle.get()


def _inputs(name, T, Dq, Dk, P, sigma=1.0):
    wl = W.custom(name, T, Dq, Dk, P, dtype="e4m3", seed=len(name) * 7 + Dq, x_sigma=sigma)
    return (wl, W.gen_rows(wl, "q", range(T)), W.gen_rows(wl, "k", range(T)),
            W.gen_gamma(wl, "q"), W.gen_gamma(wl, "k"))


def test_e4m3_round_trip_layout(qk):
    """Element order of the FP8 conversions: with gamma = 1 and rows whose
    RMS is 1, every value comes back unchanged and in place."""
    codes = np.array([0x38, 0xB8] * 8, dtype=np.uint8)        # +1, -1, ...: RMS = 1
    x = np.tile(codes, (4, 16))                               # [4, 256]
    x[:, 5] = 0x38
    xd = to_device(x)
    one = torch.ones(256, device="cuda")
    oq, ok = qk.qknorm_fwd(xd, xd.clone(), one, one, 4, 0.0)
    torch.cuda.synchronize()
    assert np.array_equal(to_host(oq), x) and np.array_equal(to_host(ok), x)


SHAPES = [
    ("decode", 64, 4096, 4096, 4),
    ("prefill", 3 * 148 + 7, 5120, 5120, 4),
    ("gqa", 301, 5120, 1024, 8),
    ("split", 257, 4096, 4096, 8),
    ("p1", 33, 4096, 4096, 1),
]


@pytest.mark.parametrize("name,T,Dq,Dk,P", SHAPES)
@pytest.mark.parametrize("variant", ["auto", "cta", "bulk", "rows", "generic"])
def test_fp8_fused_and_split(qk, orc, name, T, Dq, Dk, P, variant):
    wl, q, k, gq, gk = _inputs(name, T, Dq, Dk, P, sigma=1.5)
    vid = {"auto": -1, "cta": 0, "bulk": 3, "rows": 4, "generic": 2}[variant]
    qd, kd, gqd, gkd = to_device(q), to_device(k), to_device(gq), to_device(gk)
    qk.qknorm_force_variant(vid, 0)
    try:
        oq, ok = qk.qknorm_fwd(qd, kd, gqd, gkd, P, 1e-6)
        torch.cuda.synchronize()
    except qk.QKNormError as e:
        assert variant in ("cta", "bulk") and e.status == qk.QKNORM_ERR_UNSUPPORTED
        return
    finally:
        qk.qknorm_force_variant(qk.VARIANT_AUTO, 0)
    yq, yk, _, _ = orc.qknorm(q, k, gq, gk, P, EPS, "e4m3", nthreads=8)
    check_outputs(to_host(oq), yq, "e4m3", f"{name} q")
    check_outputs(to_host(ok), yk, "e4m3", f"{name} k")
    if variant == "auto":
        for x, xd_, g, out in ((q, qd, gqd, oq), (k, kd, gkd, ok)):
            st = qk.qknorm_partial_sumsq(xd_, P)
            y = qk.qknorm_apply(xd_, g, st, 1e-6)
            torch.cuda.synchronize()
            assert torch.equal(bits(y), bits(out))
            check_stats(st.cpu().numpy(), orc.partial_sumsq(x, P, "e4m3"), x.shape[1], P, "e4m3", name)


def test_fp8_deferred_and_headwise(qk, orc):
    wl, q, k, gq, gk = _inputs("hw8", 45, 4096, 1024, 8)
    qd = to_device(q)
    u = qk.qknorm_xgamma(qd, to_device(gq))
    r = qk.qknorm_inv_rms(qd, 8, 1e-6)
    hq, hk = qk.qknorm_headwise_fwd(qd, to_device(k), to_device(gq[:128]), to_device(gk[:128]), 128, 1e-6)
    torch.cuda.synchronize()
    check_outputs(to_host(u), orc.xgamma(q, gq, "e4m3"), "e4m3", "xgamma")
    r_or = orc.inv_rms(q, 8, EPS, "e4m3")
    assert (np.abs(r.cpu().numpy() - r_or) / r_or).max() < 1e-5
    check_outputs(to_host(hq), orc.headwise(q, gq[:128], 128, EPS, "e4m3"), "e4m3", "headwise q")
    check_outputs(to_host(hk), orc.headwise(k, gk[:128], 128, EPS, "e4m3"), "e4m3", "headwise k")
