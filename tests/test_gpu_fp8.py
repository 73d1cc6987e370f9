"""GPU parity of the FP8 E4M3 path (E4M3 in and out, fp32 statistics): the
fused kernels (every variant), the split path, the deferred steps and the
headwise form, through the C ABI, against the float64 oracle."""
import os

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
@pytest.mark.parametrize("variant", ["auto", "cta", "bulk", "rows", "pair", "gpair", "warp", "generic"])
def test_fp8_fused_and_split(qk, orc, name, T, Dq, Dk, P, variant):
    wl, q, k, gq, gk = _inputs(name, T, Dq, Dk, P, sigma=1.5)
    vid = {"auto": -1, "cta": 0, "bulk": 3, "rows": 4, "pair": 5, "gpair": 6, "warp": 1, "generic": 2}[variant]
    qd, kd, gqd, gkd = to_device(q), to_device(k), to_device(gq), to_device(gk)
    qk.qknorm_force_variant(vid, 0)
    try:
        oq, ok = qk.qknorm_fwd(qd, kd, gqd, gkd, P, 1e-6)
        torch.cuda.synchronize()
    except qk.QKNormError as e:
        assert variant in ("cta", "bulk", "pair", "gpair") and e.status == qk.QKNORM_ERR_UNSUPPORTED
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


def _code_rows(T, D, seed):
    """Rows built from E4M3 codes: every finite code, subnormal-only rows and
    rows at the largest magnitudes (NaN codes 0x7f and 0xff excluded)."""
    rng = np.random.default_rng(seed)
    finite = np.array([c for c in range(256) if c & 0x7F != 0x7F], dtype=np.uint8)
    sub = np.array([c for c in range(256) if (c & 0x78) == 0 and c & 0x7], dtype=np.uint8)
    big = np.array([c for c in range(256) if (c & 0x7F) >= 0x70 and c & 0x7F != 0x7F], dtype=np.uint8)
    x = np.empty((T, D), dtype=np.uint8)
    for t in range(T):
        pool = (finite, sub, big)[t % 3]
        x[t] = rng.choice(pool, size=D)
    x[0, :finite.size] = finite                      # each finite code at least once
    return x


@pytest.mark.parametrize("variant", ["auto", "cta", "bulk", "rows", "warp", "generic"])
def test_fp8_every_code(qk, orc, variant):
    """Every finite E4M3 code in, subnormal-only rows (whose factor is large,
    so their outputs are far from zero) and rows near +-448, with gamma of
    both signs: each variant against the oracle."""
    T, D, P = 3 * 37, 4096, 4
    q, k = _code_rows(T, D, 11), _code_rows(T, D, 12)
    rng = np.random.default_rng(13)
    gq = rng.uniform(0.5, 1.5, D).astype(np.float32) * rng.choice([-1.0, 1.0], D).astype(np.float32)
    gk = rng.uniform(0.5, 1.5, D).astype(np.float32)
    vid = {"auto": -1, "cta": 0, "bulk": 3, "rows": 4, "warp": 1, "generic": 2}[variant]
    qk.qknorm_force_variant(vid, 0)
    try:
        oq, ok = qk.qknorm_fwd(to_device(q), to_device(k), to_device(gq), to_device(gk), P, 1e-6)
        torch.cuda.synchronize()
    finally:
        qk.qknorm_force_variant(qk.VARIANT_AUTO, 0)
    yq, yk, _, _ = orc.qknorm(q, k, gq, gk, P, EPS, "e4m3", nthreads=8)
    check_outputs(to_host(oq), yq, "e4m3", "every-code q")
    check_outputs(to_host(ok), yk, "e4m3", "every-code k")


@pytest.mark.parametrize("D,P", [(4096, 4), (5120, 4), (1024, 8), (4096, 1)])
def test_fp8_variants_bit_identical(qk, D, P):
    """Every fused variant and the split path give the same bytes (one
    reduction order, one rounding of each output)."""
    T = 2 * 148 + 3
    q = _code_rows(T, D, 21 + D)
    k = _code_rows(T, D, 22 + D)
    g = torch.from_numpy(np.random.default_rng(23).uniform(-1.5, 1.5, D).astype(np.float32)).cuda()
    qd, kd = to_device(q), to_device(k)
    outs = {}
    for name, vid in (("cta", 0), ("bulk", 3), ("rows", 4), ("pair", 5), ("gpair", 6), ("warp", 1), ("generic", 2)):
        qk.qknorm_force_variant(vid, 0)
        try:
            outs[name] = qk.qknorm_fwd(qd, kd, g, g, P, 1e-6)
        except qk.QKNormError as e:
            assert name in ("cta", "bulk", "pair", "gpair") and e.status == qk.QKNORM_ERR_UNSUPPORTED
        finally:
            qk.qknorm_force_variant(qk.VARIANT_AUTO, 0)
    outs["split"] = tuple(qk.qknorm_apply(x, g, qk.qknorm_partial_sumsq(x, P), 1e-6) for x in (qd, kd))
    torch.cuda.synchronize()
    ref = outs["generic"]
    for name, (oq, ok) in outs.items():
        assert torch.equal(bits(oq), bits(ref[0])), f"{name} q"
        assert torch.equal(bits(ok), bits(ref[1])), f"{name} k"


def test_fp8_saturation(qk, orc):
    """Outputs beyond the E4M3 range saturate to +-448 with the sign of
    x * gamma, on every variant; the rest stay within one E4M3 ulp."""
    T, D, P = 150, 4096, 4
    q, k = _code_rows(T, D, 31), _code_rows(T, D, 32)
    rng = np.random.default_rng(33)
    g = rng.uniform(0.5, 1.5, D).astype(np.float32)
    g[::7] *= -300.0                                   # these channels overflow the format
    for vid in (-1, 0, 1, 2, 3, 4, 5, 6):
        qk.qknorm_force_variant(vid, 0)
        try:
            oq, ok = qk.qknorm_fwd(to_device(q), to_device(k), to_device(g), to_device(g), P, 1e-6)
            torch.cuda.synchronize()
        except qk.QKNormError as e:
            assert vid in (0, 3, 5, 6) and e.status == qk.QKNORM_ERR_UNSUPPORTED
            continue
        finally:
            qk.qknorm_force_variant(qk.VARIANT_AUTO, 0)
        for x, out in ((q, oq), (k, ok)):
            y_or, _ = orc.rmsnorm(x, g, P, EPS, "e4m3", nthreads=8)
            y = W.storage_to_f64(to_host(out), "e4m3")
            over = np.abs(y_or) > 448 * (1 + 2.0 ** -4)
            assert over.any()
            assert np.array_equal(y[over], np.sign(y_or[over]) * 448.0)
            inside = np.abs(y_or) < 448
            diff = np.abs(y[inside] - y_or[inside])
            assert (diff <= 2.0 ** -3 * np.abs(y_or[inside]) + 2.0 ** -9).all()


@pytest.mark.parametrize("name", ["prefill13b_e4m3", "split_large_e4m3", "gqa_e4m3"])
def test_fp8_bench_workloads_full_size(qk, orc, name):
    """The FP8 configurations the benchmark times, at full size and in the
    selector's launch configuration (inputs drawn on the device with the
    workload's recipe): fused == split on every row, and every row of both
    tensors against the oracle (in chunks of 2048 rows)."""
    wl = W.WORKLOADS[name]
    T = wl.Ts[0]
    dev = torch.device("cuda")
    q = W.gen_device_workload(wl, "q", T, dev)
    k = W.gen_device_workload(wl, "k", T, dev)
    gq = torch.from_numpy(W.gen_gamma(wl, "q")).to(dev)
    gk = torch.from_numpy(W.gen_gamma(wl, "k")).to(dev)
    qk.qknorm_force_variant(qk.VARIANT_AUTO, 0)
    oq, ok = qk.qknorm_fwd(q, k, gq, gk, wl.P, wl.eps)
    aq = qk.qknorm_apply(q, gq, qk.qknorm_partial_sumsq(q, wl.P), wl.eps)
    ak = qk.qknorm_apply(k, gk, qk.qknorm_partial_sumsq(k, wl.P), wl.eps)
    torch.cuda.synchronize()
    assert torch.equal(bits(aq), bits(oq)) and torch.equal(bits(ak), bits(ok))
    eps = float(np.float32(wl.eps))
    nthreads = max(1, min(32, os.cpu_count() or 1))
    chunk = 2048
    for tag, x, g, y in (("q", q, gq, oq), ("k", k, gk, ok)):
        g_host = g.cpu().numpy()
        for r0 in range(0, T, chunk):
            xs = x[r0:r0 + chunk].view(torch.uint8).cpu().numpy()          # E4M3 codes
            y_or, _ = orc.rmsnorm(xs, g_host, wl.P, eps, "e4m3", nthreads=nthreads)
            check_outputs(y[r0:r0 + chunk].view(torch.uint8).cpu().numpy(), y_or, "e4m3",
                          f"{name} {tag} rows {r0}..")
    del q, k, oq, ok, aq, ak
    torch.cuda.empty_cache()


GPAIR_SHAPES = [
    # T, Dq, Dk, P, dtype: separate warps with half slots; mixed with half slots;
    # separate, one whole slot; mixed bf16 with guarded ragged slots
    (257, 5120, 5120, 4, "e4m3"),
    (301, 5120, 1024, 8, "e4m3"),
    (199, 4096, 4096, 8, "e4m3"),
    (2 * 148 + 5, 4096, 4096, 4, "e4m3"),
    (77, 5120, 1024, 8, "bf16"),
]


@pytest.mark.parametrize("T,Dq,Dk,P,dtype", GPAIR_SHAPES)
def test_gpair_bit_identical_and_oracle(qk, orc, T, Dq, Dk, P, dtype):
    """The shard-pair ring with staged gamma on every instance: the default
    plan, forced small grids (each CTA walks many tokens through its ring) and
    row-strided inputs (Q and K inside one buffer), bit-identical to the
    generic kernel and within tolerance of the oracle."""
    wl = W.custom(f"gp{Dq}_{Dk}_{P}", T, Dq, Dk, P, dtype=dtype, seed=Dq + Dk + P + T, x_sigma=1.5)
    q, k = W.gen_rows(wl, "q", range(T)), W.gen_rows(wl, "k", range(T))
    gq, gk = W.gen_gamma(wl, "q"), W.gen_gamma(wl, "k")
    qd, kd, gqd, gkd = to_device(q), to_device(k), to_device(gq), to_device(gk)
    outs = {}
    for name, vid, grid in (("generic", 2, 0), ("gpair", 6, 0), ("gpair_g7", 6, 7), ("gpair_g148", 6, 148)):
        qk.qknorm_force_variant(vid, grid)
        try:
            outs[name] = qk.qknorm_fwd(qd, kd, gqd, gkd, P, 1e-6)
            torch.cuda.synchronize()
        finally:
            qk.qknorm_force_variant(qk.VARIANT_AUTO, 0)
    # Strided: Q and K as column slices of one [T, Dq + Dk + 64] buffer, in place.
    pad = 64
    buf = torch.cat([qd, kd, torch.zeros_like(kd[:, :pad])], dim=1).contiguous()
    qs, ks = buf[:, :Dq], buf[:, Dq:Dq + Dk]
    qk.qknorm_force_variant(6, 0)
    try:
        qk.qknorm_fwd_strided(qs, ks, gqd, gkd, P, 1e-6, out_q=qs, out_k=ks)
        torch.cuda.synchronize()
    finally:
        qk.qknorm_force_variant(qk.VARIANT_AUTO, 0)
    outs["gpair_strided"] = (qs.contiguous(), ks.contiguous())
    ref = outs["generic"]
    for name, (oq, ok) in outs.items():
        assert torch.equal(bits(oq), bits(ref[0])), f"{name} q"
        assert torch.equal(bits(ok), bits(ref[1])), f"{name} k"
    assert torch.equal(bits(buf[:, Dq + Dk:]), bits(torch.zeros_like(kd[:, :pad])))   # padding untouched
    yq, yk, _, _ = orc.qknorm(q, k, gq, gk, P, EPS, dtype, nthreads=8)
    check_outputs(to_host(ref[0]), yq, dtype, f"gpair {Dq}/{Dk} q")
    check_outputs(to_host(ref[1]), yk, dtype, f"gpair {Dq}/{Dk} k")


@pytest.mark.parametrize("T,Dq,Dk,P,dtype", [(3001, 5120, 1024, 8, "e4m3"), (2 * 1184 + 3, 5120, 5120, 4, "e4m3"),
                                             (1500, 5120, 1024, 8, "bf16")])
def test_gpair_many_launches_two_streams(qk, T, Dq, Dk, P, dtype):
    """The staged-gamma ring launched many times back to back (programmatic
    dependent launch between them), on two streams at once and with different
    grids (each CTA walking from 2 to over 400 tokens through its ring): every
    launch gives exactly the generic kernel's bits on every row."""
    wl = W.custom(f"dyn{Dq}_{Dk}_{P}", T, Dq, Dk, P, dtype=dtype, seed=T + Dq, x_sigma=1.2)
    q, k = W.gen_rows(wl, "q", range(T)), W.gen_rows(wl, "k", range(T))
    qd, kd = to_device(q), to_device(k)
    gqd, gkd = to_device(W.gen_gamma(wl, "q")), to_device(W.gen_gamma(wl, "k"))
    qk.qknorm_force_variant(2, 0)
    try:
        ref = qk.qknorm_fwd(qd, kd, gqd, gkd, P, 1e-6)
    finally:
        qk.qknorm_force_variant(qk.VARIANT_AUTO, 0)
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = []
    try:
        for i in range(24):
            qk.qknorm_force_variant(6, (0, 0, 7, 300)[i % 4])
            s = streams[i % 2]
            with torch.cuda.stream(s):
                oq, ok = torch.empty_like(qd), torch.empty_like(kd)
                qk.qknorm_fwd(qd, kd, gqd, gkd, P, 1e-6, out_q=oq, out_k=ok, stream=s.cuda_stream)
            outs.append((oq, ok))
    finally:
        qk.qknorm_force_variant(qk.VARIANT_AUTO, 0)
    torch.cuda.synchronize()
    assert qk.qknorm_device_errors() == 0
    for i, (oq, ok) in enumerate(outs):
        assert torch.equal(bits(oq), bits(ref[0])), f"launch {i} q"
        assert torch.equal(bits(ok), bits(ref[1])), f"launch {i} k"
