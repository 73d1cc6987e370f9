"""GPU edge cases through the C ABI: empty and ragged inputs, every kernel
variant (bit-identical by construction), shard shapes that reach each code
path, in-place calls, guard regions around the outputs, unchanged inputs,
and tensors of more than 2^31 elements."""
import zlib

import numpy as np
import pytest
import torch

import oracle
import qknorm_workloads as W
from gpu_util import bits, check_outputs, check_stats, to_device, to_host

pytestmark = pytest.mark.gpu

VARIANTS = ("cta", "bulk", "rows", "pair", "gpair", "warp", "generic")


@pytest.fixture(scope="module")
def qk():
    import qk_norm_attention_b200 as qk
    yield qk
    qk.qknorm_force_variant(qk.VARIANT_AUTO, 0)


@pytest.fixture(scope="module")
def orc():
    return oracle.get()


def _inputs(wl, T):
    q = W.gen_rows(wl, "q", range(T))
    k = W.gen_rows(wl, "k", range(T))
    gq, gk = W.gen_gamma(wl, "q"), W.gen_gamma(wl, "k")
    return q, k, gq, gk


def _fwd(qk, wl, q, k, gq, gk, variant=None, grid=0):
    vid = {"cta": qk.VARIANT_CTA, "warp": qk.VARIANT_WARP, "generic": qk.VARIANT_GENERIC,
           "bulk": qk.VARIANT_BULK, "rows": qk.VARIANT_ROWS, "pair": qk.VARIANT_PAIR,
           "gpair": qk.VARIANT_GPAIR, None: qk.VARIANT_AUTO}[variant]
    qk.qknorm_force_variant(vid, grid)
    try:
        oq, ok = qk.qknorm_fwd(to_device(q), to_device(k), to_device(gq), to_device(gk),
                               wl.P, wl.eps)
        torch.cuda.synchronize()
    finally:
        qk.qknorm_force_variant(qk.VARIANT_AUTO, 0)
    return oq, ok


def _check_oracle(orc, wl, q, k, gq, gk, oq, ok):
    eps = float(np.float32(wl.eps))
    yq, yk, _, _ = orc.qknorm(q, k, gq, gk, wl.P, eps, wl.dtype, nthreads=8)
    check_outputs(to_host(oq), yq, wl.dtype, f"{wl.name} q")
    check_outputs(to_host(ok), yk, wl.dtype, f"{wl.name} k")


SHAPES = [
    # name, T, Dq, Dk, P, dtype
    ("decode_odd_T", 33, 4096, 4096, 4, "bf16"),
    ("gqa_ragged_lanes", 77, 5120, 1024, 8, "bf16"),
    ("p1_two_groups", 19, 4096, 4096, 1, "bf16"),       # nv = 512 -> K = 2
    ("p16_block1024", 21, 4096, 4096, 16, "bf16"),      # 32 warps, 1 vector per lane
    ("p32_generic", 9, 4096, 4096, 32, "bf16"),         # 64 tasks -> generic
    ("wide_p1", 5, 65536, 8192, 1, "bf16"),             # K = 32 -> generic
    ("k_one_vector_shard", 13, 1024, 64, 8, "bf16"),    # K shard = one vector
    ("mixed_groups", 7, 32768, 1024, 4, "bf16"),        # K_q = 4, K_k = 1
    ("fp32_d4096", 29, 4096, 4096, 4, "f32"),
    ("fp32_p64", 6, 1024, 512, 64, "f32"),              # 4-wide shards, generic
]


@pytest.mark.parametrize("shape", SHAPES, ids=[s[0] for s in SHAPES])
def test_shapes_and_variants(qk, orc, shape):
    name, T, Dq, Dk, P, dtype = shape
    wl = W.custom(name, T, Dq, Dk, P, dtype=dtype, seed=zlib.crc32(name.encode()) % 1000)
    q, k, gq, gk = _inputs(wl, T)
    outs = {}
    for v in VARIANTS:
        try:
            outs[v] = _fwd(qk, wl, q, k, gq, gk, variant=v)
        except qk.QKNormError as e:
            # Only the register-resident kernels (cta, bulk, pair) and the
            # shared-memory staged ones (bulk, rows, pair) have shape limits.
            assert v in ("cta", "bulk", "rows", "pair", "gpair") and e.status == qk.QKNORM_ERR_UNSUPPORTED, str(e)
    base = outs["generic"]
    for v, (oq, ok) in outs.items():
        assert torch.equal(bits(oq), bits(base[0])), f"{v} Q differs from generic"
        assert torch.equal(bits(ok), bits(base[1])), f"{v} K differs from generic"
    auto = _fwd(qk, wl, q, k, gq, gk)
    assert torch.equal(bits(auto[0]), bits(base[0])) and torch.equal(bits(auto[1]), bits(base[1]))
    _check_oracle(orc, wl, q, k, gq, gk, *auto)
    # The split path agrees bit for bit with the fused path on every shape.
    for x, g, out in ((q, gq, auto[0]), (k, gk, auto[1])):
        xd = to_device(x)
        st = qk.qknorm_partial_sumsq(xd, P)
        y = qk.qknorm_apply(xd, to_device(g), st, wl.eps)
        torch.cuda.synchronize()
        assert torch.equal(bits(y), bits(out))
        S_or = orc.partial_sumsq(x, P, dtype)
        check_stats(st.cpu().numpy(), S_or, x.shape[1], P, dtype, name)


@pytest.mark.parametrize("grid", [1, 5, 148])
def test_persistent_stride_and_ragged_tail(qk, orc, grid):
    """Forced small grids: every CTA walks many tokens (prefetch path) and the
    last wave is partial; the result is bit-identical to the automatic plan."""
    wl = W.custom("stride", 3 * 148 + 7, 4096, 1024, 4, seed=31)
    q, k, gq, gk = _inputs(wl, wl.Ts[0])
    ref = _fwd(qk, wl, q, k, gq, gk)
    got = _fwd(qk, wl, q, k, gq, gk, variant="cta", grid=grid)
    assert torch.equal(bits(got[0]), bits(ref[0])) and torch.equal(bits(got[1]), bits(ref[1]))
    got_w = _fwd(qk, wl, q, k, gq, gk, variant="warp", grid=grid)
    assert torch.equal(bits(got_w[0]), bits(ref[0]))
    _check_oracle(orc, wl, q, k, gq, gk, *ref)


def test_plan_grid_tail(qk, orc):
    """T one past a multiple of the automatic persistent grid."""
    plan = qk.qknorm_launch_plan(100000, 5120, 5120, 4, qk.QKNORM_BF16)
    T = 2 * plan["grid"] + 1
    wl = W.custom("tail", T, 5120, 5120, 4, seed=32, x_sigma=1.5)
    q, k, gq, gk = _inputs(wl, T)
    oq, ok = _fwd(qk, wl, q, k, gq, gk)
    _check_oracle(orc, wl, q, k, gq, gk, oq, ok)


def test_empty_T(qk):
    e = torch.empty((0, 4096), dtype=torch.bfloat16, device="cuda")
    g = torch.ones(4096, dtype=torch.float32, device="cuda")
    oq, ok = qk.qknorm_fwd(e, e.clone(), g, g, 4, 1e-6)
    st = qk.qknorm_partial_sumsq(e, 4)
    y = qk.qknorm_apply(e, g, st, 1e-6)
    torch.cuda.synchronize()
    assert oq.shape == (0, 4096) and st.shape == (0, 4) and y.shape == (0, 4096)


def test_in_place(qk):
    wl = W.custom("inplace", 50, 2048, 1024, 4, seed=33)
    q, k, gq, gk = _inputs(wl, 50)
    ref = _fwd(qk, wl, q, k, gq, gk)
    qd, kd = to_device(q), to_device(k)
    qk.qknorm_fwd(qd, kd, to_device(gq), to_device(gk), 4, wl.eps, out_q=qd, out_k=kd)
    torch.cuda.synchronize()
    assert torch.equal(bits(qd), bits(ref[0])) and torch.equal(bits(kd), bits(ref[1]))
    xd = to_device(q)
    st = qk.qknorm_partial_sumsq(xd, 4)
    qk.qknorm_apply(xd, to_device(gq), st, wl.eps, out=xd)
    torch.cuda.synchronize()
    assert torch.equal(bits(xd), bits(ref[0]))


GUARD_CASES = [
    # variant, T, Dq, Dk, P, dtype
    (None, 37, 5120, 1024, 8, "bf16"),
    ("cta", 2 * 148 + 41, 5120, 1024, 8, "bf16"),
    ("bulk", 2 * 148 + 41, 5120, 1024, 8, "bf16"),
    ("rows", 2 * 148 + 41, 5120, 1024, 8, "bf16"),
    ("pair", 2 * 148 + 41, 5120, 1024, 8, "bf16"),
    ("generic", 2 * 148 + 41, 5120, 1024, 8, "bf16"),
    ("bulk", 2 * 148 + 41, 5120, 5120, 4, "e4m3"),     # the FP8 half-slot mode
    ("pair", 2 * 148 + 41, 5120, 1024, 8, "e4m3"),
    ("pair", 2 * 148 + 41, 5120, 4096, 8, "bf16"),     # K shards in pairs, ragged Q lanes
    (None, 2 * 148 + 41, 4096, 4096, 8, "e4m3"),       # FP8 K pairs, one vector per lane
]


@pytest.mark.parametrize("variant,T,Dq,Dk,P,dtype", GUARD_CASES)
def test_guard_regions_and_const_inputs(qk, variant, T, Dq, Dk, P, dtype):
    """Outputs sit inside larger buffers filled with a canary pattern; after
    the calls (every kernel variant, ragged lanes, tokens that wrap the
    persistent grid) the canaries and the inputs are byte-identical to before."""
    wl = W.custom("guard", T, Dq, Dk, P, dtype=dtype, seed=34)
    q, k, gq, gk = _inputs(wl, T)
    qd, kd, gqd, gkd = (to_device(a) for a in (q, k, gq, gk))
    saved = [t.clone() for t in (qd, kd, gqd, gkd)]
    pad = 4096  # elements of guard on each side (keeps 16-byte alignment)
    def canary(n):
        if dtype == "e4m3":   # the code 0xd6 (-14.0)
            return torch.full((n,), 0xD6, dtype=torch.uint8, device="cuda").view(torch.float8_e4m3fn)
        return torch.full((n,), -77.0, dtype=torch.bfloat16 if dtype == "bf16" else torch.float32,
                          device="cuda")
    bq = canary(T * Dq + 2 * pad)
    bk = canary(T * Dk + 2 * pad)
    bs = torch.full((T * P + 2 * pad,), -5.5, dtype=torch.float32, device="cuda")
    bcopy = [b.clone() for b in (bq, bk, bs)]
    oq = bq[pad:pad + T * Dq].view(T, Dq)
    ok = bk[pad:pad + T * Dk].view(T, Dk)
    st = bs[pad:pad + T * P].view(T, P)
    vid = {None: qk.VARIANT_AUTO, "cta": qk.VARIANT_CTA, "bulk": qk.VARIANT_BULK,
           "rows": qk.VARIANT_ROWS, "pair": qk.VARIANT_PAIR, "generic": qk.VARIANT_GENERIC}[variant]
    qk.qknorm_force_variant(vid, 0)
    try:
        qk.qknorm_fwd(qd, kd, gqd, gkd, P, wl.eps, out_q=oq, out_k=ok)
    finally:
        qk.qknorm_force_variant(qk.VARIANT_AUTO, 0)
    qk.qknorm_partial_sumsq(qd, P, stats=st)
    torch.cuda.synchronize()
    for b, c in zip((bq, bk, bs), bcopy):
        assert torch.equal(bits(b[:pad]), bits(c[:pad])) and torch.equal(bits(b[-pad:]), bits(c[-pad:]))
    for t, s_ in zip((qd, kd, gqd, gkd), saved):
        assert torch.equal(bits(t), bits(s_))
    ref = _fwd(qk, wl, q, k, gq, gk, variant="generic")
    assert torch.equal(bits(oq), bits(ref[0])) and torch.equal(bits(ok), bits(ref[1]))
    assert qk.qknorm_device_errors() == 0


def test_rejected_call_launches_nothing(qk):
    x = torch.randn(8, 1000, device="cuda").to(torch.bfloat16)
    g = torch.ones(1000, device="cuda")
    out = torch.full_like(x, 3.0)
    with pytest.raises(qk.QKNormError) as ei:
        qk.qknorm_fwd(x, x, g, g, 3, 1e-6, out_q=out, out_k=out.clone())   # D % P != 0
    assert ei.value.status == qk.QKNORM_ERR_INVALID_ARG
    with pytest.raises(qk.QKNormError) as ei:
        qk.qknorm_fwd(x, x, g, g, 50, 1e-6, out_q=out, out_k=out.clone())  # 20-wide shards
    assert ei.value.status == qk.QKNORM_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert bool((out == 3.0).all())


def test_more_than_2_31_elements(qk, orc):
    """Row offsets beyond 2^31 elements: T = 2^19 + 5 rows of 4096 bf16 (input
    drawn on the device); the oracle checks rows at both ends."""
    T, D, P = (1 << 19) + 5, 4096, 8
    q = W.gen_device_normal(T, D, seed=41, dtype=torch.bfloat16, device="cuda")
    k = W.gen_device_normal(T, D, seed=42, dtype=torch.bfloat16, device="cuda")
    g = torch.from_numpy(W.gen_gamma(W.custom("big", 1, D, D, P, seed=43), "q")).cuda()
    oq, ok = qk.qknorm_fwd(q, k, g, g, P, 1e-6)
    st = qk.qknorm_partial_sumsq(k, P)
    ak = qk.qknorm_apply(k, g, st, 1e-6)
    torch.cuda.synchronize()
    assert torch.equal(bits(ak), bits(ok))
    rows = torch.tensor(list(range(0, 4)) + list(range(T - 70, T)), device="cuda")
    gh = g.cpu().numpy()
    for x, y in ((q, oq), (k, ok)):
        xs = to_host(x.index_select(0, rows))
        y_or, _ = orc.rmsnorm(xs, gh, P, float(np.float32(1e-6)), "bf16")
        check_outputs(to_host(y.index_select(0, rows)), y_or, "bf16", "2^31+ rows")
    del q, k, oq, ok, ak, st
    torch.cuda.empty_cache()


@pytest.mark.parametrize("stages", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("tokens_per_stage", [1, 2])
@pytest.mark.parametrize("gamma_regs", [0, 1])
def test_bulk_ring_depths(qk, stages, tokens_per_stage, gamma_regs):
    """Every ring depth, token batch and gamma placement gives the same bits,
    with grids that make CTAs wrap the ring several times and end mid-stage."""
    wl = W.custom("ring", 2 * 148 + 37, 5120, 1024, 8, seed=35)
    q, k, gq, gk = _inputs(wl, wl.Ts[0])
    ref = _fwd(qk, wl, q, k, gq, gk, variant="generic")
    try:
        qk.qknorm_set_tuning(stages=stages, tokens_per_stage=tokens_per_stage, gamma_regs=gamma_regs)
        ring = stages * tokens_per_stage * (5120 + 1024) * 2
        if ring > 220 * 1024:      # more than one CTA's shared memory: rejected before launch
            with pytest.raises(qk.QKNormError) as ei:
                _fwd(qk, wl, q, k, gq, gk, variant="bulk")
            assert ei.value.status == qk.QKNORM_ERR_UNSUPPORTED
            return
        for grid in (0, 7, 148):
            got = _fwd(qk, wl, q, k, gq, gk, variant="bulk", grid=grid)
            assert torch.equal(bits(got[0]), bits(ref[0])) and torch.equal(bits(got[1]), bits(ref[1]))
    finally:
        qk.qknorm_set_tuning()
    assert qk.qknorm_device_errors() == 0


def test_bounded_wait_times_out_and_reports(qk):
    """A wait on an mbarrier nobody arrives on gives up after its limit, sets
    the error bit, and leaves the context usable."""
    assert qk.qknorm_device_errors(clear=True) == 0
    qk.qknorm_selftest_bounded_wait(20_000_000)        # 20 ms
    torch.cuda.synchronize()
    assert qk.qknorm_device_errors(clear=True) & 1
    assert qk.qknorm_device_errors(clear=False) == 0
    x = torch.ones(4, 256, device="cuda")               # the context still works
    g = torch.ones(256, device="cuda")
    oq, _ = qk.qknorm_fwd(x, x.clone(), g, g, 2, 0.0)
    torch.cuda.synchronize()
    assert bool((oq == 1.0).all())


@pytest.mark.parametrize("wq,wk,stages,gsm", [(1, 1, 1, 0), (1, 1, 3, 1), (2, 1, 2, 0), (5, 1, 2, 1),
                                               (3, 4, 1, 1), (7, 1, 3, 0), (0, 0, 0, -1), (0, 0, 3, 0)])
@pytest.mark.parametrize("grid", [0, 1, 5])
def test_rows_variant_rings(qk, wq, wk, stages, gsm, grid):
    """Warp-per-row kernel: any Q and K pool sizes, ring depth, gamma staging
    and grid (rows wrap the rings many times; the two pools have rings of
    their own row widths) gives the same bits as the generic kernel."""
    wl = W.custom("rows", 2 * 148 + 41, 5120, 1024, 8, seed=36)
    q, k, gq, gk = _inputs(wl, wl.Ts[0])
    ref = _fwd(qk, wl, q, k, gq, gk, variant="generic")
    try:
        qk.qknorm_set_rows_tuning(wq, wk, stages, gsm)
        got = _fwd(qk, wl, q, k, gq, gk, variant="rows", grid=grid)
    finally:
        qk.qknorm_set_rows_tuning()
    assert torch.equal(bits(got[0]), bits(ref[0])) and torch.equal(bits(got[1]), bits(ref[1]))
    assert qk.qknorm_device_errors() == 0


@pytest.mark.parametrize("T,Dq,Dk,P", [(2 * 148 + 41, 5120, 1024, 8), (700, 4096, 1024, 8),
                                        (301, 2048, 256, 4), (150, 1536, 256, 2),
                                        # K shards wider than 16 vectors: K in pairs too
                                        (2 * 148 + 41, 4096, 4096, 8), (301, 5120, 4096, 8),
                                        (150, 2048, 2048, 4), (77, 1024, 1536, 2)])
@pytest.mark.parametrize("grid,stages", [(0, 0), (1, 1), (5, 3), (0, 1)])
def test_pair_variant(qk, T, Dq, Dk, P, grid, stages):
    """The shard-pair token ring (two Q shards per warp; two K shards on lane
    halves, or in pairs like Q's when wider than 16 vectors): any grid (tokens
    wrap the ring many times) and ring depth gives the same bits as the
    generic kernel."""
    wl = W.custom("pair", T, Dq, Dk, P, seed=38 + P)
    q, k, gq, gk = _inputs(wl, wl.Ts[0])
    ref = _fwd(qk, wl, q, k, gq, gk, variant="generic")
    try:
        qk.qknorm_set_tuning(stages, 0, -1, 0)
        got = _fwd(qk, wl, q, k, gq, gk, variant="pair", grid=grid)
    finally:
        qk.qknorm_set_tuning()
    assert torch.equal(bits(got[0]), bits(ref[0])) and torch.equal(bits(got[1]), bits(ref[1]))
    assert qk.qknorm_device_errors() == 0


@pytest.mark.parametrize("variant", ["cta", "bulk", "rows", "pair", "generic"])
def test_dependent_launches_with_pdl(qk, variant):
    """Each call reads the previous call's output. With programmatic dependent
    launch every kernel waits for the previous grid before reading memory, so
    a chain launched back to back equals the same chain with a device
    synchronisation after every call, and the chain with PDL off."""
    # (the shard-pair ring needs K shards of <= 16 vectors: P = 8 there)
    wl = W.custom("chain", 3 * 148 + 5, 4096, 1024, 8 if variant == "pair" else 4, seed=37)
    q, k, gq, gk = _inputs(wl, wl.Ts[0])
    vid = {"cta": qk.VARIANT_CTA, "bulk": qk.VARIANT_BULK, "rows": qk.VARIANT_ROWS,
           "pair": qk.VARIANT_PAIR, "generic": qk.VARIANT_GENERIC}[variant]
    gqd, gkd = to_device(gq), to_device(gk)

    def chain(pdl, sync):
        qk.qknorm_set_pdl(pdl)
        qk.qknorm_force_variant(vid, 0)
        try:
            a, b = to_device(q), to_device(k)
            for _ in range(6):
                a, b = qk.qknorm_fwd(a, b, gqd, gkd, wl.P, wl.eps)
                st = qk.qknorm_partial_sumsq(a, wl.P)       # split kernels in the chain too
                a = qk.qknorm_apply(a, gqd, st, wl.eps)
                if sync:
                    torch.cuda.synchronize()
            torch.cuda.synchronize()
            return a, b
        finally:
            qk.qknorm_set_pdl(True)
            qk.qknorm_force_variant(qk.VARIANT_AUTO, 0)

    ref = chain(False, True)
    for pdl in (True, False):
        got = chain(pdl, False)
        assert torch.equal(bits(got[0]), bits(ref[0])) and torch.equal(bits(got[1]), bits(ref[1]))


@pytest.mark.parametrize("variant", ["auto", "cta", "bulk", "rows", "generic"])
@pytest.mark.parametrize("T", [37, 3 * 148 + 5])
def test_strided_qkv_in_place(qk, variant, T):
    """Q and K normalised in place inside a fused QKV buffer [T, Dq + 2 Dk]
    (row stride Dq + 2 Dk): the slices equal dense calls bit for bit, V and
    the padding are untouched; also strided in, dense out and dense in,
    strided out."""
    Dq, Dk, P = 2048, 512, 4
    wl = W.custom("qkv", T, Dq, Dk, P, seed=38)
    q, k, gq, gk = _inputs(wl, T)
    ref = _fwd(qk, wl, q, k, gq, gk, variant=None if variant == "auto" else variant)
    qd, kd = to_device(q), to_device(k)
    ld = Dq + 2 * Dk + 64                        # QKV row plus 64 elements of padding
    buf = torch.full((T, ld), 5.0, dtype=torch.bfloat16, device="cuda")
    buf[:, :Dq] = qd
    buf[:, Dq:Dq + Dk] = kd
    untouched = buf[:, Dq + Dk:].clone()
    vid = {"auto": qk.VARIANT_AUTO, "cta": qk.VARIANT_CTA, "bulk": qk.VARIANT_BULK,
           "rows": qk.VARIANT_ROWS, "generic": qk.VARIANT_GENERIC}[variant]
    gqd, gkd = to_device(gq), to_device(gk)
    qk.qknorm_force_variant(vid, 0)
    try:
        qs, ks = buf[:, :Dq], buf[:, Dq:Dq + Dk]
        dq, dk = qk.qknorm_fwd_strided(qs, ks, gqd, gkd, P, wl.eps)           # strided in, dense out
        qk.qknorm_fwd_strided(qs, ks, gqd, gkd, P, wl.eps, out_q=qs, out_k=ks)  # in place
        buf2 = torch.zeros((T, ld), dtype=torch.bfloat16, device="cuda")
        qk.qknorm_fwd_strided(qd, kd, gqd, gkd, P, wl.eps, out_q=buf2[:, :Dq],
                              out_k=buf2[:, Dq:Dq + Dk])                      # dense in, strided out
        torch.cuda.synchronize()
    finally:
        qk.qknorm_force_variant(qk.VARIANT_AUTO, 0)
    for got_q, got_k in ((dq, dk), (buf[:, :Dq], buf[:, Dq:Dq + Dk]), (buf2[:, :Dq], buf2[:, Dq:Dq + Dk])):
        assert torch.equal(bits(got_q.contiguous()), bits(ref[0]))
        assert torch.equal(bits(got_k.contiguous()), bits(ref[1]))
    assert torch.equal(bits(buf[:, Dq + Dk:]), bits(untouched))
    assert bool((buf2[:, Dq + Dk:] == 0).all())
