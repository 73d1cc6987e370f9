"""GPU parity of the decode kernels through the C ABI: the warp-per-token
kernel (one warp owns a token's Q and K rows in registers) and the
CTA-per-token kernel with and without its gamma registers, against each
other (bit for bit: one reduction order) and against the float64 oracle, at
the decode sizes (T <= 64) and through the persistent stride loop."""
import zlib

import numpy as np
import pytest
import torch

import oracle
import qknorm_workloads as W
from gpu_util import bits, check_outputs, to_device, to_host

pytestmark = pytest.mark.gpu

SHAPES = [
    # name, Dq, Dk, P, dtype, the warp kernel's (vq, vk)
    ("decode_olmo2", 4096, 4096, 4, "bf16", (4, 4)),
    ("gqa", 5120, 1024, 8, "bf16", (3, 1)),
    ("decode_e4m3", 4096, 4096, 4, "e4m3", (2, 2)),
    ("tiny_f32", 256, 256, 2, "f32", (1, 1)),
    ("ragged_k", 4096, 640, 4, "bf16", (4, 1)),      # K shards of 20 vectors: lanes 20-31 idle
]


@pytest.fixture(scope="module")
def qk():
    import qk_norm_attention_b200 as qk
    yield qk
    qk.qknorm_force_variant(qk.VARIANT_AUTO, 0)
    qk.qknorm_set_tuning()


@pytest.fixture(scope="module")
def orc():
    return oracle.get()


def _run(qk, variant, args, P, grid=0, gamma_regs=-1):
    qk.qknorm_force_variant(variant, grid)
    qk.qknorm_set_tuning(gamma_regs=gamma_regs)
    try:
        out = qk.qknorm_fwd(*args, P, 1e-6)
        torch.cuda.synchronize()
    finally:
        qk.qknorm_force_variant(qk.VARIANT_AUTO, 0)
        qk.qknorm_set_tuning()
    return out


@pytest.mark.parametrize("shape", SHAPES, ids=[s[0] for s in SHAPES])
def test_warp_kernel_plan(qk, shape):
    name, Dq, Dk, P, dtype, (vq, vk) = shape
    code = {"bf16": qk.QKNORM_BF16, "f32": qk.QKNORM_F32, "e4m3": qk.QKNORM_E4M3}[dtype]
    qk.qknorm_force_variant(qk.VARIANT_WARP, 0)
    try:
        pl = qk.qknorm_launch_plan(64, Dq, Dk, P, code)
    finally:
        qk.qknorm_force_variant(qk.VARIANT_AUTO, 0)
    assert pl["variant"] == qk.VARIANT_WARP and (pl["vmax"], pl["vmax_k"]) == (vq, vk)
    assert pl["block"] == 32 and pl["grid"] == 64


@pytest.mark.parametrize("T", [1, 8, 64, 333])
@pytest.mark.parametrize("shape", SHAPES, ids=[s[0] for s in SHAPES])
def test_decode_kernels_bit_identical_and_oracle(qk, orc, shape, T):
    name, Dq, Dk, P, dtype, _ = shape
    wl = W.custom(name, T, Dq, Dk, P, dtype=dtype, seed=zlib.crc32(name.encode()) % 997 + T)
    q, k = W.gen_rows(wl, "q", range(T)), W.gen_rows(wl, "k", range(T))
    gq, gk = W.gen_gamma(wl, "q"), W.gen_gamma(wl, "k")
    args = (to_device(q), to_device(k), to_device(gq), to_device(gk))
    outs = {
        "warp": _run(qk, qk.VARIANT_WARP, args, P),
        "warp_grid5": _run(qk, qk.VARIANT_WARP, args, P, grid=5),        # stride loop
        "cta_greg": _run(qk, qk.VARIANT_CTA, args, P, gamma_regs=1),
        "cta_l1": _run(qk, qk.VARIANT_CTA, args, P, gamma_regs=0),
        "generic": _run(qk, qk.VARIANT_GENERIC, args, P),
        "auto": _run(qk, qk.VARIANT_AUTO, args, P),
    }
    ref = outs["generic"]
    for v, (oq, ok) in outs.items():
        assert torch.equal(bits(oq), bits(ref[0])), f"{v} Q differs from generic"
        assert torch.equal(bits(ok), bits(ref[1])), f"{v} K differs from generic"
    yq, yk, _, _ = orc.qknorm(q, k, gq, gk, P, float(np.float32(1e-6)), dtype, nthreads=8)
    check_outputs(to_host(ref[0]), yq, dtype, f"{name} T={T} q")
    check_outputs(to_host(ref[1]), yk, dtype, f"{name} T={T} k")


def test_warp_kernel_strided_in_place(qk, orc):
    """Q and K as slices of one fused QKV buffer, normalised in place by the
    warp kernel: equal to the dense call, and V untouched."""
    T, Dq, Dk, P = 37, 4096, 1024, 4
    wl = W.custom("wstride", T, Dq, Dk, P, seed=88)
    q, k = W.gen_rows(wl, "q", range(T)), W.gen_rows(wl, "k", range(T))
    gq, gk = to_device(W.gen_gamma(wl, "q")), to_device(W.gen_gamma(wl, "k"))
    qkv = torch.cat([to_device(q), to_device(k), to_device(k)], dim=1).contiguous()
    v_before = qkv[:, Dq + Dk:].clone()
    ld = Dq + 2 * Dk
    qk.qknorm_force_variant(qk.VARIANT_WARP, 0)
    try:
        qs, ks = qkv[:, :Dq], qkv[:, Dq:Dq + Dk]
        qk.qknorm_fwd_strided(qs, ks, gq, gk, P, 1e-6, out_q=qs, out_k=ks)
        ref = qk.qknorm_fwd(to_device(q), to_device(k), gq, gk, P, 1e-6)
        torch.cuda.synchronize()
    finally:
        qk.qknorm_force_variant(qk.VARIANT_AUTO, 0)
    assert qkv.stride(0) == ld
    assert torch.equal(bits(qkv[:, :Dq].contiguous()), bits(ref[0]))
    assert torch.equal(bits(qkv[:, Dq:Dq + Dk].contiguous()), bits(ref[1]))
    assert torch.equal(bits(qkv[:, Dq + Dk:].contiguous()), bits(v_before))
