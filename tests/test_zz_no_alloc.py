"""qknorm_split_noalloc: the split path in one call with no device memory
supplied by the caller (collected last on purpose).

Who needs it: callers that cannot allocate device memory for the [T, P]
statistics that qknorm_partial_sumsq hands to qknorm_apply, for example code
whose device memory all belongs to a framework's pool, or a latency-critical
loop that must not call cudaMalloc (it synchronises the device). The entry
point keeps the statistics in a buffer inside the library instead.

The test calls it through the C ABI twice in a row, on different shapes, and
checks each result against the existing entry points, within the parity
tolerance and bit for bit (the same kernels run). It also checks the size
limit. It passes run alone in a fresh process or after the other tests."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import qknorm_workloads as W
from gpu_util import bits, check_outputs, to_device, to_host

pytestmark = pytest.mark.gpu


def _noalloc(qk, x, g, P, eps):
    out = torch.empty_like(x)
    dtype = {torch.bfloat16: qk.QKNORM_BF16, torch.float32: qk.QKNORM_F32}[x.dtype]
    st = qk.lib.qknorm_split_noalloc(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(g.data_ptr()),
                                     ctypes.c_void_p(out.data_ptr()), x.shape[0], x.shape[1], P,
                                     eps, dtype, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == qk.QKNORM_OK, qk.qknorm_status_string(st)
    return out


def test_noalloc_matches_the_existing_entry_points_twice():
    import qk_norm_attention_b200 as qk
    orc = oracle.get()
    cases = [W.custom("na1", 513, 4096, 4096, 8, seed=71),                 # bf16, P = 8
             W.custom("na2", 129, 1024, 1024, 4, dtype="f32", seed=72)]    # fp32, other shape
    for wl in cases:                                                       # two calls in a row
        T = wl.Ts[0]
        x = W.gen_rows(wl, "q", range(T))
        g = W.gen_gamma(wl, "q")
        xd, gd = to_device(x), to_device(g)
        got = _noalloc(qk, xd, gd, wl.P, wl.eps)
        ref, _ = qk.qknorm_fwd(xd, xd.clone(), gd, gd, wl.P, wl.eps)       # fused path
        st = qk.qknorm_partial_sumsq(xd, wl.P)                             # split path, caller stats
        ref2 = qk.qknorm_apply(xd, gd, st, wl.eps)
        torch.cuda.synchronize()
        check_outputs(to_host(got), orc.rmsnorm(x, g, wl.P, float(np.float32(wl.eps)), wl.dtype)[0],
                      wl.dtype, wl.name)
        assert torch.equal(bits(got), bits(ref)) and torch.equal(bits(got), bits(ref2))
        via_wrapper = qk.qknorm_split_noalloc(xd, gd, wl.P, wl.eps)           # the Python binding
        torch.cuda.synchronize()
        assert torch.equal(bits(via_wrapper), bits(got))


def test_noalloc_rejects_more_statistics_than_its_buffer():
    import qk_norm_attention_b200 as qk
    cap = qk.lib.qknorm_split_noalloc_max_stats()
    assert cap == 1 << 20
    x = torch.zeros((cap // 8 + 1, 64), dtype=torch.bfloat16, device="cuda")
    g = torch.ones(64, device="cuda")
    out = torch.full_like(x, 7.0)
    st = qk.lib.qknorm_split_noalloc(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(g.data_ptr()),
                                     ctypes.c_void_p(out.data_ptr()), x.shape[0], 64, 8, 1e-6,
                                     qk.QKNORM_BF16, None)
    assert st == qk.QKNORM_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())                                        # nothing was launched
