"""GPU: qknorm_fwd_host (host rows in, host rows out, chunked and pipelined
over three workspace sets and two copy streams) equals qknorm_fwd on the
device bit for bit, for chunk sizes that divide T and that leave a ragged
last chunk, pinned and pageable host memory, and calls back to back that
reuse one workspace."""
import pytest
import torch

import qknorm_workloads as W
from gpu_util import bits, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def qk():
    import qk_norm_attention_b200 as qk
    qk.qknorm_force_variant(qk.VARIANT_AUTO, 0)
    return qk


def _host(t: torch.Tensor, pinned: bool) -> torch.Tensor:
    h = t.cpu()
    return h.pin_memory() if pinned else h


@pytest.mark.parametrize("T,Dq,Dk,P,dtype,chunk,pinned", [
    (1500, 5120, 1024, 8, "bf16", 0, True),       # default chunks: 1024 + 476 tokens
    (1000, 4096, 4096, 4, "bf16", 7, True),       # many chunks, ragged last
    (333, 256, 256, 2, "f32", 100, False),        # pageable memory
    (640, 4096, 1024, 8, "e4m3", 64, True),
    (1, 4096, 4096, 4, "bf16", 0, True),
])
def test_host_path_equals_device_path(qk, T, Dq, Dk, P, dtype, chunk, pinned):
    wl = W.custom("host", T, Dq, Dk, P, dtype=dtype, seed=71)
    q, k = to_device(W.gen_rows(wl, "q", range(T))), to_device(W.gen_rows(wl, "k", range(T)))
    gq, gk = to_device(W.gen_gamma(wl, "q")), to_device(W.gen_gamma(wl, "k"))
    oq, ok = qk.qknorm_fwd(q, k, gq, gk, P, 1e-6)
    ws = torch.empty(qk.qknorm_fwd_host_workspace(Dq, Dk, q.dtype, chunk), dtype=torch.uint8,
                     device="cuda")
    qh, kh = _host(q, pinned), _host(k, pinned)
    hq, hk = qk.qknorm_fwd_host(qh, kh, gq, gk, P, 1e-6, ws, chunk_tokens=chunk)
    torch.cuda.current_stream().synchronize()
    assert torch.equal(bits(hq), bits(oq.cpu())) and torch.equal(bits(hk), bits(ok.cpu()))


def test_host_calls_back_to_back_share_a_workspace(qk):
    """Three calls enqueued without a synchronisation, one workspace: each
    call's copies into a set wait for that set's previous copy-out."""
    T, D, P = 700, 2048, 4
    wl = W.custom("host2", T, D, D, P, dtype="bf16", seed=72)
    g = to_device(W.gen_gamma(wl, "q"))
    ws = torch.empty(qk.qknorm_fwd_host_workspace(D, D, torch.bfloat16, 64), dtype=torch.uint8,
                     device="cuda")
    ins, outs, refs = [], [], []
    for i in range(3):
        x = to_device(W.gen_rows(W.custom("host2", T, D, D, P, dtype="bf16", seed=73 + i), "q", range(T)))
        refs.append(qk.qknorm_fwd(x, x, g, g, P, 1e-6)[0].cpu())
        ins.append(_host(x, True))
    for xh in ins:
        outs.append(qk.qknorm_fwd_host(xh, xh, g, g, P, 1e-6, ws, chunk_tokens=64))
    torch.cuda.current_stream().synchronize()
    for (hq, hk), ref in zip(outs, refs):
        assert torch.equal(bits(hq), bits(ref)) and torch.equal(bits(hk), bits(ref))
