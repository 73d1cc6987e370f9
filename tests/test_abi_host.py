"""Host-side checks of libqknorm (CPU only, no kernel launches): the library
loads, exports every function the header declares, validates arguments before
touching CUDA, and the selector plans the expected launches.

Argument checks use fake addresses. The few calls that pass validation reach
the CUDA runtime, which finds no device; these tests skip themselves on a
machine with a GPU, so no fake address can ever reach a kernel."""
import ctypes
import math
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qknorm.h")


@pytest.fixture(scope="module")
def qk():
    import runpy
    runpy.run_path(os.path.join(ROOT, "qk_norm_attention_b200", "csrc", "build_lib.py"))["build"]()
    import qk_norm_attention_b200 as qk
    return qk


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"QKNORM_API\s+(?:int|int64_t|const char \*)\s*(qknorm_\w+)\s*\(", src)))


def test_header_declares_the_api():
    names = declared_functions()
    for want in ("qknorm_fwd", "qknorm_partial_sumsq", "qknorm_apply", "qknorm_status_string"):
        assert want in names


def test_every_declared_symbol_is_exported(qk):
    lib = ctypes.CDLL(qk.LIBRARY)
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in qknorm.h but not exported"


def test_status_strings(qk):
    assert qk.qknorm_status_string(0) == "ok"
    for s in range(1, 5):
        assert qk.qknorm_status_string(s) not in ("ok", "unknown status")
    assert qk.qknorm_status_string(99) == "unknown status"
    assert qk.qknorm_version() // 100 == 1          # ABI major version


# ----------------------------------------------------------------- argument checks

needs_cpu = pytest.mark.skipif(
    __import__("torch").cuda.is_available(),
    reason="fake-address checks run only on machines without a GPU")

A = 0x10000          # fake, 16-byte aligned addresses far apart
B = 0x20000000
C = 0x40000000
Dd = 0x60000000
E = 0x80000000
F = 0xA0000000


def fwd(qk, q=A, k=B, gq=C, gk=Dd, oq=E, ok=F, T=4, Dq=256, Dk=256, P=2, eps=1e-6, dtype=1):
    return qk.lib.qknorm_fwd(q, k, gq, gk, oq, ok, T, Dq, Dk, P, eps, dtype, None)


@needs_cpu
@pytest.mark.parametrize("kw,status", [
    (dict(T=-1), 1), (dict(Dq=0), 1), (dict(Dk=-8), 1), (dict(P=0), 1), (dict(P=-2), 1),
    (dict(Dq=250, P=4), 1),                    # D % P != 0
    (dict(eps=-1e-6), 1), (dict(eps=math.nan), 1), (dict(eps=math.inf), 1),
    (dict(q=0), 1), (dict(k=0), 1), (dict(gq=0), 1), (dict(gk=0), 1), (dict(oq=0), 1), (dict(ok=0), 1),
    (dict(dtype=3), 3), (dict(dtype=-1), 3),
    (dict(Dq=48, Dk=48, P=2, dtype=2), 3),     # 24-wide FP8 shards (need multiples of 16)
    (dict(Dq=40, Dk=40, P=2, dtype=1), 3),     # 20-wide bf16 shards
    (dict(Dq=24, Dk=24, P=4, dtype=0), 3),     # 6-wide fp32 shards
    (dict(q=A + 2), 2), (dict(k=B + 8), 2), (dict(gq=C + 4), 2), (dict(gk=Dd + 12), 2),
    (dict(oq=E + 2), 2), (dict(ok=F + 6), 2),
    (dict(oq=A + 16), 1),                      # output overlaps its input partly
    (dict(oq=B), 1),                           # output aliases the other input
    (dict(ok=E), 1),                           # the two outputs coincide
    (dict(oq=C), 1),                           # output on gamma
    (dict(ok=A), 1),                           # K output on Q input
])
def test_fwd_rejects(qk, kw, status):
    assert fwd(qk, **kw) == status


@needs_cpu
def test_fwd_T0_is_a_noop(qk):
    assert fwd(qk, T=0, q=0, k=0, gq=0, gk=0, oq=0, ok=0) == 0


@needs_cpu
def test_split_rejects(qk):
    L = qk.lib
    assert L.qknorm_partial_sumsq(A, B, 4, 250, 4, 1, None) == 1
    assert L.qknorm_partial_sumsq(A, B, 4, 256, 4, 5, None) == 3
    assert L.qknorm_partial_sumsq(A, B, 4, 256, 64, 1, None) == 3      # 4-wide bf16 shards
    assert L.qknorm_partial_sumsq(A + 2, B, 4, 256, 4, 1, None) == 2
    assert L.qknorm_partial_sumsq(A, B + 2, 4, 256, 4, 1, None) == 2     # stats need 4-byte alignment
    assert L.qknorm_partial_sumsq(A, A + 16, 4, 256, 4, 1, None) == 1  # stats inside x
    assert L.qknorm_partial_sumsq(0, B, 4, 256, 4, 1, None) == 1
    assert L.qknorm_partial_sumsq(0, 0, 0, 256, 4, 1, None) == 0
    assert L.qknorm_apply(A, B, C, Dd, 4, 256, 4, -1.0, 1, None) == 1
    assert L.qknorm_apply(A, B, C, Dd, 4, 256, 3, 1e-6, 1, None) == 1
    assert L.qknorm_apply(A, B, C, Dd + 2, 4, 256, 4, 1e-6, 1, None) == 2
    assert L.qknorm_apply(A, B, C, B, 4, 256, 4, 1e-6, 1, None) == 1   # out on gamma
    assert L.qknorm_apply(A, B, C, C, 4, 256, 4, 1e-6, 1, None) == 1   # out on stats
    assert L.qknorm_apply(A, B, C, A + 32, 4, 256, 4, 1e-6, 1, None) == 1
    assert L.qknorm_apply(A, B, C, Dd, 4, 256, 4, 1e-6, 9, None) == 3
    assert L.qknorm_apply(A, B, C + 2, Dd, 4, 256, 4, 1e-6, 1, None) == 2   # stats need 4-byte alignment


def test_host_workspace_size(qk):
    L = qk.lib
    assert L.qknorm_fwd_host_workspace(0, 5120, 5120, 1) == 3 * 1024 * 10240 * 2
    assert L.qknorm_fwd_host_workspace(7, 256, 128, 0) == 3 * 7 * 384 * 4
    assert L.qknorm_fwd_host_workspace(7, 256, 128, 2) == 3 * 7 * 384
    assert L.qknorm_fwd_host_workspace(7, 0, 128, 1) == -1
    assert L.qknorm_fwd_host_workspace(7, 256, 128, 9) == -1


@needs_cpu
def test_fwd_host_rejects(qk):
    L = qk.lib
    ws = L.qknorm_fwd_host_workspace(4, 256, 256, 1)    # T = 4 tokens make one chunk of 4
    # q, k, gamma_q, gamma_k, out_q, out_k, T, Dq, Dk, P, eps, dtype, ws, ws_bytes, chunk, stream
    base = [A, A + 0x100000, B, B + 0x1000, C, C + 0x100000, 4, 256, 256, 4, 1e-6, 1, Dd, ws, 0, None]
    call = lambda **kw: L.qknorm_fwd_host(*[kw.get(str(i), v) for i, v in enumerate(base)])
    assert call(**{"13": ws - 16}) == 1          # workspace too small
    assert call(**{"12": Dd + 8}) == 2           # workspace not 16-byte aligned
    assert call(**{"14": -1}) == 1               # negative chunk
    assert call(**{"4": A + 64}) == 1            # out_q partly over q
    assert call(**{"5": C + 512}) == 1           # out_k over out_q
    assert call(**{"6": 0}) == 0                 # T = 0
    assert call(**{"9": 3}) == 1                 # D % P
    assert call(**{"12": 0}) == 1                # no workspace


@needs_cpu
def test_apply_tp_rejects(qk):
    L = qk.lib
    # x, gamma, stats, block stride, out, T, D_local, P_local, ranks, eps, dtype, stream
    assert L.qknorm_apply_tp(A, B, C, 0, Dd, 4, 256, 4, 0, 1e-6, 1, None) == 1    # ranks < 1
    assert L.qknorm_apply_tp(A, B, C, -1, Dd, 4, 256, 4, 2, 1e-6, 1, None) == 1   # negative stride
    assert L.qknorm_apply_tp(A, B, C, 15, Dd, 4, 256, 4, 2, 1e-6, 1, None) == 1   # blocks overlap
    assert L.qknorm_apply_tp(A, B, C + 2, 0, Dd, 4, 256, 4, 2, 1e-6, 1, None) == 2
    assert L.qknorm_apply_tp(A + 8, B, C, 0, Dd, 4, 256, 4, 2, 1e-6, 1, None) == 2
    assert L.qknorm_apply_tp(A, B, C, 0, Dd, 4, 256, 3, 2, 1e-6, 1, None) == 1    # D_local % P_local
    assert L.qknorm_apply_tp(A, B, C, 0, C + 16, 4, 256, 4, 2, 1e-6, 1, None) == 1  # out on stats
    assert L.qknorm_apply_tp(0, 0, 0, 0, 0, 0, 256, 4, 2, 1e-6, 1, None) == 0     # T = 0


@needs_cpu
def test_two_tensor_calls_reject(qk):
    """qknorm_partial_sumsq_qk and qknorm_apply_tp_qk check each tensor as the
    one-tensor calls do, and also reject overlaps across the two tensors."""
    L = qk.lib
    # q, k, stats_q, stats_k, T, Dq, Dk, P, dtype, stream  (q 2 KiB at A, k 512 B at A + 4096)
    sbase = [A, A + 4096, C, C + 4096, 4, 256, 64, 4, 1, None]
    scall = lambda **kw: L.qknorm_partial_sumsq_qk(*[kw.get(str(i), v) for i, v in enumerate(sbase)])
    assert scall(**{"4": 0}) == 0                   # T = 0
    assert scall(**{"3": C + 32}) == 1              # stats_k over stats_q
    assert scall(**{"3": A}) == 1                   # stats_k over q
    assert scall(**{"2": A + 4096}) == 1            # stats_q over k
    assert scall(**{"6": 66}) == 1                  # Dk % P
    assert scall(**{"6": 60}) == 3                  # shard width not whole 16-byte vectors
    assert scall(**{"1": A + 4104}) == 2            # k misaligned
    assert scall(**{"8": 7}) == 3                   # no such dtype
    # q, k, gq, gk, stats_q, stats_k, stride, out_q, out_k, T, Dq, Dk, P_local, ranks, eps, dtype, stream
    abase = [A, A + 4096, B, B + 4096, C, C + 16, 32, Dd, Dd + 4096, 4, 256, 64, 4, 2, 1e-6, 1, None]
    acall = lambda **kw: L.qknorm_apply_tp_qk(*[kw.get(str(i), v) for i, v in enumerate(abase)])
    assert acall(**{"9": 0}) == 0                   # T = 0
    assert acall(**{"13": 0}) == 1                  # ranks < 1
    assert acall(**{"6": -1}) == 1                  # negative stride
    assert acall(**{"6": 15}) == 1                  # blocks overlap
    assert acall(**{"8": Dd + 64}) == 1             # out_k over out_q
    assert acall(**{"7": A + 4096}) == 1            # out_q over k
    assert acall(**{"8": B}) == 1                   # out_k over gamma_q
    assert acall(**{"7": C + 16}) == 1              # out_q over stats_k
    assert acall(**{"8": A}) == 1                   # out_k over q
    assert acall(**{"14": -1.0}) == 1               # eps < 0
    assert acall(**{"8": Dd + 4100}) == 2           # out_k misaligned


@needs_cpu
def test_valid_call_without_gpu_reports_cuda_error(qk):
    """All checks pass, then the runtime finds no device: QKNORM_ERR_CUDA with text."""
    assert fwd(qk) == 4
    assert qk.qknorm_last_error() != ""


# ----------------------------------------------------------------- the selector

def test_auto_k_pairs(qk):
    """The selector puts K shards in pairs (P warps per token) for FP8 at one
    vector per lane and for ragged bf16 lanes, keeps the ring with 2P warps
    for full bf16 lanes, and gives FP8 at two or more vectors per lane the
    shard pairs with gamma staged in shared memory."""
    qk.qknorm_force_variant(qk.VARIANT_AUTO, 0)
    cases = [((65536, 4096, 4096, 8, qk.QKNORM_E4M3), (qk.VARIANT_PAIR, 1)),
             ((16384, 2048, 2048, 4, qk.QKNORM_E4M3), (qk.VARIANT_PAIR, 1)),
             ((8192, 5120, 4096, 8, qk.QKNORM_BF16), (qk.VARIANT_PAIR, 1)),
             ((16384, 4096, 4096, 4, qk.QKNORM_E4M3), (qk.VARIANT_GPAIR, 0)),
             ((65536, 4096, 4096, 8, qk.QKNORM_BF16), (qk.VARIANT_BULK, 0)),
             ((8192, 5120, 5120, 4, qk.QKNORM_E4M3), (qk.VARIANT_GPAIR, 0))]
    for shape, (variant, kp) in cases:
        pl = qk.qknorm_plan_fwd(*shape, 148, 2)
        assert (pl["variant"], pl["k_pairs"]) == (variant, kp), shape
        if variant == qk.VARIANT_PAIR:
            assert pl["block"] == shape[3] * 32 and pl["gamma_regs"] == 1


def test_plan_for_each_workload(qk):
    import qknorm_workloads as W
    qk.qknorm_force_variant(qk.VARIANT_AUTO, 0)
    dt = {"bf16": qk.QKNORM_BF16, "f32": qk.QKNORM_F32}
    want_block = {"tiny": 4 * 32, "decode": 8 * 32, "prefill13b": 8 * 32, "gqa": 16 * 32,
                  "split_large": 16 * 32}
    want_vmax = {"tiny": 1, "decode": 4, "prefill13b": 5, "gqa": 3, "split_large": 2}
    for name in want_block:
        wl = W.WORKLOADS[name]
        for T in wl.Ts:
            pl = qk.qknorm_plan_fwd(T, wl.Dq, wl.Dk, wl.P, dt[wl.dtype], 148, 4)
            # One token per CTA: registers only. Several: the token ring (one
            # token per stage, gamma in registers while vmax <= 3), or for the
            # GQA widths below 48 tokens per SM the staged-gamma shard-pair
            # ring compiled for that shape (P / 2 mixed warps per token: two Q
            # and two K shards each).
            if T <= 2 * 148:
                want = qk.VARIANT_CTA
            else:
                want = qk.VARIANT_GPAIR if name == "gqa" else qk.VARIANT_BULK
            assert pl["variant"] == want, (name, T)
            assert pl["groups_q"] == pl["groups_k"] == 1
            if want == qk.VARIANT_GPAIR:
                assert pl["block"] == wl.P // 2 * 32 and pl["mixed"] == 1 and pl["gamma_regs"] == 0
                assert (pl["vmax"], pl["vmax_k"], pl["half_slots"]) == (3, 1, 0)
                assert pl["stages"] == 2 and pl["tokens_per_stage"] == 1
                continue
            assert pl["block"] == want_block[name], name
            assert pl["vmax"] == want_vmax[name], name
            assert pl["grid"] == min(T, 148 * 4)
            if want == qk.VARIANT_BULK:
                small = want_vmax[name] <= 3
                assert pl["prefetch"] == 0 and pl["stages"] == 2
                assert pl["tokens_per_stage"] == 1
                assert pl["gamma_regs"] == (1 if small else 0)
                stage = (wl.Dq + wl.Dk) * wl.elem_bytes * pl["tokens_per_stage"]
                assert pl["smem_bytes"] >= pl["stages"] * stage
            else:
                assert pl["prefetch"] == int(T > 148 * 4) and pl["stages"] == 0


def test_full_lanes_flag(qk):
    """Guard-free kernels only where every lane holds exactly vmax vectors."""
    qk.qknorm_force_variant(qk.VARIANT_AUTO, 0)
    full = lambda *a: qk.qknorm_plan_fwd(*a, qk.QKNORM_BF16, 148)["full_lanes"]
    assert full(8, 4096, 4096, 4) == 1          # 128 vectors per shard: 4 per lane
    assert full(8, 5120, 5120, 4) == 1          # 160: 5 per lane
    assert full(8, 5120, 1024, 8) == 0          # 80 and 16: ragged
    assert full(8, 4096, 1024, 4) == 0          # 4 per lane for Q, 1 for K
    assert full(8, 4096, 4096, 1) == 1          # 512 = 2 groups x 32 lanes x 8


def test_plan_groups_and_fallbacks(qk):
    qk.qknorm_force_variant(qk.VARIANT_AUTO, 0)
    pl = qk.qknorm_plan_fwd(10, 4096, 4096, 1, qk.QKNORM_BF16, 148)      # nv = 512
    assert (pl["groups_q"], pl["vmax"], pl["block"]) == (2, 8, 4 * 32)
    pl = qk.qknorm_plan_fwd(10, 4096, 4096, 16, qk.QKNORM_BF16, 148)     # 32 tasks, 1 vector
    assert (pl["variant"], pl["block"], pl["vmax"]) == (qk.VARIANT_CTA, 1024, 1)
    pl = qk.qknorm_plan_fwd(10, 4096, 4096, 32, qk.QKNORM_BF16, 148)     # 64 tasks
    assert (pl["variant"], pl["block"]) == (qk.VARIANT_GENERIC, 256)
    pl = qk.qknorm_plan_fwd(10, 32768, 1024, 4, qk.QKNORM_BF16, 148)     # 20 tasks, vmax 8
    assert pl["variant"] == qk.VARIANT_GENERIC and pl["groups_q"] == 4
    with pytest.raises(qk.QKNormError):
        qk.qknorm_plan_fwd(10, 4096, 4096, 3, qk.QKNORM_BF16, 148)


def test_forced_variants(qk):
    try:
        qk.qknorm_force_variant(qk.VARIANT_WARP, 0)
        pl = qk.qknorm_plan_fwd(64, 4096, 4096, 4, qk.QKNORM_BF16, 148, 32)
        assert (pl["variant"], pl["block"], pl["grid"]) == (qk.VARIANT_WARP, 32, 64)
        # The register-resident warp kernel: (vectors per lane per Q shard, per K shard).
        assert (pl["vmax"], pl["vmax_k"], pl["smem_bytes"]) == (4, 4, 0)
        pl = qk.qknorm_plan_fwd(64, 5120, 1024, 8, qk.QKNORM_BF16, 148, 32)
        assert (pl["vmax"], pl["vmax_k"]) == (3, 1)
        pl = qk.qknorm_plan_fwd(64, 4096, 4096, 4, qk.QKNORM_E4M3, 148, 32)
        assert (pl["vmax"], pl["vmax_k"]) == (2, 2)
        # Beyond 32 vectors per lane (5 + 5 in 4 shards), or shards of two lane
        # groups: the looped one-warp form.
        for shape in ((5120, 5120, 4), (4096, 4096, 1)):
            pl = qk.qknorm_plan_fwd(64, *shape, qk.QKNORM_BF16, 148, 32)
            assert (pl["variant"], pl["vmax"], pl["block"]) == (qk.VARIANT_WARP, 0, 32)
        # The CTA kernel keeps gamma in registers while it is at most 32 floats
        # per lane and a CTA takes one token.
        qk.qknorm_force_variant(qk.VARIANT_CTA, 0)
        pl = qk.qknorm_plan_fwd(64, 4096, 4096, 4, qk.QKNORM_BF16, 148, 2)
        assert (pl["gamma_regs"], pl["prefetch"]) == (1, 0)
        pl = qk.qknorm_plan_fwd(64, 5120, 5120, 4, qk.QKNORM_BF16, 148, 2)    # 5 x 8 floats
        assert pl["gamma_regs"] == 0
        qk.qknorm_force_variant(qk.VARIANT_CTA, 8)
        pl = qk.qknorm_plan_fwd(64, 4096, 4096, 4, qk.QKNORM_BF16, 148, 2)    # 8 tokens per CTA
        assert (pl["gamma_regs"], pl["prefetch"]) == (0, 1)
        qk.qknorm_force_variant(qk.VARIANT_WARP, 0)
        qk.qknorm_force_variant(qk.VARIANT_CTA, 7)
        pl = qk.qknorm_plan_fwd(100, 4096, 4096, 4, qk.QKNORM_BF16, 148, 4)
        assert (pl["grid"], pl["prefetch"]) == (7, 1)
        qk.qknorm_force_variant(qk.VARIANT_CTA, 0)
        with pytest.raises(qk.QKNormError) as ei:
            qk.qknorm_plan_fwd(10, 4096, 4096, 32, qk.QKNORM_BF16, 148)
        assert ei.value.status == qk.QKNORM_ERR_UNSUPPORTED
        with pytest.raises(qk.QKNormError):
            qk.qknorm_force_variant(7, 0)
        # The shard-pair ring: P warps, GQA-like shapes only.
        qk.qknorm_force_variant(qk.VARIANT_PAIR, 0)
        pl = qk.qknorm_plan_fwd(4096, 5120, 1024, 8, qk.QKNORM_BF16, 148)
        assert (pl["variant"], pl["block"], pl["vmax"], pl["tokens_per_stage"], pl["k_pairs"]) == \
            (qk.VARIANT_PAIR, 8 * 32, 3, 1, 0)
        # K shards wider than 16 vectors go in pairs like Q's (vmax covers both tensors).
        pl = qk.qknorm_plan_fwd(4096, 5120, 4096, 8, qk.QKNORM_BF16, 148)
        assert (pl["variant"], pl["block"], pl["vmax"], pl["k_pairs"]) == (qk.VARIANT_PAIR, 8 * 32, 3, 1)
        pl = qk.qknorm_plan_fwd(4096, 4096, 4096, 8, qk.QKNORM_E4M3, 148)
        assert (pl["vmax"], pl["k_pairs"], pl["gamma_regs"]) == (1, 1, 1)
        pl = qk.qknorm_plan_fwd(4096, 4096, 4096, 4, qk.QKNORM_E4M3, 148)
        assert (pl["vmax"], pl["k_pairs"], pl["gamma_regs"]) == (2, 1, 0)   # 2 x 2 FP8 vectors: gamma via L1
        for shape in ((4096, 5120, 5120, 4), (4096, 5120, 5120, 2), (4096, 1280, 640, 5), (64, 4096, 512, 32)):
            with pytest.raises(qk.QKNormError) as ei:           # shards over 3 vectors per lane,
                qk.qknorm_plan_fwd(*shape, qk.QKNORM_BF16, 148)  # P odd, or P > 16
            assert ei.value.status == qk.QKNORM_ERR_UNSUPPORTED
        qk.qknorm_force_variant(qk.VARIANT_BULK, 0)
        qk.qknorm_set_tuning(stages=3, tokens_per_stage=2, gamma_regs=0)
        pl = qk.qknorm_plan_fwd(10, 4096, 4096, 8, qk.QKNORM_BF16, 148)   # vmax 2
        assert (pl["variant"], pl["stages"], pl["gamma_regs"], pl["tokens_per_stage"]) == \
            (qk.VARIANT_BULK, 3, 0, 2)
        assert pl["smem_bytes"] >= 3 * 2 * 2 * 4096 * 2
        assert pl["full_lanes"] == 1                        # 64 vectors = 2 per lane
        qk.qknorm_set_tuning(tokens_per_stage=2)            # vmax 8 x 2 tokens: no instance
        with pytest.raises(qk.QKNormError) as ei:
            qk.qknorm_plan_fwd(10, 4096, 4096, 2, qk.QKNORM_BF16, 148)
        assert ei.value.status == qk.QKNORM_ERR_UNSUPPORTED
        with pytest.raises(qk.QKNormError):
            qk.qknorm_set_tuning(tokens_per_stage=3)
        with pytest.raises(qk.QKNormError):
            qk.qknorm_set_tuning(tokens_per_stage=-1)
        with pytest.raises(qk.QKNormError) as ei:      # 64 tasks do not fit one CTA
            qk.qknorm_plan_fwd(10, 4096, 4096, 32, qk.QKNORM_BF16, 148)
        assert ei.value.status == qk.QKNORM_ERR_UNSUPPORTED
        with pytest.raises(qk.QKNormError):
            qk.qknorm_set_tuning(stages=17)
    finally:
        qk.qknorm_force_variant(qk.VARIANT_AUTO, 0)
        qk.qknorm_set_tuning()


def test_bulk_stages_fill_shared_memory(qk):
    """Stage count: as many token stages as fit in each CTA's share of the
    SM's 228 KiB (1 KiB reserved per CTA), at most 8. The host-only plan
    assumes 64 registers: 256 threads -> 4 CTAs per SM -> 56 KiB each ->
    two 20 KiB stages of the 13B prefill shape after the 384-byte header."""
    qk.qknorm_force_variant(qk.VARIANT_AUTO, 0)
    pl = qk.qknorm_plan_fwd(8192, 5120, 5120, 4, qk.QKNORM_BF16, 148)
    stage = 2 * 5120 * 2
    assert (pl["variant"], pl["tokens_per_stage"]) == (qk.VARIANT_BULK, 1)
    assert (pl["stages"], pl["smem_bytes"]) == (2, 1152 + 2 * stage)
    # A 1024-thread CTA (P = 16, one vector per lane) is alone on its SM:
    # two stages of one 16 KiB token (the automatic caps).
    try:
        qk.qknorm_force_variant(qk.VARIANT_BULK, 0)
        pl = qk.qknorm_plan_fwd(8192, 4096, 4096, 16, qk.QKNORM_BF16, 148)
        assert (pl["variant"], pl["stages"], pl["tokens_per_stage"]) == (qk.VARIANT_BULK, 2, 1)
        assert pl["smem_bytes"] == 1152 + 2 * 16384
    finally:
        qk.qknorm_force_variant(qk.VARIANT_AUTO, 0)


def test_rows_pools_plan(qk):
    """Warp-per-row plan: a Q pool and a K pool of warps (at least one each,
    at most 16 together), row stages per warp, CTAs that fit shared memory;
    the pools follow the widths, and a forced tuning is honoured."""
    try:
        qk.qknorm_force_variant(qk.VARIANT_ROWS, 0)
        for T, Dq, Dk, P in ((4096, 5120, 1024, 8), (65536, 4096, 4096, 8), (300, 256, 4096, 2)):
            pl = qk.qknorm_plan_fwd(T, Dq, Dk, P, qk.QKNORM_BF16, 148)
            W = pl["block"] // 32
            wq, wk = pl["q_warps"], W - pl["q_warps"]
            assert pl["variant"] == qk.VARIANT_ROWS and wq >= 1 and wk >= 1 and W <= 16
            assert pl["stages"] == 2 and pl["smem_bytes"] <= 227 * 1024
            if Dq > Dk:
                assert wq >= wk
            elif Dq < Dk:
                assert wq <= wk
            # every warp of the smaller pool gets a row, the grid stays persistent
            assert pl["grid"] <= -(-T // min(wq, wk))
        qk.qknorm_set_rows_tuning(5, 1, 3, 1)
        pl = qk.qknorm_plan_fwd(4096, 5120, 1024, 8, qk.QKNORM_BF16, 148)
        assert (pl["block"], pl["q_warps"], pl["stages"], pl["gamma_smem"]) == (192, 5, 3, 1)
        # 19 barriers (padded to 256 B), 24 KiB of gamma, 3 stages of 5 x 10 KiB
        # Q rows and of 1 x 2 KiB K rows
        assert pl["smem_bytes"] == 256 + (5120 + 1024) * 4 + 3 * (5 * 10240 + 2048)
        with pytest.raises(qk.QKNormError):
            qk.qknorm_set_rows_tuning(0, 2, 0, -1)
        with pytest.raises(qk.QKNormError):
            qk.qknorm_set_rows_tuning(9, 8, 0, -1)
        with pytest.raises(qk.QKNormError):
            qk.qknorm_set_rows_tuning(1, 1, 0, 2)
    finally:
        qk.qknorm_set_rows_tuning()
        qk.qknorm_force_variant(qk.VARIANT_AUTO, 0)


@needs_cpu
def test_deferred_entry_points_reject(qk):
    L = qk.lib
    assert L.qknorm_xgamma(A + 2, B, C, 4, 256, 1, None) == 2
    assert L.qknorm_xgamma(A, B, C, 4, 252, 1, None) == 3          # 252 not a multiple of 8
    assert L.qknorm_xgamma(A, B, A + 16, 4, 256, 1, None) == 1     # partial overlap
    assert L.qknorm_xgamma(A, B, B, 4, 256, 1, None) == 1          # out on gamma
    assert L.qknorm_xgamma(0, B, C, 4, 256, 1, None) == 1
    assert L.qknorm_xgamma(0, 0, 0, 0, 256, 1, None) == 0
    assert L.qknorm_inv_rms(A, B, 4, 256, 3, 1e-6, 1, None) == 1   # D % P
    assert L.qknorm_inv_rms(A, B, 4, 256, 4, -1.0, 1, None) == 1
    assert L.qknorm_inv_rms(A, A + 64, 4, 256, 4, 1e-6, 1, None) == 1
    assert L.qknorm_inv_rms(A, B + 4, 4, 256, 4, 1e-6, 1, None) == 2
    assert L.qknorm_inv_rms(A, B, 4, 256, 4, 1e-6, 7, None) == 3


@needs_cpu
def test_strided_checks(qk):
    """Row strides: >= the width, a multiple of the 16-byte vector; Q and K as
    slices of one fused QKV buffer may be normalised in place; an output that
    lands on another tensor's rows is rejected."""
    L = qk.lib
    Dq, Dk = 256, 128
    ld = Dq + 2 * Dk                       # one QKV row, bf16 elements
    qkv = 0x100000
    q, k, v = qkv, qkv + 2 * Dq, qkv + 2 * (Dq + Dk)

    def call(q_, k_, oq, ok, ldq=ld, ldk=ld, ldoq=ld, ldok=ld, T=16):
        return L.qknorm_fwd_strided(q_, k_, C, Dd, oq, ok, T, Dq, Dk, 2, 1e-6, 1,
                                    ldq, ldk, ldoq, ldok, None)

    assert call(q, k, q, k) == 4                          # in place: valid, then no GPU
    assert call(q, k, E, F, ldoq=Dq, ldok=Dk) == 4        # strided in, dense out: valid
    assert call(q, k, q, k, ldq=Dq - 8) == 1              # stride below the width
    assert call(q, k, q, k, ldq=ld + 4) == 2              # stride not a multiple of 8 bf16
    assert call(q, k, k, q) == 1                          # outputs on each other's input
    assert call(q, k, v, k) == 1                          # Dq-wide output from V's start reaches next Q
    assert call(q, k, q, v) == 4                          # Dk-wide K output into the V slot: disjoint rows
    assert call(q, k, q + 16, k) == 1                     # Q output shifted into its own input
    assert call(q, k, E, F, ldoq=Dq, ldok=Dk, T=0) == 0


@needs_cpu
def test_headwise_checks(qk):
    L = qk.lib

    def call(Hq=8, Hk=2, hd=128, T=4, ldq=None, ldk=None, ldoq=None, ldok=None, q=A, k=B, oq=E, ok=F,
             eps=1e-6, dtype=1):
        ldq = ldq or Hq * hd
        ldk = ldk or Hk * hd
        return L.qknorm_headwise_fwd(q, k, C, Dd, oq, ok, T, Hq, Hk, hd, eps, dtype, ldq, ldk,
                                     ldoq or Hq * hd, ldok or Hk * hd, None)

    assert call() == 4                                  # valid: the runtime finds no device
    assert call(Hq=0) == 1 and call(hd=0) == 1 and call(T=-1) == 1
    assert call(hd=100) == 3                            # not a multiple of 8 bf16
    assert call(hd=8 * 257) == 3                        # more than 256 vectors per head
    assert call(ldq=8 * 128 - 8) == 1                   # stride below the width
    assert call(ldq=8 * 128 + 4) == 2
    assert call(eps=-1.0) == 1 and call(dtype=3) == 3
    assert call(oq=B) == 1                              # output on the other input
    assert call(T=0, q=0, k=0, oq=0, ok=0) == 0


def test_two_tensor_wrappers_check_metadata(qk):
    """The Python wrappers of the two-tensor calls reject mismatched shapes and
    host tensors before calling into the library."""
    import torch
    q, k = torch.zeros(4, 256, dtype=torch.bfloat16), torch.zeros(4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        qk.qknorm_partial_sumsq_qk(q, torch.zeros(5, 64, dtype=torch.bfloat16), 4)   # row counts differ
    with pytest.raises(ValueError):
        qk.qknorm_partial_sumsq_qk(q, k, 4)                                         # host tensors
    g = torch.ones(256)
    with pytest.raises(ValueError):
        qk.qknorm_apply_tp_qk(q, k, g, g[:64], torch.zeros(2, 4, 4), 1e-6)          # stats not 4-D
    with pytest.raises(ValueError):
        qk.qknorm_apply_tp_qk(q, k, g, g[:64], torch.zeros(2, 3, 4, 4), 1e-6)       # not [ranks, 2, ...]
    with pytest.raises(ValueError):
        qk.qknorm_apply_tp_qk(q, k, g, g[:64], torch.zeros(2, 2, 4, 4), 1e-6)       # host tensors


def test_noalloc_wrapper_checks_metadata(qk):
    """The Python wrapper of qknorm_split_noalloc rejects a gamma of the wrong
    dtype or length and an out of the wrong shape or dtype, and host tensors,
    before calling into the library."""
    import torch
    x = torch.zeros(4, 256, dtype=torch.bfloat16)
    g = torch.ones(256)
    with pytest.raises(TypeError):
        qk.qknorm_split_noalloc(x, g.to(torch.bfloat16), 4, 1e-6)              # bf16 gamma
    with pytest.raises(ValueError):
        qk.qknorm_split_noalloc(x, g[:128], 4, 1e-6)                           # short gamma
    with pytest.raises(ValueError):
        qk.qknorm_split_noalloc(x, g, 4, 1e-6, out=torch.zeros(2, 256, dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        qk.qknorm_split_noalloc(x, g, 4, 1e-6, out=torch.zeros(4, 256))        # fp32 out
    with pytest.raises(TypeError):
        qk.qknorm_split_noalloc(x.to(torch.float16), g, 4, 1e-6)               # unsupported dtype
    with pytest.raises(ValueError):
        qk.qknorm_split_noalloc(x, g, 4, 1e-6)                                 # host tensors


def test_gpair_plans(qk):
    """The shard-pair ring with staged gamma: separate warps for Q and K of one
    geometry, mixed warps (both tensors) otherwise; FP8 splits a last slot of
    at most 16 vectors in lane halves; the selector takes it for FP8, and for
    bf16 where an instance is compiled for the exact shape (GQA widths, P = 8)."""
    qk.qknorm_force_variant(qk.VARIANT_GPAIR, 0)
    try:
        pl = qk.qknorm_plan_fwd(8192, 5120, 5120, 4, qk.QKNORM_E4M3, 148)     # 80 vectors per shard
        assert (pl["variant"], pl["block"], pl["vmax"], pl["vmax_k"], pl["half_slots"], pl["mixed"]) == \
            (qk.VARIANT_GPAIR, 4 * 32, 2, 2, 3, 0)
        pl = qk.qknorm_plan_fwd(4096, 5120, 1024, 8, qk.QKNORM_E4M3, 148)     # 40 and 8 vectors
        assert (pl["block"], pl["vmax"], pl["vmax_k"], pl["half_slots"], pl["mixed"]) == (4 * 32, 1, 0, 3, 1)
        pl = qk.qknorm_plan_fwd(4096, 5120, 1024, 8, qk.QKNORM_BF16, 148)     # 80 and 16: guarded slots
        assert (pl["block"], pl["vmax"], pl["vmax_k"], pl["half_slots"], pl["mixed"]) == (4 * 32, 3, 1, 0, 1)
        assert pl["stages"] == 2 and pl["smem_bytes"] > 24 * 1024            # gamma is staged
        qk.qknorm_set_tuning(stages=3)
        assert qk.qknorm_plan_fwd(4096, 5120, 1024, 8, qk.QKNORM_E4M3, 148)["stages"] == 3
        qk.qknorm_set_tuning()
        for bad in ((5120, 5120, 4, qk.QKNORM_BF16),    # no instance
                    (3072, 3072, 3, qk.QKNORM_E4M3),    # odd P
                    (4096, 4096, 1, qk.QKNORM_E4M3)):   # one shard
            with pytest.raises(qk.QKNormError) as ei:
                qk.qknorm_plan_fwd(4096, *bad, 148)
            assert ei.value.status == qk.QKNORM_ERR_UNSUPPORTED
    finally:
        qk.qknorm_force_variant(qk.VARIANT_AUTO, 0)
        qk.qknorm_set_tuning()
    assert qk.qknorm_plan_fwd(4096, 5120, 1024, 8, qk.QKNORM_E4M3, 148)["variant"] == qk.VARIANT_GPAIR
    assert qk.qknorm_plan_fwd(4096, 5120, 1024, 8, qk.QKNORM_BF16, 148)["variant"] == qk.VARIANT_GPAIR
    assert qk.qknorm_plan_fwd(48 * 148, 5120, 1024, 8, qk.QKNORM_BF16, 148)["variant"] == qk.VARIANT_PAIR
    assert qk.qknorm_plan_fwd(4096, 5120, 768, 8, qk.QKNORM_BF16, 148)["variant"] == qk.VARIANT_PAIR   # 12 K vectors
    assert qk.qknorm_plan_fwd(8192, 5120, 5120, 4, qk.QKNORM_E4M3, 148)["variant"] == qk.VARIANT_GPAIR
    assert qk.qknorm_plan_fwd(8192, 4096, 4096, 4, qk.QKNORM_E4M3, 148)["variant"] == qk.VARIANT_GPAIR
    assert qk.qknorm_plan_fwd(65536, 4096, 4096, 8, qk.QKNORM_E4M3, 148)["variant"] == qk.VARIANT_PAIR
    assert qk.qknorm_plan_fwd(8192, 5120, 5120, 4, qk.QKNORM_BF16, 148)["variant"] == qk.VARIANT_BULK
    assert qk.qknorm_plan_fwd(64, 5120, 1024, 8, qk.QKNORM_E4M3, 148)["variant"] == qk.VARIANT_CTA
