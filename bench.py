#!/usr/bin/env python
"""Benchmark of layerwise QK-Norm on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

A step is one fused QK-Norm pass (qknorm_fwd: Algorithm 1 Phases A-C for Q
and K, launch chosen by the selector) over the 13B-shaped prefill batch:
T = 8192 tokens per GPU, Dq = Dk = 5120, bf16, P = 4, eps = 1e-6. Tokens are
independent, so N GPUs each run their own batch (weak scaling, no collective
on the data path); value = algorithmic bytes of all ranks / max-over-ranks
device time. The split path, the decode latencies and the GQA shapes are
measured after the timed region and reported beside it.

--impl reference times the float64 CPU oracle (the only reference this
method has) on the same workload, a bounded sample of rows per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import qknorm_workloads as W  # noqa: E402

METRIC = "QK-Norm GB/s and % of B200 HBM peak (prefill); μs/call at decode T≤64"
HEADLINE = "prefill13b"
FALLBACK_HBM_GBS = 6650.0

KERNEL_OF_VARIANT = {0: "fused_cta", 1: "fused_warp", 2: "fused_generic", 6: "fused_gpair",
                     3: "fused_bulk", 4: "fused_rows", 5: "fused_pair"}

# dram bytes per launch of the headline kernel from one ncu capture, and the
# hash of the kernel sources it was taken with (None until captured).
# Taken from an ncu --set full capture of one launch of the 13B-shaped
# prefill (cold caches, serialised): dram__bytes_read.sum 167,838,208 +
# dram__bytes_write.sum 113,555,968 (about 54 MB of the writes were still in
# L2 when the kernel ended).
NCU_TRAFFIC = {"src_sha": "6db328ea93242283", "bytes_per_launch": 281394176,
               "plan": {"variant": 3, "block": 256, "grid": 296, "vmax": 5, "stages": 2,
                        "tokens_per_stage": 1, "gamma_regs": 0, "full_lanes": 1}}


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("native", "reference"), default="native")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the decode / GQA / split measurements after the timed region")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(W.WORKLOADS),
                    help="workload of the timed region (default: the 13B-shaped prefill); "
                         "the largest T of the workload is used")
    ap.add_argument("--variant", default="auto",
                    choices=("auto", "cta", "warp", "generic", "bulk", "rows", "pair", "gpair"),
                    help="force a kernel variant (for profiling; default: the selector's choice)")
    ap.add_argument("--path", default="fused", choices=("fused", "split", "headwise"),
                    help="what a step runs: qknorm_fwd (default), the split path "
                         "(qknorm_partial_sumsq then qknorm_apply, for Q and for K: 4 launches), "
                         "or headwise QK-Norm over heads of 128 (qknorm_headwise_fwd)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="tokens per GPU of the timed region (default: the workload's largest T); "
                         "a smaller T gives a small case for profiling")
    return ap.parse_args(argv)


VARIANT_IDS = {"auto": -1, "cta": 0, "warp": 1, "generic": 2, "bulk": 3, "rows": 4, "pair": 5, "gpair": 6}


# The source of the headline kernel (the fused_bulk template, from its
# declaration to the next section of its file) and of the device helpers it
# uses. The traffic figure is valid while they are unchanged AND the launch
# plan equals the one captured (the plan is the selector's, in qknorm_api.cu).
HEADLINE_SOURCES = (
    ("qknorm_fused_bulk.cu", "template <class Tag, int VMAX, bool GREG, int TB, int MODE, int MAXT>",
     "// ---------------------------------------------------------------- warp per row"),
    ("qknorm_bulk.cuh", None, None),
    ("qknorm_device.cuh", None, None),
)


def kernel_src_sha() -> str:
    csrc = os.path.join(ROOT, "qk_norm_attention_b200", "csrc")
    h = hashlib.sha256()
    for f, start, end in HEADLINE_SOURCES:
        with open(os.path.join(csrc, f), "rb") as fh:
            text = fh.read()
        if start is not None:
            i = text.index(start.encode())
            text = text[i:text.index(end.encode(), i)]
        h.update(f.encode() + b"\0" + text)
    return h.hexdigest()[:16]


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured (MEASURED_PEAKS.json hbm_gbs: STREAM-style copy)"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback (6.65 TB/s earlier measurement on this pool)"


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# ----------------------------------------------------------------------------- distributed

class Dist:
    """Rank bookkeeping. Under torchrun (WORLD_SIZE > 1) an NCCL process group
    with a short timeout carries the barriers and the max-over-ranks reduction."""

    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None

    def init(self, backend: str):
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist

    def barrier(self):
        if self.pg is not None:
            self.pg.barrier()

    def max(self, value: float, device) -> float:
        if self.pg is None:
            return value
        import torch
        t = torch.tensor([value], dtype=torch.float64, device=device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()


def shard_tokens(T_global: int, world: int, rank: int):
    """Contiguous token range [start, stop) of this rank (the remainder goes to
    the first ranks)."""
    base, rem = divmod(T_global, world)
    start = rank * base + min(rank, rem)
    return start, start + base + (1 if rank < rem else 0)


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        "sw_power_cap": 0x4, "hw_slowdown": 0x8, "sync_boost": 0x10,
        "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, index: int, period_s: float = 0.005):
        self.index = index
        self.period = period_s
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self.error = None
        self._stop = threading.Event()
        self._thread = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # NVML absent: report it instead of clocks
            self.error = f"{type(e).__name__}: {e}"
            return self
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()
        return self

    def _run(self):
        n = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append(n.nvmlDeviceGetClockInfo(self._h, n.NVML_CLOCK_SM))
                mask = n.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for name, bit in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception as e:
                self.error = f"{type(e).__name__}: {e}"
                return
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()
        return False

    def summary(self):
        out = {"sm_mhz": statistics.median(self.samples) if self.samples else None,
               "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
               "samples": len(self.samples), "source": "NVML, sampled during the timed region"}
        if self.error:
            out["error"] = self.error
        return out


def nvml_index(torch, device) -> int:
    """NVML index of a CUDA device (honours CUDA_VISIBLE_DEVICES)."""
    fn = getattr(torch.cuda, "_get_nvml_device_index", None)
    try:
        return int(fn(device)) if fn else int(device.index or 0)
    except Exception:
        return int(device.index or 0)


# ----------------------------------------------------------------------------- native arm

class Fused:
    """Raw C-ABI call of qknorm_fwd for one buffer set (no per-call Python
    marshalling beyond ctypes)."""

    def __init__(self, qk, bufs, T, Dq, Dk, P, eps, dtype_code, stream):
        q, k, gq, gk, oq, ok = bufs
        self.fn = qk.lib.qknorm_fwd
        self.args = (q.data_ptr(), k.data_ptr(), gq.data_ptr(), gk.data_ptr(), oq.data_ptr(),
                     ok.data_ptr(), T, Dq, Dk, P, eps, dtype_code, stream)
        self.qk = qk

    def __call__(self):
        st = self.fn(*self.args)
        if st != 0:
            raise RuntimeError(f"qknorm_fwd: {self.qk.qknorm_status_string(st)} "
                               f"{self.qk.qknorm_last_error()}")


class Split:
    """The split path for one buffer set through the raw C ABI: statistics of
    Q and K (qknorm_partial_sumsq), then the apply step of each (qknorm_apply)."""

    def __init__(self, qk, bufs, stats, T, Dq, Dk, P, eps, dtype_code, stream):
        q, k, gq, gk, oq, ok = bufs
        sq, sk = stats
        L = qk.lib
        self.calls = [
            (L.qknorm_partial_sumsq, (q.data_ptr(), sq.data_ptr(), T, Dq, P, dtype_code, stream)),
            (L.qknorm_partial_sumsq, (k.data_ptr(), sk.data_ptr(), T, Dk, P, dtype_code, stream)),
            (L.qknorm_apply, (q.data_ptr(), gq.data_ptr(), sq.data_ptr(), oq.data_ptr(), T, Dq, P, eps,
                              dtype_code, stream)),
            (L.qknorm_apply, (k.data_ptr(), gk.data_ptr(), sk.data_ptr(), ok.data_ptr(), T, Dk, P, eps,
                              dtype_code, stream)),
        ]
        self.qk = qk

    def __call__(self):
        for fn, a in self.calls:
            st = fn(*a)
            if st != 0:
                raise RuntimeError(f"split path: {self.qk.qknorm_status_string(st)} "
                                   f"{self.qk.qknorm_last_error()}")


HEAD_DIM = 128


class Headwise:
    """Headwise QK-Norm for one buffer set through the raw C ABI: Q and K rows
    as heads of HEAD_DIM values, gamma [HEAD_DIM] per tensor."""

    def __init__(self, qk, bufs, T, Dq, Dk, eps, dtype_code, stream):
        q, k, gq, gk, oq, ok = bufs
        self.fn = qk.lib.qknorm_headwise_fwd
        self.args = (q.data_ptr(), k.data_ptr(), gq.data_ptr(), gk.data_ptr(), oq.data_ptr(),
                     ok.data_ptr(), T, Dq // HEAD_DIM, Dk // HEAD_DIM, HEAD_DIM, eps, dtype_code,
                     Dq, Dk, Dq, Dk, stream)
        self.qk = qk

    def __call__(self):
        st = self.fn(*self.args)
        if st != 0:
            raise RuntimeError(f"headwise: {self.qk.qknorm_status_string(st)} {self.qk.qknorm_last_error()}")


def device_inputs(torch, wl, T, device, row0=0):
    """q, k (bf16 or fp32) drawn on the device with the workload's recipe, and
    gamma; rows start at row0."""
    from qknorm_workloads import gen_gamma

    def dev(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
        return torch.from_numpy(a).to(device)

    q = W.gen_device_workload(wl, "q", T, device, row0)
    k = W.gen_device_workload(wl, "k", T, device, row0)
    return q, k, dev(gen_gamma(wl, "q")), dev(gen_gamma(wl, "k"))


def time_launches(torch, calls, steps, stream, per_launch=True):
    """Run `calls` round-robin for `steps` launches; returns (total_ms, [per-launch ms]).
    With per_launch=False only two events bracket the launches (nothing is
    recorded between them) and the list is empty."""
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps if per_launch else 0)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(steps):
        if per_launch:
            ev[i][0].record(stream)
        calls[i % len(calls)]()
        if per_launch:
            ev[i][1].record(stream)
    t1.record(stream)
    t1.synchronize()
    return t0.elapsed_time(t1), [a.elapsed_time(b) for a, b in ev]


def latency_us(torch, qk, wl, T, device, n_eager=400, n_graph=100, graph_reps=10):
    """µs per qknorm_fwd call at a small T: back-to-back eager launches through
    ctypes, and the same calls replayed from a CUDA graph."""
    stream = torch.cuda.current_stream(device)
    q, k, gq, gk = device_inputs(torch, wl, T, device)
    bufs = (q, k, gq, gk, torch.empty_like(q), torch.empty_like(k))
    dt = {"bf16": qk.QKNORM_BF16, "f32": qk.QKNORM_F32, "e4m3": qk.QKNORM_E4M3}[wl.dtype]
    f = Fused(qk, bufs, T, wl.Dq, wl.Dk, wl.P, wl.eps, dt, stream.cuda_stream)
    for _ in range(50):
        f()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(n_eager):
        f()
    t1.record(stream)
    t1.synchronize()
    eager = t0.elapsed_time(t1) * 1000.0 / n_eager
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fc = Fused(qk, bufs, T, wl.Dq, wl.Dk, wl.P, wl.eps, dt,
                   torch.cuda.current_stream(device).cuda_stream)
        for _ in range(n_graph):
            fc()
    g.replay()
    torch.cuda.synchronize()
    t0.record(stream)
    for _ in range(graph_reps):
        g.replay()
    t1.record(stream)
    t1.synchronize()
    graph = t0.elapsed_time(t1) * 1000.0 / (n_graph * graph_reps)
    del g
    return {"eager_us": round(eager, 3), "graph_us": round(graph, 3)}


def decode_c_abi(wl):
    """The decode sizes timed by the C++ program built beside the library
    (qknorm_fwd called from C, no Python): device us per call and host us
    per call, back to back on one stream."""
    exe = os.path.join(ROOT, "qk_norm_attention_b200", "decode_bench")
    if not os.path.exists(exe):
        return {"unavailable": "decode_bench not built"}
    import subprocess
    r = subprocess.run([exe, str(wl.Dq), str(wl.P), "2000"], capture_output=True, text=True, timeout=120)
    if r.returncode != 0:
        return {"unavailable": r.stderr.strip()[-200:]}
    out = json.loads(r.stdout)
    out["how"] = "C++ program through the C ABI: 2000 back-to-back calls per T, CUDA events (device) and steady_clock (host)"
    return out


def copy_floor(peak):
    """A plain streaming copy and a plain streaming read of the byte counts
    the workloads move in one launch (the yardstick built beside the
    library, `copy_floor`): device us per launch, back to back with eight
    rotating buffer sets, and the fraction of the measured peak they reach.
    Sizes: 21 MB (one tensor-parallel rank's statistics read at 8 ranks),
    42 MB (its apply), 50.3 MB (FP8 GQA, T = 4096), 100.7 MB (GQA),
    168 MB (FP8 13B), 336 MB (13B)."""
    exe = os.path.join(ROOT, "qk_norm_attention_b200", "copy_floor")
    if not os.path.exists(exe):
        return {"unavailable": "copy_floor not built"}
    import subprocess
    sizes = ["21", "42", "50.3", "100.7", "168", "336"]
    r = subprocess.run([exe, *sizes], capture_output=True, text=True, timeout=120)
    if r.returncode != 0:
        return {"unavailable": r.stderr.strip()[-200:]}
    out = json.loads(r.stdout)
    for kind in ("copy", "read"):
        out[kind] = {mb: {"us": us, "pct_hbm_peak": round(100 * float(mb) * 1e6 / (us * 1e3) / peak, 1)}
                     for mb, us in out[kind].items()}
    out["how"] = ("grid-stride kernels, 256 threads x 8 blocks per SM, four 16-byte streaming loads in "
                  "flight per thread, PDL; copy MB = bytes read + bytes written")
    return out


def throughput(torch, qk, wl, T, device, sets, steps=50):
    """GB/s of the fused path on T tokens with `sets` rotating buffer sets."""
    stream = torch.cuda.current_stream(device)
    dt = {"bf16": qk.QKNORM_BF16, "f32": qk.QKNORM_F32, "e4m3": qk.QKNORM_E4M3}[wl.dtype]
    q, k, gq, gk = device_inputs(torch, wl, T, device)
    calls = []
    for s in range(sets):
        qs, ks = (q, k) if s == 0 else (q.clone(), k.clone())
        calls.append(Fused(qk, (qs, ks, gq, gk, torch.empty_like(q), torch.empty_like(k)), T,
                           wl.Dq, wl.Dk, wl.P, wl.eps, dt, stream.cuda_stream))
    for i in range(10):
        calls[i % sets]()
    torch.cuda.synchronize()
    total, _ = time_launches(torch, calls, steps, stream, per_launch=False)
    ms = total / steps
    nbytes = W.fused_bytes(T, wl.Dq, wl.Dk, wl.elem_bytes)
    return {"T": T, "us_per_call": round(ms * 1000, 3), "GB_s": round(nbytes / ms / 1e6, 1),
            "algorithmic_bytes": nbytes, "buffer_sets": sets}


def deferred_steps(torch, qk, device, peak, steps=100):
    """qknorm_xgamma and qknorm_inv_rms on the 13B-shaped Q tensor (T = 8192,
    D = 5120, bf16, P = 4), three rotating inputs (> L2)."""
    wl = W.WORKLOADS["prefill13b"]
    T, D, P = wl.Ts[0], wl.Dq, wl.P
    stream = torch.cuda.current_stream(device)
    h = stream.cuda_stream
    x = W.gen_device_workload(wl, "q", T, device)
    xs = [x, x.clone(), x.clone()]
    g = torch.from_numpy(W.gen_gamma(wl, "q")).to(device)
    us = [torch.empty_like(x) for _ in xs]
    rs = [torch.empty(T, dtype=torch.float32, device=device) for _ in xs]
    L = qk.lib

    def xg(i):
        def f():
            if L.qknorm_xgamma(xs[i].data_ptr(), g.data_ptr(), us[i].data_ptr(), T, D, 1, h) != 0:
                raise RuntimeError("qknorm_xgamma failed")
        return f

    def ir(i):
        def f():
            if L.qknorm_inv_rms(xs[i].data_ptr(), rs[i].data_ptr(), T, D, P, wl.eps, 1, h) != 0:
                raise RuntimeError("qknorm_inv_rms failed")
        return f

    out = {"workload": "13B-shaped Q tensor: T=8192, D=5120, bf16, P=4"}
    for name, calls, nbytes in (("xgamma", [xg(i) for i in range(3)], 2 * T * D * 2 + 4 * D),
                                ("inv_rms", [ir(i) for i in range(3)], T * D * 2 + 4 * T)):
        for i in range(6):
            calls[i % 3]()
        torch.cuda.synchronize()
        tot, _ = time_launches(torch, calls, steps, stream, per_launch=False)
        ms = tot / steps
        out[name] = {"us_per_call": round(ms * 1000, 2), "GB_s": round(nbytes / ms / 1e6, 1),
                     "pct_hbm_peak": round(100 * nbytes / ms / 1e6 / peak, 1),
                     "algorithmic_bytes": nbytes}
    return out


def _fp8_case(torch, qk, device, peak, wl, gq, gk, steps):
    """Time qknorm_fwd in FP8 E4M3 on wl's first T over rotating buffer sets."""
    T = wl.Ts[0]
    stream = torch.cuda.current_stream(device)
    q = W.gen_device_workload(wl, "q", T, device)
    k = W.gen_device_workload(wl, "k", T, device)
    nbytes = W.fused_bytes(T, wl.Dq, wl.Dk, 1)
    n = buffer_sets(nbytes)
    sets = [(q, k)] + [(q.clone(), k.clone()) for _ in range(n - 1)]
    calls = [Fused(qk, (a, b, gq, gk, torch.empty_like(a), torch.empty_like(b)), T, wl.Dq, wl.Dk,
                   wl.P, wl.eps, qk.QKNORM_E4M3, stream.cuda_stream) for a, b in sets]
    for i in range(10):
        calls[i % n]()
    torch.cuda.synchronize()
    tot, _ = time_launches(torch, calls, steps, stream, per_launch=False)
    ms = tot / steps
    plan = qk.qknorm_launch_plan(T, wl.Dq, wl.Dk, wl.P, qk.QKNORM_E4M3)
    return {"us_per_call": round(ms * 1000, 2), "GB_s": round(nbytes / ms / 1e6, 1),
            "pct_hbm_peak": round(100 * nbytes / ms / 1e6 / peak, 1),
            "tokens_per_s": round(T / ms * 1000, 1), "algorithmic_bytes": nbytes,
            "kernel": KERNEL_OF_VARIANT.get(plan["variant"], "?")}


def fp8_prefill(torch, qk, device, peak, steps=200):
    """The 13B-shaped prefill (T = 8192, Dq = Dk = 5120, P = 4) in FP8 E4M3:
    E4M3 in and out, fp32 statistics; half the bytes of the bf16 step. Also
    the large split shape in FP8 (T = 65536, D = 4096, P = 8: one vector per
    lane, where the shard-pair ring takes Q and K) and the GQA shape in FP8
    (T = 4096, Dq = 5120, Dk = 1024, P = 8)."""
    wl = W.WORKLOADS["prefill13b_e4m3"]
    gq = torch.from_numpy(W.gen_gamma(wl, "q")).to(device)
    gk = torch.from_numpy(W.gen_gamma(wl, "k")).to(device)
    out = {"workload": "13B-shaped prefill in FP8 E4M3: T=8192, Dq=Dk=5120, P=4"}
    out.update(_fp8_case(torch, qk, device, peak, wl, gq, gk, steps))
    wl8 = W.WORKLOADS["split_large_e4m3"]
    g8q = torch.from_numpy(W.gen_gamma(wl8, "q")).to(device)
    g8k = torch.from_numpy(W.gen_gamma(wl8, "k")).to(device)
    r = {"workload": "T=65536, Dq=Dk=4096, P=8 in FP8 E4M3"}
    r.update(_fp8_case(torch, qk, device, peak, wl8, g8q, g8k, steps // 4))
    out["split_large_e4m3"] = r
    wlg = W.WORKLOADS["gqa_e4m3"]
    ggq = torch.from_numpy(W.gen_gamma(wlg, "q")).to(device)
    ggk = torch.from_numpy(W.gen_gamma(wlg, "k")).to(device)
    r = {"workload": "GQA-shaped prefill in FP8 E4M3: T=4096, Dq=5120, Dk=1024, P=8"}
    r.update(_fp8_case(torch, qk, device, peak, wlg, ggq, ggk, steps))
    out["gqa_e4m3"] = r
    return out


def tp_rank_step(torch, qk, device, peak, steps=100):
    """One rank's kernels of the tensor-parallel form at the 13B shape (T =
    8192, Dq = Dk = 5120, P = 8) for a group of `ranks` GPUs: the statistics
    of its Q and K slices, then the apply step of each, as two launches
    (qknorm_partial_sumsq_qk, qknorm_apply_tp_qk: what qknorm_tp_fwd runs) and
    as four one-tensor launches. The all-gather between them needs several
    GPUs and is not timed here; the gathered sums are those of the emulated
    group, computed beforehand."""
    T, D, P = 8192, 5120, 8
    stream = torch.cuda.current_stream(device)
    h = stream.cuda_stream
    L = qk.lib
    wl = W.custom("tp", T, D, D, P, dtype="bf16", seed=9)
    q = W.gen_device_workload(wl, "q", T, device)
    k = W.gen_device_workload(wl, "k", T, device)
    g = torch.rand(D, device=device) + 0.5
    out = {}

    def ok(rc):
        if rc != 0:
            raise RuntimeError(qk.qknorm_status_string(rc))

    for ranks in (2, 4, 8):
        Dl, Pl = D // ranks, P // ranks
        qs = [q[:, r * Dl:(r + 1) * Dl].contiguous() for r in range(ranks)]
        ks = [k[:, r * Dl:(r + 1) * Dl].contiguous() for r in range(ranks)]
        gathered = torch.stack([qk.qknorm_partial_sumsq_qk(a, b, Pl) for a, b in zip(qs, ks)])
        gl = g[:Dl].contiguous()
        sets = [(qs[r], ks[r], torch.empty_like(qs[r]), torch.empty_like(ks[r]),
                 torch.empty((2, T, Pl), dtype=torch.float32, device=device)) for r in range(ranks)]
        stride = gathered.stride(0)
        gq_, gk_ = gathered[:, 0].data_ptr(), gathered[:, 1].data_ptr()

        # The raw C-ABI calls of one step, arguments marshalled once (as in
        # Fused / Split), so the eager loop times the kernels, not Python.
        def calls_two(a, b, oa, ob, st, hs):
            return [(L.qknorm_partial_sumsq_qk, (a.data_ptr(), b.data_ptr(), st[0].data_ptr(), st[1].data_ptr(),
                                                 T, Dl, Dl, Pl, 1, hs)),
                    (L.qknorm_apply_tp_qk, (a.data_ptr(), b.data_ptr(), gl.data_ptr(), gl.data_ptr(), gq_, gk_,
                                            stride, oa.data_ptr(), ob.data_ptr(), T, Dl, Dl, Pl, ranks, 1e-6,
                                            1, hs))]

        def calls_four(a, b, oa, ob, st, hs):
            return [(L.qknorm_partial_sumsq, (a.data_ptr(), st[0].data_ptr(), T, Dl, Pl, 1, hs)),
                    (L.qknorm_partial_sumsq, (b.data_ptr(), st[1].data_ptr(), T, Dl, Pl, 1, hs)),
                    (L.qknorm_apply_tp, (a.data_ptr(), gl.data_ptr(), gq_, stride, oa.data_ptr(), T, Dl, Pl,
                                         ranks, 1e-6, 1, hs)),
                    (L.qknorm_apply_tp, (b.data_ptr(), gl.data_ptr(), gk_, stride, ob.data_ptr(), T, Dl, Pl,
                                         ranks, 1e-6, 1, hs))]

        def as_step(calls):
            def step():
                for fn, args in calls:
                    ok(fn(*args))
            return step

        step_two = lambda *st: as_step(calls_two(*st, h))
        step_four = lambda *st: as_step(calls_four(*st, h))

        nbytes = 2 * (3 * T * Dl * 2 + 4 * T * Pl + 4 * ranks * T * Pl + 4 * Dl)
        res = {}
        for label, mk in (("two_launches", step_two), ("four_launches", step_four)):
            calls = [mk(*st) for st in sets]        # the ranks' slices rotate (inputs beyond L2)
            for i in range(10):
                calls[i % ranks]()
            torch.cuda.synchronize()
            tot, _ = time_launches(torch, calls, steps, stream, per_launch=False)
            ms = tot / steps
            res[label] = {"us_per_step": round(ms * 1000, 2), "GB_s": round(nbytes / ms / 1e6, 1),
                          "pct_hbm_peak": round(100 * nbytes / ms / 1e6 / peak, 1)}
        # The two-launch step of every rank's slices captured in one CUDA graph
        # (how a serving step runs), replayed; us per step.
        side = torch.cuda.Stream(device)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=side):
                hs = side.cuda_stream
                for rep in range(4):
                    for st in sets:
                        as_step(calls_two(*st, hs))()
        stream.wait_stream(side)
        graph.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(10):
            graph.replay()
        e1.record(stream)
        e1.synchronize()
        gms = e0.elapsed_time(e1) / (10 * 4 * ranks)
        del graph
        out[str(ranks)] = dict(res["two_launches"], four_launches=res["four_launches"],
                               graph={"us_per_step": round(gms * 1000, 2), "GB_s": round(nbytes / gms / 1e6, 1),
                                      "pct_hbm_peak": round(100 * nbytes / gms / 1e6 / peak, 1)},
                               algorithmic_bytes=nbytes, exchange_bytes_per_rank=2 * 4 * T * Pl)
        del qs, ks, gathered, sets
    return {"workload": "13B-shaped Q and K (T=8192, D=5120, P=8) split over a tensor-parallel group; "
                        "one rank's statistics + apply kernels (Q and K in one launch each), "
                        "the all-gather not timed",
            "ranks": out}


def headwise(torch, qk, device, peak, steps=100):
    """Headwise QK-Norm: T = 8192 tokens, Hq = 32 and Hk = 8 heads of 128
    (bf16), gamma [128] per tensor, three rotating buffer sets."""
    T, Hq, Hk, hd = 8192, 32, 8, 128
    wl = W.custom("headwise", T, Hq * hd, Hk * hd, Hq, seed=7)
    stream = torch.cuda.current_stream(device)
    h = stream.cuda_stream
    q = W.gen_device_workload(wl, "q", T, device)
    k = W.gen_device_workload(wl, "k", T, device)
    g = torch.ones(hd, dtype=torch.float32, device=device)
    sets = [(q, k)] + [(q.clone(), k.clone()) for _ in range(2)]
    outs = [(torch.empty_like(a), torch.empty_like(b)) for a, b in sets]
    L = qk.lib

    def call(i):
        (a, b), (oa, ob) = sets[i], outs[i]

        def f():
            if L.qknorm_headwise_fwd(a.data_ptr(), b.data_ptr(), g.data_ptr(), g.data_ptr(),
                                     oa.data_ptr(), ob.data_ptr(), T, Hq, Hk, hd, 1e-6, 1,
                                     Hq * hd, Hk * hd, Hq * hd, Hk * hd, h) != 0:
                raise RuntimeError("qknorm_headwise_fwd failed")
        return f

    calls = [call(i) for i in range(3)]
    for i in range(6):
        calls[i % 3]()
    torch.cuda.synchronize()
    tot, _ = time_launches(torch, calls, steps, stream, per_launch=False)
    ms = tot / steps
    nbytes = W.fused_bytes(T, Hq * hd, Hk * hd, 2)
    return {"workload": "T=8192, Hq=32, Hk=8, head_dim=128, bf16", "us_per_call": round(ms * 1000, 2),
            "GB_s": round(nbytes / ms / 1e6, 1), "pct_hbm_peak": round(100 * nbytes / ms / 1e6 / peak, 1),
            "algorithmic_bytes": nbytes}


def split_path(torch, qk, device, peak, steps=20):
    """The split path (stats + apply for Q and K: 4 launches) and the fused path
    on the large-prefill workload, T = 65536, D = 4096, P = 8, bf16."""
    wl = W.WORKLOADS["split_large"]
    T = wl.Ts[0]
    stream = torch.cuda.current_stream(device)
    h = stream.cuda_stream
    q, k, gq, gk = device_inputs(torch, wl, T, device)
    oq, ok, aq, ak = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(q), torch.empty_like(k))
    sq = torch.empty((T, wl.P), dtype=torch.float32, device=device)
    sk = torch.empty_like(sq)
    L = qk.lib
    D, P, eps = wl.Dq, wl.P, wl.eps

    def check(st):
        if st != 0:
            raise RuntimeError(qk.qknorm_status_string(st))

    def stats_q():
        check(L.qknorm_partial_sumsq(q.data_ptr(), sq.data_ptr(), T, D, P, 1, h))

    def stats_k():
        check(L.qknorm_partial_sumsq(k.data_ptr(), sk.data_ptr(), T, D, P, 1, h))

    def apply_q():
        check(L.qknorm_apply(q.data_ptr(), gq.data_ptr(), sq.data_ptr(), aq.data_ptr(), T, D, P, eps, 1, h))

    def apply_k():
        check(L.qknorm_apply(k.data_ptr(), gk.data_ptr(), sk.data_ptr(), ak.data_ptr(), T, D, P, eps, 1, h))

    fused = Fused(qk, (q, k, gq, gk, oq, ok), T, D, D, P, eps, 1, h)
    seq = [stats_q, stats_k, apply_q, apply_k]
    for _ in range(3):
        for c in seq + [fused]:
            c()
    torch.cuda.synchronize()
    same = bool(torch.equal(aq.view(torch.int16), oq.view(torch.int16)) and
                torch.equal(ak.view(torch.int16), ok.view(torch.int16)))
    split_total, _ = time_launches(torch, seq, 4 * steps, stream, per_launch=False)
    fused_total, _ = time_launches(torch, [fused], steps, stream, per_launch=False)
    split_ms = split_total / steps
    fused_ms = fused_total / steps
    # Breakdown of the split step by kernel (event pair around each launch).
    _, per_split = time_launches(torch, seq, 4 * steps, stream, per_launch=True)
    st_ms = statistics.mean(per_split[0::4] + per_split[1::4])
    ap_ms = statistics.mean(per_split[2::4] + per_split[3::4])
    b_split = 2 * W.split_bytes(T, D, P, 2)
    b_fused = W.fused_bytes(T, D, D, 2)
    b_stats = W.stats_bytes(T, D, P, 2)
    b_apply = W.apply_bytes(T, D, P, 2)
    return {
        "workload": wl.note, "fused_equals_split_bitwise": same,
        "split": {"ms_per_step": round(split_ms, 4), "GB_s": round(b_split / split_ms / 1e6, 1),
                  "pct_hbm_peak": round(100 * b_split / split_ms / 1e6 / peak, 1),
                  "algorithmic_bytes": b_split,
                  "stats_kernel": {"us": round(st_ms * 1000, 2),
                                   "GB_s": round(b_stats / st_ms / 1e6, 1)},
                  "apply_kernel": {"us": round(ap_ms * 1000, 2),
                                   "GB_s": round(b_apply / ap_ms / 1e6, 1)}},
        "fused": {"ms_per_step": round(fused_ms, 4), "GB_s": round(b_fused / fused_ms / 1e6, 1),
                  "pct_hbm_peak": round(100 * b_fused / fused_ms / 1e6 / peak, 1),
                  "algorithmic_bytes": b_fused},
    }


# ----------------------------------------------------------------------------- CPU oracle

def oracle_rows_rate(wl, n_rows, nthreads, target_s, headwise=False):
    """Run the float64 oracle on n_rows tokens of Q and K (layerwise, or
    headwise over heads of HEAD_DIM) until target_s has passed; returns
    (passes, seconds)."""
    import oracle
    orc = oracle.get()
    rows = np.arange(n_rows)
    q, k = W.gen_rows(wl, "q", rows), W.gen_rows(wl, "k", rows)
    gq, gk = W.gen_gamma(wl, "q"), W.gen_gamma(wl, "k")
    eps = float(np.float32(wl.eps))
    passes, t0 = 0, time.perf_counter()
    while True:
        if headwise:
            orc.headwise(q, gq[:HEAD_DIM], HEAD_DIM, eps, wl.dtype, nthreads=nthreads)
            orc.headwise(k, gk[:HEAD_DIM], HEAD_DIM, eps, wl.dtype, nthreads=nthreads)
        else:
            orc.qknorm(q, k, gq, gk, wl.P, eps, wl.dtype, nthreads=nthreads)
        passes += 1
        el = time.perf_counter() - t0
        if el >= target_s:
            return passes, el


def cpu_baseline(wl, T, target_s=10.0, headwise=False):
    cores = host_cores()
    n = min(T, 2048)
    passes, el = oracle_rows_rate(wl, n, cores, target_s, headwise)
    nbytes = passes * W.fused_bytes(n, wl.Dq, wl.Dk, wl.elem_bytes)
    what = f", headwise over heads of {HEAD_DIM}" if headwise else ""
    return {"value": round(nbytes / el / 1e9, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} of the {T} tokens (Q and K rows{what}), {passes} passes in {el:.1f} s, "
                      f"float64 C oracle with OpenMP over tokens on {cores} threads ({cpu_model()})",
            "tokens_per_s": round(passes * n / el, 1)}


L2_BYTES = 126 * 1024 * 1024


def buffer_sets(set_bytes: int) -> int:
    """Rotating buffer sets so that the sets together exceed L2 at least twice."""
    return max(2, -(-2 * L2_BYTES // max(1, set_bytes)))


def config_of(wl, T, world):
    nbytes = W.fused_bytes(T, wl.Dq, wl.Dk, wl.elem_bytes)
    n = buffer_sets(nbytes)
    return {"workload": wl.note, "T_per_gpu": T, "global_tokens": T * world, "Dq": wl.Dq,
            "Dk": wl.Dk, "P": wl.P, "eps": wl.eps, "storage": wl.dtype,
            "accumulation": "fp32", "parallelism": f"token-sharded dp{world} (no collective)",
            "l2": f"inputs larger than L2: {n} rotating buffer sets of {nbytes / 1e6:.0f} MB "
                  f"(inputs + outputs) each, {n * nbytes / 1e6:.0f} MB in all vs 132 MB of L2"}


def run_reference(args, dist):
    """The oracle as the reference arm: rank 0 only, a bounded sample per step."""
    if dist.rank != 0:
        return 0
    # The native arm's workload, token count and path (the split path computes
    # what the fused one does; headwise has its own oracle function).
    wl = W.WORKLOADS[args.workload]
    T = args.tokens if args.tokens > 0 else max(wl.Ts)
    hw = args.path == "headwise"
    cores = host_cores()
    # Calibrate: rows per step so that warmup + steps take about two minutes.
    p, el = oracle_rows_rate(wl, 64, cores, 0.5, hw)
    per_row = el / (p * 64)
    budget = 120.0 / max(1, args.steps + args.warmup)
    n = int(min(T, max(16, budget / per_row)))
    import oracle
    orc = oracle.get()
    rows = np.arange(n)
    q, k = W.gen_rows(wl, "q", rows), W.gen_rows(wl, "k", rows)
    gq, gk = W.gen_gamma(wl, "q"), W.gen_gamma(wl, "k")
    eps = float(np.float32(wl.eps))

    def step():
        if hw:
            orc.headwise(q, gq[:HEAD_DIM], HEAD_DIM, eps, wl.dtype, nthreads=cores)
            orc.headwise(k, gk[:HEAD_DIM], HEAD_DIM, eps, wl.dtype, nthreads=cores)
        else:
            orc.qknorm(q, k, gq, gk, wl.P, eps, wl.dtype, nthreads=cores)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    nbytes = W.fused_bytes(n, wl.Dq, wl.Dk, wl.elem_bytes)
    value = args.steps * nbytes / el / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(el * 1000 / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(config_of(wl, T, args.gpus), path=args.path),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"{n} of the {T} tokens (Q and K rows{', headwise' if hw else ''}) "
                                   f"per step, float64 C "
                                   f"oracle, OpenMP over tokens on {cores} threads ({cpu_model()})"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_native(args, dist):
    import torch
    import qk_norm_attention_b200 as qk

    device = torch.device("cuda", dist.local_rank)
    torch.cuda.set_device(device)
    dist.init("nccl")
    wl = W.WORKLOADS[args.workload]
    T = args.tokens if args.tokens > 0 else max(wl.Ts)   # tokens per GPU (weak scaling)
    split = args.path == "split"
    hw = args.path == "headwise"
    if hw and (wl.Dq % HEAD_DIM or wl.Dk % HEAD_DIM):
        raise SystemExit(f"--path headwise needs widths that are multiples of {HEAD_DIM}")
    row0, _ = shard_tokens(T * dist.world, dist.world, dist.rank)
    stream = torch.cuda.current_stream(device)
    peak, peak_src = hbm_peak()
    dt = {"bf16": qk.QKNORM_BF16, "f32": qk.QKNORM_F32, "e4m3": qk.QKNORM_E4M3}[wl.dtype]
    qk.qknorm_force_variant(VARIANT_IDS[args.variant], 0)

    q, k, gq, gk = device_inputs(torch, wl, T, device, row0)
    if hw:      # one gamma of head_dim per tensor
        gq, gk = gq[:HEAD_DIM].contiguous(), gk[:HEAD_DIM].contiguous()
    nsets = buffer_sets(W.fused_bytes(T, wl.Dq, wl.Dk, wl.elem_bytes))
    sets = [(q, k)] + [(q.clone(), k.clone()) for _ in range(nsets - 1)]
    def step_of(bufs):
        if split:
            st = (torch.empty((T, wl.P), dtype=torch.float32, device=device),
                  torch.empty((T, wl.P), dtype=torch.float32, device=device))
            return Split(qk, bufs, st, T, wl.Dq, wl.Dk, wl.P, wl.eps, dt, stream.cuda_stream)
        if hw:
            return Headwise(qk, bufs, T, wl.Dq, wl.Dk, wl.eps, dt, stream.cuda_stream)
        return Fused(qk, bufs, T, wl.Dq, wl.Dk, wl.P, wl.eps, dt, stream.cuda_stream)

    calls = [step_of((a, b, gq, gk, torch.empty_like(a), torch.empty_like(b))) for a, b in sets]
    plan = (qk.qknorm_launch_plan(T, wl.Dq, wl.Dk, wl.P, dt) if not hw else
            {"kernel": "headwise_k", "head_dim": HEAD_DIM, "heads_q": wl.Dq // HEAD_DIM,
             "heads_k": wl.Dk // HEAD_DIM})
    for i in range(max(3, args.warmup)):
        calls[i % len(calls)]()
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(nvml_index(torch, device)) as clk:
        total_ms, _ = time_launches(torch, calls, args.steps, stream, per_launch=False)
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    step_ms = dist.max(total_ms / args.steps, device)
    if split:
        nbytes = (W.split_bytes(T, wl.Dq, wl.P, wl.elem_bytes) +
                  W.split_bytes(T, wl.Dk, wl.P, wl.elem_bytes))
    else:
        nbytes = W.fused_bytes(T, wl.Dq, wl.Dk, wl.elem_bytes)
    value = dist.world * nbytes / step_ms / 1e6          # GB/s, all ranks
    # A fused step is one launch of the kernel, so its average duration over
    # the timed region is the step time (launch gaps included). A split step is
    # four launches; its figure is for the four together.
    achieved = nbytes / step_ms / 1e6                    # GB/s
    # Reference only: the same launches with an event pair around each one.
    _, per = time_launches(torch, calls, min(args.steps, 200), stream, per_launch=True)
    kern_ms = dist.max(statistics.mean(per), device)

    # End to end through the same C ABI: pinned host -> device, kernel, device -> host.
    e2e_steps = max(3, min(args.steps, 30))
    qh, kh = q.cpu().pin_memory(), k.cpu().pin_memory()
    oqh = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    okh = torch.empty(k.shape, dtype=k.dtype).pin_memory()
    qd, kd = sets[1]
    oqd, okd = (torch.empty_like(q), torch.empty_like(k))
    f = step_of((qd, kd, gq, gk, oqd, okd))
    if split or hw:
        e2e_path = f"pinned host -> device copies, the {args.path} path, device -> pinned host"

        def e2e_step():
            qd.copy_(qh, non_blocking=True)
            kd.copy_(kh, non_blocking=True)
            f()
            oqh.copy_(oqd, non_blocking=True)
            okh.copy_(okd, non_blocking=True)
    else:
        # The library's host-buffer entry point: chunks of 1024 tokens copied
        # in, normalised and copied out, the two copy directions overlapping.
        e2e_path = ("qknorm_fwd_host: pinned host rows in, 1024-token chunks over 3 device "
                    "workspace sets, host->device copy / kernel / device->host copy overlapped")
        ws = torch.empty(qk.qknorm_fwd_host_workspace(wl.Dq, wl.Dk, q.dtype), dtype=torch.uint8,
                         device=device)
        hargs = (qh.data_ptr(), kh.data_ptr(), gq.data_ptr(), gk.data_ptr(), oqh.data_ptr(),
                 okh.data_ptr(), T, wl.Dq, wl.Dk, wl.P, wl.eps, dt, ws.data_ptr(), ws.numel(), 0,
                 stream.cuda_stream)

        def e2e_step():
            st = qk.lib.qknorm_fwd_host(*hargs)
            if st != 0:
                raise RuntimeError(f"qknorm_fwd_host: {qk.qknorm_status_string(st)}")

    e2e_step()
    torch.cuda.synchronize()
    dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    e1.synchronize()
    e2e_ms = dist.max(e0.elapsed_time(e1) / e2e_steps, device)
    h2d = (qh.numel() + kh.numel()) * qh.element_size()
    d2h = (oqh.numel() + okh.numel()) * oqh.element_size()
    e2e_ok = True
    if not split and not hw:      # the host outputs of the last step equal the device path's
        f()
        torch.cuda.synchronize()
        e2e_ok = bool(torch.equal(oqh.view(torch.uint8), oqd.cpu().view(torch.uint8)) and
                      torch.equal(okh.view(torch.uint8), okd.cpu().view(torch.uint8)))
    del qh, kh, oqh, okh

    extras = {}
    qk.qknorm_force_variant(-1, 0)
    if dist.rank == 0 and not args.no_extras:
        dec = W.WORKLOADS["decode"]
        extras["decode_us_per_call"] = {str(t): latency_us(torch, qk, dec, t, device) for t in dec.Ts}
        extras["decode_c_abi"] = decode_c_abi(dec)
        gqa = W.WORKLOADS["gqa"]
        extras["gqa"] = {"us_per_call": {str(t): latency_us(torch, qk, gqa, t, device)
                                         for t in gqa.Ts if t <= 256},
                         "T4096": throughput(torch, qk, gqa, 4096, device, sets=4)}
        extras["gqa"]["T4096"]["pct_hbm_peak"] = round(100 * extras["gqa"]["T4096"]["GB_s"] / peak, 1)
        extras["split_large"] = split_path(torch, qk, device, peak)
        extras["deferred"] = deferred_steps(torch, qk, device, peak)
        extras["headwise"] = headwise(torch, qk, device, peak)
        extras["fp8_prefill13b"] = fp8_prefill(torch, qk, device, peak)
        extras["tp_rank"] = tp_rank_step(torch, qk, device, peak)
        extras["copy_floor"] = copy_floor(peak)
    dist.barrier()

    traffic = None
    if (not split and not hw and args.workload == HEADLINE and T == max(wl.Ts) and
            NCU_TRAFFIC["src_sha"] == kernel_src_sha() and NCU_TRAFFIC["bytes_per_launch"] and
            all(plan.get(key) == val for key, val in NCU_TRAFFIC["plan"].items())):
        traffic = NCU_TRAFFIC["bytes_per_launch"]
    kernel = ("stats_k + apply_k (split path, 4 launches per step)" if split
              else "headwise_k (qknorm_headwise_fwd)" if hw
              else KERNEL_OF_VARIANT.get(plan["variant"], "?") + " (qknorm_fwd)")
    line = {
        "impl": "native",
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s",
        "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(step_ms, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
        "config": dict(config_of(wl, T, dist.world), path=args.path),
        "pct_hbm_peak": round(100 * value / dist.world / peak, 2),
        "tokens_per_s": round(dist.world * T / step_ms * 1000, 1),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "kernel": kernel,
                     "peak_source": peak_src,
                     "algorithmic_bytes_per_launch": nbytes,
                     "launch_us": round(step_ms * 1000, 3),
                     "launch_us_event_pair": round(kern_ms * 1000, 3),
                     "how": "achieved = algorithmic bytes / (timed-region events / steps); "
                            "launch_us_event_pair = mean of per-launch event pairs (separate pass)"},
        "e2e": {"value": round(dist.world * nbytes / e2e_ms / 1e6, 2), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 4), "steps": e2e_steps,
                "path": e2e_path, "outputs_equal_device_path": e2e_ok},
        "gpu_launches": args.steps * (4 if split else 1),
        "clocks": clk.summary(),
        "plan": plan,
    }
    line.update(extras)
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, T, headwise=hw)
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dist.close()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.steps < 1 or args.warmup < 0:
        raise SystemExit("--steps must be >= 1 and --warmup >= 0")
    dist = Dist()
    if args.impl == "reference":
        return run_reference(args, dist)
    return run_native(args, dist)


if __name__ == "__main__":
    sys.exit(main())
