"""Seeded synthetic inputs for the layerwise QK-Norm workloads.

This module holds no QK-Norm arithmetic. It names the five workload shapes,
draws their random numbers, and rounds them to the storage type (fp32 or
bf16). The CUDA path's tests and benchmark and the float64 oracle both take
their inputs from here, so both sides see exactly the same stored values.

Recipe (the same for every workload):

* Row blocks. Rows (tokens) are drawn in blocks of ``ROW_BLOCK`` rows. Block
  ``b`` of tensor ``X`` uses its own PCG64 stream seeded with
  ``SeedSequence([seed, tensor_code(X), b])``, so any subset of rows can be
  regenerated on its own and equals the same rows of the full tensor.
* Values. ``x = sigma * N(0, 1)`` in float64. Workloads with outliers scale a
  fixed set of ``round(frac * D)`` channels (drawn without replacement from
  ``SeedSequence([seed, tensor_code(X), OUTLIER_KEY])``) by ``factor``.
  Workloads with a per-token scale multiply row ``t`` of both Q and K by
  ``s_t = 10 ** U(-2, 2)``, drawn per row block from
  ``SeedSequence([seed, SCALE_KEY, b])``.
* gamma. ``U(lo, hi)`` or ``N(mean, std)`` in float64, from
  ``SeedSequence([seed, tensor_code(X), GAMMA_KEY])``, rounded to fp32.
* Storage. float64 -> fp32 by round-to-nearest-even (numpy ``astype``); bf16
  keeps the top 16 bits of that fp32 value after round-to-nearest-even on the
  dropped 16 bits. bf16 arrays are returned as their ``uint16`` bit patterns.

The second parameter of every normal distribution is a standard deviation.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional, Sequence, Tuple

import numpy as np

ROW_BLOCK = 256
OUTLIER_KEY = 1_000_003
SCALE_KEY = 1_000_033
GAMMA_KEY = 1_000_037
TENSOR_CODE = {"q": 11, "k": 13}

DTYPE_BYTES = {"f32": 4, "bf16": 2, "e4m3": 1}


def _e4m3_table():
    """The 253 distinct finite FP8 E4M3 values (+0 only), ascending, and their codes."""
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F and c != 0x80], dtype=np.uint8)
    e = (codes.astype(np.int64) >> 3) & 15
    m = codes.astype(np.int64) & 7
    mag = np.where(e == 0, m * 2.0 ** -9, (1 + m / 8.0) * 2.0 ** (e - 7))
    vals = np.where(codes >> 7, -mag, mag)
    order = np.argsort(vals, kind="stable")
    return vals[order], codes[order]


_E4M3_VALS, _E4M3_CODES = _e4m3_table()


@dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, shard count, epsilon and value recipe."""

    name: str
    Ts: Tuple[int, ...]
    Dq: int
    Dk: int
    P: int
    eps: float
    dtype: str  # "f32" or "bf16"
    seed: int
    x_sigma: float = 1.0
    outlier_frac: float = 0.0
    outlier_factor: float = 1.0
    token_scale_log10: Optional[Tuple[float, float]] = None
    gamma: Tuple[str, float, float] = ("uniform", 0.5, 1.5)
    note: str = field(default="", compare=False)

    @property
    def elem_bytes(self) -> int:
        return DTYPE_BYTES[self.dtype]


# The five workloads. Shapes are OLMo2/OLMo3-style projected Q/K widths; the
# values stand in for real activations (no weights or datasets are used).
WORKLOADS = {
    "tiny": Workload(
        "tiny", Ts=(4,), Dq=256, Dk=256, P=2, eps=1e-6, dtype="f32", seed=0,
        gamma=("normal", 1.0, 0.1),
        note="tiny oracle check: T=4, Dq=Dk=256, fp32, P=2"),
    "decode": Workload(
        "decode", Ts=(1, 8, 32, 64), Dq=4096, Dk=4096, P=4, eps=1e-6,
        dtype="bf16", seed=2, outlier_frac=0.01, outlier_factor=20.0,
        note="OLMo2-7B-shaped decode: D=4096, bf16, P=4, 1% outlier channels x20"),
    "prefill13b": Workload(
        "prefill13b", Ts=(8192,), Dq=5120, Dk=5120, P=4, eps=1e-6,
        dtype="bf16", seed=3, x_sigma=1.5,
        note="13B-shaped prefill: T=8192, D=5120, bf16, P=4"),
    "gqa": Workload(
        "gqa", Ts=(1, 32, 256, 4096), Dq=5120, Dk=1024, P=8, eps=1e-6,
        dtype="bf16", seed=4,
        note="GQA-shaped: Dq=5120 (40x128), Dk=1024 (8x128), bf16, P=8"),
    "prefill13b_e4m3": Workload(
        "prefill13b_e4m3", Ts=(8192,), Dq=5120, Dk=5120, P=4, eps=1e-6,
        dtype="e4m3", seed=3, x_sigma=1.5,
        note="13B-shaped prefill in FP8 E4M3: T=8192, D=5120, P=4"),
    "gqa_e4m3": Workload(
        "gqa_e4m3", Ts=(4096,), Dq=5120, Dk=1024, P=8, eps=1e-6,
        dtype="e4m3", seed=13, x_sigma=1.5,
        note="GQA-shaped prefill in FP8 E4M3: T=4096, Dq=5120, Dk=1024, P=8"),
    "split_large": Workload(
        "split_large", Ts=(65536,), Dq=4096, Dk=4096, P=8, eps=1e-5,
        dtype="bf16", seed=5, token_scale_log10=(-2.0, 2.0),
        note="large prefill, split path: T=65536, D=4096, bf16, P=8, "
             "per-token scale log-uniform in [0.01, 100]"),
    "split_large_e4m3": Workload(
        "split_large_e4m3", Ts=(65536,), Dq=4096, Dk=4096, P=8, eps=1e-6,
        dtype="e4m3", seed=12, x_sigma=1.5,
        note="large prefill in FP8 E4M3: T=65536, D=4096, P=8 (one 16-byte vector per lane per shard)"),
}


def _rng(*keys: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(keys))))


def to_storage(x64: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 values to the storage type.

    fp32: round-to-nearest-even. bf16: fp32 first, then round-to-nearest-even
    on the low 16 bits; the result is the uint16 bit pattern. Finite inputs only.
    """
    if dtype == "e4m3":
        return _to_e4m3(np.ascontiguousarray(x64, dtype=np.float64))
    f32 = np.ascontiguousarray(x64, dtype=np.float64).astype(np.float32)
    if dtype == "f32":
        return f32
    if dtype != "bf16":
        raise ValueError(f"unknown dtype {dtype!r}")
    # For finite values bits <= 0xFF7FFFFF, so bits + 0x8000 fits in 32 bits.
    bits = f32.view(np.uint32)
    odd = (bits >> 16) & 1
    bits += 0x7FFF
    bits += odd
    bits >>= 16
    return bits.astype(np.uint16)


def _to_e4m3(x: np.ndarray) -> np.ndarray:
    """float64 -> FP8 E4M3 codes: round to nearest, ties to the even code
    (mantissa LSB 0), saturating to +-448 (finite inputs only)."""
    v, c = _E4M3_VALS, _E4M3_CODES
    xc = np.clip(x, v[0], v[-1])
    hi = np.clip(np.searchsorted(v, xc, side="left"), 1, len(v) - 1)
    lo = hi - 1
    dlo, dhi = xc - v[lo], v[hi] - xc
    pick_hi = (dhi < dlo) | ((dhi == dlo) & ((c[hi] & 1) == 0))
    out = np.where(pick_hi, c[hi], c[lo]).astype(np.uint8)
    out[x == 0] = 0
    return out


def storage_to_f64(s: np.ndarray, dtype: str) -> np.ndarray:
    """Exact widening of stored values to float64 (bf16 bits -> fp32 -> f64)."""
    if dtype == "f32":
        return s.astype(np.float64)
    if dtype == "e4m3":
        e = (s.astype(np.int64) >> 3) & 15
        m = s.astype(np.int64) & 7
        mag = np.where(e == 0, m * 2.0 ** -9, (1 + m / 8.0) * 2.0 ** (e - 7))
        return np.where(s >> 7, -mag, mag)
    bits = s.astype(np.uint32) << 16
    return bits.view(np.float32).astype(np.float64)


def outlier_channels(wl: Workload, tensor: str, D: int) -> np.ndarray:
    n = int(round(wl.outlier_frac * D))
    if n == 0:
        return np.zeros(0, dtype=np.int64)
    return np.sort(_rng(wl.seed, TENSOR_CODE[tensor], OUTLIER_KEY).choice(D, size=n, replace=False))


def _block_scales(wl: Workload, b: int) -> np.ndarray:
    lo, hi = wl.token_scale_log10
    return 10.0 ** _rng(wl.seed, SCALE_KEY, b).uniform(lo, hi, size=ROW_BLOCK)


def token_scales(wl: Workload, rows: Sequence[int]) -> np.ndarray:
    """Per-token scale s_t for the given rows (ones if the workload has none)."""
    rows = np.asarray(rows, dtype=np.int64)
    if wl.token_scale_log10 is None:
        return np.ones(len(rows))
    out = np.empty(len(rows))
    for b in np.unique(rows // ROW_BLOCK):
        sel = (rows // ROW_BLOCK) == b
        out[sel] = _block_scales(wl, int(b))[rows[sel] % ROW_BLOCK]
    return out


def gen_rows_f64(wl: Workload, tensor: str, rows: Sequence[int]) -> np.ndarray:
    """float64 values (before storage rounding) of the given rows of Q or K."""
    D = wl.Dq if tensor == "q" else wl.Dk
    rows = np.asarray(rows, dtype=np.int64)
    out = np.empty((len(rows), D))
    cols = outlier_channels(wl, tensor, D)
    blk = np.empty((ROW_BLOCK, D))
    for b in np.unique(rows // ROW_BLOCK):
        sel = (rows // ROW_BLOCK) == b
        _rng(wl.seed, TENSOR_CODE[tensor], int(b)).standard_normal(out=blk)
        blk *= wl.x_sigma
        if cols.size:
            blk[:, cols] *= wl.outlier_factor
        if wl.token_scale_log10 is not None:
            blk *= _block_scales(wl, int(b))[:, None]
        out[sel] = blk[rows[sel] % ROW_BLOCK]
    return out


def gen_rows(wl: Workload, tensor: str, rows: Sequence[int]) -> np.ndarray:
    """Stored values (fp32 array, or bf16 as uint16 bits) of the given rows."""
    return to_storage(gen_rows_f64(wl, tensor, rows), wl.dtype)


def gen_tensor(wl: Workload, tensor: str, T: int) -> np.ndarray:
    """All T rows of Q or K in storage form, [T, D]."""
    D = wl.Dq if tensor == "q" else wl.Dk
    dt = {"f32": np.float32, "bf16": np.uint16, "e4m3": np.uint8}[wl.dtype]
    out = np.empty((T, D), dtype=dt)
    for start in range(0, T, ROW_BLOCK):
        stop = min(T, start + ROW_BLOCK)
        out[start:stop] = gen_rows(wl, tensor, np.arange(start, stop))
    return out


def gen_gamma(wl: Workload, tensor: str) -> np.ndarray:
    """The fp32 weight vector gamma of Q or K."""
    D = wl.Dq if tensor == "q" else wl.Dk
    kind, a, b = wl.gamma
    rng = _rng(wl.seed, TENSOR_CODE[tensor], GAMMA_KEY)
    g = rng.uniform(a, b, size=D) if kind == "uniform" else rng.normal(a, b, size=D)
    return g.astype(np.float32)


def custom(name: str, T: int, Dq: int, Dk: int, P: int, dtype: str = "bf16",
           eps: float = 1e-6, seed: int = 1234, **kw) -> Workload:
    """A workload of arbitrary shape (for edge-case tests)."""
    return Workload(name, Ts=(T,), Dq=Dq, Dk=Dk, P=P, eps=eps, dtype=dtype, seed=seed, **kw)


def fused_bytes(T: int, Dq: int, Dk: int, elem_bytes: int) -> int:
    """Minimum bytes the fused pass must move: x read and y written once, gamma once."""
    return T * (Dq + Dk) * 2 * elem_bytes + 4 * (Dq + Dk)


def split_bytes(T: int, D: int, P: int, elem_bytes: int) -> int:
    """Minimum bytes of the split path for ONE tensor: x read twice, y written,
    the [T, P] fp32 statistics written once and read once, gamma once."""
    return 3 * T * D * elem_bytes + 2 * 4 * T * P + 4 * D


def stats_bytes(T: int, D: int, P: int, elem_bytes: int) -> int:
    """Bytes of the statistics pass alone: x read once, [T, P] fp32 written."""
    return T * D * elem_bytes + 4 * T * P


def apply_bytes(T: int, D: int, P: int, elem_bytes: int) -> int:
    """Bytes of the apply pass alone: x read, y written, stats read, gamma."""
    return 2 * T * D * elem_bytes + 4 * T * P + 4 * D


def gen_device_normal(T: int, D: int, seed: int, dtype, device, sigma: float = 1.0):
    """Large synthetic input drawn on the device with torch's seeded generator
    (N(0, sigma) in fp32, then rounded to `dtype`); for sizes too large to draw
    on the host in reasonable time. Rows needed by the oracle are copied back
    from the returned tensor."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    x = torch.empty((T, D), dtype=dtype, device=device)
    step = max(1, (1 << 28) // D)
    for t0 in range(0, T, step):
        t1 = min(T, t0 + step)
        x[t0:t1] = (torch.randn((t1 - t0, D), generator=gen, device=device) * sigma).to(dtype)
    return x


def gen_device_workload(wl: Workload, tensor: str, T: int, device, row0: int = 0):
    """The workload's recipe drawn on the device with torch's seeded generator:
    N(0, sigma), the same outlier channels, a per-token log-uniform scale when
    the workload has one, rounded to the storage dtype. The values differ from
    gen_tensor's (another random stream) but follow the same distribution; it
    serves timing runs, where drawing on the host would take too long."""
    import torch
    D = wl.Dq if tensor == "q" else wl.Dk
    tdt = {"bf16": torch.bfloat16, "f32": torch.float32, "e4m3": torch.float8_e4m3fn}[wl.dtype]
    gen = torch.Generator(device=device)
    gen.manual_seed(wl.seed * 1_000_003 + TENSOR_CODE[tensor] * 7919 + row0)
    sgen = torch.Generator(device=device)
    sgen.manual_seed(wl.seed * 1_000_003 + SCALE_KEY + row0)
    cols = torch.from_numpy(outlier_channels(wl, tensor, D)).to(device)
    x = torch.empty((T, D), dtype=tdt, device=device)
    step = max(1, (1 << 26) // D)
    for t0 in range(0, T, step):
        t1 = min(T, t0 + step)
        blk = torch.randn((t1 - t0, D), generator=gen, device=device) * wl.x_sigma
        if cols.numel():
            blk[:, cols] *= wl.outlier_factor
        if wl.token_scale_log10 is not None:
            lo, hi = wl.token_scale_log10
            u = torch.rand((t1 - t0, 1), generator=sgen, device=device) * (hi - lo) + lo
            blk *= torch.pow(10.0, u)
        x[t0:t1] = blk.to(tdt)
    return x
