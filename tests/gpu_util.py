"""Helpers for the GPU parity tests: host<->device transfer of stored values,
the tolerances, and error statistics against the float64 oracle.

Tolerances
----------
* bf16 outputs: |y - y_oracle| <= 2^-7 |y_oracle| + 2^-133 (one bf16 ulp of
  relative error; the absolute floor is the bf16 subnormal quantum and only
  matters for y ~ 0). The kernel rounds an fp32 value to bf16 once (at most
  half an ulp, 2^-9 relative) and the fp32 work before it adds ~1e-6, so the
  bound has a 4x margin.
* fp32 outputs: |y - y_oracle| <= 1e-5 |y_oracle|, and y_oracle = 0 gives 0.
* FP8 E4M3 outputs: |y - y_oracle| <= 2^-3 |y_oracle| + 2^-9. Rounding to
  nearest costs at most 2^-4 relative on normals (3 mantissa bits) and 2^-10
  absolute on subnormals (quantum 2^-9), so the bound has a 2x margin.
* fp32 shard sums: all terms are non-negative, so the relative error of a
  sum formed by a tree of depth n is at most n u / (1 - n u), u = 2^-24. A
  term passes through vec - 1 fma roundings, at most vmax chain additions,
  5 butterfly additions and K group additions: n = vec + vmax + K + 5.
"""
from __future__ import annotations

import numpy as np
import torch

U24 = 2.0 ** -24


def to_device(a: np.ndarray, device="cuda") -> torch.Tensor:
    """Stored values (fp32, bf16 bits as uint16, E4M3 codes as uint8) -> CUDA tensor."""
    if a.dtype == np.uint8:
        return torch.from_numpy(np.ascontiguousarray(a)).view(torch.float8_e4m3fn).to(device)
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def to_host(t: torch.Tensor) -> np.ndarray:
    """CUDA tensor -> stored values (fp32 array, or bf16 bits as uint16)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def bits(t: torch.Tensor) -> torch.Tensor:
    """The raw bit patterns of a tensor (for bit-for-bit comparisons)."""
    return t.view({1: torch.uint8, 2: torch.int16, 4: torch.int32}[t.element_size()])


def widen(a: np.ndarray) -> np.ndarray:
    if a.dtype == np.uint8:
        import qknorm_workloads
        return qknorm_workloads.storage_to_f64(a, "e4m3")
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def rtol_of(dtype: str) -> float:
    return {"bf16": 2.0 ** -7, "e4m3": 2.0 ** -3}.get(dtype, 1e-5)


def check_outputs(y_dev_stored: np.ndarray, y_oracle: np.ndarray, dtype: str, what: str = ""):
    """Assert the element-wise bound; return (max_abs, mae, rmse, max_rel, exact_rate)."""
    y = widen(y_dev_stored)
    diff = np.abs(y - y_oracle)
    if dtype == "bf16":
        bound = 2.0 ** -7 * np.abs(y_oracle) + 2.0 ** -133
    elif dtype == "e4m3":
        # One E4M3 ulp of relative error (3 mantissa bits), and the smallest
        # subnormal 2^-9 as the absolute floor; outputs must be inside +-448.
        assert np.abs(y_oracle).max() < 448, "outputs beyond the E4M3 range"
        bound = 2.0 ** -3 * np.abs(y_oracle) + 2.0 ** -9
    else:
        bound = 1e-5 * np.abs(y_oracle)
    bad = diff > bound
    if bad.any():
        idx = np.argwhere(bad)[0]
        raise AssertionError(
            f"{what}: {int(bad.sum())} elements out of tolerance; first at {tuple(idx)}: "
            f"gpu {y[tuple(idx)]!r} oracle {y_oracle[tuple(idx)]!r}")
    rel = diff / np.maximum(np.abs(y_oracle), 1e-300)
    exact = None
    if dtype == "bf16":
        ref_bits = rne_bf16(y_oracle)
        exact = float(np.mean(ref_bits == y_dev_stored))
    return (float(diff.max()), float(diff.mean()), float(np.sqrt(np.mean(diff ** 2))),
            float(rel.max()), exact)


def rne_bf16(y64: np.ndarray) -> np.ndarray:
    """Round float64 to bf16 bits (through fp32), for the exact-match rate."""
    f32 = y64.astype(np.float32)
    bits = f32.view(np.uint32).astype(np.uint64)
    return ((bits + 0x7FFF + ((bits >> 16) & 1)) >> 16).astype(np.uint16)


def stats_depth(D: int, P: int, dtype: str) -> int:
    vec = {"bf16": 8, "e4m3": 16}.get(dtype, 4)
    nv = D // P // vec
    K = max(1, -(-nv // 256))
    vmax = -(-nv // (32 * K))
    return vec + vmax + K + 5


def check_stats(S_dev: np.ndarray, S_oracle: np.ndarray, D: int, P: int, dtype: str, what=""):
    n = stats_depth(D, P, dtype)
    tol = n * U24 / (1 - n * U24)
    err = np.abs(S_dev.astype(np.float64) - S_oracle)
    bound = tol * S_oracle
    bad = err > bound
    if bad.any():
        idx = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: shard sum out of tolerance at {tuple(idx)}: "
                             f"gpu {S_dev[tuple(idx)]!r} oracle {S_oracle[tuple(idx)]!r} (n={n})")
    return float(np.max(err / np.maximum(S_oracle, 1e-300))) if err.size else 0.0
