"""Float64 CPU oracle for layerwise QK-Norm (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package. The product path (``qk_norm_attention_b200``)
never imports it and shares no code with it.

The arithmetic lives in ``qknorm_oracle.c`` (plain C loops in double, built
here with gcc); this module only builds it, loads it with ctypes and converts
numpy arrays. What it computes follows the SwiftQK technical review
("SwiftQK: When Normalization Becomes the Bottleneck of Tensor Parallelism"):
Eq. (1) in "Prerequisites", and Section 3, Algorithm 1, Phases A-C.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "qknorm_oracle.c")
LIBRARY = os.path.join(_HERE, "liboracle.so")

_DTYPE_CODE = {"f32": 0, "bf16": 1, "e4m3": 2}
_STORAGE = {"f32": np.float32, "bf16": np.uint16, "e4m3": np.uint8}


def build(force: bool = False, source: str = SOURCE, output: str = LIBRARY) -> str:
    """Compile the oracle with gcc (OpenMP over tokens). Returns the library path."""
    if (not force and os.path.exists(output)
            and os.path.getmtime(output) >= os.path.getmtime(source)):
        return output
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-o", output, source, "-lm"]
    subprocess.run(cmd, check=True)
    return output


class Oracle:
    """ctypes front end of one compiled oracle library."""

    def __init__(self, path: Optional[str] = None):
        self.path = path or build()
        lib = ctypes.CDLL(self.path)
        i64, vp, dp = ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p
        lib.qko_partial_sumsq.argtypes = [vp, ctypes.c_int, i64, i64, i64, dp, ctypes.c_int]
        lib.qko_partial_sumsq.restype = ctypes.c_int
        lib.qko_rmsnorm.argtypes = [vp, ctypes.c_int, vp, i64, i64, i64, ctypes.c_double,
                                    dp, dp, ctypes.c_int]
        lib.qko_rmsnorm.restype = ctypes.c_int
        lib.qko_xgamma.argtypes = [vp, ctypes.c_int, vp, i64, i64, dp, ctypes.c_int]
        lib.qko_xgamma.restype = ctypes.c_int
        lib.qko_has_openmp.restype = ctypes.c_int
        self._lib = lib

    @property
    def has_openmp(self) -> bool:
        return bool(self._lib.qko_has_openmp())

    @staticmethod
    def _prep(x: np.ndarray, dtype: str) -> np.ndarray:
        want = _STORAGE[dtype]
        if x.ndim != 2 or x.dtype != want:
            raise ValueError(f"x must be a 2-D {want.__name__} array for dtype {dtype}")
        return np.ascontiguousarray(x)

    def partial_sumsq(self, x: np.ndarray, P: int, dtype: str, nthreads: int = 1) -> np.ndarray:
        """S[t, p]: float64 sum of squares of shard p of row t (Algorithm 1, Phase A)."""
        x = self._prep(x, dtype)
        T, D = x.shape
        S = np.empty((T, P), dtype=np.float64)
        rc = self._lib.qko_partial_sumsq(x.ctypes.data, _DTYPE_CODE[dtype], T, D, P,
                                         S.ctypes.data, nthreads)
        if rc != 0:
            raise ValueError("oracle rejected the arguments")
        return S

    def rmsnorm(self, x: np.ndarray, gamma: np.ndarray, P: int, eps: float, dtype: str,
                nthreads: int = 1, want_y: bool = True) -> Tuple[Optional[np.ndarray], np.ndarray]:
        """(y, r): y[t, j] = (x[t, j] * gamma[j]) * r[t], r[t] = 1/sqrt(S[t]/D + eps).

        ``eps`` is used as given (pass ``float(np.float32(eps))`` to match a
        kernel that receives fp32). ``y`` is float64 and unrounded.
        """
        x = self._prep(x, dtype)
        T, D = x.shape
        g = np.ascontiguousarray(gamma, dtype=np.float32)
        if g.shape != (D,):
            raise ValueError("gamma must have shape [D]")
        y = np.empty((T, D), dtype=np.float64) if want_y else None
        r = np.empty(T, dtype=np.float64)
        rc = self._lib.qko_rmsnorm(x.ctypes.data, _DTYPE_CODE[dtype], g.ctypes.data, T, D, P,
                                   float(eps), y.ctypes.data if want_y else None,
                                   r.ctypes.data, nthreads)
        if rc != 0:
            raise ValueError("oracle rejected the arguments")
        return y, r

    def xgamma(self, x: np.ndarray, gamma: np.ndarray, dtype: str, nthreads: int = 1) -> np.ndarray:
        """u[t, j] = x[t, j] * gamma[j] in float64 (the weight multiply alone)."""
        x = self._prep(x, dtype)
        T, D = x.shape
        g = np.ascontiguousarray(gamma, dtype=np.float32)
        if g.shape != (D,):
            raise ValueError("gamma must have shape [D]")
        u = np.empty((T, D), dtype=np.float64)
        if self._lib.qko_xgamma(x.ctypes.data, _DTYPE_CODE[dtype], g.ctypes.data, T, D,
                                u.ctypes.data, nthreads) != 0:
            raise ValueError("oracle rejected the arguments")
        return u

    def inv_rms(self, x: np.ndarray, P: int, eps: float, dtype: str, nthreads: int = 1) -> np.ndarray:
        """r[t] = 1/sqrt(S[t]/D + eps) alone (the per-token dynamic statistic)."""
        D = x.shape[1]
        _, r = self.rmsnorm(x, np.ones(D, dtype=np.float32), P, eps, dtype, nthreads, want_y=False)
        return r

    def headwise(self, x: np.ndarray, gamma: np.ndarray, head_dim: int, eps: float, dtype: str,
                 nthreads: int = 1) -> np.ndarray:
        """Headwise RMSNorm: each head's head_dim values normalised on their
        own (the same RMSNorm on rows of length head_dim), gamma [head_dim]
        shared by the heads. x [T, H*head_dim] -> y [T, H*head_dim], float64."""
        x = self._prep(x, dtype)
        T, D = x.shape
        if D % head_dim:
            raise ValueError("width must be a multiple of head_dim")
        y, _ = self.rmsnorm(np.ascontiguousarray(x.reshape(T * (D // head_dim), head_dim)),
                            gamma, 1, eps, dtype, nthreads)
        return y.reshape(T, D)

    def qknorm(self, q, k, gamma_q, gamma_k, P, eps, dtype, nthreads: int = 1):
        """Layerwise QK-Norm: the RMSNorm above applied to Q and, on its own, to K."""
        yq, rq = self.rmsnorm(q, gamma_q, P, eps, dtype, nthreads)
        yk, rk = self.rmsnorm(k, gamma_k, P, eps, dtype, nthreads)
        return yq, yk, rq, rk


_default: Optional[Oracle] = None


def get() -> Oracle:
    """The oracle built from this directory's source (built on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default
