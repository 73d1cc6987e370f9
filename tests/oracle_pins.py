"""Pins that tie the float64 oracle to facts fixed outside it.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError
when the oracle disagrees with:

* the values the SwiftQK technical review prints for its worked example
  (Section 4b, Eqs. (2)-(8)), stored in ``golden/worked_example.txt``;
* exact rational arithmetic (``fractions.Fraction``) and a 50-digit decimal
  square root on tiny inputs (brute force);
* a library routine the special case P = 1 reduces to
  (``torch.nn.functional.rms_norm`` in float64);
* closed forms of Eq. (1): unit RMS of the output when gamma = 1, the constant
  row, the scale law r(c x) = 1 / sqrt(c^2 m + eps);
* invariants the review states: the per-shard sums add up to the unsharded
  sum for every shard count (Section 4b, "Sanity check against the
  un-sharded computation"), and a per-token positive pre-scale cancels
  exactly (the deferred normalisation of the "deferred attention RMSNorm"
  pull request).

The same functions run against copies of the oracle with planted mistakes
(``test_oracle_mutants.py``) to show that each plausible mistake fails one.
"""
from __future__ import annotations

import math
import os
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np

import qknorm_workloads as W

U53 = 2.0 ** -53
GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ----------------------------------------------------------------------------- helpers

def load_worked_example():
    """Parse golden/worked_example.txt into {name: (decimals or None, [values])}."""
    out = {}
    with open(os.path.join(GOLDEN, "worked_example.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, dec, *vals = line.split()
            out[name] = (None if dec == "exact" else int(dec), [float(v) for v in vals])
    return out


def widen(x, dtype):
    return W.storage_to_f64(x, dtype)



def exact_shard_sums(row64, P):
    """Exact Fraction sum of squares of each shard of one widened row."""
    D = len(row64)
    w = D // P
    return [sum((Fraction(float(v)) ** 2 for v in row64[p * w:(p + 1) * w]), Fraction(0))
            for p in range(P)]


def dec_sqrt(fr: Fraction) -> Decimal:
    getcontext().prec = 50
    return (Decimal(fr.numerator) / Decimal(fr.denominator)).sqrt()


def exact_y(row64, gamma32, eps: float):
    """y_j of Eq. (1) from exact sums and a 50-digit root; returns (y list, r)."""
    getcontext().prec = 50
    D = len(row64)
    S = sum((Fraction(float(v)) ** 2 for v in row64), Fraction(0))
    m_eps = S / D + Fraction(eps)
    r = Decimal(1) / dec_sqrt(m_eps)
    y = [float(Decimal(float(row64[j])) * Decimal(float(gamma32[j])) * r) for j in range(D)]
    return y, float(r)


def rel_err(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.maximum(np.abs(b), np.finfo(np.float64).tiny)
    return float(np.max(np.abs(a - b) / den)) if a.size else 0.0


def tiny_inputs(T=4):
    wl = W.WORKLOADS["tiny"]
    q = W.gen_rows(wl, "q", range(T))
    k = W.gen_rows(wl, "k", range(T))
    return wl, q, k, W.gen_gamma(wl, "q"), W.gen_gamma(wl, "k")


def tiny_q(T=4):
    """Rows of the tiny workload's Q and its gamma (fp32)."""
    wl, q, k, gq, gk = tiny_inputs(T)
    return q, gq


def bf16_inputs(T, D, seed, sigma=1.0):
    wl = W.custom("pin", T, D, D, 1, dtype="bf16", seed=seed, x_sigma=sigma)
    return W.gen_rows(wl, "q", range(T)), W.gen_gamma(wl, "q")


# ----------------------------------------------------------------------------- pins

def pin_worked_example(orc):
    """Section 4b, Eqs. (2)-(8): shard sums, global sum, factor and outputs."""
    g = load_worked_example()
    x = np.array([g["x"][1]], dtype=np.float64)
    D = int(g["H_total"][1][0])
    P = int(g["shards"][1][0])
    eps = g["eps"][1][0]
    gamma = np.ones(D, dtype=np.float32)
    for dtype in ("f32", "bf16"):
        xs = W.to_storage(x, dtype)
        assert np.array_equal(widen(xs, dtype), x), "example values must be exact in storage"
        S = orc.partial_sumsq(xs, P, dtype)[0]
        assert list(S) == g["S_local"][1], f"S_local {list(S)} != Eqs. (3),(4)"
        assert float(np.sum(S)) == g["S_global"][1][0]
        y, r = orc.rmsnorm(xs, gamma, P, eps, dtype)
        r = float(r[0])
        # Eq. (6): printed to 4 decimals.
        assert abs(r - g["rms_inv"][1][0]) <= 0.5e-4, f"RMS_inv {r}"
        assert abs(1.0 / r - g["sqrt_mean_eps"][1][0]) <= 0.5e-4, f"sqrt {1.0 / r}"
        # The mean the page prints is exact: 1/r^2 - eps recovers it to rounding.
        assert abs((1.0 / r ** 2 - eps) - g["mean"][1][0]) <= 1e-12
        # Eqs. (7),(8): 3 decimals of y formed with RMS^-1 rounded to 4 decimals.
        for j, (yj, pj) in enumerate(zip(y[0], g["y"][1])):
            tol = 0.5e-3 + 0.5e-4 * abs(x[0, j]) + 1e-12
            assert abs(yj - pj) <= tol, f"y[{j}] = {yj} vs printed {pj}"


def pin_shard_sums_exact(orc):
    """Phase A against exact rationals, for every power-of-two shard count."""
    wl, q, k, gq, gk = tiny_inputs(2)
    for x in (q, k):
        x64 = widen(x, "f32")
        D = x.shape[1]
        P = 1
        while P <= D:
            S = orc.partial_sumsq(x, P, "f32")
            w = D // P
            for t in range(x.shape[0]):
                ex = exact_shard_sums(x64[t], P)
                for p in range(P):
                    bound = max(w - 1, 1) * U53 * float(ex[p]) * 1.0000001
                    assert abs(Fraction(float(S[t, p])) - ex[p]) <= Fraction(bound), \
                        f"S[{t},{p}] (P={P}) off the exact shard sum"
            P *= 2


def pin_one_hot_shards(orc):
    """A row with one nonzero element puts v^2 in exactly one shard: j // w."""
    D, P = 48, 6
    w = D // P
    for dtype in ("f32", "bf16"):
        rows = np.zeros((D, D))
        for j in range(D):
            rows[j, j] = -1.5 if j % 2 else 2.25
        xs = W.to_storage(rows, dtype)
        S = orc.partial_sumsq(xs, P, dtype)
        for j in range(D):
            want = np.zeros(P)
            want[j // w] = rows[j, j] ** 2
            assert np.array_equal(S[j], want), f"{dtype}: element {j} landed in the wrong shard"


def pin_additivity_over_P(orc):
    """The factor does not depend on how many shards the width is cut into."""
    for dtype, (x, g) in (("f32", tiny_q(4)),
                          ("bf16", bf16_inputs(5, 1280, seed=7))):
        D = x.shape[1]
        _, r1 = orc.rmsnorm(x, g, 1, 1e-6, dtype)
        for P in [p for p in range(1, D + 1) if D % p == 0]:
            SP = orc.partial_sumsq(x, P, dtype)
            S1 = orc.partial_sumsq(x, 1, dtype)[:, 0]
            assert rel_err(SP.sum(axis=1), S1) <= 2 * D * U53, f"sum of shards != full sum, P={P}"
            _, rP = orc.rmsnorm(x, g, P, 1e-6, dtype)
            assert rel_err(rP, r1) <= 2 * D * U53, f"factor changes with P={P}"


def pin_bruteforce(orc):
    """Every output of 4-token inputs against exact sums and a 50-digit root."""
    wl, q, k, gq, gk = tiny_inputs(4)
    cases = [(q, gq, wl.P, "f32"), (k, gk, wl.P, "f32")]
    xb, gb = bf16_inputs(4, 8, seed=11)
    gb = W.to_storage(np.linspace(0.5, 1.5, 8) * np.array([1, -1, 1, 1, -1, 1, 1, 1]), "f32")
    cases.append((xb, gb, 2, "bf16"))
    for eps in (1e-6, 0.3):
        for x, g, P, dtype in cases:
            y, r = orc.rmsnorm(x, g, P, eps, dtype)
            x64 = widen(x, dtype)
            D = x.shape[1]
            tol = (D + 8) * U53
            for t in range(x.shape[0]):
                ye, re = exact_y(x64[t], g, eps)
                assert rel_err([r[t]], [re]) <= tol, f"r[{t}]"
                assert rel_err(y[t], ye) <= tol, f"y[{t}] ({dtype}, eps={eps})"


def pin_library_rms_norm(orc):
    """P = 1 is textbook RMSNorm: torch.nn.functional.rms_norm in float64.
    Any P gives the same result, since the shard sums add up (Section 4b)."""
    import torch
    for dtype, (x, g) in (("f32", tiny_q(4)),
                          ("bf16", bf16_inputs(9, 5120, seed=3, sigma=1.5))):
        x64 = torch.from_numpy(widen(x, dtype))
        D = x.shape[1]
        for eps in (1e-6, 1e-5, 0.2):
            ref = torch.nn.functional.rms_norm(x64, (D,), weight=torch.from_numpy(g.astype(np.float64)),
                                               eps=eps).numpy()
            for P in (1, 2, 4, 8):
                y, _ = orc.rmsnorm(x, g, P, eps, dtype)
                assert rel_err(y, ref) <= 4 * (D + 8) * U53, f"{dtype} P={P} eps={eps}"


def pin_unit_rms(orc):
    """Eq. (1) with gamma = 1: mean_j y_j^2 = m / (m + eps); exactly 1 at eps = 0."""
    for dtype, (x, _) in (("f32", tiny_q(4)), ("bf16", bf16_inputs(6, 4096, seed=5))):
        D = x.shape[1]
        ones = np.ones(D, dtype=np.float32)
        x64 = widen(x, dtype)
        for eps in (0.0, 1e-6, 0.25, 3.0):
            y, _ = orc.rmsnorm(x, ones, 4, eps, dtype)
            for t in range(x.shape[0]):
                m = math.fsum(float(v) ** 2 for v in x64[t]) / D
                got = math.fsum(float(v) ** 2 for v in y[t]) / D
                assert abs(got - m / (m + eps)) <= 4 * (D + 8) * U53, f"{dtype} eps={eps} t={t}"


def pin_constant_row(orc):
    """x_j = c for all j: y_j = gamma_j * c / sqrt(c^2 + eps)."""
    getcontext().prec = 50
    D, P = 64, 4
    g = W.to_storage(np.linspace(-2.0, 2.0, D), "f32")
    for dtype in ("f32", "bf16"):
        for c in (1.5, -0.25, 96.0):
            xs = W.to_storage(np.full((1, D), c), dtype)
            for eps in (1e-6, 0.5):
                y, _ = orc.rmsnorm(xs, g, P, eps, dtype)
                den = (Decimal(c) * Decimal(c) + Decimal(eps)).sqrt()
                want = [float(Decimal(float(gj)) * Decimal(c) / den) for gj in g]
                assert rel_err(y[0], want) <= 8 * U53, f"{dtype} c={c} eps={eps}"


def pin_scale_law(orc):
    """y(c x) = y(x) for c = 2^k at eps = 0 (bitwise: powers of two commute with
    rounding); with eps > 0, r(c x) = 1 / sqrt(c^2 m + eps)."""
    for dtype, (x, g) in (("f32", tiny_q(4)), ("bf16", bf16_inputs(4, 4096, seed=8))):
        x64 = widen(x, dtype)
        D = x.shape[1]
        y0, r0 = orc.rmsnorm(x, g, 4, 0.0, dtype)
        for kexp in (-4, -1, 3, 4):
            c = 2.0 ** kexp
            xc = W.to_storage(x64 * c, dtype)
            assert np.array_equal(widen(xc, dtype), x64 * c)
            yc, rc = orc.rmsnorm(xc, g, 4, 0.0, dtype)
            assert np.array_equal(yc, y0), f"{dtype}: y(2^{kexp} x) != y(x) at eps=0"
            for eps in (1e-5, 0.5):
                _, r1 = orc.rmsnorm(x, g, 4, eps, dtype)
                _, r2 = orc.rmsnorm(xc, g, 4, eps, dtype)
                for t in range(x.shape[0]):
                    m = math.fsum(float(v) ** 2 for v in x64[t]) / D
                    assert rel_err([r1[t]], [1 / math.sqrt(m + eps)]) <= (D + 8) * U53
                    assert rel_err([r2[t]], [1 / math.sqrt(c * c * m + eps)]) <= (D + 8) * U53


def pin_deferred_prescale(orc):
    """A per-token positive pre-scale s_t (the deferred inverse RMS of an earlier
    norm) cancels when the row is normalised again: y(s_t z_t) = y(z_t) at eps = 0
    (bitwise for s_t = 2^k_t); at eps > 0, r(s z) = 1/sqrt(s^2 m + eps)."""
    for dtype, (x, g) in (("f32", tiny_q(4)), ("bf16", bf16_inputs(8, 4096, seed=12))):
        x64 = widen(x, dtype)
        T, D = x.shape
        kexp = np.array([(-3, 5, 0, 2, -6, 1, 4, -2)[t % 8] for t in range(T)], dtype=np.float64)
        s = 2.0 ** kexp
        xs = W.to_storage(x64 * s[:, None], dtype)
        y0, _ = orc.rmsnorm(x, g, 8 if D % 8 == 0 else 2, 0.0, dtype)
        y1, _ = orc.rmsnorm(xs, g, 8 if D % 8 == 0 else 2, 0.0, dtype)
        assert np.array_equal(y0, y1), f"{dtype}: per-token pre-scale did not cancel"
        _, r1 = orc.rmsnorm(xs, g, 2, 1e-5, dtype)
        for t in range(T):
            m = math.fsum(float(v) ** 2 for v in x64[t]) / D
            assert rel_err([r1[t]], [1 / math.sqrt(s[t] ** 2 * m + 1e-5)]) <= (D + 8) * U53


def pin_row_independence(orc):
    """Each row uses only its own sum: a row's output does not change when the
    other rows do, and stacked rows equal rows normalised one at a time."""
    wl, q, k, gq, gk = tiny_inputs(4)
    y_all, r_all = orc.rmsnorm(q, gq, 2, 1e-6, "f32")
    for t in range(4):
        y_t, r_t = orc.rmsnorm(q[t:t + 1].copy(), gq, 2, 1e-6, "f32")
        assert np.array_equal(y_t[0], y_all[t]) and r_t[0] == r_all[t], f"row {t}"


def pin_xgamma(orc):
    """The weight multiply alone: exact products of stored values (a double
    product of a bf16 or fp32 value and an fp32 weight is exact); gamma = 1
    returns x; y = xgamma * r where r is the factor (Eq. (1) factorises)."""
    for dtype, (x, g) in (("f32", tiny_q(4)), ("bf16", bf16_inputs(5, 1280, seed=13))):
        x64 = widen(x, dtype)
        u = orc.xgamma(x, g, dtype)
        for t in range(x.shape[0]):
            for j in (0, 1, x.shape[1] // 2, x.shape[1] - 1):
                assert Fraction(float(u[t, j])) == Fraction(float(x64[t, j])) * Fraction(float(g[j]))
        assert np.array_equal(orc.xgamma(x, np.ones(x.shape[1], np.float32), dtype), x64)
        y, r = orc.rmsnorm(x, g, 4, 1e-6, dtype)
        assert np.array_equal(y, u * r[:, None])      # same two roundings: (x*g) then *r
        assert np.array_equal(orc.inv_rms(x, 4, 1e-6, dtype), r)


def pin_headwise(orc):
    """Headwise form (one factor per head, gamma of head_dim shared by the
    heads): torch rms_norm over the last axis of [T, H, head_dim]; a one-hot
    head; heads independent of one another; unit RMS per head at gamma = 1."""
    import torch
    T, H, hd = 3, 5, 64
    x, _ = bf16_inputs(T, H * hd, seed=14)
    g = W.gen_gamma(W.custom("hw", 1, hd, hd, 1, seed=15), "q")
    x64 = widen(x, "bf16")
    for eps in (1e-6, 0.5):
        y = orc.headwise(x, g, hd, eps, "bf16")
        ref = torch.nn.functional.rms_norm(torch.from_numpy(x64).view(T, H, hd), (hd,),
                                           weight=torch.from_numpy(g.astype(np.float64)), eps=eps)
        assert rel_err(y, ref.reshape(T, H * hd).numpy()) <= 4 * (hd + 8) * U53
        ones = orc.headwise(x, np.ones(hd, np.float32), hd, eps, "bf16").reshape(T, H, hd)
        m = (x64.reshape(T, H, hd) ** 2).mean(axis=2)
        assert rel_err((ones ** 2).mean(axis=2), m / (m + eps)) <= 4 * (hd + 8) * U53
    one = np.zeros((1, H * hd))
    one[0, 2 * hd + 7] = 3.0
    y = orc.headwise(W.to_storage(one, "bf16"), g, hd, 1e-6, "bf16")
    want = np.zeros((1, H * hd))
    want[0, 2 * hd + 7] = float(g[7]) * 3.0 / math.sqrt(9.0 / hd + 1e-6)
    assert rel_err(y[0, 2 * hd + 7:2 * hd + 8], want[0, 2 * hd + 7:2 * hd + 8]) <= 8 * U53
    assert np.count_nonzero(y) == 1
    x2 = x.copy()
    x2[:, 3 * hd:4 * hd] = W.to_storage(np.full((T, hd), 0.75), "bf16")
    y1, y2 = orc.headwise(x, g, hd, 1e-6, "bf16"), orc.headwise(x2, g, hd, 1e-6, "bf16")
    keep = np.r_[0:3 * hd, 4 * hd:H * hd]
    assert np.array_equal(y1[:, keep], y2[:, keep])


def pin_qknorm(orc):
    """Layerwise QK-Norm of a layer: one factor over the whole Q row with
    gamma_q and, separately, one over the whole K row with gamma_k (the
    review's "Prerequisites", layerwise QK-Norm; Eq. (1) once per tensor).
    Each output, and each factor, is checked against exact sums and a 50-digit
    root of its OWN tensor with its OWN weight: the tiny workload (Dq == Dk,
    gamma_q != gamma_k) and a bf16 GQA-like case with Dk < Dq. A swapped
    weight, swapped outputs or K normalised with Q's statistic fails here
    even when the two widths are equal."""
    wl, q, k, gq, gk = tiny_inputs(4)
    assert not np.array_equal(gq, gk)
    cases = [(q, k, gq, gk, wl.P, "f32")]
    wq = W.custom("pinqk", 3, 48, 16, 2, dtype="bf16", seed=19)
    qb, kb = W.gen_rows(wq, "q", range(3)), W.gen_rows(wq, "k", range(3))
    gqb = W.to_storage(np.linspace(0.5, 1.5, 48), "f32")
    gkb = W.to_storage(np.linspace(-2.0, -0.25, 16), "f32")
    cases.append((qb, kb, gqb, gkb, 2, "bf16"))
    # Equal widths, the same rows in Q and K, different weights: only the
    # weights tell the two outputs apart.
    cases.append((q, q.copy(), gq, gk, wl.P, "f32"))
    for xq, xk, g_q, g_k, P, dtype in cases:
        for eps in (1e-6, 0.3):
            yq, yk, rq, rk = orc.qknorm(xq, xk, g_q, g_k, P, eps, dtype)
            assert yq.shape == xq.shape and yk.shape == xk.shape
            for x, g, y, r, name in ((xq, g_q, yq, rq, "q"), (xk, g_k, yk, rk, "k")):
                x64 = widen(x, dtype)
                tol = (x.shape[1] + 8) * U53
                for t in range(x.shape[0]):
                    ye, re = exact_y(x64[t], g, eps)
                    assert rel_err([r[t]], [re]) <= tol, f"qknorm r_{name}[{t}] ({dtype})"
                    assert rel_err(y[t], ye) <= tol, f"qknorm y_{name}[{t}] ({dtype}, eps={eps})"


def e4m3_inputs(T, D, seed, sigma=1.0):
    wl = W.custom("pin8", T, D, D, 1, dtype="e4m3", seed=seed, x_sigma=sigma)
    return W.gen_rows(wl, "q", range(T)), W.gen_gamma(wl, "q")


def pin_e4m3(orc):
    """FP8 E4M3 storage: codes fixed by the format (1.0 = 0x38, 448 = 0x7E,
    2^-9 = 0x01 the smallest subnormal, 2^-6 = 0x08 the smallest normal,
    -2 = 0xC0) widen exactly; torch's own float8_e4m3fn widening agrees on
    every finite code; RMSNorm of FP8 rows matches torch rms_norm and exact
    rational arithmetic."""
    import torch
    known = {0x38: 1.0, 0x7E: 448.0, 0x01: 2.0 ** -9, 0x08: 2.0 ** -6, 0xC0: -2.0, 0x00: 0.0}
    for code, val in known.items():
        x = np.zeros((1, 16), np.uint8)
        x[0, 3] = code
        S = orc.partial_sumsq(x, 1, "e4m3")[0, 0]
        assert S == val * val, (hex(code), S)
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    x = np.tile(codes[:, None], (1, 16))
    g1 = np.ones(16, np.float32)
    u = orc.xgamma(x, g1, "e4m3")
    assert np.array_equal(u[:, 0], ref)
    for xs, g in (e4m3_inputs(6, 512, seed=16), e4m3_inputs(4, 48, seed=17, sigma=40.0)):
        x64 = widen(xs, "e4m3")
        D = xs.shape[1]
        for P in (1, 2, 4):
            y, r = orc.rmsnorm(xs, g, P, 1e-6, "e4m3")
            t = torch.nn.functional.rms_norm(torch.from_numpy(x64), (D,),
                                             weight=torch.from_numpy(g.astype(np.float64)), eps=1e-6)
            assert rel_err(y, t.numpy()) <= 4 * (D + 8) * U53
        for t in range(xs.shape[0]):
            ye, re = exact_y(x64[t], g, 1e-6)
            assert rel_err(y[t], ye) <= (D + 8) * U53


ALL_PINS = [
    pin_worked_example,
    pin_shard_sums_exact,
    pin_one_hot_shards,
    pin_additivity_over_P,
    pin_bruteforce,
    pin_library_rms_norm,
    pin_unit_rms,
    pin_constant_row,
    pin_scale_law,
    pin_deferred_prescale,
    pin_row_independence,
    pin_xgamma,
    pin_headwise,
    pin_qknorm,
    pin_e4m3,
]
