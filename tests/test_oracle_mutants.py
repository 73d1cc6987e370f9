"""Planted mistakes in the oracle must each fail at least one pin (CPU only).

Each mutant is a copy of ``oracle/qknorm_oracle.c`` with one plausible
mistake (a dropped term, a wrong divisor, a misplaced epsilon, a wrong index
or stride), compiled to its own library in a temporary directory. The test
passes when some pin of ``oracle_pins`` rejects the mutant, which shows that
the pins would catch that mistake in the real oracle.
"""
import importlib.util
import os

import pytest

import oracle
import oracle_pins

MUTANTS = {
    # Phase B divisor: the shard width instead of the full width.
    "mean_over_shard_width": [("S / (double)D;", "S / (double)(D / P);")],
    # eps added outside the root.
    "eps_outside_sqrt": [("1.0 / sqrt(m + eps)", "1.0 / (sqrt(m) + eps)")],
    # eps dropped.
    "eps_dropped": [("1.0 / sqrt(m + eps)", "1.0 / sqrt(m)")],
    # eps added to the sum instead of the mean.
    "eps_on_sum": [("double m = S / (double)D;", "double m = (S + eps) / (double)D;"),
                   ("1.0 / sqrt(m + eps)", "1.0 / sqrt(m)")],
    # The root instead of its inverse.
    "rms_not_inverse": [("1.0 / sqrt(m + eps)", "sqrt(m + eps)")],
    # gamma indexed back to front.
    "gamma_reversed": [("(double)gamma[j]", "(double)gamma[D - 1 - j]")],
    # gamma dropped from the weight multiply.
    "gamma_dropped": [("* (double)gamma[j]", "* 1.0")],
    # Last element of every shard skipped.
    "shard_short_by_one": [("j < p * w + w;", "j < p * w + w - 1;")],
    # Shards start one element late.
    "shard_offset": [("int64_t j = p * w;", "int64_t j = p * w + (p > 0);")],
    # Last shard left out of the global sum.
    "last_shard_dropped": [("S += s;", "if (p < P - 1) S += s;")],
    # Sum of values instead of squares.
    "square_dropped": [("s += v * v;", "s += v;")],
    # Signed square.
    "signed_square": [("s += v * v;", "s += v * fabs(v);")],
    # Row stride counted in elements, not bytes.
    "row_stride_elements": [("(size_t)t * (size_t)D * es", "(size_t)t * (size_t)D")],
    # bf16 widened from the wrong bit position.
    "bf16_shift": [("<< 16;", "<< 15;")],
    # bf16 sign bit lost.
    "bf16_sign": [("(uint32_t)((const uint16_t *)x)[i] << 16;",
                   "((uint32_t)((const uint16_t *)x)[i] & 0x7fffu) << 16;")],
    # FP8 exponent bias off by one.
    "e4m3_bias": [("ldexp(1.0 + m / 8.0, e - 7)", "ldexp(1.0 + m / 8.0, e - 8)")],
    # FP8 subnormals scaled like normals.
    "e4m3_subnormal": [("ldexp((double)m, -9)", "ldexp((double)m, -10)")],
    # Outputs written to the first row only.
    "y_row_stride": [("y[t * D + j] = u * rt;", "y[j] = u * rt;")],
}


def _build_mutant(tmpdir, name, edits):
    with open(oracle.SOURCE) as f:
        src = f.read()
    for old, new in edits:
        assert old in src, f"mutant {name}: pattern {old!r} not in the oracle source"
        src = src.replace(old, new)
    path = os.path.join(tmpdir, f"{name}.c")
    with open(path, "w") as f:
        f.write(src)
    return oracle.build(force=True, source=path, output=os.path.join(tmpdir, f"lib{name}.so"))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    lib = _build_mutant(str(tmp_path), name, MUTANTS[name])
    orc = oracle.Oracle(lib)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(orc)
        except (AssertionError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"no pin rejects the planted mistake {name}"


# Mistakes in the Python front end's composition of Q and K (Oracle.qknorm in
# oracle/__init__.py): each is an edit of that file's text, loaded as its own
# module over the real compiled oracle.
PY_MUTANTS = {
    # Q normalised with K's weight and K with Q's.
    "qknorm_gamma_swapped": [("self.rmsnorm(q, gamma_q,", "self.rmsnorm(q, gamma_k,"),
                             ("self.rmsnorm(k, gamma_k,", "self.rmsnorm(k, gamma_q,")],
    # (yk, yq) returned in place of (yq, yk).
    "qknorm_outputs_swapped": [("return yq, yk, rq, rk", "return yk, yq, rk, rq")],
    # K normalised with Q's statistic (the factor of the wrong tensor).
    "qknorm_k_uses_q_factor": [("return yq, yk, rq, rk",
                                "return yq, yk * (rq / rk)[:, None], rq, rq")],
    # eps dropped for K only.
    "qknorm_k_eps_dropped": [("self.rmsnorm(k, gamma_k, P, eps,", "self.rmsnorm(k, gamma_k, P, 0.0,")],
}


def _load_py_mutant(tmpdir, name, edits):
    src_path = os.path.join(os.path.dirname(oracle.SOURCE), "__init__.py")
    with open(src_path) as f:
        src = f.read()
    for old, new in edits:
        assert old in src, f"mutant {name}: pattern {old!r} not in the oracle front end"
        src = src.replace(old, new)
    path = os.path.join(tmpdir, f"oracle_{name}.py")
    with open(path, "w") as f:
        f.write(src)
    spec = importlib.util.spec_from_file_location(f"oracle_{name}", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.Oracle(oracle.build())


@pytest.mark.parametrize("name", sorted(PY_MUTANTS))
def test_front_end_mutant_is_caught(tmp_path, name):
    orc = _load_py_mutant(str(tmp_path), name, PY_MUTANTS[name])
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(orc)
        except (AssertionError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"no pin rejects the planted mistake {name}"
