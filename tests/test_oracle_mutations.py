"""The oracle's pins catch plausible mistakes.

Each mutant below is a copy of oracle/kvq_oracle.c with one deliberate slip
(a dropped sign, a transposed operand, an offset bin, a wrong rounding, a
missing scale, a swapped parameter ...).  It is compiled on the CPU into a
temporary library and the whole pin suite (tests/test_oracle_pins.py) is run
against it through KVQ_ORACLE_LIB; the suite must fail for every mutant.
"""
import os
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "kvq_oracle.c")

MUTANTS = {
    "no_sign": ("y[k] = s[k] * half_to_double(x_half[k]);", "y[k] = half_to_double(x_half[k]);"),
    "angle_offset": ("double t = (theta + PI) * (double)L", "double t = (theta + PI / 2) * (double)L"),
    "pair_transposed": ("double theta = atan2(v, u);", "double theta = atan2(u, v);"),
    "bin_edge_not_centre": ("return -PI + (a + 0.5) * 2.0 * PI", "return -PI + (a + 0.0) * 2.0 * PI"),
    "lin8_truncates": ("double q = floor(vq + 0.5);\n                c = q > 255.0",
                       "double q = floor(vq);\n                c = q > 255.0"),
    "lin8_255_levels": ("double vq = 255.0 * r[i] / M;", "double vq = 256.0 * r[i] / M;"),
    "log4_nibbles_swapped": ("norm_row[i / 2] |= (uint8_t)(c << (4 * (i % 2)));",
                             "norm_row[i / 2] |= (uint8_t)(c << (4 * (1 - i % 2)));"),
    "log4_lo_hi_swapped": ("put_half(param_row, lmin);\n        put_half(param_row + 2, lmax);",
                           "put_half(param_row, lmax);\n        put_half(param_row + 2, lmin);"),
    "unrotate_unscaled": ("x[k] = s[k] * w[k] / sqrt((double)d);", "x[k] = s[k] * w[k];"),
    "hadamard_or": ("popcount((unsigned)(j & k))", "popcount((unsigned)(j | k))"),
    "max_is_last": ("mx = r[i] > mx ? r[i] : mx;", "mx = r[i];"),
    "packing_reversed": ("put_bits(words, (long)i * b, b, (uint32_t)a[i]);",
                         "put_bits(words, (long)(P - 1 - i) * b, b, (uint32_t)a[i]);"),
    "softmax_unnormalised": ("o[j] += scores_tmp[t] / den * vhat[t * d + j];",
                             "o[j] += scores_tmp[t] * vhat[t * d + j];"),
    "zero_pair_not_special": ("if (u == 0.0 && v == 0.0) {", "if (0) {"),
    "rotated_cos_sin_swapped": ("sc += rh[i] * (qr[2 * i] * cos(th) + qr[2 * i + 1] * sin(th));",
                                "sc += rh[i] * (qr[2 * i] * sin(th) + qr[2 * i + 1] * cos(th));"),
    "log4_floor_missing": ("l[i] = log2(fmax(r[i], ldexp(1.0, -24)));", "l[i] = log2(r[i]);"),
    "rotate_scale_sqrt2": ("z[j] = zt[j] / sqrt((double)d);", "z[j] = zt[j] / sqrt((double)(2 * d));"),
    # the edge flags decide which GPU/oracle code differences the parity rule excuses
    "lin8_norm_flag_never": (
        "if (fabs((vq - floor(vq)) - 0.5) < EDGE_TOL * fmax(vq, 1.0)) fl[i] |= FLAG_NORM;",
        "if (0) fl[i] |= FLAG_NORM;"),
    "lin8_norm_flag_always": (
        "if (fabs((vq - floor(vq)) - 0.5) < EDGE_TOL * fmax(vq, 1.0)) fl[i] |= FLAG_NORM;",
        "fl[i] |= FLAG_NORM;"),
    "lin8_norm_tol_x1e3": ("< EDGE_TOL * fmax(vq, 1.0))", "< 1e3 * EDGE_TOL * fmax(vq, 1.0))"),
    "log4_norm_flag_never": (
        "if (fabs((vq - floor(vq)) - 0.5) < EDGE_TOL * fmax(fabs(vq), 1.0)) fl[i] |= FLAG_NORM;",
        "if (0) fl[i] |= FLAG_NORM;"),
    "log4_norm_flag_always": (
        "if (fabs((vq - floor(vq)) - 0.5) < EDGE_TOL * fmax(fabs(vq), 1.0)) fl[i] |= FLAG_NORM;",
        "fl[i] |= FLAG_NORM;"),
    "log4_norm_tol_x1e3": ("< EDGE_TOL * fmax(fabs(vq), 1.0))",
                           "< 1e3 * EDGE_TOL * fmax(fabs(vq), 1.0))"),
    "param_flag_never": ("int pflag = near_half_midpoint(mx, EDGE_TOL);", "int pflag = 0;"),
    "param_flag_always": ("norm_row[i] = (uint8_t)c;\n            if (pflag) fl[i] |= FLAG_PARAM;",
                          "norm_row[i] = (uint8_t)c;\n            fl[i] |= FLAG_PARAM;"),
    "param_tol_x1e3": ("int pflag = near_half_midpoint(mx, EDGE_TOL);",
                       "int pflag = near_half_midpoint(mx, 1e3 * EDGE_TOL);"),
    "midpoint_wrong_upper_neighbour": ("double up = half_to_double((uint16_t)(h + 1));",
                                       "double up = half_to_double((uint16_t)(h + 2));"),
    "midpoint_wrong_lower_neighbour": ("double dn = half_to_double((uint16_t)(h - 1));",
                                       "double dn = half_to_double((uint16_t)(h - 2));"),
    "log4_param_hi_ignored": (
        "near_half_midpoint(lmin, EDGE_TOL) || near_half_midpoint(lmax, EDGE_TOL)",
        "near_half_midpoint(lmin, EDGE_TOL)"),
    "log4_param_lo_ignored": (
        "near_half_midpoint(lmin, EDGE_TOL) || near_half_midpoint(lmax, EDGE_TOL)",
        "near_half_midpoint(lmax, EDGE_TOL)"),
}


def _run_mutant(name, old, new, tmp):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site of {name} not unique"
    path_c = os.path.join(tmp, f"{name}.c")
    path_so = os.path.join(tmp, f"lib{name}.so")
    open(path_c, "w").write(src.replace(old, new))
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared",
                           "-o", path_so, path_c, "-lm"])
    env = dict(os.environ, KVQ_ORACLE_LIB=path_so)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return name, r.returncode, r.stdout[-400:]


def test_every_mutant_fails_a_pin():
    with tempfile.TemporaryDirectory() as tmp:
        with ThreadPoolExecutor(min(8, os.cpu_count() or 1)) as ex:
            results = list(ex.map(lambda kv: _run_mutant(kv[0], *kv[1], tmp), MUTANTS.items()))
    survivors = [(n, out) for n, rc, out in results if rc == 0]
    assert not survivors, f"mutants not caught by any pin: {survivors}"
    assert all(rc == 1 for _, rc, _ in results), results


if __name__ == "__main__":
    pytest.main([__file__, "-q"])
