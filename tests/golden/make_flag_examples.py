"""Writes tests/golden/flag_examples.json: vectors built by hand so that a norm
code or an fp16 parameter of the codec lies exactly on (or just off) one of its
rounding edges, with the flags and codes the definition implies.

Codec ("TurboAngle: Near-Lossless KV Cache Compression via Uniform Angle
Quantization", Abstract): z = H D x / sqrt(d), pairs (z[2i], z[2i+1]), 8-bit
linear key norms c = floor(255 r / M + 1/2) with M = fp16(max r), 4-bit log
value norms c = floor(15 (l - LO) / (HI - LO) + 1/2) with l = log2 r and
LO / HI = fp16(min / max l).  The flags are the oracle's reading of where two
correct implementations may differ: a norm code within 1e-6 (relative to
max(|v|, 1)) of its rounding edge, and a vector whose fp16 parameter lies
within 1e-6 (relative) of an fp16 rounding midpoint.

Construction: d = 16, D = I, the rotated vector z is chosen (integer pairs),
and x = H z / 4 (H H = 16 I, so H x / sqrt(16) = z).  Every x entry is an
exact fp16 value (checked: multiples of 1/4 below 512, of 1/2 below 1024).  Angles
use L = 3, whose bin edges (theta = -pi/3, pi/3, pi) are far from every pair
used here.  Nothing in this script calls the oracle: the expected codes and
flags are worked out in exact rational arithmetic, or with 60-digit decimal
logarithms where a logarithm is involved, and every decision is checked to sit
either exactly on an edge or well clear of the 1e-6 band.

Run from the repository root: python tests/golden/make_flag_examples.py
"""
from __future__ import annotations

import json
import math
import os
from decimal import Decimal, getcontext
from fractions import Fraction

getcontext().prec = 60
D16 = 16
TOL = Decimal("1e-6")
HERE = os.path.dirname(os.path.abspath(__file__))


def sylvester(d):
    H = [[1]]
    while len(H) < d:
        H = [row + row for row in H] + [row + [-v for v in row] for row in H]
    return H


def fp16_grid(v: Fraction):
    """(below, above): the adjacent fp16 values around |v| > 0 (normal range)."""
    a = abs(v)
    e = math.floor(math.log2(a))
    if Fraction(2) ** e > a:
        e -= 1
    if Fraction(2) ** (e + 1) <= a:
        e += 1
    ulp = Fraction(2) ** (max(e, -14) - 10)
    lo = (a // ulp) * ulp
    return lo, lo + ulp


def is_fp16(v: Fraction) -> bool:
    if v == 0:
        return True
    lo, _ = fp16_grid(v)
    return lo == abs(v) and abs(v) <= 65504


def fp16_round(v: Decimal):
    """Round-to-nearest-even of a positive or negative Decimal to fp16; returns
    (value, bits)."""
    neg = v < 0
    a = Fraction(abs(v))
    lo, hi = fp16_grid(a)
    if a - lo < hi - a:
        r = lo
    elif a - lo > hi - a:
        r = hi
    else:  # tie: the even mantissa
        ulp = hi - lo
        r = lo if (lo / ulp) % 2 == 0 else hi
    e = math.floor(math.log2(r))
    if Fraction(2) ** e > r:
        e -= 1
    mant = int(r / Fraction(2) ** e * 1024) - 1024
    bits = ((e + 15) << 10) | mant
    if neg:
        bits |= 0x8000
    return (-r if neg else r), bits


def midpoint_distance(v: Decimal) -> Decimal:
    """Distance of |v| to the nearest midpoint between two adjacent fp16 values."""
    a = Fraction(abs(v))
    lo, hi = fp16_grid(a)
    ulp = hi - lo
    cands = [lo - ulp / 2, lo + ulp / 2, hi + ulp / 2]
    return min(abs(Decimal(c.numerator) / Decimal(c.denominator) - abs(v)) for c in cands)


def log2d(x: Decimal) -> Decimal:
    return x.ln() / Decimal(2).ln()


def build_x(pairs):
    z = [c for p in pairs for c in p]
    H = sylvester(D16)
    x = [Fraction(sum(H[k][j] * z[j] for j in range(D16)), 4) for k in range(D16)]
    assert all(is_fp16(v) for v in x), x
    return [float(v) for v in x]


def angle_codes(pairs, L):
    out = []
    for a, b in pairs:
        if a == 0 and b == 0:
            out.append(0)
            continue
        t = (math.atan2(b, a) + math.pi) * L / (2 * math.pi)
        f = t - math.floor(t)
        assert 1e-3 < f < 1 - 1e-3, "angle too close to a bin edge for this example"
        out.append(int(math.floor(t)) % L)
    return out


def edge_state(v: Decimal):
    """('edge'|'clear', code): exactly on a .5 edge, or further than 1e-5 of
    max(|v|, 1) from it (so no fp64 evaluation can land on the other side of
    the 1e-6 band)."""
    fl = v - v.to_integral_value(rounding="ROUND_FLOOR")
    dist = abs(fl - Decimal("0.5"))
    scale = max(abs(v), Decimal(1))
    if dist < Decimal("1e-40"):
        return "edge", None
    assert dist > Decimal("1e-5") * scale, (v, dist)
    return "clear", int((v + Decimal("0.5")).to_integral_value(rounding="ROUND_FLOOR"))


def lin8(pairs, L=3):
    r = [Decimal(a * a + b * b).sqrt() for a, b in pairs]
    rmax = max(r)
    M, M_bits = fp16_round(rmax)
    Md = Decimal(M.numerator) / Decimal(M.denominator)
    pflag = midpoint_distance(rmax) <= TOL * rmax
    if not pflag:
        assert midpoint_distance(rmax) > Decimal("1e-5") * rmax, "parameter too close to call"
    flags, codes = [], []
    for ri in r:
        v = Decimal(255) * ri / Md
        st, c = edge_state(v)
        if c is not None:
            c = min(c, 255)
        flags.append((2 if st == "edge" else 0) | (4 if pflag else 0))
        codes.append(c)
    return dict(mode=0, L=L, x=build_x(pairs), z_pairs=[list(p) for p in pairs],
                angles=angle_codes(pairs, L), flags=flags, codes=codes, params=[M_bits])


def log4(pairs, L=3):
    r = [Decimal(a * a + b * b).sqrt() for a, b in pairs]
    assert all(ri > 0 for ri in r), "no zero pairs here (their logarithm is the floor)"
    l = [log2d(ri) for ri in r]
    lmin, lmax = min(l), max(l)
    LO, LO_bits = fp16_round(lmin) if lmin != 0 else (Fraction(0), 0)
    HI, HI_bits = fp16_round(lmax) if lmax != 0 else (Fraction(0), 0)
    LOd = Decimal(LO.numerator) / Decimal(LO.denominator)
    HId = Decimal(HI.numerator) / Decimal(HI.denominator)

    def near(v):
        if v == 0:
            return False
        dist = midpoint_distance(v)
        if dist <= TOL * abs(v):
            return True
        assert dist > Decimal("1e-5") * abs(v), "parameter too close to call"
        return False
    pflag = near(lmin) or near(lmax)
    flags, codes = [], []
    for li in l:
        v = Decimal(15) * (li - LOd) / (HId - LOd)
        st, c = edge_state(v)
        if c is not None:
            c = max(0, min(15, c))
        flags.append((2 if st == "edge" else 0) | (4 if pflag else 0))
        codes.append(c)
    return dict(mode=1, L=L, x=build_x(pairs), z_pairs=[list(p) for p in pairs],
                angles=angle_codes(pairs, L), flags=flags, codes=codes,
                params=[LO_bits, HI_bits])


def search_log4_near_midpoint(which):
    """A pair (a, b) whose log2 norm lies within 5e-7 (relative) of an fp16
    midpoint, beside power-of-two norms (exact logarithms) that keep it the
    largest (which='hi') or the smallest (which='lo') log-norm."""
    best = None
    for a in range(1, 120):
        for b in range(0, a + 1):
            r = Decimal(a * a + b * b).sqrt()
            l = log2d(r)
            if l <= 0:
                continue
            if (which == "hi" and not (64 < r < 128)) or (which == "lo" and not (32 < r < 64)):
                continue
            rel = midpoint_distance(l) / abs(l)
            if rel < Decimal("5e-7") and (best is None or rel < best[0]):
                best = (rel, a, b)
    assert best, which
    return best


def main():
    ex = []
    # 1. LIN8, pair 0 exactly on a rounding edge: M = 128 (pair 1), r0 = 64,
    #    255 * 64 / 128 = 127.5.  Pair 2 = (64, 1): r = sqrt(4097) = 64.0078,
    #    v = 127.5156, 0.0156 from the edge (outside 1e-6 * 127.5, inside
    #    1e-3 * 127.5).  The others: v = 63.75, 191.25, 31.875, 159.375, 95.625.
    ex.append(dict(name="lin8_norm_edge_and_near_miss",
                   **lin8([(64, 0), (128, 0), (64, 1), (32, 0), (96, 0), (16, 0), (80, 0),
                           (48, 0)])))
    # 2. LIN8, max r = 2055 (3-4-5 triangle times 411), the midpoint of fp16
    #    2054 and 2056: round to even gives M = 2056 (0x6804); every pair
    #    carries the parameter flag (detected against the lower neighbour).
    ex.append(dict(name="lin8_param_midpoint_rounds_up",
                   **lin8([(1233, 1644), (1, 0), (0, 0), (0, 0), (0, 0), (0, 0), (0, 0), (0, 0)])))
    # 3. LIN8, max r = 2053 = hypot(1475, 1428), the midpoint of fp16 2052 and
    #    2054: M = 2052 (0x6802, even); flag found against the upper neighbour.
    ex.append(dict(name="lin8_param_midpoint_rounds_down",
                   **lin8([(1475, 1428), (1, 0), (0, 0), (0, 0), (0, 0), (0, 0), (0, 0), (0, 0)])))
    # 4. LOG4, LO = log2 64 = 6, HI = log2 128 = 7 (exact), pair 3 = (64, 64):
    #    l = 6.5, v = 15 * 0.5 = 7.5 exactly (edge).  Pair 2 = (63, 65):
    #    r^2 = 8194, l = 6.5 + 1.76e-4, v = 7.5026 (outside 1e-6 * 7.5, inside
    #    1e-3 * 7.5).
    ex.append(dict(name="log4_norm_edge_and_near_miss",
                   **log4([(64, 0), (128, 0), (63, 65), (64, 64), (64, 0), (64, 0), (64, 0),
                           (64, 0)])))
    # 5./6. LOG4 with HI (resp. LO) within 5e-7 of an fp16 midpoint (found by a
    #    search over integer pairs, checked with 60-digit logarithms).
    _, a, b = search_log4_near_midpoint("hi")
    ex.append(dict(name="log4_param_hi_near_midpoint",
                   **log4([(a, b), (64, 0), (64, 0), (32, 0), (64, 0), (16, 0), (64, 0),
                           (32, 0)])))
    _, a, b = search_log4_near_midpoint("lo")
    ex.append(dict(name="log4_param_lo_near_midpoint",
                   **log4([(a, b), (64, 0), (128, 0), (64, 0), (128, 0), (64, 0), (128, 0),
                           (64, 0)])))
    # 7. A generic vector: nothing near an edge, M = 128 exactly (its nearest
    #    fp16 midpoints, 127.96875 and 128.0625, are 2.4e-4 of M away).
    ex.append(dict(name="lin8_generic_no_flags",
                   **lin8([(100, 0), (128, 0), (70, 3), (33, 0), (90, 0), (17, 0), (81, 0),
                           (41, 0)])))
    doc = {
        "source": __doc__.strip().split("\n\n")[0] + " Written by tests/golden/make_flag_examples.py.",
        "d": D16, "signs": [1] * D16,
        "flag_bits": {"angle": 1, "norm": 2, "param": 4},
        "codes_note": "codes[i] is null where the pair is flagged for its norm (either side of "
                      "the edge is correct); params are the fp16 bit patterns (LIN8: M; LOG4: "
                      "LO, HI)",
        "examples": ex,
    }
    with open(os.path.join(HERE, "flag_examples.json"), "w") as f:
        json.dump(doc, f, indent=1)
        f.write("\n")


if __name__ == "__main__":
    main()
