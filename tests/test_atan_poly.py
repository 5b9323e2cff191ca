"""The odd polynomial the encode kernel uses for atan (kvq_atan_poly.h),
evaluated in float32 the way the kernel evaluates it (octant reduction,
Horner in t^2, fp32 constants), stays within the angle slack the kernel's
bin-edge margin assumes (1.5e-6 rad) of the true atan2."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "decode_attention_rand_b200", "csrc", "kvq_atan_poly.h")
SLACK = 1.5e-6


def coefficients():
    text = open(HDR).read()
    found = dict(re.findall(r"#define KVQ_ATAN_C(\d+) ([-0-9.e]+)f", text))
    return np.array([float(found[str(k)]) for k in range(len(found))], np.float32)


def atan2_poly32(y, x, c):
    f = np.float32
    y, x = y.astype(f), x.astype(f)
    ax, ay = np.abs(x), np.abs(y)
    mx, mn = np.maximum(ax, ay), np.minimum(ax, ay)
    t = (mn * (f(1) / mx)).astype(f)
    t2 = (t * t).astype(f)
    p = np.full_like(t, c[-1])
    for k in range(len(c) - 2, -1, -1):
        p = (p * t2 + c[k]).astype(f)
    th = (p * t).astype(f)
    th = np.where(ay > ax, (f(1.5707963267948966) - th).astype(f), th)
    th = np.where(x < 0, (f(np.pi) - th).astype(f), th)
    return np.where(y < 0, -th, th)


def test_polynomial_error_within_slack():
    c = coefficients()
    assert len(c) == 8
    rng = np.random.default_rng(0)
    ang = np.concatenate([rng.uniform(-np.pi, np.pi, 2_000_000),
                          np.arange(-8, 9) * np.pi / 8])  # octant boundaries
    r = rng.lognormal(0, 3, ang.size)
    x, y = (r * np.cos(ang)).astype(np.float32), (r * np.sin(ang)).astype(np.float32)
    ok = (x != 0) | (y != 0)
    got = atan2_poly32(y[ok], x[ok], c).astype(np.float64)
    want = np.arctan2(y[ok].astype(np.float64), x[ok].astype(np.float64))
    err = np.abs(np.angle(np.exp(1j * (got - want))))
    assert err.max() < SLACK / 3, err.max()
