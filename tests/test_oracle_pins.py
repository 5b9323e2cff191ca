"""Pins of the fp64 oracle against facts fixed outside the oracle itself.

Each test checks the oracle against something other than its own formula:
a hand-worked example, an independent construction (Kronecker product,
numpy's fp16 rounding), a closed-form bound, an invariant, a special case or
brute force on tiny inputs.  Together they are chosen so that a plausible
slip anywhere in the oracle (a dropped sign, a transposed pair, an offset
bin, a wrong rounding, a missing scale) fails at least one of them; the
mutation tests run exactly these pins against deliberately broken copies.

Method: "TurboAngle: Near-Lossless KV Cache Compression via Uniform Angle
Quantization", Abstract (random diagonal + FWHT, consecutive pairs, uniform
angles, 8-bit K / 4-bit log-space V norms, per-layer L_K / L_V).
"""
import json
import math
import os

import numpy as np
import pytest

import oracle as O

HERE = os.path.dirname(os.path.abspath(__file__))
GOLD = json.load(open(os.path.join(HERE, "golden", "hand_examples.json")))


def _rng(seed=0):
    return np.random.default_rng(seed)


def _rand_signs(rng, d):
    return np.where(rng.integers(0, 2, d) == 0, 1, -1).astype(np.int8)


def _sylvester(d):
    H = np.array([[1]], dtype=np.int64)
    while H.shape[0] < d:
        H = np.kron(np.array([[1, 1], [1, -1]], dtype=np.int64), H)
    return H


# --------------------------------------------------------------- rotation --

@pytest.mark.parametrize("d", [2, 4, 8, 16, 32, 64, 128, 256])
def test_hadamard_is_sylvester_and_orthogonal(d):
    """H from the oracle equals the Kronecker power of [[1,1],[1,-1]], and
    H H = d I exactly (integer arithmetic)."""
    ones = np.ones(d, np.int8)
    H = O.rotate(np.eye(d), ones, scaled=False).T  # column k = H e_k
    assert np.array_equal(H, _sylvester(d).astype(np.float64))
    Hi = H.astype(np.int64)
    assert np.array_equal(Hi @ Hi, d * np.eye(d, dtype=np.int64))


@pytest.mark.parametrize("d", [4, 8, 64, 128, 256])
def test_rotation_preserves_norm_and_inverts(d):
    rng = _rng(d)
    s = _rand_signs(rng, d)
    x = rng.standard_normal((16, d))
    z = O.rotate(x, s, scaled=True)
    assert np.allclose(np.linalg.norm(z, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    assert np.allclose(O.unrotate(z, s), x, atol=1e-13)
    # D is applied once: H D x equals H (s * x) with D = I
    assert np.allclose(z, O.rotate(x * s, np.ones(d, np.int8), scaled=True), atol=1e-13)


@pytest.mark.parametrize("d", [4, 8])
def test_dot_product_identity_brute_force(d):
    """q . k = (H D q) . (H D k) / d for every one of the 2^d sign patterns."""
    rng = _rng(100 + d)
    q = rng.standard_normal(d)
    k = rng.standard_normal(d)
    for pattern in range(2 ** d):
        s = np.array([-1 if (pattern >> j) & 1 else 1 for j in range(d)], np.int8)
        zq = O.rotate(q, s, scaled=False)[0]
        zk = O.rotate(k, s, scaled=False)[0]
        assert math.isclose(float(zq @ zk) / d, float(q @ k), rel_tol=1e-12, abs_tol=1e-12)
        # and the 1/sqrt(d)-scaled rotation is an isometry of the dot product
        sq = O.rotate(q, s)[0]
        sk = O.rotate(k, s)[0]
        assert math.isclose(float(sq @ sk), float(q @ k), rel_tol=1e-12, abs_tol=1e-12)


# ---------------------------------------------------------- hand examples --

@pytest.mark.parametrize("ex", GOLD["examples"], ids=lambda e: e["name"])
def test_hand_examples(ex):
    d = ex["d"]
    s = np.array(ex["signs"], np.int8)
    x = np.array(ex["x"], np.float16)
    z = O.rotate(x.astype(np.float64), s)[0]
    assert np.allclose(z, ex["z"], atol=1e-15)
    for L, want in ex.get("codes", {}).items():
        c = O.encode(x[None], s, int(L), O.MODE_LIN8)
        a, _, _ = O.unpack(c)
        assert a[0].tolist() == want, (L, a[0].tolist(), want)
        assert not (c.flags[0] & O.FLAG_ANGLE).any()
    for L in ex.get("edge_L", []):
        c = O.encode(x[None], s, int(L), O.MODE_LIN8)
        assert (c.flags[0] & O.FLAG_ANGLE).all(), "an exact bin edge must be flagged"
    for L, row in ex.get("angle_row", {}).items():
        c = O.encode(x[None], s, int(L), O.MODE_LIN8)
        assert c.angles[0].tolist() == row
    if "lin8" in ex:
        c = O.encode(x[None], s, 8, O.MODE_LIN8)
        M_bits = int(c.params[0, 0]) | (int(c.params[0, 1]) << 8)
        assert M_bits == ex["lin8"]["M_bits"]
        assert c.norms[0].tolist() == ex["lin8"]["c"]
        _, _, rh = O.unpack(c)
        M = O.half_bits_to_double(M_bits)
        assert np.allclose(rh[0], np.array(ex["lin8"]["c"]) * M / 255.0, rtol=1e-15)
    if "log4" in ex:
        c = O.encode(x[None], s, 8, O.MODE_LOG4)
        p = c.params[0]
        assert int(p[0]) | int(p[1]) << 8 == ex["log4"]["LO_bits"]
        assert int(p[2]) | int(p[3]) << 8 == ex["log4"]["HI_bits"]
        _, cc, _ = O.unpack(c)
        assert cc[0].tolist() == ex["log4"]["c"]
        if "norm_row" in ex["log4"]:
            assert c.norms[0].tolist() == ex["log4"]["norm_row"]
            assert c.params[0].tolist() == ex["log4"]["param_row"]


FLAGS = json.load(open(os.path.join(HERE, "golden", "flag_examples.json")))


@pytest.mark.parametrize("ex", FLAGS["examples"], ids=lambda e: e["name"])
def test_norm_and_parameter_flags(ex):
    """The oracle's norm-edge and fp16-midpoint flags on vectors built to sit
    exactly on a rounding edge, just off it (a few 1e-4 .. 1e-2 away, outside
    the 1e-6 band), or on / within 5e-7 of an fp16 rounding midpoint of the
    parameter (tests/golden/make_flag_examples.py derives every expectation
    in exact or 60-digit arithmetic).  Exact edges must be flagged, near
    misses must not, a midpoint parameter flags every pair of its vector, and
    codes away from every edge are the definition's."""
    d = FLAGS["d"]
    s = np.array(FLAGS["signs"], np.int8)
    x = np.array(ex["x"], np.float16)
    assert np.array_equal(x.astype(np.float64), np.array(ex["x"]))  # exact fp16 inputs
    z = O.rotate(x.astype(np.float64), s)[0]
    assert np.array_equal(z, np.array(ex["z_pairs"], np.float64).ravel())
    c = O.encode(x[None], s, ex["L"], ex["mode"])
    assert c.flags[0].tolist() == ex["flags"]
    a, cc, _ = O.unpack(c)
    assert a[0].tolist() == ex["angles"]
    for got, want in zip(cc[0].tolist(), ex["codes"]):
        if want is not None:
            assert got == want
    p = c.params[0]
    bits = [int(p[2 * i]) | int(p[2 * i + 1]) << 8 for i in range(len(ex["params"]))]
    assert bits == ex["params"]


def test_packing_layout():
    g = GOLD["packing"]
    d, L = g["d"], g["L"]
    ab = O.row_bytes(d, L, O.MODE_LOG4, 0)
    assert ab == 4
    codes = O.Codes(d, L, O.MODE_LOG4, np.array([g["angle_row"]], np.uint8),
                    np.array([g["log4_norm_row"]], np.uint8),
                    np.array([[0, 0, 0, 0x3C]], np.uint8))  # LO = 0, HI = 1.0
    a, c, rh = O.unpack(codes)
    assert a[0].tolist() == g["codes"]
    assert c[0].tolist() == g["log4_codes"]
    assert np.allclose(rh[0], 2.0 ** (np.array(g["log4_codes"]) / 15.0), rtol=1e-15)


def test_row_bytes_and_bit_accounting():
    """Bytes per token and the angle-bits accounting of the TurboAngle
    abstract: angle bits per element = (log2 L_K + log2 L_V) / 4."""
    assert [O.angle_bits(L) for L in (2, 3, 4, 5, 128, 129, 256, 65536)] == \
        [1, 2, 2, 3, 7, 8, 8, 16]
    assert O.angle_bits(1) < 0 and O.angle_bits(65537) < 0
    k = sum(O.row_bytes(128, 128, O.MODE_LIN8, w) for w in range(3))
    v = sum(O.row_bytes(128, 64, O.MODE_LOG4, w) for w in range(3))
    assert (k, v) == (122, 84)
    assert O.row_bytes(64, 32, O.MODE_LOG4, 0) == 20
    assert O.row_bytes(16, 3, O.MODE_LIN8, 0) == 4  # 16 bits padded to a word
    # per-layer early-boost: 4 of 32 layers at 256/256, the rest at 128/64
    per_layer = [(8 + 8) / 4] * 4 + [(7 + 6) / 4] * 28
    angle_bits = sum(per_layer) / 32
    assert 3.28 <= angle_bits <= 3.67  # the abstract's early-boost range
    total = angle_bits + (8 + 4) / 4 + (16 + 32) / 256  # + norms + fp16 params
    assert abs(total - 6.56) < 0.1  # consistent with the abstract's 6.56


# ------------------------------------------------------------ fp16 edges --

def test_fp16_rounding_matches_numpy():
    rng = _rng(7)
    vals = list(rng.standard_normal(20000) * 10.0 ** rng.integers(-8, 5, 20000))
    # exact midpoints and double-rounding traps (a float32 detour would fail)
    for h in rng.integers(1, 0x7BFE, 3000):
        a = float(np.array(h, np.uint16).view(np.float16))
        b = float(np.array(h + 1, np.uint16).view(np.float16))
        m = 0.5 * (a + b)
        vals += [m, np.nextafter(m, np.inf), np.nextafter(m, -np.inf), -m]
    for v in vals:
        assert O.double_to_half_bits(v) == int(np.array(v).astype(np.float16).view(np.uint16)), v
        h = int(np.array(v).astype(np.float16).view(np.uint16))
        assert O.half_bits_to_double(h) == float(np.array(h, np.uint16).view(np.float16))


# ------------------------------------------------------------ codec bounds --

def _vectors(n, d, seed, outliers=True):
    rng = _rng(seed)
    x = rng.standard_normal((n, d))
    if outliers:
        x[:, 3 % d] *= 20.0
        x[:, 77 % d] *= 20.0
    return x.astype(np.float16), _rand_signs(rng, d)


def _exact_pairs(x16, s):
    z = O.rotate(x16.astype(np.float64), s)
    u, v = z[:, 0::2], z[:, 1::2]
    return np.hypot(u, v), np.arctan2(v, u)


@pytest.mark.parametrize("L", [3, 8, 64, 128, 256, 1000])
def test_angle_error_at_most_pi_over_L(L):
    x, s = _vectors(400, 64, L)
    c = O.encode(x, s, L, O.MODE_LIN8)
    a, _, _ = O.unpack(c)
    r, th = _exact_pairs(x, s)
    thh = -np.pi + (a + 0.5) * 2 * np.pi / L
    err = np.abs(np.angle(np.exp(1j * (th - thh))))
    assert err.max() <= np.pi / L + 1e-12
    assert a.min() >= 0 and a.max() < L


def test_code_is_the_bin_containing_theta():
    """Brute force: the code is the unique bin [edge_a, edge_a+1) holding theta,
    found by scanning all L edges (no floor formula)."""
    L = 12
    x, s = _vectors(200, 16, 5)
    c = O.encode(x, s, L, O.MODE_LIN8)
    a, _, _ = O.unpack(c)
    _, th = _exact_pairs(x, s)
    edges = -np.pi + np.arange(L + 1) * 2 * np.pi / L
    for i in range(th.shape[0]):
        for j in range(th.shape[1]):
            if c.flags[i, j] & O.FLAG_ANGLE:
                continue
            k = [b for b in range(L) if edges[b] <= th[i, j] < edges[b + 1]]
            want = k[0] if k else 0  # theta == pi wraps to bin 0
            assert a[i, j] == want


def test_norm_code_bounds():
    """LIN8: |r - r^| <= M/510 + |max r - M|, codes are round-half-up of
    255 r / M.  LOG4: |log2 r - log2 r^| <= (HI - LO)/30 (+ the fp16 rounding
    of HI) for every r >= 2^LO, codes in 0..15."""
    x, s = _vectors(500, 128, 11)
    r, _ = _exact_pairs(x, s)
    c8 = O.encode(x, s, 128, O.MODE_LIN8)
    _, c, rh = O.unpack(c8)
    M = np.array([O.half_bits_to_double(int(p[0]) | int(p[1]) << 8) for p in c8.params])
    bound = M[:, None] / 510 + np.abs(r.max(1) - M)[:, None]
    assert np.all(np.abs(r - rh) <= bound * (1 + 1e-12) + 1e-15)
    want = np.minimum(255, np.floor(255 * r / M[:, None] + 0.5))
    flagged = (c8.flags & (O.FLAG_NORM | O.FLAG_PARAM)) != 0
    assert np.all((c == want) | flagged)
    # M is the fp16 rounding (numpy's) of the largest exact pair norm
    pflag = (c8.flags[:, 0] & O.FLAG_PARAM) != 0
    assert np.all((M == r.max(1).astype(np.float16).astype(np.float64)) | pflag)
    c4 = O.encode(x, s, 64, O.MODE_LOG4)
    _, c, rh = O.unpack(c4)
    LO = np.array([O.half_bits_to_double(int(p[0]) | int(p[1]) << 8) for p in c4.params])
    HI = np.array([O.half_bits_to_double(int(p[2]) | int(p[3]) << 8) for p in c4.params])
    lr = np.log2(np.maximum(r, 2.0 ** -24))
    pflag = (c4.flags[:, 0] & O.FLAG_PARAM) != 0
    assert np.all((LO == lr.min(1).astype(np.float16).astype(np.float64)) | pflag)
    assert np.all((HI == lr.max(1).astype(np.float16).astype(np.float64)) | pflag)
    err = np.abs(lr - np.log2(rh))
    bound = (HI - LO)[:, None] / 30 + np.maximum(lr.max(1) - HI, 0)[:, None] + 1e-12
    ok = lr >= LO[:, None]
    assert np.all(err[ok] <= np.broadcast_to(bound, err.shape)[ok])
    assert c.min() >= 0 and c.max() <= 15


def test_codec_error_from_codes_alone():
    """|x - x^|^2 = sum_i r_i^2 + r^_i^2 - 2 r_i r^_i cos(theta_i - theta^_i):
    the dequantized vector (through the inverse rotation) agrees with the
    per-pair reconstruction read from the codes."""
    for mode, L in ((O.MODE_LIN8, 128), (O.MODE_LOG4, 64), (O.MODE_LIN8, 5)):
        x, s = _vectors(300, 128, 13 + L)
        c = O.encode(x, s, L, mode)
        a, _, rh = O.unpack(c)
        r, th = _exact_pairs(x, s)
        thh = -np.pi + (a + 0.5) * 2 * np.pi / L
        want = (r ** 2 + rh ** 2 - 2 * r * rh * np.cos(th - thh)).sum(1)
        xh = O.dequant(c, s)
        got = ((x.astype(np.float64) - xh) ** 2).sum(1)
        assert np.allclose(got, want, rtol=1e-9, atol=1e-9)


def test_exact_round_trip_as_L_grows():
    """Unquantized norms: |x - x^| <= (pi / L) |x| and the error halves when L
    doubles (the round trip becomes exact as L grows)."""
    x, s = _vectors(200, 128, 17)
    xn = np.linalg.norm(x.astype(np.float64), axis=1)
    prev = None
    for b in range(4, 17):
        L = 2 ** b
        c = O.encode(x, s, L, O.MODE_EXACT)
        xh = O.dequant(c, s)
        e = np.linalg.norm(x.astype(np.float64) - xh, axis=1)
        assert np.all(e <= np.pi / L * xn * (1 + 1e-9))
        tot = float(e.sum() / xn.sum())
        if prev is not None:
            assert 1.6 < prev / tot < 2.4, (L, prev / tot)
        prev = tot
    assert prev < 1e-4


def test_zero_and_tiny_vectors():
    d = 16
    s = np.ones(d, np.int8)
    z = np.zeros((1, d), np.float16)
    c = O.encode(z, s, 128, O.MODE_LIN8)
    a, cc, rh = O.unpack(c)
    assert a.sum() == 0 and cc.sum() == 0 and c.params.sum() == 0
    c = O.encode(z, s, 128, O.MODE_LOG4)
    a, cc, rh = O.unpack(c)
    LO = O.half_bits_to_double(int(c.params[0, 0]) | int(c.params[0, 1]) << 8)
    assert LO == -24.0 and cc.sum() == 0
    tiny = np.zeros((1, d), np.float16)
    tiny[0, 5] = np.float16(2.0 ** -24)  # smallest subnormal
    c = O.encode(tiny, s, 64, O.MODE_LIN8)
    # every rotated pair is +-(1, -1) 2^-24 / 4 (a single odd channel maps to the
    # diagonals -pi/4, 3pi/4, which are bin edges at L = 64: t = 24 or 56, so
    # every angle is flagged); r = 2^-24 sqrt(2) / 4 = 2.1e-8 is below half the
    # smallest fp16 subnormal (2.98e-8): M rounds to +0, every norm code is 0,
    # and 2.1e-8 lies 8.7e-9 from that midpoint, far outside 1e-6 relative
    assert (c.flags == O.FLAG_ANGLE).all()
    assert c.params.sum() == 0 and c.norms.sum() == 0
    xh = O.dequant(c, s)
    assert np.all(xh == 0)


def test_uniform_angles_after_rotation():
    """Rotated pairs are roughly uniform on the circle (TurboAngle abstract) for
    keys whose energy is spread over channels: chi-square of the L = 128 codes
    over 2^20 pairs, isotropic and per-channel lognormal(0, 0.5) scaled keys.
    (A single dominant input channel k is different: every rotated pair is then
    +-(1, 1) (k even) or +-(1, -1) (k odd) times x_k / sqrt(d), so outlier
    channels pull the angles towards the diagonals; see the next test.)"""
    from scipy.stats import chisquare
    rng = _rng(3)
    n = 2 ** 20 // 64
    s = _rand_signs(rng, 128)
    for scale in (np.ones(128), rng.lognormal(0, 0.5, 128)):
        x = rng.standard_normal((n, 128)) * scale
        c = O.encode(x.astype(np.float16), s, 128, O.MODE_LIN8)
        a, _, _ = O.unpack(c)
        counts = np.bincount(a.ravel(), minlength=128)
        assert chisquare(counts).pvalue > 1e-3


def test_single_channel_maps_to_diagonals():
    """Closed form of H D e_k: pair i of the rotated unit vector is
    s_k (H[2i][k], H[2i+1][k]) / sqrt(d) = +-(1, (-1)^k) / sqrt(d), so its angle
    is a diagonal: pi/4 or -3pi/4 for even k, -pi/4 or 3pi/4 for odd k.  With
    L = 12 no diagonal is a bin edge, so the codes are exact."""
    d, L = 32, 12
    rng = _rng(4)
    s = _rand_signs(rng, d)
    even = {int(np.floor((t + np.pi) * L / (2 * np.pi))) for t in (np.pi / 4, -3 * np.pi / 4)}
    odd = {int(np.floor((t + np.pi) * L / (2 * np.pi))) for t in (-np.pi / 4, 3 * np.pi / 4)}
    for k in range(d):
        x = np.zeros((1, d), np.float16)
        x[0, k] = 3.0
        c = O.encode(x, s, L, O.MODE_LIN8)
        a, cc, _ = O.unpack(c)
        assert set(a[0].tolist()) <= (odd if k % 2 else even), k
        assert np.all(cc[0] == 255)  # all pairs have the same norm


# -------------------------------------------------------------- attention --

def _cache(T, d, LK, LV, seed):
    xk, sk = _vectors(T, d, seed)
    rng = _rng(seed + 1)
    xv = rng.standard_normal((T, d)).astype(np.float16)
    sv = _rand_signs(rng, d)
    kc = O.encode(xk, sk, LK, O.MODE_LIN8)
    vc = O.encode(xv, sv, LV, O.MODE_LOG4)
    return kc, vc, sk, sv


@pytest.mark.parametrize("d,T", [(8, 5), (16, 33), (128, 200)])
def test_materialised_attention_equals_rotated_streaming(d, T):
    """The textbook attention on dequantized vectors equals the streaming
    rotated-domain computation from the codes (q rotated once, cos/sin of the
    bin centres, online softmax, one inverse rotation per head)."""
    kc, vc, sk, sv = _cache(T, d, 128, 64, d + T)
    q = _rng(5).standard_normal((4, d))
    tau = 1 / math.sqrt(d)
    o1 = O.attend(q, O.dequant(kc, sk), O.dequant(vc, sv), tau)
    o2 = O.attend_rotated(q, sk, sv, kc, vc, tau)
    assert np.allclose(o1, o2, rtol=1e-10, atol=1e-12)


def test_attention_special_cases():
    d, T = 64, 50
    kc, vc, sk, sv = _cache(T, d, 128, 64, 21)
    kh, vh = O.dequant(kc, sk), O.dequant(vc, sv)
    q = _rng(6).standard_normal((3, d))
    # one token: the output is that token's value
    assert np.allclose(O.attend(q, kh[:1], vh[:1], 0.1), np.repeat(vh[:1], 3, 0), atol=1e-14)
    # equal scores (q = 0): the output is the mean value
    assert np.allclose(O.attend(np.zeros((1, d)), kh, vh, 1.0)[0], vh.mean(0), atol=1e-13)
    # no tokens: zeros
    assert np.all(O.attend(q, kh[:0], vh[:0], 0.1) == 0)
    # token order does not matter
    perm = _rng(8).permutation(T)
    assert np.allclose(O.attend(q, kh, vh, 0.1), O.attend(q, kh[perm], vh[perm], 0.1),
                       atol=1e-13)
    # a dominant score picks its token: q along k^_7 with a large scale
    qd = kh[7:8] / np.linalg.norm(kh[7])
    sc = (kh @ qd[0])
    gap = sc[7] - np.max(np.delete(sc, 7))
    if gap > 0:
        o = O.attend(qd, kh, vh, 60.0 / gap)
        assert np.allclose(o[0], vh[7], atol=1e-6 * np.abs(vh).max())
    # scores shift-invariance: adding a multiple of nothing; scaling tau by 0 gives mean
    assert np.allclose(O.attend(q, kh, vh, 0.0)[1], vh.mean(0), atol=1e-13)


def test_zero_parameter_is_stored_as_plus_zero():
    """A vector whose pair norms are all exactly 1 has log2 r = 0, so LO = HI = 0;
    fp64 rounding of the logarithm can come out as -1.6e-16, and the stored
    parameter must still be +0 (bits 0x0000), not -0."""
    d = 128
    x = np.zeros((1, d), np.float16)
    x[0, 78] = 8.0  # r = 8 sqrt(2) / sqrt(128) = 1 for every pair
    for seed in range(4):
        s = _rand_signs(_rng(seed), d)
        c = O.encode(x, s, 64, O.MODE_LOG4)
        assert c.params[0].tolist() == [0, 0, 0, 0]
