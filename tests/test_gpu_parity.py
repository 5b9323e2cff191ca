"""GPU parity: the CUDA library (through its C ABI) against the fp64 oracle.

Rules (per code / per output vector):
  - angle codes, norm codes and fp16 parameters bit-exact, except values the
    oracle flags within 1e-6 of a decision edge, and at most 1e-5 of all codes
    may differ;
  - dequantized vectors and attention outputs within relative L2 2e-3 of the
    oracle, both sides computed on the same (oracle-encoded) codes.
Inputs are seeded synthetic tensors (decode_attention_rand_b200.synth); every
expected value comes from oracle/.
"""
import json
import math
import os

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle as O
from decode_attention_rand_b200 import build as kbuild
from decode_attention_rand_b200 import kvq, synth

from kvq_testutil import REL_L2_TOL, compare_codes, plane_rows, put_rows, rel_l2

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    kbuild.build()
    kvq.lib()
    return torch.device("cuda:0")


def _signs(seed, d):
    rng = np.random.default_rng(seed)
    return np.where(rng.integers(0, 2, d) == 0, 1, -1).astype(np.int8)


def _dev_signs(s):
    return torch.from_numpy(np.ascontiguousarray(s)).cuda()


def _rand_x(B, H, T, d, seed, outliers=True, scale=1.0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((B, H, T, d)) * scale
    if outliers and d > 8:
        x[..., 3] *= 20.0
        x[..., min(77, d - 1)] *= 20.0
    return x.astype(np.float16)


def gpu_encode(x16: np.ndarray, s: np.ndarray, L: int, mode: int, cap=None, pos0=0):
    B, H, T, d = x16.shape
    cap = cap or ((pos0 + T + 15) // 16 * 16)
    c = kvq.codec(d, L, mode)
    plane = kvq.alloc_plane(c, B, H, cap)
    xd = torch.from_numpy(x16).cuda()
    kvq.encode(c, _dev_signs(s), xd, plane, pos0)
    torch.cuda.synchronize()
    return c, plane


def check_encode(x16, s, L, mode, pos0=0, cap=None):
    B, H, T, d = x16.shape
    c, plane = gpu_encode(x16, s, L, mode, cap, pos0)
    oc = O.encode(x16, s, L, mode)
    stats = compare_codes(plane_rows(plane, t_range=(pos0, pos0 + T)), oc)
    # rows outside [pos0, pos0 + T) are untouched
    for w in range(3):
        r = plane.rows(w)
        assert int(r[:, :, :pos0].count_nonzero()) == 0
        assert int(r[:, :, pos0 + T:].count_nonzero()) == 0
    return stats, c, plane, oc


# ------------------------------------------------------------------ encode --

def test_encode_hand_examples(dev):
    gold = json.load(open(os.path.join(HERE, "golden", "hand_examples.json")))
    for ex in gold["examples"]:
        s = np.array(ex["signs"], np.int8)
        x = np.array(ex["x"], np.float16).reshape(1, 1, 1, -1)
        for L, want in ex.get("codes", {}).items():
            c, plane = gpu_encode(x, s, int(L), O.MODE_LIN8)
            from kvq_testutil import unpack_rows
            a, _, _ = unpack_rows(*plane_rows(plane, t_range=(0, 1)), 4, int(L), O.MODE_LIN8)
            assert a[0].tolist() == want, (ex["name"], L)
        if "lin8" in ex:
            c, plane = gpu_encode(x, s, 8, O.MODE_LIN8)
            rows = plane_rows(plane, t_range=(0, 1))
            assert rows[1][0].tolist() == ex["lin8"]["c"]
            assert int(rows[2][0].view("<u2")[0]) == ex["lin8"]["M_bits"]
        if "log4" in ex and "param_row" in ex["log4"]:
            c, plane = gpu_encode(x, s, 8, O.MODE_LOG4)
            rows = plane_rows(plane, t_range=(0, 1))
            assert rows[1][0].tolist() == ex["log4"]["norm_row"]
            assert rows[2][0].tolist() == ex["log4"]["param_row"]


@pytest.mark.parametrize("d", [4, 8, 16, 32, 64, 128, 256])
@pytest.mark.parametrize("L", [2, 3, 5, 8, 16, 24, 40, 64, 128, 200, 256, 1000, 65536])
def test_encode_sweep(dev, d, L):
    s = _signs(d * 7 + L, d)
    x = _rand_x(2, 3, 37, d, seed=d * 1000 + L)
    for mode in (O.MODE_LIN8, O.MODE_LOG4):
        check_encode(x, s, L, mode, pos0=5, cap=48)


def test_encode_append_one_token(dev):
    d, L = 128, 128
    s = _signs(1, d)
    x = _rand_x(2, 4, 40, d, seed=2)
    c = kvq.codec(d, L, O.MODE_LIN8)
    plane = kvq.alloc_plane(c, 2, 4, 48)
    xd = torch.from_numpy(x).cuda()
    sd = _dev_signs(s)
    kvq.encode(c, sd, xd[:, :, :39].contiguous(), plane, 0)
    kvq.encode(c, sd, xd[:, :, 39:].contiguous(), plane, 39)  # T = 1 append
    torch.cuda.synchronize()
    compare_codes(plane_rows(plane, t_range=(0, 40)), O.encode(x, s, L, O.MODE_LIN8))


@pytest.mark.parametrize("T,pos0", [(37, 5), (1, 47)])
def test_encode_kv_equals_two_encodes(dev, T, pos0):
    """kvq_encode_kv writes exactly what kvq_encode writes for K and V
    separately (a prefill slice and a one-token append), and both match the
    oracle."""
    d, B, H, cap = 128, 2, 3, 48
    sk, sv = _signs(11, d), _signs(12, d)
    k = _rand_x(B, H, T, d, seed=13)
    v = _rand_x(B, H, T, d, seed=14, outliers=False)
    kc, vc = kvq.codec(d, 128, O.MODE_LIN8), kvq.codec(d, 64, O.MODE_LOG4)
    skd, svd = _dev_signs(sk), _dev_signs(sv)
    kd, vd = torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda()
    K1, V1 = kvq.alloc_plane(kc, B, H, cap), kvq.alloc_plane(vc, B, H, cap)
    K2, V2 = kvq.alloc_plane(kc, B, H, cap), kvq.alloc_plane(vc, B, H, cap)
    kvq.encode_kv(kc, skd, kd, K1, vc, svd, vd, V1, pos0)
    kvq.encode(kc, skd, kd, K2, pos0)
    kvq.encode(vc, svd, vd, V2, pos0)
    torch.cuda.synchronize()
    for w in range(3):
        assert torch.equal(K1.rows(w), K2.rows(w))
        assert torch.equal(V1.rows(w), V2.rows(w))
    compare_codes(plane_rows(K1, t_range=(pos0, pos0 + T)), O.encode(k, sk, 128, O.MODE_LIN8))
    compare_codes(plane_rows(V1, t_range=(pos0, pos0 + T)), O.encode(v, sv, 64, O.MODE_LOG4))


def test_encode_kv_rejects_mismatched_head_dims(dev):
    kc, vc = kvq.codec(128, 128, O.MODE_LIN8), kvq.codec(64, 64, O.MODE_LOG4)
    K, V = kvq.alloc_plane(kc, 1, 1, 16), kvq.alloc_plane(vc, 1, 1, 16)
    k = torch.zeros((1, 1, 1, 128), dtype=torch.float16, device="cuda")
    v = torch.zeros((1, 1, 1, 64), dtype=torch.float16, device="cuda")
    s = torch.ones(128, dtype=torch.int8, device="cuda")
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_encode_kv(kc, s, k, K.c(), vc, s, v, V.c(), 1, 1, 1, 0)
    assert "head_dim" in str(e.value)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_encode_edge_cases(dev, d):
    s = _signs(3, d)
    xs = []
    xs.append(np.zeros((1, d)))                          # all-zero vector
    one = np.zeros((8, d))
    for i in range(8):                                   # one channel: pairs on diagonals,
        one[i, i * 13 % d] = 2.0 ** (i - 3)              # exact bin edges when 8 | L
    xs.append(one)
    xs.append(np.full((2, d), 2.0 ** -24))               # subnormal fp16
    big = np.zeros((2, d))
    big[:, :] = 60000.0                                  # near fp16 max: M saturates
    xs.append(big)
    xs.append(np.tile([1.0, -1.0], (3, d // 2)))         # structured
    rng = np.random.default_rng(9)
    xs.append(rng.standard_normal((4, d)) * 1e-4)        # tiny norms (log floor)
    sparse = np.zeros((4, d))
    sparse[:, [0, 1]] = [[3.0, 1.0], [1.0, 3.0], [-2.0, 2.0], [0.5, -0.25]]
    xs.append(sparse)
    x = np.concatenate(xs).astype(np.float16)[None, None]
    for L in (4, 8, 16, 24, 40, 128, 200, 256, 3, 65536):
        for mode in (O.MODE_LIN8, O.MODE_LOG4):
            check_encode(x, s, L, mode)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_encode_every_vector_in_doubt(dev, d):
    """Every vector has pairs exactly on bin edges (one nonzero channel: its
    rotated pairs lie on multiples of pi/4, edges when 8 | L), so the
    streaming pass marks all of them and the fixup pass re-encodes them all:
    its per-warp queue fills and wraps many times over."""
    n = 3000
    s = _signs(d + 5, d)
    rng = np.random.default_rng(d)
    x = np.zeros((n, d))
    x[np.arange(n), rng.integers(0, d, n)] = rng.choice([-1, 1], n) * 2.0 ** rng.integers(-6, 6, n)
    x = x.astype(np.float16)[None, None]
    for L, mode in ((128, O.MODE_LIN8), (64, O.MODE_LOG4), (256, O.MODE_LIN8)):
        stats, *_ = check_encode(x, s, L, mode)
        assert stats["vectors"] == n


def test_encode_distributions_llama_layer(dev):
    """Full Llama-7B-shaped layer (8 KV heads x 4096 tokens, d = 128), K with
    lognormal channel scales and outliers, V ~ N(0,1): every code checked."""
    w = synth.WORKLOADS["llama7b_layer_b1_hq32_hkv8_d128_ctx4096"]
    sk, sv = synth.layer_signs(w, 0)
    for kind, L, mode, s in ((synth.KIND_K, 128, O.MODE_LIN8, sk), (synth.KIND_V, 64, O.MODE_LOG4, sv)):
        x = synth.kv(w, 0, kind, device="cuda").cpu().numpy()
        stats, *_ = check_encode(x, s, L, mode)
        assert stats["vectors"] == 8 * 4096
        # near-edge values are re-decided exactly, so even flagged codes agree here
        assert stats["mismatches"] == 0, stats


# ----------------------------------------------------------------- dequant --

@pytest.mark.parametrize("d", [4, 16, 64, 128, 256])
@pytest.mark.parametrize("L", [2, 3, 5, 16, 24, 64, 128, 256, 5000, 65536])
def test_dequant_sweep(dev, d, L):
    s = _signs(d + L, d)
    x = _rand_x(2, 2, 21, d, seed=5 * d + L)
    for mode in (O.MODE_LIN8, O.MODE_LOG4):
        oc = O.encode(x, s, L, mode)
        c = kvq.codec(d, L, mode)
        plane = kvq.alloc_plane(c, 2, 2, 32)
        n = 0
        for b in range(2):
            for h in range(2):
                put_rows(plane, oc.take(slice(n, n + 21)), b, h, 3)
                n += 21
        y = kvq.dequant(c, _dev_signs(s), plane, 21, pos0=3)
        torch.cuda.synchronize()
        got = y.cpu().numpy().astype(np.float64).reshape(-1, d)
        want = O.dequant(oc, s)
        err = rel_l2(got, want)
        assert err.max() <= REL_L2_TOL, (mode, err.max())


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("B,H,T,pos0", [(1, 1, 3, 0), (1, 3, 7, 5), (3, 2, 13, 1), (2, 5, 101, 17)])
def test_dequant_fast_ragged_tiles(dev, d, B, H, T, pos0):
    """The fast dequant (32 elements per lane, d/32 lanes per vector, 32*32/d
    vectors per warp tile, the lane-bit butterflies after a transposition
    through shared memory) on vector counts that leave the last warp tile
    partly filled, fewer vectors than one tile included, with rows read from
    an offset position of each (b, KV head) run."""
    s = _signs(d + B * 7 + T, d)
    x = _rand_x(B, H, T, d, seed=d * 3 + T)
    n = B * H * T
    for L, mode in ((128, O.MODE_LIN8), (64, O.MODE_LOG4), (256, O.MODE_LIN8), (16, O.MODE_LOG4)):
        oc = O.encode(x, s, L, mode)
        c = kvq.codec(d, L, mode)
        plane = kvq.alloc_plane(c, B, H, (pos0 + T + 15) // 16 * 16 + 16)
        k = 0
        for b in range(B):
            for h in range(H):
                put_rows(plane, oc.take(slice(k, k + T)), b, h, pos0)
                k += T
        y = kvq.dequant(c, _dev_signs(s), plane, T, pos0=pos0)
        torch.cuda.synchronize()
        got = y.cpu().numpy().astype(np.float64).reshape(-1, d)
        assert got.shape[0] == n
        err = rel_l2(got, O.dequant(oc, s))
        assert err.max() <= REL_L2_TOL, (L, mode, err.max())


# ------------------------------------------------------------------ decode --

def run_decode_case(B, H_q, H_kv, d, ctx_lens, LK, LV, seed=0, splits=None, cap=None,
                    out_dtype=kvq.OUT_FP32, q_scale=1.0, tau=None, mode_k=O.MODE_LIN8,
                    mode_v=O.MODE_LOG4):
    maxc = max(ctx_lens) if len(ctx_lens) else 0
    cap = cap or max(16, (maxc + 15) // 16 * 16)
    G = H_q // H_kv
    sk, sv = _signs(seed + 11, d), _signs(seed + 12, d)
    xk = _rand_x(B, H_kv, cap, d, seed=seed + 1)
    xv = _rand_x(B, H_kv, cap, d, seed=seed + 2, outliers=False)
    q = (np.random.default_rng(seed + 3).standard_normal((B, H_q, d)) * q_scale).astype(np.float16)
    kc, vc = kvq.codec(d, LK, mode_k), kvq.codec(d, LV, mode_v)
    Kp, Vp = kvq.alloc_plane(kc, B, H_kv, cap), kvq.alloc_plane(vc, B, H_kv, cap)
    kcodes = O.encode(xk, sk, LK, mode_k)
    vcodes = O.encode(xv, sv, LV, mode_v)
    for b in range(B):
        for h in range(H_kv):
            sl = slice((b * H_kv + h) * cap, (b * H_kv + h + 1) * cap)
            put_rows(Kp, kcodes.take(sl), b, h, 0)
            put_rows(Vp, vcodes.take(sl), b, h, 0)
    tau = tau if tau is not None else 1.0 / math.sqrt(d)
    ctx_t = torch.tensor(ctx_lens, dtype=torch.int32, device="cuda")
    qd = torch.from_numpy(q).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = kvq.decode_attn(qd, kc, vc, _dev_signs(sk), _dev_signs(sv), Kp, Vp, ctx_t, maxc, tau,
                          num_splits=splits, err_word=err, out_dtype=out_dtype)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy().astype(np.float64)
    want = np.zeros((B, H_q, d))
    for b in range(B):
        for h in range(H_kv):
            base = (b * H_kv + h) * cap
            T = ctx_lens[b]
            kh = O.dequant(kcodes.take(slice(base, base + T)), sk)
            vh = O.dequant(vcodes.take(slice(base, base + T)), sv)
            want[b, h * G:(h + 1) * G] = O.attend(q[b, h * G:(h + 1) * G].astype(np.float64),
                                                   kh, vh, tau)
    return got, want, int(err.item())


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_decode_gqa_sweep(dev, d, G):
    H_kv = 2
    got, want, err = run_decode_case(3, G * H_kv, H_kv, d, [1, 77, 300], 128, 64, seed=d + G)
    e = rel_l2(got, want)
    assert err == 0
    assert e.max() <= REL_L2_TOL, e.max()


@pytest.mark.parametrize("d,G,LK,LV,mk,mv", [
    (4, 1, 2, 3, O.MODE_LIN8, O.MODE_LOG4),        # the smallest head
    (8, 3, 16, 16, O.MODE_LIN8, O.MODE_LOG4),      # G not a power of two
    (16, 2, 128, 64, O.MODE_LOG4, O.MODE_LIN8),    # norm modes swapped
    (32, 4, 1000, 24, O.MODE_LIN8, O.MODE_LOG4),
    (64, 16, 128, 64, O.MODE_LIN8, O.MODE_LOG4),   # G 16: two head chunks
    (128, 4, 512, 64, O.MODE_LIN8, O.MODE_LOG4),   # L past the staged kernel's 256
    (128, 6, 65536, 5000, O.MODE_LOG4, O.MODE_LOG4),  # sincospif past the 4096 table
    (256, 4, 128, 64, O.MODE_LIN8, O.MODE_LOG4),
    (256, 1, 4096, 2, O.MODE_LIN8, O.MODE_LIN8),
])
def test_decode_every_codec(dev, d, G, LK, LV, mk, mv):
    """Decode over codecs outside the staged kernel's set (the generic
    kernel) against the oracle: ragged lengths, an empty sequence, two split
    counts."""
    H_kv = 2
    for splits in (None, 3):
        got, want, err = run_decode_case(4, G * H_kv, H_kv, d, [1, 77, 300, 0], LK, LV,
                                         seed=d + G + LK, splits=splits, mode_k=mk, mode_v=mv)
        assert err == 0
        assert rel_l2(got, want)[:3].max() <= REL_L2_TOL, (splits, rel_l2(got, want))
        assert np.all(got[3] == 0)


@pytest.mark.parametrize("G,LK,LV", [(4, 128, 64), (2, 32, 128), (1, 64, 32), (4, 100, 20)])
def test_decode_multi_wave(dev, G, LK, LV):
    """Launches of more than one wave of CTAs (here 8 x 4 x 6 = 192 > 148)
    with G up to 4 and 5..7-bit codes: the one-CTA instance with 256-token
    tiles on this contiguous cache (splits of 336 tokens; the two-CTAs-per-SM
    instance serves paged caches: test_paged); against the oracle."""
    B, H_kv = 8, 4
    got, want, err = run_decode_case(B, G * H_kv, H_kv, 128,
                                     [2000, 1, 129, 1500, 0, 1800, 64, 333],
                                     LK, LV, seed=G + LK, splits=6)
    assert err == 0
    e = rel_l2(got, want)
    assert e[[0, 1, 2, 3, 5, 6, 7]].max() <= REL_L2_TOL, e
    assert np.all(got[4] == 0)


@pytest.mark.parametrize("LK,LV", [(256, 256), (128, 64), (32, 5), (2, 2), (200, 33)])
def test_decode_codebooks(dev, LK, LV):
    got, want, _ = run_decode_case(2, 8, 2, 128, [129, 64], LK, LV, seed=LK + LV)
    assert rel_l2(got, want).max() <= REL_L2_TOL


@pytest.mark.parametrize("splits", [1, 2, 3, 7, 20])
def test_decode_splits(dev, splits):
    got, want, _ = run_decode_case(2, 8, 2, 128, [333, 17], 128, 64, seed=4, splits=splits)
    assert rel_l2(got, want).max() <= REL_L2_TOL


def test_decode_split_invariance(dev):
    outs = [run_decode_case(1, 8, 2, 64, [500], 128, 64, seed=8, splits=s)[0] for s in (1, 4, 16)]
    for o in outs[1:]:
        assert rel_l2(o, outs[0]).max() < 1e-5


@pytest.mark.parametrize("ctx_lens,splits,H_kv,G,d,LK,LV", [
    ([300, 129, 1, 0], None, 2, 4, 128, 128, 64),  # ragged, a one-token sequence, an empty one
    ([256, 128], 2, 2, 4, 128, 128, 64),  # new token on the first row of a tile / of a split
    ([257, 200], 3, 2, 4, 128, 128, 64),
    ([4096], None, 8, 4, 128, 128, 64),   # the Llama-shaped layer
    ([1000, 513], 1, 1, 8, 128, 128, 64),  # one split: the held tile is not the first
    ([300, 129, 1, 0], 3, 2, 3, 256, 128, 64),  # the generic kernel (append launched first)
    ([4096, 3000, 1], 20, 4, 4, 128, 128, 64),  # multi-wave: two CTAs per SM, append first
    ([200, 64], None, 2, 4, 32, 512, 32),
])
def test_decode_step_equals_append_then_decode(dev, ctx_lens, splits, H_kv, G, d, LK, LV):
    """kvq_decode_step writes the new token's codes exactly as kvq_encode_kv
    does and returns exactly what kvq_decode_attn returns on the appended
    cache; the appended cache also matches the oracle."""
    B = len(ctx_lens)
    H_q = G * H_kv
    cap = (max(ctx_lens) + 16 + 15) // 16 * 16
    sk, sv = _signs(31, d), _signs(32, d)
    k = _rand_x(B, H_kv, cap, d, seed=33)
    v = _rand_x(B, H_kv, cap, d, seed=34, outliers=False)
    kc, vc = kvq.codec(d, LK, O.MODE_LIN8), kvq.codec(d, LV, O.MODE_LOG4)
    skd, svd = _dev_signs(sk), _dev_signs(sv)
    kd, vd = torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda()
    # reference: every position encoded; step: the new positions blanked first
    Kr, Vr = kvq.alloc_plane(kc, B, H_kv, cap), kvq.alloc_plane(vc, B, H_kv, cap)
    Ks, Vs = kvq.alloc_plane(kc, B, H_kv, cap), kvq.alloc_plane(vc, B, H_kv, cap)
    for P, c, x, sg in ((Kr, kc, kd, skd), (Vr, vc, vd, svd), (Ks, kc, kd, skd), (Vs, vc, vd, svd)):
        kvq.encode(c, sg, x, P, 0)
    k_new = torch.zeros((B, H_kv, d), dtype=torch.float16, device="cuda")
    v_new = torch.zeros_like(k_new)
    for b, n in enumerate(ctx_lens):
        if n >= 1:
            k_new[b] = kd[b, :, n - 1]
            v_new[b] = vd[b, :, n - 1]
            for P in (Ks, Vs):
                for w in range(3):
                    P.rows(w)[b, :, n - 1] = 0xA5
    ctx = torch.tensor(ctx_lens, dtype=torch.int32, device="cuda")
    q = torch.from_numpy(np.random.default_rng(35).standard_normal((B, H_q, d)).astype(np.float16)).cuda()
    maxc = max(ctx_lens)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out_s = kvq.decode_step(q, k_new, v_new, kc, vc, skd, svd, Ks, Vs, ctx, maxc, num_splits=splits,
                            err_word=err)
    out_r = kvq.decode_attn(q, kc, vc, skd, svd, Kr, Vr, ctx, maxc, num_splits=splits)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for w in range(3):
        assert torch.equal(Ks.rows(w), Kr.rows(w)), ("K", w)
        assert torch.equal(Vs.rows(w), Vr.rows(w)), ("V", w)
    assert torch.equal(out_s, out_r)
    compare_codes(plane_rows(Ks, t_range=(0, cap)), O.encode(k, sk, LK, O.MODE_LIN8))
    compare_codes(plane_rows(Vs, t_range=(0, cap)), O.encode(v, sv, LV, O.MODE_LOG4))


def test_decode_step_prepared_call_equals_call(dev):
    """DecodeStepCall (arguments marshalled once) runs the same C entry point:
    on twin caches it writes the same codes and returns the same output as
    kvq_decode_step, and repeated calls keep doing so."""
    d, B, H_kv, G = 128, 2, 2, 4
    H_q, cap = G * H_kv, 512
    kc, vc = kvq.codec(d, 128, O.MODE_LIN8), kvq.codec(d, 64, O.MODE_LOG4)
    skd, svd = _dev_signs(_signs(41, d)), _dev_signs(_signs(42, d))
    kd = torch.from_numpy(_rand_x(B, H_kv, cap, d, seed=43)).cuda()
    vd = torch.from_numpy(_rand_x(B, H_kv, cap, d, seed=44, outliers=False)).cuda()
    planes = []
    for _ in range(2):
        K, V = kvq.alloc_plane(kc, B, H_kv, cap), kvq.alloc_plane(vc, B, H_kv, cap)
        kvq.encode(kc, skd, kd, K, 0)
        kvq.encode(vc, svd, vd, V, 0)
        planes.append((K, V))
    q = torch.randn((B, H_q, d), dtype=torch.float16, device="cuda")
    k_new = torch.randn((B, H_kv, d), dtype=torch.float16, device="cuda")
    v_new = torch.randn((B, H_kv, d), dtype=torch.float16, device="cuda")
    ctx = torch.tensor([400, 129], dtype=torch.int32, device="cuda")
    S, tau = 3, 1 / math.sqrt(d)
    ws = [kvq.DecodeWorkspace(B, H_q, d, S) for _ in range(2)]
    outs = [torch.empty((B, H_q, d), dtype=torch.float32, device="cuda") for _ in range(2)]
    (K0, V0), (K1, V1) = planes
    Kc0, Vc0, Kc1, Vc1 = K0.c(), V0.c(), K1.c(), V1.c()
    call = kvq.DecodeStepCall(q, k_new, v_new, kc, vc, skd, svd, Kc1, Vc1, ctx, B, H_q, H_kv,
                              cap, tau, S, ws[1].buf, ws[1].nbytes, None, outs[1], kvq.OUT_FP32)
    for _ in range(2):
        kvq.kvq_decode_step(q, k_new, v_new, kc, vc, skd, svd, Kc0, Vc0, ctx, B, H_q, H_kv, cap,
                            tau, S, ws[0].buf, ws[0].nbytes, None, outs[0], kvq.OUT_FP32)
        call()
        torch.cuda.synchronize()
        assert torch.equal(outs[0], outs[1])
        for w in range(3):
            assert torch.equal(K0.rows(w), K1.rows(w)) and torch.equal(V0.rows(w), V1.rows(w))


def test_decode_step_host_equals_device_step(dev):
    """kvq_decode_step_host (inputs and output in pinned host memory, copies
    on the stream, or read and written by the kernel itself) equals
    kvq_decode_step on twin caches, through the prepared-call wrapper too."""
    d, B, H_kv, G = 128, 2, 2, 4
    H_q, cap = G * H_kv, 512
    kc, vc = kvq.codec(d, 128, O.MODE_LIN8), kvq.codec(d, 64, O.MODE_LOG4)
    skd, svd = _dev_signs(_signs(51, d)), _dev_signs(_signs(52, d))
    kd = torch.from_numpy(_rand_x(B, H_kv, cap, d, seed=53)).cuda()
    vd = torch.from_numpy(_rand_x(B, H_kv, cap, d, seed=54, outliers=False)).cuda()
    planes = []
    for _ in range(4):
        K, V = kvq.alloc_plane(kc, B, H_kv, cap), kvq.alloc_plane(vc, B, H_kv, cap)
        kvq.encode(kc, skd, kd, K, 0)
        kvq.encode(vc, svd, vd, V, 0)
        planes.append((K, V, K.c(), V.c()))
    nq, nk = B * H_q * d, B * H_kv * d
    hin = torch.randn(nq + 2 * nk, dtype=torch.float16).pin_memory()
    din = torch.empty(nq + 2 * nk, dtype=torch.float16, device="cuda")
    q, k_new, v_new = (hin[:nq].cuda().view(B, H_q, d), hin[nq:nq + nk].cuda().view(B, H_kv, d),
                       hin[nq + nk:].cuda().view(B, H_kv, d))
    ctx = torch.tensor([333, 129], dtype=torch.int32, device="cuda")
    S, tau = 2, 1 / math.sqrt(d)
    ws = [kvq.DecodeWorkspace(B, H_q, d, S) for _ in range(4)]
    out_ref = torch.empty((B, H_q, d), dtype=torch.float16, device="cuda")
    kvq.kvq_decode_step(q, k_new, v_new, kc, vc, skd, svd, planes[0][2], planes[0][3], ctx, B, H_q,
                        H_kv, cap, tau, S, ws[0].buf, ws[0].nbytes, None, out_ref, kvq.OUT_FP16)
    hout = [torch.empty((B, H_q, d), dtype=torch.float16).pin_memory() for _ in range(2)]
    dout = [torch.empty((B, H_q, d), dtype=torch.float16, device="cuda") for _ in range(2)]
    kvq.kvq_decode_step_host(hin, din, hout[0], dout[0], kc, vc, skd, svd, planes[1][2],
                             planes[1][3], ctx, B, H_q, H_kv, cap, tau, S, ws[1].buf, ws[1].nbytes,
                             None, kvq.OUT_FP16)
    call = kvq.DecodeStepHostCall(hin, din, hout[1], dout[1], kc, vc, skd, svd, planes[2][2],
                                  planes[2][3], ctx, B, H_q, H_kv, cap, tau, S, ws[2].buf,
                                  ws[2].nbytes, None, kvq.OUT_FP16)
    call()
    # no device buffers: the kernel reads and writes the page-locked host memory
    hout.append(torch.empty((B, H_q, d), dtype=torch.float16).pin_memory())
    kvq.kvq_decode_step_host(hin, None, hout[2], None, kc, vc, skd, svd, planes[3][2],
                             planes[3][3], ctx, B, H_q, H_kv, cap, tau, S, ws[3].buf,
                             ws[3].nbytes, None, kvq.OUT_FP16)
    torch.cuda.synchronize()
    ref = out_ref.cpu()
    for h in hout:
        assert torch.equal(h, ref)
    for w in range(3):
        for P in planes[1:]:
            assert torch.equal(P[0].rows(w), planes[0][0].rows(w))
            assert torch.equal(P[1].rows(w), planes[0][1].rows(w))


def test_decode_step_clipped_context_appends_nothing(dev):
    d, B, H_kv, cap = 128, 1, 2, 64
    kc, vc = kvq.codec(d, 128, O.MODE_LIN8), kvq.codec(d, 64, O.MODE_LOG4)
    K, V = kvq.alloc_plane(kc, B, H_kv, cap), kvq.alloc_plane(vc, B, H_kv, cap)
    s = _dev_signs(_signs(36, d))
    k_new = torch.ones((B, H_kv, d), dtype=torch.float16, device="cuda")
    q = torch.ones((B, 4 * H_kv, d), dtype=torch.float16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ctx = torch.tensor([cap + 5], dtype=torch.int32, device="cuda")
    kvq.decode_step(q, k_new, k_new, kc, vc, s, s, K, V, ctx, cap, err_word=err)
    torch.cuda.synchronize()
    assert int(err.item()) & kvq.KVQ_DEVERR_CTX_RANGE
    for w in range(3):
        assert int(K.rows(w).count_nonzero()) == 0 and int(V.rows(w).count_nonzero()) == 0


def test_decode_fp16_output_and_scale(dev):
    got, want, _ = run_decode_case(2, 16, 2, 128, [250, 99], 128, 64, seed=6,
                                   out_dtype=kvq.OUT_FP16, q_scale=3.0, tau=0.2)
    assert rel_l2(got, want).max() <= REL_L2_TOL


def test_decode_empty_and_clipped_context(dev):
    # ctx_len 0 gives zeros; a ctx_len above capacity is clipped and flagged
    got, want, err = run_decode_case(2, 4, 1, 64, [0, 32], 128, 64, seed=7)
    assert np.all(got[0] == 0)
    assert rel_l2(got[1], want[1]).max() <= REL_L2_TOL and err == 0
    B, d = 1, 64
    kc, vc = kvq.codec(d, 128, 0), kvq.codec(d, 64, 1)
    Kp, Vp = kvq.alloc_plane(kc, B, 1, 32), kvq.alloc_plane(vc, B, 1, 32)
    q = torch.zeros((B, 1, d), dtype=torch.float16, device="cuda")
    errw = torch.zeros(1, dtype=torch.int32, device="cuda")
    s = _dev_signs(_signs(1, d))
    out = kvq.decode_attn(q, kc, vc, s, s, Kp, Vp, torch.tensor([99], dtype=torch.int32,
                                                               device="cuda"), 64, 0.125,
                          err_word=errw)
    torch.cuda.synchronize()
    assert int(errw.item()) & kvq.KVQ_DEVERR_CTX_RANGE
    assert torch.isfinite(out).all()


def test_decode_deterministic(dev):
    a = run_decode_case(2, 8, 2, 128, [300, 300], 128, 64, seed=9)[0]
    b = run_decode_case(2, 8, 2, 128, [300, 300], 128, 64, seed=9)[0]
    assert np.array_equal(a, b)


# --------------------------------------------------- workloads (full sizes) --

def _plane_for(w, layer, kind, dev_signs, L, mode, cap):
    c = kvq.codec(w.d, L, mode)
    p = kvq.alloc_plane(c, w.B, w.H_kv, cap)
    x = synth.kv(w, layer, kind, device="cuda", T=w.ctx)
    kvq.encode(c, dev_signs, x, p, 0)
    return c, p, x


def test_workload_tiny_round_trip_and_decode_step(dev):
    """1 layer, B 1, 2 KV / 4 query heads, d 128, 256 tokens, L_K = L_V = 128:
    prefill 255 tokens, append the 256th (T = 1), round-trip through dequant,
    then one decode step over all 256 tokens."""
    w = synth.WORKLOADS["tiny_b1_hq4_hkv2_d128_ctx256"]
    sk, sv = synth.layer_signs(w, 0)
    K = synth.kv(w, 0, synth.KIND_K, device="cuda")
    V = synth.kv(w, 0, synth.KIND_V, device="cuda")
    q = synth.queries(w, 0, device="cuda")
    kc, vc = kvq.codec(128, 128, 0), kvq.codec(128, 128, 1)
    Kp, Vp = kvq.alloc_plane(kc, 1, 2, 256), kvq.alloc_plane(vc, 1, 2, 256)
    skd, svd = _dev_signs(sk), _dev_signs(sv)
    for c, p, x, s in ((kc, Kp, K, skd), (vc, Vp, V, svd)):
        kvq.encode(c, s, x[:, :, :255].contiguous(), p, 0)
        kvq.encode(c, s, x[:, :, 255:].contiguous(), p, 255)
    torch.cuda.synchronize()
    Kh, Vh = K.cpu().numpy(), V.cpu().numpy()
    ok_ = O.encode(Kh, sk, 128, O.MODE_LIN8)
    ov_ = O.encode(Vh, sv, 128, O.MODE_LOG4)
    compare_codes(plane_rows(Kp), ok_)
    compare_codes(plane_rows(Vp), ov_)
    # round trip: GPU dequant of the oracle's codes vs the oracle's dequant
    for c, p, oc, s, sd in ((kc, Kp, ok_, sk, skd), (vc, Vp, ov_, sv, svd)):
        for h in range(2):
            put_rows(p, oc.take(slice(h * 256, (h + 1) * 256)), 0, h, 0)
        y = kvq.dequant(c, sd, p, 256).cpu().numpy().astype(np.float64).reshape(-1, 128)
        assert rel_l2(y, O.dequant(oc, s)).max() <= REL_L2_TOL
    ctx = torch.tensor([256], dtype=torch.int32, device="cuda")
    out = kvq.decode_attn(q, kc, vc, skd, svd, Kp, Vp, ctx, 256).cpu().numpy()
    qh = q.cpu().numpy().astype(np.float64)
    for h in range(2):
        kh = O.dequant(ok_.take(slice(h * 256, (h + 1) * 256)), sk)
        vh = O.dequant(ov_.take(slice(h * 256, (h + 1) * 256)), sv)
        want = O.attend(qh[0, 2 * h:2 * h + 2], kh, vh, 1 / math.sqrt(128))
        assert rel_l2(out[0, 2 * h:2 * h + 2], want).max() <= REL_L2_TOL


def _check_decode_workload(w, layers, samples, seed=0):
    """Full-size layers: GPU-encode the whole layer, compare sampled (b, kv
    head) slices with the oracle's codes, overwrite those slices with the
    oracle's codes, run the decode launch the bench times (default splits)
    and compare the sampled heads with oracle attention; every other head
    must be finite and inside the convex hull bound max_t |v^_t|."""
    rng = np.random.default_rng(seed)
    cap = w.ctx
    sm = torch.cuda.get_device_properties(0).multi_processor_count
    S = kvq.kvq_decode_num_splits(w.B, w.H_kv, w.ctx, sm)
    ws = kvq.DecodeWorkspace(w.B, w.H_q, w.d, S)
    tau = 1.0 / math.sqrt(w.d)
    for layer in layers:
        sk, sv = synth.layer_signs(w, layer)
        skd, svd = _dev_signs(sk), _dev_signs(sv)
        kc, Kp, K = _plane_for(w, layer, synth.KIND_K, skd, w.L_K[layer], 0, cap)
        vc, Vp, V = _plane_for(w, layer, synth.KIND_V, svd, w.L_V[layer], 1, cap)
        q = synth.queries(w, layer, device="cuda")
        picks = [(int(rng.integers(0, w.B)), int(rng.integers(0, w.H_kv))) for _ in range(samples)]
        oracle_codes = {}
        for b, h in picks:
            xk = K[b, h].cpu().numpy()
            xv = V[b, h].cpu().numpy()
            okc = O.encode(xk, sk, w.L_K[layer], 0)
            ovc = O.encode(xv, sv, w.L_V[layer], 1)
            compare_codes(plane_rows(Kp, (b, b + 1), (h, h + 1)), okc)
            compare_codes(plane_rows(Vp, (b, b + 1), (h, h + 1)), ovc)
            put_rows(Kp, okc, b, h, 0)
            put_rows(Vp, ovc, b, h, 0)
            oracle_codes[(b, h)] = (okc, ovc)
        del K, V
        ctx = torch.full((w.B,), w.ctx, dtype=torch.int32, device="cuda")
        out = kvq.decode_attn(q, kc, vc, skd, svd, Kp, Vp, ctx, w.ctx, tau, num_splits=S,
                              workspace=ws)
        torch.cuda.synchronize()
        o = out.cpu().numpy().astype(np.float64)
        assert np.isfinite(o).all()
        qh = q.cpu().numpy().astype(np.float64)
        G = w.G
        for (b, h), (okc, ovc) in oracle_codes.items():
            kh, vh = O.dequant(okc, sk), O.dequant(ovc, sv)
            want = O.attend(qh[b, h * G:(h + 1) * G], kh, vh, tau)
            e = rel_l2(o[b, h * G:(h + 1) * G], want)
            assert e.max() <= REL_L2_TOL, (layer, b, h, e.max())
            vmax = np.linalg.norm(vh, axis=1).max()
            assert np.linalg.norm(o[b, h * G:(h + 1) * G], axis=1).max() <= vmax * (1 + 1e-3)
        del Kp, Vp
        torch.cuda.empty_cache()


def test_workload_llama7b_layer_full(dev):
    w = synth.WORKLOADS["llama7b_layer_b1_hq32_hkv8_d128_ctx4096"]
    _check_decode_workload(w, [0], samples=8)


def test_workload_mistral7b_32layers_sampled(dev):
    w = synth.WORKLOADS["mistral7b_32layers_b8_hq32_hkv8_d128_ctx32768"]
    _check_decode_workload(w, [0, 3, 4, 31], samples=2, seed=3)


def test_workload_tinyllama_long_context_sampled(dev):
    w = synth.WORKLOADS["tinyllama_22layers_b4_hq32_hkv4_d64_ctx65536"]
    _check_decode_workload(w, [0, 1, 2, 21], samples=2, seed=5)


def test_workload_prefill_encode_dequant_sampled(dev):
    """Prefill workload at full per-layer size (16 x 8 x 8192 vectors of d 128
    per K/V): GPU encode of a whole layer, sampled slices against the oracle,
    then GPU dequant of the oracle's codes of those slices."""
    w = synth.WORKLOADS["prefill_32layers_b16_t8192_hkv8_d128"]
    rng = np.random.default_rng(1)
    for layer in (0, 31):
        sk, sv = synth.layer_signs(w, layer)
        for kind, L, mode, s in ((synth.KIND_K, 128, 0, sk), (synth.KIND_V, 64, 1, sv)):
            sd = _dev_signs(s)
            c, p, x = _plane_for(w, layer, kind, sd, L, mode, w.ctx)
            picks = {}
            for _ in range(2):
                b, h = int(rng.integers(0, w.B)), int(rng.integers(0, w.H_kv))
                oc = O.encode(x[b, h].cpu().numpy(), s, L, mode)
                compare_codes(plane_rows(p, (b, b + 1), (h, h + 1)), oc)
                put_rows(p, oc, b, h, 0)
                picks[(b, h)] = oc
            y = kvq.dequant(c, sd, p, w.ctx)
            torch.cuda.synchronize()
            assert torch.isfinite(y).all()
            for (b, h), oc in picks.items():
                yb = y[b, h].cpu().numpy().astype(np.float64)
                assert rel_l2(yb, O.dequant(oc, s)).max() <= REL_L2_TOL
            del p, x, y
            torch.cuda.empty_cache()
