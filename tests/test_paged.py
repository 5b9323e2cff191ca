"""Paged K/V planes: kvq_encode_kv_paged, kvq_decode_attn_paged and
kvq_decode_step_paged against the contiguous forms on the same rows.

The pages hold whole 128-token tiles; the rows of each sequence are spread
over a shuffled page table (with pages of other sequences and unused pages in
between), so any mix-up of pages, heads or offsets changes the result."""
import ctypes as C
import math

import numpy as np
import pytest

from decode_attention_rand_b200 import kvq

FAKE = 1 << 20


def _codecs(d=128):
    return kvq.codec(d, 128, kvq.KVQ_NORM_LIN8), kvq.codec(d, 64, kvq.KVQ_NORM_LOG4)


def _paged(page_tokens=128, max_pages=4, num_pages=16, pages=FAKE):
    return kvq.kvq_paged_plane(FAKE, FAKE, FAKE, pages, page_tokens, max_pages, num_pages)


@pytest.mark.parametrize("kw,msg", [
    (dict(page_tokens=100), "multiple of 128"),
    (dict(page_tokens=0), "multiple of 128"),
    (dict(pages=None), "NULL pool or page table"),
    (dict(max_pages=0), "must be positive"),
])
def test_paged_plane_checks(kw, msg):
    kc, vc = _codecs()
    K, V = _paged(**kw), _paged()
    ws = kvq.kvq_decode_workspace_bytes(1, 8, 128, 2)
    rc = kvq.lib().kvq_decode_attn_paged(FAKE, C.byref(kc), C.byref(vc), FAKE, FAKE, C.byref(K),
                                         C.byref(V), FAKE, 1, 8, 2, 256, 0.1, 2, FAKE, ws, None,
                                         FAKE, 0, None)
    assert rc == kvq.KVQ_EINVAL
    assert msg in kvq.kvq_last_error()


def test_paged_encode_checks_capacity():
    kc, vc = _codecs()
    K, V = _paged(max_pages=2), _paged(max_pages=2)  # capacity 256
    rc = kvq.lib().kvq_encode_kv_paged(C.byref(kc), FAKE, FAKE, C.byref(K), C.byref(vc), FAKE,
                                       FAKE, C.byref(V), 1, 2, 10, 250, None, None)
    assert rc == kvq.KVQ_EINVAL
    assert "exceed capacity" in kvq.kvq_last_error()


# ------------------------------------------------------------------- GPU --

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from decode_attention_rand_b200 import build as kbuild
    kbuild.build()
    kvq.lib()
    return torch.device("cuda:0")


def _signs(seed, d):
    rng = np.random.default_rng(seed)
    return torch.from_numpy(np.where(rng.integers(0, 2, d) == 0, 1, -1).astype(np.int8)).cuda()


def _setup(B, H_kv, d, max_pages, page_tokens=128, spare=3, seed=0):
    """Contiguous planes filled with encoded random K/V, and paged planes holding
    the same rows under a shuffled page table."""
    kc, vc = _codecs(d)
    cap = max_pages * page_tokens
    rng = np.random.default_rng(seed)
    k = torch.from_numpy(rng.standard_normal((B, H_kv, cap, d)).astype(np.float16)).cuda()
    v = torch.from_numpy(rng.standard_normal((B, H_kv, cap, d)).astype(np.float16)).cuda()
    k[..., 3] *= 20
    sk, sv = _signs(seed + 1, d), _signs(seed + 2, d)
    Kc, Vc = kvq.alloc_plane(kc, B, H_kv, cap), kvq.alloc_plane(vc, B, H_kv, cap)
    kvq.encode(kc, sk, k, Kc, 0)
    kvq.encode(vc, sv, v, Vc, 0)
    num_pages = B * max_pages + spare
    table = rng.permutation(num_pages)[:B * max_pages].reshape(B, max_pages)
    Kp = kvq.alloc_paged_plane(kc, H_kv, page_tokens, num_pages, table)
    Vp = kvq.alloc_paged_plane(vc, H_kv, page_tokens, num_pages, table)
    for P, Cn in ((Kp, Kc), (Vp, Vc)):
        for w in range(3):
            for b in range(B):
                for i in range(max_pages):
                    P.rows(w)[int(table[b, i])] = Cn.rows(w)[b, :, i * page_tokens:(i + 1) * page_tokens]
    return kc, vc, sk, sv, k, v, Kc, Vc, Kp, Vp, table


def _same_rows(P, Cn, table, page_tokens=128):
    B, max_pages = table.shape
    for w in range(3):
        for b in range(B):
            for i in range(max_pages):
                got = P.rows(w)[int(table[b, i])]
                want = Cn.rows(w)[b, :, i * page_tokens:(i + 1) * page_tokens]
                if not torch.equal(got, want):
                    return False
    return True


def _ws(B, H_q, d, S):
    return kvq.DecodeWorkspace(B, H_q, d, S, "cuda")


@pytest.mark.gpu
@pytest.mark.parametrize("S", [1, 2, 3, 6])
def test_paged_decode_equals_contiguous(dev, S):
    B, H_kv, G, d, max_pages = 3, 2, 4, 128, 6
    kc, vc, sk, sv, k, v, Kc, Vc, Kp, Vp, table = _setup(B, H_kv, d, max_pages, seed=S)
    H_q = G * H_kv
    q = torch.randn((B, H_q, d), dtype=torch.float16, device="cuda")
    ctx = torch.tensor([300, 129, 768], dtype=torch.int32, device="cuda")
    maxc, tau = 768, 1 / math.sqrt(d)  # 768 / S is a whole number of tiles for these S
    out_c = kvq.decode_attn(q, kc, vc, sk, sv, Kc, Vc, ctx, maxc, tau, num_splits=S)
    ws = _ws(B, H_q, d, S)
    out_p = torch.empty_like(out_c)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvq.kvq_decode_attn_paged(q, kc, vc, sk, sv, Kp.c(), Vp.c(), ctx, B, H_q, H_kv, maxc, tau, S,
                              ws.buf, ws.nbytes, err, out_p, kvq.OUT_FP32)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(out_p, out_c)


@pytest.mark.gpu
def test_paged_decode_unaligned_split_count(dev):
    # 5 splits of 768 tokens: the paged form starts its splits on whole tiles,
    # the contiguous one on 16-token rows: the same attention up to rounding
    B, H_kv, G, d, max_pages = 2, 2, 4, 128, 6
    kc, vc, sk, sv, k, v, Kc, Vc, Kp, Vp, table = _setup(B, H_kv, d, max_pages, seed=9)
    H_q = G * H_kv
    q = torch.randn((B, H_q, d), dtype=torch.float16, device="cuda")
    ctx = torch.tensor([700, 401], dtype=torch.int32, device="cuda")
    out_c = kvq.decode_attn(q, kc, vc, sk, sv, Kc, Vc, ctx, 768, None, num_splits=5)
    ws = _ws(B, H_q, d, 5)
    out_p = torch.empty_like(out_c)
    kvq.kvq_decode_attn_paged(q, kc, vc, sk, sv, Kp.c(), Vp.c(), ctx, B, H_q, H_kv, 768,
                              1 / math.sqrt(d), 5, ws.buf, ws.nbytes, None, out_p, kvq.OUT_FP32)
    torch.cuda.synchronize()
    rel = ((out_p - out_c).double().norm(dim=-1) / out_c.double().norm(dim=-1)).max().item()
    assert rel < 1e-5


@pytest.mark.gpu
def test_paged_encode_kv_equals_contiguous(dev):
    B, H_kv, d, max_pages = 2, 3, 128, 4
    kc, vc, sk, sv, k, v, Kc, Vc, Kp, Vp, table = _setup(B, H_kv, d, max_pages, seed=5)
    # overwrite tokens 50 .. 349 (three pages) of both layouts with new vectors
    rng = np.random.default_rng(6)
    kn = torch.from_numpy(rng.standard_normal((B, H_kv, 300, d)).astype(np.float16)).cuda()
    vn = torch.from_numpy(rng.standard_normal((B, H_kv, 300, d)).astype(np.float16)).cuda()
    kvq.encode_kv(kc, sk, kn, Kc, vc, sv, vn, Vc, 50)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvq.kvq_encode_kv_paged(kc, sk, kn, Kp.c(), vc, sv, vn, Vp.c(), B, H_kv, 300, 50, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert _same_rows(Kp, Kc, table) and _same_rows(Vp, Vc, table)


@pytest.mark.gpu
def test_paged_decode_step_equals_contiguous(dev):
    B, H_kv, G, d, max_pages = 3, 2, 4, 128, 4
    kc, vc, sk, sv, k, v, Kc, Vc, Kp, Vp, table = _setup(B, H_kv, d, max_pages, seed=7)
    H_q = G * H_kv
    q = torch.randn((B, H_q, d), dtype=torch.float16, device="cuda")
    k_new = torch.randn((B, H_kv, d), dtype=torch.float16, device="cuda")
    v_new = torch.randn((B, H_kv, d), dtype=torch.float16, device="cuda")
    ctx = torch.tensor([129, 256, 384], dtype=torch.int32, device="cuda")  # page edges
    S = 2
    out_c = kvq.decode_step(q, k_new, v_new, kc, vc, sk, sv, Kc, Vc, ctx, 512, num_splits=S)
    ws = _ws(B, H_q, d, S)
    out_p = torch.empty_like(out_c)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvq.kvq_decode_step_paged(q, k_new, v_new, kc, vc, sk, sv, Kp.c(), Vp.c(), ctx, B, H_q, H_kv,
                              512, 1 / math.sqrt(d), S, ws.buf, ws.nbytes, err, out_p,
                              kvq.OUT_FP32)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert _same_rows(Kp, Kc, table) and _same_rows(Vp, Vc, table)
    assert torch.equal(out_p, out_c)


@pytest.mark.gpu
def test_paged_bad_page_entry_is_reported(dev):
    B, H_kv, G, d, max_pages = 1, 2, 4, 128, 2
    kc, vc, sk, sv, k, v, Kc, Vc, Kp, Vp, table = _setup(B, H_kv, d, max_pages, seed=8)
    Kp.pages[0, 1] = 10_000  # beyond the pool
    H_q = G * H_kv
    q = torch.randn((B, H_q, d), dtype=torch.float16, device="cuda")
    ctx = torch.tensor([256], dtype=torch.int32, device="cuda")
    ws = _ws(B, H_q, d, 1)
    out = torch.empty((B, H_q, d), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvq.kvq_decode_attn_paged(q, kc, vc, sk, sv, Kp.c(), Vp.c(), ctx, B, H_q, H_kv, 256,
                              1 / math.sqrt(d), 1, ws.buf, ws.nbytes, err, out, kvq.OUT_FP32)
    torch.cuda.synchronize()
    assert int(err.item()) & kvq.KVQ_DEVERR_PAGE_RANGE
    assert torch.isfinite(out).all()


# --------------------------------------------------- against the oracle --
# The tests above pin the paged forms to the contiguous ones; these compare
# them with the fp64 oracle directly, reading the codes through the page
# table on the host.

import oracle as O  # noqa: E402

from kvq_testutil import REL_L2_TOL, compare_codes, paged_rows, rel_l2  # noqa: E402


def _gather(P, table, b, t0, t1):
    """O.Codes of tokens t0 .. t1-1 of every KV head of sequence b, read
    through the page table; rows in (h, t) order."""
    rows = paged_rows(P, table, b, t0, t1)
    c = P.codec
    return O.Codes(c.head_dim, c.L, c.norm_mode, *rows)


def _oracle_attend_paged(q, Kp, Vp, table, sk, sv, ctx_lens, G, tau):
    B, H_q, d = q.shape
    H_kv = H_q // G
    want = np.zeros((B, H_q, d))
    for b in range(B):
        n = int(ctx_lens[b])
        kcodes, vcodes = _gather(Kp, table, b, 0, n), _gather(Vp, table, b, 0, n)
        for h in range(H_kv):
            kh = O.dequant(kcodes.take(slice(h * n, (h + 1) * n)), sk)
            vh = O.dequant(vcodes.take(slice(h * n, (h + 1) * n)), sv)
            want[b, h * G:(h + 1) * G] = O.attend(q[b, h * G:(h + 1) * G].astype(np.float64),
                                                   kh, vh, tau)
    return want


@pytest.mark.gpu
@pytest.mark.parametrize("S", [1, 4])
def test_paged_decode_matches_oracle(dev, S):
    """Paged decode attention over ragged sequences (a one-token sequence, one
    ending on a page's first row, one spanning six pages) against textbook
    attention on the oracle's dequantization of the rows the table maps."""
    B, H_kv, G, d, max_pages = 3, 2, 4, 128, 6
    kc, vc, sk, sv, k, v, Kc, Vc, Kp, Vp, table = _setup(B, H_kv, d, max_pages, seed=20 + S)
    H_q = G * H_kv
    qn = np.random.default_rng(21).standard_normal((B, H_q, d)).astype(np.float16)
    q = torch.from_numpy(qn).cuda()
    ctx_lens = [1, 129, 768]
    ctx = torch.tensor(ctx_lens, dtype=torch.int32, device="cuda")
    tau = 1 / math.sqrt(d)
    ws = _ws(B, H_q, d, S)
    out = torch.empty((B, H_q, d), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvq.kvq_decode_attn_paged(q, kc, vc, sk, sv, Kp.c(), Vp.c(), ctx, B, H_q, H_kv, 768, tau, S,
                              ws.buf, ws.nbytes, err, out, kvq.OUT_FP32)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    want = _oracle_attend_paged(qn, Kp, Vp, table, sk.cpu().numpy(), sv.cpu().numpy(), ctx_lens,
                                G, tau)
    assert rel_l2(out.cpu().numpy(), want).max() <= REL_L2_TOL


@pytest.mark.gpu
def test_paged_encode_matches_oracle(dev):
    """kvq_encode_kv_paged over tokens 50 .. 349 (three pages, both page
    boundaries crossed): the codes the table maps equal the oracle's codes of
    the same vectors, under the parity rule."""
    B, H_kv, d, max_pages = 2, 3, 128, 4
    kc, vc, sk, sv, k, v, Kc, Vc, Kp, Vp, table = _setup(B, H_kv, d, max_pages, seed=25)
    rng = np.random.default_rng(26)
    kn = rng.standard_normal((B, H_kv, 300, d)).astype(np.float16)
    kn[..., 5] *= 20
    vn = rng.standard_normal((B, H_kv, 300, d)).astype(np.float16)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvq.kvq_encode_kv_paged(kc, sk, torch.from_numpy(kn).cuda(), Kp.c(), vc, sv,
                            torch.from_numpy(vn).cuda(), Vp.c(), B, H_kv, 300, 50, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for P, x, s, c in ((Kp, kn, sk, kc), (Vp, vn, sv, vc)):
        want = O.encode(x, s.cpu().numpy(), c.L, c.norm_mode)
        for b in range(B):
            got = _gather(P, table, b, 50, 350)
            rows = slice(b * H_kv * 300, (b + 1) * H_kv * 300)
            compare_codes((got.angles, got.norms, got.params), want.take(rows))


@pytest.mark.gpu
def test_paged_decode_step_matches_oracle(dev):
    """The fused paged step with appends on a page's first row (ctx 129), its
    last row (ctx 256) and mid-page (ctx 300): the appended rows equal the
    oracle's codes of the new vectors, and the output equals textbook
    attention over the oracle's dequantization of the mapped rows."""
    B, H_kv, G, d, max_pages = 3, 2, 4, 128, 4
    kc, vc, sk, sv, k, v, Kc, Vc, Kp, Vp, table = _setup(B, H_kv, d, max_pages, seed=27)
    H_q = G * H_kv
    rng = np.random.default_rng(28)
    qn = rng.standard_normal((B, H_q, d)).astype(np.float16)
    kn = rng.standard_normal((B, H_kv, d)).astype(np.float16)
    kn[..., 9] *= 20
    vn = rng.standard_normal((B, H_kv, d)).astype(np.float16)
    ctx_lens = [129, 256, 300]
    ctx = torch.tensor(ctx_lens, dtype=torch.int32, device="cuda")
    S, tau = 3, 1 / math.sqrt(d)
    ws = _ws(B, H_q, d, S)
    out = torch.empty((B, H_q, d), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvq.kvq_decode_step_paged(torch.from_numpy(qn).cuda(), torch.from_numpy(kn).cuda(),
                              torch.from_numpy(vn).cuda(), kc, vc, sk, sv, Kp.c(), Vp.c(), ctx,
                              B, H_q, H_kv, 512, tau, S, ws.buf, ws.nbytes, err, out,
                              kvq.OUT_FP32)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for P, x, s, c in ((Kp, kn, sk, kc), (Vp, vn, sv, vc)):
        want = O.encode(x, s.cpu().numpy(), c.L, c.norm_mode)
        for b, n in enumerate(ctx_lens):
            got = _gather(P, table, b, n - 1, n)
            compare_codes((got.angles, got.norms, got.params),
                          want.take(slice(b * H_kv, (b + 1) * H_kv)))
    want = _oracle_attend_paged(qn, Kp, Vp, table, sk.cpu().numpy(), sv.cpu().numpy(), ctx_lens,
                                G, tau)
    assert rel_l2(out.cpu().numpy(), want).max() <= REL_L2_TOL


@pytest.mark.gpu
def test_paged_multi_wave_step_matches_oracle(dev):
    """A paged step of more than one wave of CTAs (3 x 2 x 28 = 168 > 148
    SMs, G 4, 7/6-bit codes): the two-CTAs-per-SM decode after its own append
    launch, the decode waiting for the append only before the tile that holds
    the new row.  Appends on a page's first row, mid-page and the last row of
    the last page; codes and output against the oracle."""
    B, H_kv, G, d, max_pages = 3, 2, 4, 128, 28
    kc, vc, sk, sv, k, v, Kc, Vc, Kp, Vp, table = _setup(B, H_kv, d, max_pages, seed=31)
    H_q = G * H_kv
    rng = np.random.default_rng(32)
    qn = rng.standard_normal((B, H_q, d)).astype(np.float16)
    kn = rng.standard_normal((B, H_kv, d)).astype(np.float16)
    kn[..., 11] *= 20
    vn = rng.standard_normal((B, H_kv, d)).astype(np.float16)
    cap = max_pages * 128
    ctx_lens = [3073, 2000, cap]
    ctx = torch.tensor(ctx_lens, dtype=torch.int32, device="cuda")
    S, tau = 28, 1 / math.sqrt(d)
    ws = _ws(B, H_q, d, S)
    out = torch.empty((B, H_q, d), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvq.kvq_decode_step_paged(torch.from_numpy(qn).cuda(), torch.from_numpy(kn).cuda(),
                              torch.from_numpy(vn).cuda(), kc, vc, sk, sv, Kp.c(), Vp.c(), ctx,
                              B, H_q, H_kv, cap, tau, S, ws.buf, ws.nbytes, err, out,
                              kvq.OUT_FP32)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for P, x, s, c in ((Kp, kn, sk, kc), (Vp, vn, sv, vc)):
        want = O.encode(x, s.cpu().numpy(), c.L, c.norm_mode)
        for b, n in enumerate(ctx_lens):
            got = _gather(P, table, b, n - 1, n)
            compare_codes((got.angles, got.norms, got.params),
                          want.take(slice(b * H_kv, (b + 1) * H_kv)))
    want = _oracle_attend_paged(qn, Kp, Vp, table, sk.cpu().numpy(), sv.cpu().numpy(), ctx_lens,
                                G, tau)
    assert rel_l2(out.cpu().numpy(), want).max() <= REL_L2_TOL
