"""The decode loop as a serving system runs it: several layers and several
generated tokens of kvq_decode_step captured in one CUDA graph, every launch a
programmatic dependent of the one before it (the library sets that up), one
cache per layer growing by one token per step.

A step's kernel may start its setup while the previous one still runs, and
reads the row the previous step appended.  An ordering mistake in that chain
would show here and in no eager, one-call-at-a-time test.  Every appended row
is compared with the oracle's codes of the same vector, and every step's
output with textbook attention over the oracle's dequantization of the rows
the GPU holds after the replay (rows below each step's length never change
after that step)."""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle as O
from decode_attention_rand_b200 import build as kbuild
from decode_attention_rand_b200 import kvq

from kvq_testutil import REL_L2_TOL, compare_codes, paged_rows, plane_rows, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    kbuild.build()
    kvq.lib()
    return torch.device("cuda:0")


def _signs(rng, d):
    return np.where(rng.integers(0, 2, d) == 0, 1, -1).astype(np.int8)


@pytest.mark.parametrize("splits,base", [(3, 300), (16, 4090), (40, 4090), (2, 1500)])
def test_graph_of_chained_steps_matches_oracle(dev, splits, base):
    """3 layers x 4 steps, B 2, 2 KV heads, G 4, d 128; the first case
    splits 300..303 tokens three ways (last-CTA combine), the second takes
    16 splits (one cluster per KV head) over 4090..4093 tokens, the third 40
    splits (160 CTAs, more than one wave), all three with 128-token tiles
    (splits of at most 256 tokens); the fourth two splits of about 750
    tokens (256-token tiles for layers 1 and 2, 128-token tiles for layer
    0's 8-bit codes)."""
    layers, steps, B, H_kv, G, d = 3, 4, 2, 2, 4, 128
    H_q = G * H_kv
    cap = (base + steps + 15) // 16 * 16
    rng = np.random.default_rng(splits)
    tau = 1 / math.sqrt(d)
    kcs = [kvq.codec(d, (256, 128, 128)[l], kvq.KVQ_NORM_LIN8) for l in range(layers)]
    vcs = [kvq.codec(d, (256, 64, 32)[l], kvq.KVQ_NORM_LOG4) for l in range(layers)]
    sk = [_signs(rng, d) for _ in range(layers)]
    sv = [_signs(rng, d) for _ in range(layers)]
    skd = [torch.from_numpy(s).cuda() for s in sk]
    svd = [torch.from_numpy(s).cuda() for s in sv]
    planes = []
    for l in range(layers):
        k = rng.standard_normal((B, H_kv, cap, d)).astype(np.float16)
        k[..., 3] *= 20
        v = rng.standard_normal((B, H_kv, cap, d)).astype(np.float16)
        K, V = kvq.alloc_plane(kcs[l], B, H_kv, cap), kvq.alloc_plane(vcs[l], B, H_kv, cap)
        # tokens 0 .. base-2 are cached; the steps append base-1 .. base+steps-2
        kvq.encode(kcs[l], skd[l], torch.from_numpy(k[:, :, :base - 1].copy()).cuda(), K, 0)
        kvq.encode(vcs[l], svd[l], torch.from_numpy(v[:, :, :base - 1].copy()).cuda(), V, 0)
        planes.append((K, V))
    q = rng.standard_normal((steps, layers, B, H_q, d)).astype(np.float16)
    kn = rng.standard_normal((steps, layers, B, H_kv, d)).astype(np.float16)
    kn[..., 7] *= 20
    vn = rng.standard_normal((steps, layers, B, H_kv, d)).astype(np.float16)
    qd, knd, vnd = (torch.from_numpy(a).cuda() for a in (q, kn, vn))
    ctx = [torch.full((B,), base + s, dtype=torch.int32, device="cuda") for s in range(steps)]
    out = torch.zeros((steps, layers, B, H_q, d), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = kvq.DecodeWorkspace(B, H_q, d, splits)
    calls = [[kvq.DecodeStepCall(qd[s, l], knd[s, l], vnd[s, l], kcs[l], vcs[l], skd[l], svd[l],
                                 planes[l][0].c(), planes[l][1].c(), ctx[s], B, H_q, H_kv,
                                 base + steps, tau, splits, ws.buf, ws.nbytes, err, out[s, l],
                                 kvq.OUT_FP32)
              for l in range(layers)] for s in range(steps)]
    torch.cuda.synchronize()
    stream = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for s in range(steps):
            for l in range(layers):
                calls[s][l](torch.cuda.current_stream())
    g.replay()
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    got = out.cpu().numpy()
    for l in range(layers):
        K, V = planes[l]
        kc, vc = kcs[l], vcs[l]
        # appended rows: position base-1+s holds step s's new token
        for P, x, s_, c in ((K, kn, sk[l], kc), (V, vn, sv[l], vc)):
            rows = plane_rows(P, t_range=(base - 1, base - 1 + steps))  # (b, h, t) order
            want = O.encode(np.ascontiguousarray(x[:, l].transpose(1, 2, 0, 3)), s_, c.L,
                            c.norm_mode)
            compare_codes(rows, want)
        kcodes = O.Codes(d, kc.L, kc.norm_mode, *plane_rows(K, t_range=(0, base + steps - 1)))
        vcodes = O.Codes(d, vc.L, vc.norm_mode, *plane_rows(V, t_range=(0, base + steps - 1)))
        n_all = base + steps - 1
        for s in range(steps):
            n = base + s
            want = np.zeros((B, H_q, d))
            for b in range(B):
                for h in range(H_kv):
                    r0 = (b * H_kv + h) * n_all
                    kh = O.dequant(kcodes.take(slice(r0, r0 + n)), sk[l])
                    vh = O.dequant(vcodes.take(slice(r0, r0 + n)), sv[l])
                    want[b, h * G:(h + 1) * G] = O.attend(
                        q[s, l, b, h * G:(h + 1) * G].astype(np.float64), kh, vh, tau)
            assert rel_l2(got[s, l], want).max() <= REL_L2_TOL, (l, s)
    # a second replay appends the same rows again and returns the same outputs
    first = out.clone()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, first)
    del g


def test_graph_of_chained_paged_steps_matches_oracle(dev):
    """The same chain on paged caches with more than one wave of CTAs (3 x 2 x
    28 = 168): each layer's step is an append launch followed by the
    two-CTAs-per-SM decode as its programmatic dependent, which starts before
    the append ends and waits for it only before the tile holding the new
    row.  2 layers x 3 steps, ragged lengths, shuffled page tables; appended
    rows and outputs against the oracle."""
    layers, steps, B, H_kv, G, d, pt, max_pages, S = 2, 3, 3, 2, 4, 128, 128, 28, 28
    H_q, cap = G * H_kv, max_pages * 128
    base = [3000, 1500, cap - steps + 1]
    rng = np.random.default_rng(77)
    tau = 1 / math.sqrt(d)
    kcs = [kvq.codec(d, 128, kvq.KVQ_NORM_LIN8) for _ in range(layers)]
    vcs = [kvq.codec(d, (64, 32)[l], kvq.KVQ_NORM_LOG4) for l in range(layers)]
    sk = [_signs(rng, d) for _ in range(layers)]
    sv = [_signs(rng, d) for _ in range(layers)]
    skd = [torch.from_numpy(x).cuda() for x in sk]
    svd = [torch.from_numpy(x).cuda() for x in sv]
    num_pages = B * max_pages + 2
    planes, tables = [], []
    for l in range(layers):
        table = rng.permutation(num_pages)[:B * max_pages].reshape(B, max_pages)
        Kp = kvq.alloc_paged_plane(kcs[l], H_kv, pt, num_pages, table)
        Vp = kvq.alloc_paged_plane(vcs[l], H_kv, pt, num_pages, table)
        # every position but the ones the steps append holds an encoded vector
        T0 = max(base) - 1
        k = rng.standard_normal((B, H_kv, T0, d)).astype(np.float16)
        k[..., 3] *= 20
        v = rng.standard_normal((B, H_kv, T0, d)).astype(np.float16)
        kvq.kvq_encode_kv_paged(kcs[l], skd[l], torch.from_numpy(k).cuda(), Kp.c(), vcs[l],
                                svd[l], torch.from_numpy(v).cuda(), Vp.c(), B, H_kv, T0, 0)
        planes.append((Kp, Vp))
        tables.append(table)
    q = rng.standard_normal((steps, layers, B, H_q, d)).astype(np.float16)
    kn = rng.standard_normal((steps, layers, B, H_kv, d)).astype(np.float16)
    kn[..., 7] *= 20
    vn = rng.standard_normal((steps, layers, B, H_kv, d)).astype(np.float16)
    qd, knd, vnd = (torch.from_numpy(a).cuda() for a in (q, kn, vn))
    ctx = [torch.tensor([n + s for n in base], dtype=torch.int32, device="cuda")
           for s in range(steps)]
    out = torch.zeros((steps, layers, B, H_q, d), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = kvq.DecodeWorkspace(B, H_q, d, S)
    pc = [(P[0].c(), P[1].c()) for P in planes]
    torch.cuda.synchronize()
    stream = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for s in range(steps):
            for l in range(layers):
                kvq.kvq_decode_step_paged(qd[s, l], knd[s, l], vnd[s, l], kcs[l], vcs[l], skd[l],
                                          svd[l], pc[l][0], pc[l][1], ctx[s], B, H_q, H_kv, cap,
                                          tau, S, ws.buf, ws.nbytes, err, out[s, l],
                                          kvq.OUT_FP32, torch.cuda.current_stream())
    g.replay()
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    got = out.cpu().numpy()
    for l in range(layers):
        Kp, Vp = planes[l]
        kc, vc = kcs[l], vcs[l]
        for b in range(B):
            n_all = base[b] + steps - 1
            for P, x, s_, c in ((Kp, kn, sk[l], kc), (Vp, vn, sv[l], vc)):
                rows = paged_rows(P, tables[l], b, base[b] - 1, n_all)  # (h, t) order
                want = O.encode(np.ascontiguousarray(x[:, l, b].transpose(1, 0, 2)), s_, c.L,
                                c.norm_mode)
                compare_codes(rows, want)
            kcodes = O.Codes(d, kc.L, kc.norm_mode, *paged_rows(Kp, tables[l], b, 0, n_all))
            vcodes = O.Codes(d, vc.L, vc.norm_mode, *paged_rows(Vp, tables[l], b, 0, n_all))
            for s in range(steps):
                n = base[b] + s
                want = np.zeros((H_q, d))
                for h in range(H_kv):
                    kh = O.dequant(kcodes.take(slice(h * n_all, h * n_all + n)), sk[l])
                    vh = O.dequant(vcodes.take(slice(h * n_all, h * n_all + n)), sv[l])
                    want[h * G:(h + 1) * G] = O.attend(
                        q[s, l, b, h * G:(h + 1) * G].astype(np.float64), kh, vh, tau)
                assert rel_l2(got[s, l, b], want).max() <= REL_L2_TOL, (l, b, s)
    del g
