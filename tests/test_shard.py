"""Context-sharded decode: the cached context of each sequence spread over
several ranks, each decoding its own tokens to split partials
(kvq_decode_attn_partials), the partials exchanged and merged
(kvq_decode_merge_partials).

On the GPU the ranks are emulated one after another on one device (each
"rank" its own planes holding a slice of every sequence, some slices empty):
the merged output must equal textbook attention over the oracle's
dequantization of the whole context, and the single-GPU decode of the whole
cache up to rounding.  On the host, two gloo ranks check the exchange's rank
order, and the new calls' argument checks run without a GPU."""
import ctypes as C
import math
import multiprocessing as mp
import os
import socket
import sys

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle as O
from decode_attention_rand_b200 import kvq, shard

from kvq_testutil import REL_L2_TOL, put_rows, rel_l2

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 0x10000  # 16-byte aligned, never dereferenced


# ------------------------------------------------------------------ host --

def _merge_rc(**kw):
    return kvq.lib().kvq_decode_merge_partials(
        kw.get("parts", FAKE), kw.get("n", 2), kw.get("B", 1), kw.get("H_q", 8),
        kw.get("d", 128), kw.get("S", 4), kw.get("signs", FAKE), kw.get("out", FAKE),
        kw.get("out_dtype", 1), None)


@pytest.mark.parametrize("kw,msg", [
    (dict(n=0), "n_parts"),
    (dict(d=48), "power of two"),
    (dict(d=512), "power of two"),
    (dict(S=0), "num_splits"),
    (dict(n=1000, S=100), "16384"),
    (dict(out_dtype=3), "out_dtype"),
    (dict(parts=None), "NULL"),
    (dict(parts=FAKE + 4), "16-byte"),
])
def test_merge_rejects_bad_arguments(kw, msg):
    assert _merge_rc(**kw) == kvq.KVQ_EINVAL
    assert msg in kvq.kvq_last_error()


def test_partials_checks_as_decode():
    """kvq_decode_attn_partials validates like kvq_decode_attn (no output
    argument); a valid call reaches its launch (here failed on the host)."""
    kc, vc = kvq.codec(128, 128, kvq.KVQ_NORM_LIN8), kvq.codec(128, 64, kvq.KVQ_NORM_LOG4)
    K = kvq.kvq_plane(FAKE, FAKE, FAKE, 256)
    V = kvq.kvq_plane(FAKE, FAKE, FAKE, 256)
    L = kvq.lib()
    ws = kvq.kvq_decode_workspace_bytes(1, 8, 128, 2)

    def call(H_q=8, H_kv=2, ws_bytes=ws):
        return L.kvq_decode_attn_partials(FAKE, C.byref(kc), C.byref(vc), FAKE, FAKE, C.byref(K),
                                          C.byref(V), FAKE, 1, H_q, H_kv, 32, 0.1, 2, FAKE,
                                          ws_bytes, None, None)

    assert call(H_q=6, H_kv=4) == kvq.KVQ_EINVAL
    assert call(ws_bytes=100) == kvq.KVQ_EINVAL and "workspace" in kvq.kvq_last_error()
    kvq.kvq_test_control(kvq.KVQ_TEST_FAIL_LAUNCHES, 1)
    try:
        assert call() == kvq.KVQ_ECUDA
        assert kvq.kvq_last_error().startswith("kvq_decode_attn_partials")
    finally:
        kvq.kvq_test_control(kvq.KVQ_TEST_RESET, 0)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gather_rank(rank, port, out):
    os.environ.update(WORLD_SIZE="2", RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from decode_attention_rand_b200 import shard as sh
    dist.init_process_group("gloo", rank=rank, world_size=2)
    buf = torch.full((48,), 10 * rank + 1, dtype=torch.uint8)
    buf[0] = rank
    got = sh.gather_partials(buf)
    out.put((rank, tuple(got.shape), got[:, 0].tolist(), got[:, 1].tolist()))
    dist.destroy_process_group()


@pytest.mark.skipif(torch.cuda.is_available(), reason="the host (gloo) path of the exchange")
def test_gather_partials_in_rank_order_gloo():
    spawn = mp.get_context("spawn")
    q = spawn.Queue()
    port = _free_port()
    procs = [spawn.Process(target=_gather_rank, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, shape, first, second in got:
        assert shape == (2, 48)
        assert first == [0, 1] and second == [1, 11]


# ------------------------------------------------------------------- GPU --

@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from decode_attention_rand_b200 import build as kbuild
    kbuild.build()
    kvq.lib()
    return torch.device("cuda:0")


def _signs(rng, d):
    return np.where(rng.integers(0, 2, d) == 0, 1, -1).astype(np.int8)


@pytest.mark.gpu
@pytest.mark.parametrize("d,G,LK,LV,N,S", [
    (128, 4, 128, 64, 3, 4),    # the staged kernel, one CTA per SM
    (64, 8, 256, 256, 2, 3),    # staged, one shared table
    (32, 2, 1000, 24, 3, 2),    # the runtime-width kernel
])
def test_context_sharded_decode_matches_oracle(dev, d, G, LK, LV, N, S):
    B, H_kv = 3, 2
    H_q = G * H_kv
    ctx_lens = [700, 129, 300]
    cap = 704
    rng = np.random.default_rng(d + G + N)
    sk, sv = _signs(rng, d), _signs(rng, d)
    skd, svd = torch.from_numpy(sk).cuda(), torch.from_numpy(sv).cuda()
    xk = rng.standard_normal((B, H_kv, cap, d)).astype(np.float16)
    xk[..., 1] *= 20
    xv = rng.standard_normal((B, H_kv, cap, d)).astype(np.float16)
    q = rng.standard_normal((B, H_q, d)).astype(np.float16)
    qd = torch.from_numpy(q).cuda()
    kc, vc = kvq.codec(d, LK, kvq.KVQ_NORM_LIN8), kvq.codec(d, LV, kvq.KVQ_NORM_LOG4)
    kcodes = O.encode(xk, sk, LK, kc.norm_mode)
    vcodes = O.encode(xv, sv, LV, vc.norm_mode)
    tau = 1 / math.sqrt(d)
    # rank r holds tokens [bounds[r][b], bounds[r+1][b]) of sequence b; some
    # ranges are empty (sequence 1 on the last rank)
    cuts = [[0] * B] + [[min(n, (r + 1) * (n // N + 37)) for n in ctx_lens] for r in range(N - 1)]
    cuts.append(list(ctx_lens))
    parts = []
    for r in range(N):
        lo, hi = cuts[r], cuts[r + 1]
        n_loc = [hi[b] - lo[b] for b in range(B)]
        cap_r = max(16, (max(n_loc) + 15) // 16 * 16)
        Kr, Vr = kvq.alloc_plane(kc, B, H_kv, cap_r), kvq.alloc_plane(vc, B, H_kv, cap_r)
        for b in range(B):
            for h in range(H_kv):
                base = (b * H_kv + h) * cap
                if n_loc[b]:
                    put_rows(Kr, kcodes.take(slice(base + lo[b], base + hi[b])), b, h, 0)
                    put_rows(Vr, vcodes.take(slice(base + lo[b], base + hi[b])), b, h, 0)
        ctx_r = torch.tensor(n_loc, dtype=torch.int32, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        ws = shard.decode_attn_partials(qd, kc, vc, skd, svd, Kr, Vr, ctx_r, max(n_loc), S, tau,
                                        err_word=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        parts.append(ws.buf[:ws.nbytes].clone())
    got = shard.merge_partials(torch.stack(parts), B, H_q, d, S, svd).cpu().numpy()
    want = np.zeros((B, H_q, d))
    for b in range(B):
        for h in range(H_kv):
            base = (b * H_kv + h) * cap
            n = ctx_lens[b]
            kh = O.dequant(kcodes.take(slice(base, base + n)), sk)
            vh = O.dequant(vcodes.take(slice(base, base + n)), sv)
            want[b, h * G:(h + 1) * G] = O.attend(q[b, h * G:(h + 1) * G].astype(np.float64),
                                                   kh, vh, tau)
    assert rel_l2(got, want).max() <= REL_L2_TOL
    # the single-GPU decode of the whole cache agrees to rounding
    Kf, Vf = kvq.alloc_plane(kc, B, H_kv, cap), kvq.alloc_plane(vc, B, H_kv, cap)
    for b in range(B):
        for h in range(H_kv):
            sl = slice((b * H_kv + h) * cap, (b * H_kv + h + 1) * cap)
            put_rows(Kf, kcodes.take(sl), b, h, 0)
            put_rows(Vf, vcodes.take(sl), b, h, 0)
    ctx = torch.tensor(ctx_lens, dtype=torch.int32, device="cuda")
    full = kvq.decode_attn(qd, kc, vc, skd, svd, Kf, Vf, ctx, max(ctx_lens), tau,
                           num_splits=S).cpu().numpy()
    assert rel_l2(got, full.astype(np.float64)).max() <= 1e-5


@pytest.mark.gpu
def test_merge_of_empty_parts_is_zero(dev):
    """Every rank holds no token of any sequence: the merged output is 0, as
    for an empty context on one GPU."""
    B, H_q, d, S = 2, 8, 128, 2
    ws = kvq.DecodeWorkspace(B, H_q, d, S)
    kc, vc = kvq.codec(d, 128, kvq.KVQ_NORM_LIN8), kvq.codec(d, 64, kvq.KVQ_NORM_LOG4)
    K, V = kvq.alloc_plane(kc, B, 2, 16), kvq.alloc_plane(vc, B, 2, 16)
    q = torch.randn((B, H_q, d), dtype=torch.float16, device="cuda")
    signs = torch.ones(d, dtype=torch.int8, device="cuda")
    ctx = torch.zeros(B, dtype=torch.int32, device="cuda")
    shard.decode_attn_partials(q, kc, vc, signs, signs, K, V, ctx, 16, S, workspace=ws)
    parts = torch.stack([ws.buf[:ws.nbytes].clone() for _ in range(3)])
    out = shard.merge_partials(parts, B, H_q, d, S, signs)
    torch.cuda.synchronize()
    assert bool((out == 0).all())


@pytest.mark.gpu
def test_bench_shard_case_runs(dev):
    """bench.py's context-sharded case (ranks emulated on this GPU) on the
    Llama-shaped layer split three ways: one JSON line with the whole step's
    and the merge's times and the bytes the merge moves."""
    import json
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--case", "shard_layer",
                        "--workload", "llama7b_layer_b1_hq32_hkv8_d128_ctx4096", "--parts", "3",
                        "--steps", "2"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    assert "3 parts" in res["case"]
    assert res["us_per_launch"] > 0 and res["merge_us"] > 0
    S = int(res["case"].split(" splits")[0].split()[-1])
    assert res["merge_bytes"] == 3 * kvq.kvq_decode_workspace_bytes(1, 32, 128, S) + 32 * 128 * 2
