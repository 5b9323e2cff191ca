"""Host-side checks of libkvq.so that need no GPU: it builds for sm_100a, it
loads, it exports every function include/kvq.h declares, its layout queries
agree with the byte layout, and invalid arguments are rejected before any
CUDA call (no compute call is made here)."""
import ctypes as C
import os

import numpy as np
import pytest

from decode_attention_rand_b200 import build as kbuild
from decode_attention_rand_b200 import kvq

import oracle as O


@pytest.fixture(scope="module", autouse=True)
def built():
    kbuild.build()
    return kvq.lib()


def test_exports_every_declared_function():
    names = kvq.header_functions()
    assert {"kvq_encode", "kvq_dequant", "kvq_decode_attn", "kvq_last_error"} <= set(names)
    L = C.CDLL(kvq.LIB_PATH)
    for n in names:
        assert hasattr(L, n), n
    assert kvq.kvq_version() >= 10000


def test_binding_signatures_match_the_header():
    """Every ctypes signature of the binding has as many parameters as the
    declaration in include/kvq.h (a missing or extra argument would shift
    every later one)."""
    import re
    text = re.sub(r"/\*.*?\*/", "", open(kvq.HEADER).read(), flags=re.S)
    decls = {}
    for m in re.finditer(r"\b(kvq_\w+)\s*\(([^;{]*?)\)\s*;", text):
        params = m.group(2).strip()
        decls[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    assert set(kvq._SIGNATURES) == set(decls)  # every entry point has its ctypes signature
    for name, (_, argtypes) in kvq._SIGNATURES.items():
        assert len(argtypes) == decls[name], name
    assert set(decls) == set(kvq.header_functions())


def test_angle_bits_and_row_bytes_match_layout():
    for L in [2, 3, 4, 5, 7, 8, 100, 128, 129, 255, 256, 4096, 65535, 65536]:
        assert kvq.kvq_angle_bits(L) == O.angle_bits(L)
    assert kvq.kvq_angle_bits(1) < 0 and kvq.kvq_angle_bits(65537) < 0
    for d in [4, 8, 16, 32, 64, 128, 256]:
        for L in [2, 3, 5, 32, 64, 128, 256, 1000, 65536]:
            for mode in (kvq.KVQ_NORM_LIN8, kvq.KVQ_NORM_LOG4):
                c = kvq.codec(d, L, mode)
                for w in range(3):
                    assert kvq.kvq_row_bytes(c, w) == O.row_bytes(d, L, mode, w)
    assert kvq.kvq_row_bytes(kvq.codec(48, 16, 0), 0) < 0
    assert kvq.kvq_row_bytes(kvq.codec(64, 16, 7), 1) < 0


def test_split_heuristic():
    for B, H, ctx, sm in [(1, 8, 4096, 148), (8, 8, 32768, 148), (4, 4, 65536, 148),
                          (1, 2, 256, 148), (1, 1, 1, 148), (64, 8, 100, 148)]:
        s = kvq.kvq_decode_num_splits(B, H, ctx, sm)
        assert 1 <= s <= max(1, (ctx + 127) // 128)
        assert s == kvq.kvq_decode_num_splits(B, H, ctx, sm)
        assert B * H * s <= 8 * sm + B * H
    # the model: waves x (tokens per CTA + 512), minimised, fewer CTAs on ties
    def cost(B, H, ctx, s, sm=148):
        return -(-(B * H * s) // sm) * (-(-ctx // s) + 512)
    for B, H, ctx in [(8, 8, 32768), (4, 4, 65536), (1, 8, 4096), (2, 8, 4096), (16, 8, 8192)]:
        s = kvq.kvq_decode_num_splits(B, H, ctx, 148)
        best = min(cost(B, H, ctx, t) for t in range(1, -(-ctx // 128) + 1)
                   if B * H * t <= 8 * 148 + B * H)
        assert cost(B, H, ctx, s) == best, (B, H, ctx, s)
    # the decode workloads: one wave of 144 CTAs of 228 tokens each for the
    # Llama-shaped layer (16 splits ran 8 % slower), about four waves for the
    # Mistral-shaped one, one wave of 144 for the TinyLlama-shaped one
    assert kvq.kvq_decode_num_splits(1, 8, 4096, 148) == 18
    assert kvq.kvq_decode_num_splits(8, 8, 32768, 148) == 9
    assert kvq.kvq_decode_num_splits(4, 4, 65536, 148) == 9
    assert kvq.kvq_decode_num_splits(0, 8, 100, 148) == 1
    # counters (B*H_q int32, rounded to 16 bytes), (m, l) per split, acc per split
    # (the (m, l) block is rounded to 4 floats so the accumulators stay 16-byte aligned)
    assert kvq.kvq_decode_workspace_bytes(2, 8, 128, 3) == 4 * (16 + 2 * 8 * 3 * 2 + 2 * 8 * 3 * 128)
    assert kvq.kvq_decode_workspace_bytes(1, 3, 64, 1) == 4 * (4 + 8 + 3 * 64)


FAKE = 1 << 20  # 16-byte aligned non-NULL addresses; never dereferenced


def _plane(cap=32, base=FAKE):
    return kvq.kvq_plane(base, base + 4096, base + 8192, cap)


@pytest.mark.parametrize("case", [
    dict(codec=(100, 128, 0), msg="head_dim"),
    dict(codec=(128, 1, 0), msg="L = 1"),
    dict(codec=(128, 70000, 0), msg="L = 70000"),
    dict(codec=(128, 128, 3), msg="norm_mode"),
    dict(plane=kvq.kvq_plane(FAKE + 4, FAKE, FAKE, 32), msg="aligned"),
    dict(plane=kvq.kvq_plane(FAKE, FAKE, FAKE, 40), msg="capacity"),
    dict(plane=kvq.kvq_plane(0, FAKE, FAKE, 32), msg="NULL"),
    dict(T=20, pos0=20, msg="exceed capacity"),
    dict(T=-1, msg="negative"),
    dict(x=FAKE + 2, msg="x must be 16-byte aligned"),
])
def test_encode_rejects_bad_arguments(case):
    c = kvq.codec(*case.get("codec", (128, 128, 0)))
    p = case.get("plane", _plane())
    rc = kvq.lib().kvq_encode(C.byref(c), FAKE, case.get("x", FAKE), 1, 2, case.get("T", 4),
                              case.get("pos0", 0), C.byref(p), None)
    assert rc in (kvq.KVQ_EINVAL, kvq.KVQ_EUNSUPPORTED)
    assert case["msg"] in kvq.kvq_last_error()


@pytest.mark.parametrize("case", [
    dict(vc=(64, 64, 1), msg="head_dim"),
    dict(k=FAKE + 2, msg="k must be 16-byte aligned"),
    dict(v=FAKE + 8, msg="v must be 16-byte aligned"),
    dict(vc=(128, 1, 1), msg="L = 1"),
    dict(T=40, msg="exceed capacity"),
])
def test_encode_kv_rejects_bad_arguments(case):
    kc = kvq.codec(*case.get("kc", (128, 128, 0)))
    vc = kvq.codec(*case.get("vc", (128, 64, 1)))
    K, V = _plane(), _plane(base=FAKE + (1 << 16))
    rc = kvq.lib().kvq_encode_kv(C.byref(kc), FAKE, case.get("k", FAKE), C.byref(K), C.byref(vc),
                                 FAKE, case.get("v", FAKE), C.byref(V), 1, 2, case.get("T", 4), 0,
                                 None)
    assert rc in (kvq.KVQ_EINVAL, kvq.KVQ_EUNSUPPORTED)
    assert case["msg"] in kvq.kvq_last_error()


def test_encode_kv_empty_is_ok_without_gpu():
    kc, vc = kvq.codec(128, 128, 0), kvq.codec(128, 64, 1)
    K, V = _plane(), _plane()
    assert kvq.lib().kvq_encode_kv(C.byref(kc), None, None, C.byref(K), C.byref(vc), None, None,
                                   C.byref(V), 0, 2, 4, 0, None) == 0
    assert kvq.kvq_last_error() == ""


def test_encode_and_dequant_empty_is_ok_without_gpu():
    c = kvq.codec(128, 128, 0)
    p = _plane()
    assert kvq.lib().kvq_encode(C.byref(c), None, None, 0, 2, 4, 0, C.byref(p), None) == 0
    assert kvq.lib().kvq_dequant(C.byref(c), None, C.byref(p), 1, 2, 0, 0, None, None) == 0
    assert kvq.kvq_last_error() == ""


def _decode_rc(**kw):
    kc = kvq.codec(*kw.get("kc", (128, 128, 0)))
    vc = kvq.codec(*kw.get("vc", (128, 64, 1)))
    K, V = kw.get("K", _plane()), kw.get("V", _plane())
    B, H_q, H_kv = kw.get("B", 1), kw.get("H_q", 8), kw.get("H_kv", 2)
    S = kw.get("S", 2)
    ws = kw.get("ws", kvq.kvq_decode_workspace_bytes(B, H_q, kc.head_dim, S))
    return kvq.lib().kvq_decode_attn(FAKE, C.byref(kc), C.byref(vc), FAKE, FAKE, C.byref(K),
                                     C.byref(V), FAKE, B, H_q, H_kv, kw.get("max_ctx", 32),
                                     kw.get("scale", 0.1), S, kw.get("wsp", FAKE), ws, None,
                                     FAKE, kw.get("out_dtype", 0), None)


@pytest.mark.parametrize("kw,status,msg", [
    (dict(H_q=6, H_kv=4), kvq.KVQ_EINVAL, "multiple"),
    (dict(vc=(64, 64, 1)), kvq.KVQ_EINVAL, "head_dim differ"),
    (dict(V=_plane(48)), kvq.KVQ_EINVAL, "capacity differ"),
    (dict(S=0), kvq.KVQ_EINVAL, "num_splits"),
    (dict(ws=100), kvq.KVQ_EINVAL, "workspace"),
    (dict(wsp=FAKE + 8), kvq.KVQ_EINVAL, "workspace not 16-byte"),
    (dict(out_dtype=3), kvq.KVQ_EINVAL, "out_dtype"),
    (dict(scale=float("nan")), kvq.KVQ_EINVAL, "softmax_scale"),
    (dict(max_ctx=-1), kvq.KVQ_EINVAL, "negative"),
    (dict(max_ctx=1 << 31, S=1), kvq.KVQ_EINVAL, "exceeds 2^30"),
])
def test_decode_rejects_bad_arguments(kw, status, msg):
    assert _decode_rc(**kw) == status
    assert msg in kvq.kvq_last_error()


@pytest.mark.parametrize("kw", [
    dict(H_q=32, H_kv=2),                          # G 16
    dict(H_q=6, H_kv=2),                           # G 3
    dict(kc=(4, 2, 0), vc=(4, 3, 1)),              # the smallest head
    dict(kc=(32, 128, 0), vc=(32, 64, 1)),
    dict(kc=(256, 65536, 1), vc=(256, 5000, 0)),   # log K norms, linear V norms
    dict(kc=(128, 512, 0)),
])
def test_decode_accepts_every_codec(kw):
    """Decode takes every codec encode takes (head_dim 4..256, any G, L up to
    65536, either norm mode for K and V): the arguments pass every check and
    the call reaches its launch (here made to fail on the host, so nothing
    runs)."""
    kvq.kvq_test_control(kvq.KVQ_TEST_FAIL_LAUNCHES, 1)
    try:
        assert _decode_rc(**kw) == kvq.KVQ_ECUDA
        assert "injected" in kvq.kvq_last_error()
    finally:
        kvq.kvq_test_control(kvq.KVQ_TEST_RESET, 0)


@pytest.mark.parametrize("k,v,msg", [
    (None, FAKE, "NULL k_new"),
    (FAKE + 8, FAKE, "16-byte aligned"),
    (FAKE, FAKE + 4, "16-byte aligned"),
])
def test_decode_step_rejects_bad_new_tokens(k, v, msg):
    kc, vc = kvq.codec(128, 128, 0), kvq.codec(128, 64, 1)
    K, V = _plane(), _plane()
    ws = kvq.kvq_decode_workspace_bytes(1, 8, 128, 2)
    rc = kvq.lib().kvq_decode_step(FAKE, k, v, C.byref(kc), C.byref(vc), FAKE, FAKE, C.byref(K),
                                   C.byref(V), FAKE, 1, 8, 2, 32, 0.1, 2, FAKE, ws, None, FAKE, 0,
                                   None)
    assert rc == kvq.KVQ_EINVAL
    assert msg in kvq.kvq_last_error()


def test_decode_step_shares_the_decode_checks():
    kc, vc = kvq.codec(128, 128, 0), kvq.codec(64, 64, 1)
    K, V = _plane(), _plane()
    rc = kvq.lib().kvq_decode_step(FAKE, FAKE, FAKE, C.byref(kc), C.byref(vc), FAKE, FAKE,
                                   C.byref(K), C.byref(V), FAKE, 1, 8, 2, 32, 0.1, 2, FAKE, 1 << 20,
                                   None, FAKE, 0, None)
    assert rc == kvq.KVQ_EINVAL
    assert "kvq_decode_step: K and V head_dim differ" in kvq.kvq_last_error()


@pytest.mark.parametrize("bufs,msg", [
    ((None, FAKE, FAKE, FAKE), "NULL host buffer"),
    ((FAKE, FAKE, None, FAKE), "NULL host buffer"),
    ((FAKE, None, FAKE, FAKE), "both device buffers or neither"),
    ((FAKE, FAKE + 8, FAKE, FAKE), "16-byte aligned"),
    ((FAKE, FAKE, FAKE, FAKE + 4), "16-byte aligned"),
])
def test_decode_step_host_rejects_bad_buffers(bufs, msg):
    kc, vc = kvq.codec(128, 128, 0), kvq.codec(128, 64, 1)
    K, V = _plane(), _plane()
    ws = kvq.kvq_decode_workspace_bytes(1, 8, 128, 2)
    rc = kvq.lib().kvq_decode_step_host(*bufs, C.byref(kc), C.byref(vc), FAKE, FAKE, C.byref(K),
                                        C.byref(V), FAKE, 1, 8, 2, 32, 0.1, 2, FAKE, ws, None, 0,
                                        None)
    assert rc == kvq.KVQ_EINVAL
    assert msg in kvq.kvq_last_error()


def test_decode_step_host_without_device_buffers_needs_mapped_memory():
    # FAKE is no page-locked allocation: refused before any launch
    kc, vc = kvq.codec(128, 128, 0), kvq.codec(128, 64, 1)
    K, V = _plane(), _plane()
    ws = kvq.kvq_decode_workspace_bytes(1, 8, 128, 2)
    rc = kvq.lib().kvq_decode_step_host(FAKE, None, FAKE, None, C.byref(kc), C.byref(vc), FAKE,
                                        FAKE, C.byref(K), C.byref(V), FAKE, 1, 8, 2, 32, 0.1, 2,
                                        FAKE, ws, None, 0, None)
    assert rc == kvq.KVQ_EINVAL
    assert "page-locked" in kvq.kvq_last_error()


def test_decode_step_host_checks_before_copying():
    # an argument error is reported before any copy or launch (no GPU here)
    kc, vc = kvq.codec(128, 128, 0), kvq.codec(64, 64, 1)
    K, V = _plane(), _plane()
    rc = kvq.lib().kvq_decode_step_host(FAKE, FAKE, FAKE, FAKE, C.byref(kc), C.byref(vc), FAKE,
                                        FAKE, C.byref(K), C.byref(V), FAKE, 1, 8, 2, 32, 0.1, 2,
                                        FAKE, 1 << 20, None, 0, None)
    assert rc == kvq.KVQ_EINVAL
    assert "kvq_decode_step_host: K and V head_dim differ" in kvq.kvq_last_error()


def test_error_state_is_per_thread():
    import threading
    c = kvq.codec(128, 1, 0)
    p = _plane()
    kvq.lib().kvq_encode(C.byref(c), FAKE, FAKE, 1, 1, 1, 0, C.byref(p), None)
    seen = {}

    def other():
        seen["msg"] = kvq.kvq_last_error()

    t = threading.Thread(target=other)
    t.start()
    t.join()
    assert seen["msg"] == "" and "L = 1" in kvq.kvq_last_error()


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(kvq, "LIB_PATH", str(tmp_path / "nope.so"))
    monkeypatch.setattr(kvq, "_lib", None)
    with pytest.raises(kvq.KvqError):
        kvq.lib()
