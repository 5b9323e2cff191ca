"""Failure detection without a GPU fault.

Two kinds of failure are made on purpose, neither of which can fault, trap or
hang a GPU:
  - a launch failure injected on the host (kvq_test_control with
    KVQ_TEST_FAIL_LAUNCHES): the call must return KVQ_ECUDA with a message,
    queue nothing, and leave the library usable;
  - a device wait that gives up (KVQ_TEST_WAIT_LIMIT 0: every tile wait of the
    decode kernel fails at once, while the copies already issued are still
    drained with the normal limit): the kernel must set KVQ_DEVERR_TIMEOUT,
    write a finite output, and the next launch must be correct again.
The CPU tests run the argument checks with fake, aligned, never dereferenced
pointers; the injected failure is reported before anything touches the GPU.
"""
import ctypes as C
import math

import numpy as np
import pytest

from decode_attention_rand_b200 import kvq

FAKE = 1 << 20  # aligned, never dereferenced


@pytest.fixture
def controls():
    kvq.lib()
    yield
    kvq.kvq_test_control(kvq.KVQ_TEST_RESET, 0)


def test_control_rejects_unknown_key_and_negative_value(controls):
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_test_control(99, 1)
    assert e.value.status == kvq.KVQ_EINVAL and "unknown key" in str(e.value)
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_test_control(kvq.KVQ_TEST_WAIT_LIMIT, -1)
    assert e.value.status == kvq.KVQ_EINVAL


def _fake_plane():
    return kvq.kvq_plane(FAKE, FAKE, FAKE, 256)


def test_injected_launch_failure_maps_to_ecuda(controls):
    """Each call that would launch a kernel consumes one injected failure and
    returns KVQ_ECUDA; argument errors are still reported first, without
    consuming one."""
    L = kvq.lib()
    kc, vc = kvq.codec(128, 128, kvq.KVQ_NORM_LIN8), kvq.codec(128, 64, kvq.KVQ_NORM_LOG4)
    K, V = _fake_plane(), _fake_plane()
    kvq.kvq_test_control(kvq.KVQ_TEST_FAIL_LAUNCHES, 4)
    # an argument error comes first and does not consume the injection
    rc = L.kvq_encode(C.byref(kc), FAKE, FAKE, 1, 2, 10, 250, C.byref(K), None)
    assert rc == kvq.KVQ_EINVAL and "exceed capacity" in kvq.kvq_last_error()
    calls = [
        ("kvq_encode", lambda: L.kvq_encode(C.byref(kc), FAKE, FAKE, 1, 2, 10, 0, C.byref(K),
                                            None)),
        ("kvq_encode_kv", lambda: L.kvq_encode_kv(C.byref(kc), FAKE, FAKE, C.byref(K),
                                                  C.byref(vc), FAKE, FAKE, C.byref(V), 1, 2, 1,
                                                  5, None)),
        ("kvq_dequant", lambda: L.kvq_dequant(C.byref(kc), FAKE, C.byref(K), 1, 2, 10, 0, FAKE,
                                              None)),
        ("kvq_decode_attn", lambda: L.kvq_decode_attn(
            FAKE, C.byref(kc), C.byref(vc), FAKE, FAKE, C.byref(K), C.byref(V), FAKE, 1, 8, 2,
            256, 0.1, 2, FAKE, kvq.kvq_decode_workspace_bytes(1, 8, 128, 2), None, FAKE, 0,
            None)),
    ]
    for name, call in calls:
        assert call() == kvq.KVQ_ECUDA, name
        msg = kvq.kvq_last_error()
        assert msg.startswith(name) and "injected" in msg, msg
    # all four consumed: a reset leaves nothing pending
    kvq.kvq_test_control(kvq.KVQ_TEST_RESET, 0)
    rc = L.kvq_encode(C.byref(kc), FAKE, FAKE, 1, 2, 10, 250, C.byref(K), None)
    assert rc == kvq.KVQ_EINVAL


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


def _layer(B=1, H_kv=8, G=4, d=128, ctx=4096, seed=0):
    rng = np.random.default_rng(seed)
    kc, vc = kvq.codec(d, 128, kvq.KVQ_NORM_LIN8), kvq.codec(d, 64, kvq.KVQ_NORM_LOG4)
    sk = torch.from_numpy(np.where(rng.integers(0, 2, d) == 0, 1, -1).astype(np.int8)).cuda()
    sv = torch.from_numpy(np.where(rng.integers(0, 2, d) == 0, 1, -1).astype(np.int8)).cuda()
    Kp, Vp = kvq.alloc_plane(kc, B, H_kv, ctx), kvq.alloc_plane(vc, B, H_kv, ctx)
    k = torch.from_numpy(rng.standard_normal((B, H_kv, ctx, d)).astype(np.float16)).cuda()
    v = torch.from_numpy(rng.standard_normal((B, H_kv, ctx, d)).astype(np.float16)).cuda()
    kvq.encode(kc, sk, k, Kp, 0)
    kvq.encode(vc, sv, v, Vp, 0)
    q = torch.from_numpy(rng.standard_normal((B, G * H_kv, d)).astype(np.float16)).cuda()
    ctx_t = torch.full((B,), ctx, dtype=torch.int32, device="cuda")
    return kc, vc, sk, sv, Kp, Vp, q, ctx_t


@pytest.mark.gpu
@pytest.mark.parametrize("splits", [8, 20])  # one cluster per KV head / last-CTA combine
def test_decode_wait_timeout_is_reported(dev, controls, splits):
    kc, vc, sk, sv, Kp, Vp, q, ctx = _layer()
    ref = kvq.decode_attn(q, kc, vc, sk, sv, Kp, Vp, ctx, 4096, num_splits=splits)
    kvq.kvq_test_control(kvq.KVQ_TEST_WAIT_LIMIT, 0)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = kvq.decode_attn(q, kc, vc, sk, sv, Kp, Vp, ctx, 4096, num_splits=splits, err_word=err)
    torch.cuda.synchronize()
    assert int(err.item()) & kvq.KVQ_DEVERR_TIMEOUT
    assert torch.isfinite(out).all()
    # every CTA gave up: nothing was accumulated
    assert bool((out == 0).all())
    # the limit restored, the same launch is correct again (the context survived)
    kvq.kvq_test_control(kvq.KVQ_TEST_RESET, 0)
    err.zero_()
    again = kvq.decode_attn(q, kc, vc, sk, sv, Kp, Vp, ctx, 4096, num_splits=splits,
                            err_word=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(again, ref)


@pytest.mark.gpu
def test_decode_step_wait_timeout_still_appends(dev, controls):
    """The fused step writes the new token before its tile loop: with every
    tile wait failing, the row is still written (the same bytes as a normal
    step) and the timeout reported."""
    kc, vc, sk, sv, Kp, Vp, q, ctx = _layer(B=2, H_kv=2, ctx=512, seed=3)
    K2, V2 = (kvq.alloc_plane(c, 2, 2, 512) for c in (kc, vc))
    for A, Bp in ((K2, Kp), (V2, Vp)):
        for w in range(3):
            Bp.rows(w)[:, :, 511] = 0x5A
            A.rows(w).copy_(Bp.rows(w))
    k_new = torch.randn((2, 2, 128), dtype=torch.float16, device="cuda")
    v_new = torch.randn((2, 2, 128), dtype=torch.float16, device="cuda")
    kvq.kvq_test_control(kvq.KVQ_TEST_WAIT_LIMIT, 0)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = kvq.decode_step(q, k_new, v_new, kc, vc, sk, sv, Kp, Vp, ctx, 512, num_splits=3,
                          err_word=err)
    torch.cuda.synchronize()
    assert int(err.item()) & kvq.KVQ_DEVERR_TIMEOUT
    assert torch.isfinite(out).all()
    kvq.kvq_test_control(kvq.KVQ_TEST_RESET, 0)
    kvq.decode_step(q, k_new, v_new, kc, vc, sk, sv, K2, V2, ctx, 512, num_splits=3)
    torch.cuda.synchronize()
    for A, Bp in ((K2, Kp), (V2, Vp)):
        for w in range(3):
            assert torch.equal(A.rows(w), Bp.rows(w))


@pytest.mark.gpu
def test_injected_failure_queues_nothing_and_library_recovers(dev, controls):
    kc, vc, sk, sv, Kp, Vp, q, ctx = _layer(B=1, H_kv=2, ctx=256, seed=5)
    ref = kvq.decode_attn(q, kc, vc, sk, sv, Kp, Vp, ctx, 256, num_splits=2)
    out = torch.full_like(ref, 7.0)
    kvq.kvq_test_control(kvq.KVQ_TEST_FAIL_LAUNCHES, 1)
    with pytest.raises(kvq.KvqError) as e:
        kvq.decode_attn(q, kc, vc, sk, sv, Kp, Vp, ctx, 256, num_splits=2, out=out)
    assert e.value.status == kvq.KVQ_ECUDA
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())  # nothing ran
    kvq.decode_attn(q, kc, vc, sk, sv, Kp, Vp, ctx, 256, num_splits=2, out=out)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    assert math.isfinite(float(out.abs().max()))


def test_profile_ranges_do_not_change_results_on_host():
    """KVQ_PROFILE brackets each call's launches with an NVTX range; a call
    made with it set (in a fresh process, where it is read) returns what it
    returns without it (here: the argument errors and the launch outcome on a
    machine without a GPU are unchanged)."""
    import subprocess
    import sys
    code = (
        "import ctypes as C; from decode_attention_rand_b200 import kvq\n"
        "kc, vc = kvq.codec(128, 128, 0), kvq.codec(128, 64, 1)\n"
        f"K = kvq.kvq_plane({FAKE}, {FAKE}, {FAKE}, 256)\n"
        f"rc = kvq.lib().kvq_encode(C.byref(kc), {FAKE}, {FAKE}, 1, 2, 10, 250, C.byref(K), None)\n"
        "print(rc, kvq.kvq_last_error())\n"
    )
    outs = []
    for env in ({"KVQ_PROFILE": "1"}, {"KVQ_PROFILE": "0"}):
        import os
        r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                           env={**os.environ, **env}, timeout=300,
                           cwd=os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
        assert r.returncode == 0, r.stderr[-2000:]
        outs.append(r.stdout.strip())
    assert outs[0] == outs[1] and outs[0].startswith(str(kvq.KVQ_EINVAL))


@pytest.mark.gpu
def test_debug_checks_report_corrupted_rows(dev, controls):
    """With the KVQ_DEBUG checks on, a clean cache reports nothing; a NaN
    parameter (the streaming encoder's in-doubt marker, never left in a
    finished cache) or an angle code >= L (L = 100 leaves codes 100..127
    unused) sets KVQ_DEVERR_BAD_CODE; a decode step does not check the row it
    is about to append."""
    d, B, H_kv, G, n = 128, 2, 2, 4, 300
    rng = np.random.default_rng(41)
    kc, vc = kvq.codec(d, 100, kvq.KVQ_NORM_LIN8), kvq.codec(d, 64, kvq.KVQ_NORM_LOG4)
    sk = torch.from_numpy(np.where(rng.integers(0, 2, d) == 0, 1, -1).astype(np.int8)).cuda()
    sv = torch.from_numpy(np.where(rng.integers(0, 2, d) == 0, 1, -1).astype(np.int8)).cuda()
    K, V = kvq.alloc_plane(kc, B, H_kv, 320), kvq.alloc_plane(vc, B, H_kv, 320)
    kvq.encode(kc, sk, torch.from_numpy(rng.standard_normal((B, H_kv, 320, d)).astype(np.float16)).cuda(), K, 0)
    kvq.encode(vc, sv, torch.from_numpy(rng.standard_normal((B, H_kv, 320, d)).astype(np.float16)).cuda(), V, 0)
    q = torch.from_numpy(rng.standard_normal((B, G * H_kv, d)).astype(np.float16)).cuda()
    ctx = torch.full((B,), n, dtype=torch.int32, device="cuda")
    kvq.kvq_test_control(kvq.KVQ_TEST_DEBUG_CHECKS, 1)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")

    def run():
        err.zero_()
        kvq.decode_attn(q, kc, vc, sk, sv, K, V, ctx, n, num_splits=2, err_word=err)
        torch.cuda.synchronize()
        return int(err.item())
    assert run() == 0
    V.rows(2)[1, 1, 17] = torch.tensor([0x00, 0x7E, 0x00, 0x3C], dtype=torch.uint8)  # LO = NaN
    assert run() & kvq.KVQ_DEVERR_BAD_CODE
    kvq.encode(vc, sv, torch.from_numpy(rng.standard_normal((B, H_kv, 320, d)).astype(np.float16)).cuda(), V, 0)
    assert run() == 0
    K.rows(0)[0, 0, 5, 0] = 0x7F  # pair 0's 7-bit code = 127 >= L
    assert run() & kvq.KVQ_DEVERR_BAD_CODE
    # rows past the context are not looked at
    kvq.encode(kc, sk, torch.from_numpy(rng.standard_normal((B, H_kv, 320, d)).astype(np.float16)).cuda(), K, 0)
    K.rows(2)[:, :, n:] = 0xFF  # NaN M beyond ctx
    assert run() == 0
    # the row a step appends holds garbage until the step writes it
    K.rows(2)[:, :, n - 1] = 0xFF
    err.zero_()
    kvq.decode_step(q, q[:, :H_kv].contiguous(), q[:, :H_kv].contiguous(), kc, vc, sk, sv, K, V,
                    ctx, n, num_splits=2, err_word=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    kvq.kvq_test_control(kvq.KVQ_TEST_DEBUG_CHECKS, 0)
    K.rows(2)[0, 0, 3] = 0xFF
    assert run() == 0  # checks off: not looked at
