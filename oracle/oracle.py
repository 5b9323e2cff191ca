"""ctypes wrapper of the fp64 oracle (test infrastructure only).

Every function here is argument marshalling around ``kvq_oracle.c`` plus a
thread pool over independent vectors or heads; all arithmetic is in the C file.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np

MODE_LIN8 = 0
MODE_LOG4 = 1
MODE_EXACT = 2  # oracle only: norms stored as fp64 (used by the round-trip pins)

FLAG_ANGLE = 1
FLAG_NORM = 2
FLAG_PARAM = 4

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvq_oracle.c")
_LIB = os.path.join(_HERE, "libkvq_oracle.so")
_lock = threading.Lock()
_lib = None

_u8p = C.POINTER(C.c_uint8)
_i8p = C.POINTER(C.c_int8)
_u16p = C.POINTER(C.c_uint16)
_i32p = C.POINTER(C.c_int32)
_f64p = C.POINTER(C.c_double)


def build(force: bool = False) -> str:
    """Compile kvq_oracle.c into libkvq_oracle.so (plain gcc, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
             "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    """The loaded oracle library.  KVQ_ORACLE_LIB may name another build of
    kvq_oracle.c (the mutation tests load deliberately broken copies)."""
    global _lib
    with _lock:
        if _lib is None:
            path = os.environ.get("KVQ_ORACLE_LIB") or build()
            L = C.CDLL(path)
            L.kvq_oracle_angle_bits.restype = C.c_int
            L.kvq_oracle_angle_bits.argtypes = [C.c_int]
            L.kvq_oracle_row_bytes.restype = C.c_long
            L.kvq_oracle_row_bytes.argtypes = [C.c_int, C.c_int, C.c_int, C.c_int]
            L.kvq_oracle_double_to_half.restype = C.c_uint16
            L.kvq_oracle_double_to_half.argtypes = [C.c_double]
            L.kvq_oracle_half_to_double.restype = C.c_double
            L.kvq_oracle_half_to_double.argtypes = [C.c_uint16]
            L.kvq_oracle_rotate.restype = None
            L.kvq_oracle_rotate.argtypes = [_f64p, _i8p, C.c_int, C.c_int, _f64p]
            L.kvq_oracle_unrotate.restype = None
            L.kvq_oracle_unrotate.argtypes = [_f64p, _i8p, C.c_int, _f64p]
            L.kvq_oracle_encode_batch.restype = C.c_int
            L.kvq_oracle_encode_batch.argtypes = [_u16p, C.c_long, _i8p, C.c_int, C.c_int,
                                                  C.c_int, _u8p, _u8p, _u8p, _u8p]
            L.kvq_oracle_unpack.restype = C.c_int
            L.kvq_oracle_unpack.argtypes = [_u8p, _u8p, _u8p, C.c_int, C.c_int, C.c_int,
                                            _i32p, _i32p, _f64p]
            L.kvq_oracle_theta_hat.restype = C.c_double
            L.kvq_oracle_theta_hat.argtypes = [C.c_int, C.c_int]
            L.kvq_oracle_dequant_rotated.restype = C.c_int
            L.kvq_oracle_dequant_rotated.argtypes = [_u8p, _u8p, _u8p, C.c_int, C.c_int,
                                                     C.c_int, _f64p]
            L.kvq_oracle_dequant_batch.restype = C.c_int
            L.kvq_oracle_dequant_batch.argtypes = [_u8p, _u8p, _u8p, C.c_long, _i8p, C.c_int,
                                                   C.c_int, C.c_int, _f64p]
            L.kvq_oracle_attend.restype = None
            L.kvq_oracle_attend.argtypes = [_f64p, _f64p, _f64p, C.c_int, C.c_long, C.c_int,
                                            C.c_double, _f64p, _f64p]
            L.kvq_oracle_attend_rotated.restype = C.c_int
            L.kvq_oracle_attend_rotated.argtypes = [
                _f64p, C.c_int, C.c_int, C.c_double, _i8p, _i8p,
                C.c_int, C.c_int, _u8p, _u8p, _u8p,
                C.c_int, C.c_int, _u8p, _u8p, _u8p, C.c_long, _f64p]
            _lib = L
    return _lib


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def _ptr(a: np.ndarray, t):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(t)


def _chunks(n: int, threads: int):
    threads = max(1, min(threads, n))
    step = (n + threads - 1) // threads
    return [(i, min(n, i + step)) for i in range(0, n, step)]


def angle_bits(L: int) -> int:
    return lib().kvq_oracle_angle_bits(int(L))


def row_bytes(d: int, L: int, mode: int, which: int) -> int:
    return int(lib().kvq_oracle_row_bytes(int(d), int(L), int(mode), int(which)))


def double_to_half_bits(x: float) -> int:
    return int(lib().kvq_oracle_double_to_half(float(x)))


def half_bits_to_double(h: int) -> float:
    return float(lib().kvq_oracle_half_to_double(int(h)))


def theta_hat(a: int, L: int) -> float:
    return float(lib().kvq_oracle_theta_hat(int(a), int(L)))


def _signs(s) -> np.ndarray:
    s = np.ascontiguousarray(np.asarray(s, dtype=np.int8))
    assert np.all(np.abs(s) == 1), "signs must be +1 / -1"
    return s


def rotate(x: np.ndarray, s, scaled: bool = True) -> np.ndarray:
    """H D x (/ sqrt(d) when scaled) for each row of x (fp64)."""
    x = np.ascontiguousarray(np.atleast_2d(np.asarray(x, dtype=np.float64)))
    s = _signs(s)
    out = np.empty_like(x)
    for i in range(x.shape[0]):
        lib().kvq_oracle_rotate(_ptr(x[i], _f64p), _ptr(s, _i8p), x.shape[1], int(scaled),
                                _ptr(out[i], _f64p))
    return out


def unrotate(z: np.ndarray, s) -> np.ndarray:
    """D H z / sqrt(d) for each row of z (fp64)."""
    z = np.ascontiguousarray(np.atleast_2d(np.asarray(z, dtype=np.float64)))
    s = _signs(s)
    out = np.empty_like(z)
    for i in range(z.shape[0]):
        lib().kvq_oracle_unrotate(_ptr(z[i], _f64p), _ptr(s, _i8p), z.shape[1],
                                  _ptr(out[i], _f64p))
    return out


@dataclass
class Codes:
    """Packed rows of n tokens of one codec, in the library's byte layout."""
    d: int
    L: int
    mode: int
    angles: np.ndarray  # uint8 [n, row_bytes(0)]
    norms: np.ndarray   # uint8 [n, row_bytes(1)]
    params: np.ndarray  # uint8 [n, row_bytes(2)]
    flags: np.ndarray | None = None  # uint8 [n, d/2]

    @property
    def n(self) -> int:
        return self.angles.shape[0]

    def take(self, idx) -> "Codes":
        f = None if self.flags is None else np.ascontiguousarray(self.flags[idx])
        return Codes(self.d, self.L, self.mode, np.ascontiguousarray(self.angles[idx]),
                     np.ascontiguousarray(self.norms[idx]), np.ascontiguousarray(self.params[idx]),
                     f)


def encode(x_half: np.ndarray, s, L: int, mode: int, threads: int | None = None) -> Codes:
    """Encode rows of fp16 vectors (any leading shape, last dim d)."""
    x = np.ascontiguousarray(np.asarray(x_half, dtype=np.float16))
    d = x.shape[-1]
    x = x.reshape(-1, d)
    n = x.shape[0]
    s = _signs(s)
    assert s.shape[0] == d
    ab, nb, pb = (row_bytes(d, L, mode, w) for w in range(3))
    if min(ab, nb, pb) < 0:
        raise ValueError(f"unsupported codec d={d} L={L} mode={mode}")
    angles = np.zeros((n, ab), np.uint8)
    norms = np.zeros((n, nb), np.uint8)
    params = np.zeros((n, max(pb, 0)), np.uint8)
    flags = np.zeros((n, d // 2), np.uint8)
    xb = x.view(np.uint16)
    L_ = lib()

    def run(lo, hi):
        if hi <= lo:
            return 0
        return L_.kvq_oracle_encode_batch(
            _ptr(xb[lo:hi], _u16p), hi - lo, _ptr(s, _i8p), d, int(L), int(mode),
            _ptr(angles[lo:hi], _u8p), _ptr(norms[lo:hi], _u8p),
            _ptr(params[lo:hi], _u8p) if pb > 0 else C.cast(None, _u8p),
            _ptr(flags[lo:hi], _u8p))

    _run_parallel(run, n, threads)
    return Codes(d, int(L), int(mode), angles, norms, params, flags)


def _run_parallel(fn, n, threads):
    threads = default_threads() if threads is None else threads
    parts = _chunks(n, threads) if n > 0 else []
    if len(parts) <= 1:
        rcs = [fn(lo, hi) for lo, hi in parts]
    else:
        with ThreadPoolExecutor(len(parts)) as ex:
            rcs = list(ex.map(lambda p: fn(*p), parts))
    if any(rc != 0 for rc in rcs):
        raise RuntimeError("oracle call failed")


def unpack(codes: Codes):
    """(angle codes int32 [n,P], norm codes int32 [n,P], rhat fp64 [n,P])."""
    n, P = codes.n, codes.d // 2
    a = np.zeros((n, P), np.int32)
    c = np.zeros((n, P), np.int32)
    rh = np.zeros((n, P), np.float64)
    L_ = lib()
    for v in range(n):
        rc = L_.kvq_oracle_unpack(_ptr(codes.angles[v], _u8p), _ptr(codes.norms[v], _u8p),
                                  _ptr(codes.params[v], _u8p) if codes.params.shape[1] else
                                  C.cast(None, _u8p),
                                  codes.d, codes.L, codes.mode, _ptr(a[v], _i32p),
                                  _ptr(c[v], _i32p), _ptr(rh[v], _f64p))
        if rc:
            raise RuntimeError("unpack failed")
    return a, c, rh


def dequant_rotated(codes: Codes) -> np.ndarray:
    n, d = codes.n, codes.d
    out = np.zeros((n, d), np.float64)
    L_ = lib()
    for v in range(n):
        rc = L_.kvq_oracle_dequant_rotated(
            _ptr(codes.angles[v], _u8p), _ptr(codes.norms[v], _u8p),
            _ptr(codes.params[v], _u8p) if codes.params.shape[1] else C.cast(None, _u8p),
            d, codes.L, codes.mode, _ptr(out[v], _f64p))
        if rc:
            raise RuntimeError("dequant failed")
    return out


def dequant(codes: Codes, s, threads: int | None = None) -> np.ndarray:
    """Original-domain dequantized vectors, fp64 [n, d]."""
    n, d = codes.n, codes.d
    s = _signs(s)
    out = np.zeros((n, d), np.float64)
    L_ = lib()
    pb = codes.params.shape[1]

    def run(lo, hi):
        if hi <= lo:
            return 0
        return L_.kvq_oracle_dequant_batch(
            _ptr(codes.angles[lo:hi], _u8p), _ptr(codes.norms[lo:hi], _u8p),
            _ptr(codes.params[lo:hi], _u8p) if pb else C.cast(None, _u8p), hi - lo,
            _ptr(s, _i8p), d, codes.L, codes.mode, _ptr(out[lo:hi], _f64p))

    _run_parallel(run, n, threads)
    return out


def attend(q: np.ndarray, khat: np.ndarray, vhat: np.ndarray, tau: float) -> np.ndarray:
    """Textbook softmax attention of q [G,d] over khat, vhat [T,d] (fp64)."""
    q = np.ascontiguousarray(np.atleast_2d(np.asarray(q, np.float64)))
    khat = np.ascontiguousarray(np.asarray(khat, np.float64))
    vhat = np.ascontiguousarray(np.asarray(vhat, np.float64))
    G, d = q.shape
    T = khat.shape[0]
    out = np.zeros((G, d), np.float64)
    tmp = np.zeros(max(T, 1), np.float64)
    lib().kvq_oracle_attend(_ptr(q, _f64p), _ptr(khat.reshape(-1) if T else tmp, _f64p),
                            _ptr(vhat.reshape(-1) if T else tmp, _f64p), G, T, d, float(tau),
                            _ptr(tmp, _f64p), _ptr(out, _f64p))
    return out


def attend_rotated(q: np.ndarray, sk, sv, kcodes: Codes, vcodes: Codes, tau: float) -> np.ndarray:
    """Streaming rotated-domain attention straight from codes (pin of attend)."""
    q = np.ascontiguousarray(np.atleast_2d(np.asarray(q, np.float64)))
    G, d = q.shape
    sk, sv = _signs(sk), _signs(sv)
    out = np.zeros((G, d), np.float64)
    T = kcodes.n
    dummy = np.zeros(16, np.uint8)

    def p(a):
        return _ptr(a, _u8p) if a.size else _ptr(dummy, _u8p)

    rc = lib().kvq_oracle_attend_rotated(
        _ptr(q, _f64p), G, d, float(tau), _ptr(sk, _i8p), _ptr(sv, _i8p),
        kcodes.L, kcodes.mode, p(kcodes.angles), p(kcodes.norms), p(kcodes.params),
        vcodes.L, vcodes.mode, p(vcodes.angles), p(vcodes.norms), p(vcodes.params), T,
        _ptr(out, _f64p))
    if rc:
        raise RuntimeError("attend_rotated failed")
    return out
