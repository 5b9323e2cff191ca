"""Thin ctypes binding of libkvq.so (include/kvq.h).

Argument marshalling only: every step of encode, dequant and decode attention
runs in the CUDA kernels of libkvq.so.  PyTorch provides device memory and
streams.  The functions named ``kvq_*`` mirror the C entry points one to one
(they take the same arguments, as ctypes values or torch tensors, and raise
KvqError on a non-OK status); DecodeStepCall and DecodeStepHostCall are
kvq_decode_step / kvq_decode_step_host with their arguments marshalled once
for per-token reuse; the small helpers below them only allocate caller-owned
buffers with torch and fill the C structs.

A missing or unloadable libkvq.so raises at first use: there is no fallback.
"""
from __future__ import annotations

import ctypes as C
import os
import re
import threading
from dataclasses import dataclass

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkvq.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "kvq.h")

KVQ_OK, KVQ_EINVAL, KVQ_EUNSUPPORTED, KVQ_ECUDA, KVQ_ETIMEOUT = 0, -1, -2, -3, -4
KVQ_NORM_LIN8, KVQ_NORM_LOG4 = 0, 1
KVQ_DEVERR_CTX_RANGE, KVQ_DEVERR_TIMEOUT, KVQ_DEVERR_PAGE_RANGE = 0x1, 0x2, 0x4
KVQ_DEVERR_BAD_CODE = 0x8
KVQ_TEST_RESET, KVQ_TEST_FAIL_LAUNCHES, KVQ_TEST_WAIT_LIMIT, KVQ_TEST_DEBUG_CHECKS = 0, 1, 2, 3
OUT_FP16, OUT_FP32 = 0, 1


class KvqError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"kvq status {status}: {message}")
        self.status = status


class kvq_codec(C.Structure):
    _fields_ = [("head_dim", C.c_int32), ("L", C.c_int32), ("norm_mode", C.c_int32)]


class kvq_plane(C.Structure):
    _fields_ = [("angles", C.c_void_p), ("norms", C.c_void_p), ("params", C.c_void_p),
                ("capacity", C.c_int64)]


class kvq_paged_plane(C.Structure):
    _fields_ = [("angles", C.c_void_p), ("norms", C.c_void_p), ("params", C.c_void_p),
                ("pages", C.c_void_p), ("page_tokens", C.c_int32), ("max_pages", C.c_int32),
                ("num_pages", C.c_int64)]


_lock = threading.Lock()
_lib = None

_SIGNATURES = {
    "kvq_version": (C.c_int32, []),
    "kvq_last_error": (C.c_char_p, []),
    "kvq_test_control": (C.c_int, [C.c_int32, C.c_int64]),
    "kvq_angle_bits": (C.c_int32, [C.c_int32]),
    "kvq_row_bytes": (C.c_int64, [C.POINTER(kvq_codec), C.c_int32]),
    "kvq_encode": (C.c_int, [C.POINTER(kvq_codec), C.c_void_p, C.c_void_p, C.c_int32, C.c_int32,
                             C.c_int32, C.c_int64, C.POINTER(kvq_plane), C.c_void_p]),
    "kvq_encode_kv": (C.c_int, [C.POINTER(kvq_codec), C.c_void_p, C.c_void_p, C.POINTER(kvq_plane),
                                C.POINTER(kvq_codec), C.c_void_p, C.c_void_p, C.POINTER(kvq_plane),
                                C.c_int32, C.c_int32, C.c_int32, C.c_int64, C.c_void_p]),
    "kvq_dequant": (C.c_int, [C.POINTER(kvq_codec), C.c_void_p, C.POINTER(kvq_plane), C.c_int32,
                              C.c_int32, C.c_int32, C.c_int64, C.c_void_p, C.c_void_p]),
    "kvq_decode_num_splits": (C.c_int32, [C.c_int32, C.c_int32, C.c_int64, C.c_int32]),
    "kvq_decode_workspace_bytes": (C.c_int64, [C.c_int32, C.c_int32, C.c_int32, C.c_int32]),
    "kvq_decode_attn_noalloc": (C.c_int, [C.c_void_p, C.POINTER(kvq_codec), C.POINTER(kvq_codec),
                                          C.c_void_p, C.c_void_p, C.POINTER(kvq_plane),
                                          C.POINTER(kvq_plane), C.c_void_p, C.c_int32, C.c_int32,
                                          C.c_int32, C.c_int64, C.c_float, C.c_int32, C.c_void_p,
                                          C.c_void_p, C.c_int32, C.c_void_p]),
    "kvq_decode_step": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.POINTER(kvq_codec),
                                  C.POINTER(kvq_codec), C.c_void_p, C.c_void_p,
                                  C.POINTER(kvq_plane), C.POINTER(kvq_plane), C.c_void_p,
                                  C.c_int32, C.c_int32, C.c_int32, C.c_int64, C.c_float, C.c_int32,
                                  C.c_void_p, C.c_int64, C.c_void_p, C.c_void_p, C.c_int32,
                                  C.c_void_p]),
    "kvq_decode_step_host": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                       C.POINTER(kvq_codec), C.POINTER(kvq_codec), C.c_void_p,
                                       C.c_void_p, C.POINTER(kvq_plane), C.POINTER(kvq_plane),
                                       C.c_void_p, C.c_int32, C.c_int32, C.c_int32, C.c_int64,
                                       C.c_float, C.c_int32, C.c_void_p, C.c_int64, C.c_void_p,
                                       C.c_int32, C.c_void_p]),
    "kvq_encode_kv_paged": (C.c_int, [C.POINTER(kvq_codec), C.c_void_p, C.c_void_p,
                                      C.POINTER(kvq_paged_plane), C.POINTER(kvq_codec),
                                      C.c_void_p, C.c_void_p, C.POINTER(kvq_paged_plane),
                                      C.c_int32, C.c_int32, C.c_int32, C.c_int64, C.c_void_p,
                                      C.c_void_p]),
    "kvq_decode_attn_paged": (C.c_int, [C.c_void_p, C.POINTER(kvq_codec), C.POINTER(kvq_codec),
                                        C.c_void_p, C.c_void_p, C.POINTER(kvq_paged_plane),
                                        C.POINTER(kvq_paged_plane), C.c_void_p, C.c_int32,
                                        C.c_int32, C.c_int32, C.c_int64, C.c_float, C.c_int32,
                                        C.c_void_p, C.c_int64, C.c_void_p, C.c_void_p, C.c_int32,
                                        C.c_void_p]),
    "kvq_decode_step_paged": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.POINTER(kvq_codec),
                                        C.POINTER(kvq_codec), C.c_void_p, C.c_void_p,
                                        C.POINTER(kvq_paged_plane), C.POINTER(kvq_paged_plane),
                                        C.c_void_p, C.c_int32, C.c_int32, C.c_int32, C.c_int64,
                                        C.c_float, C.c_int32, C.c_void_p, C.c_int64, C.c_void_p,
                                        C.c_void_p, C.c_int32, C.c_void_p]),
    "kvq_decode_attn": (C.c_int, [C.c_void_p, C.POINTER(kvq_codec), C.POINTER(kvq_codec),
                                  C.c_void_p, C.c_void_p, C.POINTER(kvq_plane),
                                  C.POINTER(kvq_plane), C.c_void_p, C.c_int32, C.c_int32,
                                  C.c_int32, C.c_int64, C.c_float, C.c_int32, C.c_void_p,
                                  C.c_int64, C.c_void_p, C.c_void_p, C.c_int32, C.c_void_p]),
    "kvq_decode_attn_partials": (C.c_int, [C.c_void_p, C.POINTER(kvq_codec),
                                           C.POINTER(kvq_codec), C.c_void_p, C.c_void_p,
                                           C.POINTER(kvq_plane), C.POINTER(kvq_plane),
                                           C.c_void_p, C.c_int32, C.c_int32, C.c_int32,
                                           C.c_int64, C.c_float, C.c_int32, C.c_void_p,
                                           C.c_int64, C.c_void_p, C.c_void_p]),
    "kvq_decode_merge_partials": (C.c_int, [C.c_void_p, C.c_int32, C.c_int32, C.c_int32,
                                            C.c_int32, C.c_int32, C.c_void_p, C.c_void_p,
                                            C.c_int32, C.c_void_p]),
}


def lib():
    """The loaded libkvq.so (raises if it is missing or does not load)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise KvqError(KVQ_EUNSUPPORTED,
                               f"{LIB_PATH} is missing; build it with "
                               "`python -m decode_attention_rand_b200.build`")
            L = C.CDLL(LIB_PATH)
            for name, (res, args) in _SIGNATURES.items():
                f = getattr(L, name)
                f.restype = res
                f.argtypes = args
            _lib = L
    return _lib


def header_functions() -> list[str]:
    """Names of the functions include/kvq.h declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z0-9_]+)\s*\(", text)))


def _check(rc: int):
    if rc != KVQ_OK:
        raise KvqError(rc, lib().kvq_last_error().decode())


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ------------------------------------------------------------------ C ABI --

def kvq_version() -> int:
    return lib().kvq_version()


def kvq_last_error() -> str:
    return lib().kvq_last_error().decode()


def kvq_test_control(key: int, value: int):
    _check(lib().kvq_test_control(key, value))


def kvq_angle_bits(L: int) -> int:
    return lib().kvq_angle_bits(L)


def kvq_row_bytes(codec: kvq_codec, which: int) -> int:
    return lib().kvq_row_bytes(C.byref(codec), which)


def kvq_encode(codec: kvq_codec, signs, x, B: int, H_kv: int, T: int, pos0: int,
               out: kvq_plane, stream=None):
    _check(lib().kvq_encode(C.byref(codec), _ptr(signs), _ptr(x), B, H_kv, T, pos0,
                            C.byref(out), _stream(stream)))


def kvq_encode_kv(kc: kvq_codec, signs_k, k, K: kvq_plane, vc: kvq_codec, signs_v, v,
                  V: kvq_plane, B: int, H_kv: int, T: int, pos0: int, stream=None):
    _check(lib().kvq_encode_kv(C.byref(kc), _ptr(signs_k), _ptr(k), C.byref(K), C.byref(vc),
                               _ptr(signs_v), _ptr(v), C.byref(V), B, H_kv, T, pos0,
                               _stream(stream)))


def kvq_dequant(codec: kvq_codec, signs, plane: kvq_plane, B: int, H_kv: int, T: int,
                pos0: int, y, stream=None):
    _check(lib().kvq_dequant(C.byref(codec), _ptr(signs), C.byref(plane), B, H_kv, T, pos0,
                             _ptr(y), _stream(stream)))


def kvq_decode_num_splits(B: int, H_kv: int, max_ctx: int, sm_count: int) -> int:
    return lib().kvq_decode_num_splits(B, H_kv, max_ctx, sm_count)


def kvq_decode_workspace_bytes(B: int, H_q: int, head_dim: int, num_splits: int) -> int:
    return lib().kvq_decode_workspace_bytes(B, H_q, head_dim, num_splits)


def kvq_decode_step(q, k_new, v_new, kc: kvq_codec, vc: kvq_codec, signs_k, signs_v,
                    K: kvq_plane, V: kvq_plane, ctx_len, B: int, H_q: int, H_kv: int,
                    max_ctx: int, softmax_scale: float, num_splits: int, workspace, ws_bytes: int,
                    err_word, out, out_dtype: int, stream=None):
    _check(lib().kvq_decode_step(_ptr(q), _ptr(k_new), _ptr(v_new), C.byref(kc), C.byref(vc),
                                 _ptr(signs_k), _ptr(signs_v), C.byref(K), C.byref(V),
                                 _ptr(ctx_len), B, H_q, H_kv, max_ctx, softmax_scale, num_splits,
                                 _ptr(workspace), ws_bytes, _ptr(err_word), _ptr(out), out_dtype,
                                 _stream(stream)))


def kvq_decode_step_host(in_host, in_dev, out_host, out_dev, kc: kvq_codec, vc: kvq_codec,
                         signs_k, signs_v, K: kvq_plane, V: kvq_plane, ctx_len, B: int, H_q: int,
                         H_kv: int, max_ctx: int, softmax_scale: float, num_splits: int, workspace,
                         ws_bytes: int, err_word, out_dtype: int, stream=None):
    _check(lib().kvq_decode_step_host(_ptr(in_host), _ptr(in_dev), _ptr(out_host), _ptr(out_dev),
                                      C.byref(kc), C.byref(vc), _ptr(signs_k), _ptr(signs_v),
                                      C.byref(K), C.byref(V), _ptr(ctx_len), B, H_q, H_kv,
                                      max_ctx, softmax_scale, num_splits, _ptr(workspace),
                                      ws_bytes, _ptr(err_word), out_dtype, _stream(stream)))


class DecodeStepHostCall:
    """kvq_decode_step_host with its arguments marshalled once (host and
    device buffers fixed for the life of the object), for a serving loop that
    feeds each token's inputs from host memory."""

    def __init__(self, in_host, in_dev, out_host, out_dev, kc: kvq_codec, vc: kvq_codec,
                 signs_k, signs_v, K: kvq_plane, V: kvq_plane, ctx_len, B: int, H_q: int,
                 H_kv: int, max_ctx: int, softmax_scale: float, num_splits: int, workspace,
                 ws_bytes: int, err_word, out_dtype: int):
        self._kc, self._vc, self._K, self._V = kc, vc, K, V  # keep the structs alive
        self._fn = lib().kvq_decode_step_host
        self._args = (_ptr(in_host), _ptr(in_dev), _ptr(out_host), _ptr(out_dev), C.byref(kc),
                      C.byref(vc), _ptr(signs_k), _ptr(signs_v), C.byref(K), C.byref(V),
                      _ptr(ctx_len), B, H_q, H_kv, max_ctx, C.c_float(softmax_scale),
                      num_splits, _ptr(workspace), ws_bytes, _ptr(err_word), out_dtype)

    def __call__(self, stream=None):
        _check(self._fn(*self._args, _stream(stream)))


class DecodeStepCall:
    """kvq_decode_step with its arguments marshalled once, for a serving loop
    that calls it every token on the same buffers: the pointers, sizes and
    codec structs are converted to ctypes values here, and each call passes
    them unchanged (only the stream may vary).  The buffers must stay alive
    and in place while the object is used."""

    def __init__(self, q, k_new, v_new, kc: kvq_codec, vc: kvq_codec, signs_k, signs_v,
                 K: kvq_plane, V: kvq_plane, ctx_len, B: int, H_q: int, H_kv: int,
                 max_ctx: int, softmax_scale: float, num_splits: int, workspace, ws_bytes: int,
                 err_word, out, out_dtype: int):
        self._kc, self._vc, self._K, self._V = kc, vc, K, V  # keep the structs alive
        self._fn = lib().kvq_decode_step
        self._args = (_ptr(q), _ptr(k_new), _ptr(v_new), C.byref(kc), C.byref(vc),
                      _ptr(signs_k), _ptr(signs_v), C.byref(K), C.byref(V), _ptr(ctx_len),
                      B, H_q, H_kv, max_ctx, C.c_float(softmax_scale), num_splits,
                      _ptr(workspace), ws_bytes, _ptr(err_word), _ptr(out), out_dtype)

    def __call__(self, stream=None):
        _check(self._fn(*self._args, _stream(stream)))


def kvq_encode_kv_paged(kc: kvq_codec, signs_k, k, K: kvq_paged_plane, vc: kvq_codec, signs_v,
                        v, V: kvq_paged_plane, B: int, H_kv: int, T: int, pos0: int,
                        err_word=None, stream=None):
    _check(lib().kvq_encode_kv_paged(C.byref(kc), _ptr(signs_k), _ptr(k), C.byref(K),
                                     C.byref(vc), _ptr(signs_v), _ptr(v), C.byref(V), B, H_kv, T,
                                     pos0, _ptr(err_word), _stream(stream)))


def kvq_decode_attn_paged(q, kc: kvq_codec, vc: kvq_codec, signs_k, signs_v, K: kvq_paged_plane,
                          V: kvq_paged_plane, ctx_len, B: int, H_q: int, H_kv: int, max_ctx: int,
                          softmax_scale: float, num_splits: int, workspace, ws_bytes: int,
                          err_word, out, out_dtype: int, stream=None):
    _check(lib().kvq_decode_attn_paged(_ptr(q), C.byref(kc), C.byref(vc), _ptr(signs_k),
                                       _ptr(signs_v), C.byref(K), C.byref(V), _ptr(ctx_len), B,
                                       H_q, H_kv, max_ctx, softmax_scale, num_splits,
                                       _ptr(workspace), ws_bytes, _ptr(err_word), _ptr(out),
                                       out_dtype, _stream(stream)))


def kvq_decode_step_paged(q, k_new, v_new, kc: kvq_codec, vc: kvq_codec, signs_k, signs_v,
                          K: kvq_paged_plane, V: kvq_paged_plane, ctx_len, B: int, H_q: int,
                          H_kv: int, max_ctx: int, softmax_scale: float, num_splits: int,
                          workspace, ws_bytes: int, err_word, out, out_dtype: int, stream=None):
    _check(lib().kvq_decode_step_paged(_ptr(q), _ptr(k_new), _ptr(v_new), C.byref(kc),
                                       C.byref(vc), _ptr(signs_k), _ptr(signs_v), C.byref(K),
                                       C.byref(V), _ptr(ctx_len), B, H_q, H_kv, max_ctx,
                                       softmax_scale, num_splits, _ptr(workspace), ws_bytes,
                                       _ptr(err_word), _ptr(out), out_dtype, _stream(stream)))


def kvq_decode_attn_partials(q, kc: kvq_codec, vc: kvq_codec, signs_k, signs_v, K: kvq_plane,
                             V: kvq_plane, ctx_len, B: int, H_q: int, H_kv: int, max_ctx: int,
                             softmax_scale: float, num_splits: int, workspace, ws_bytes: int,
                             err_word=None, stream=None):
    _check(lib().kvq_decode_attn_partials(_ptr(q), C.byref(kc), C.byref(vc), _ptr(signs_k),
                                          _ptr(signs_v), C.byref(K), C.byref(V), _ptr(ctx_len),
                                          B, H_q, H_kv, max_ctx, softmax_scale, num_splits,
                                          _ptr(workspace), ws_bytes, _ptr(err_word),
                                          _stream(stream)))


def kvq_decode_merge_partials(parts, n_parts: int, B: int, H_q: int, head_dim: int,
                              num_splits: int, signs_v, out, out_dtype: int, stream=None):
    _check(lib().kvq_decode_merge_partials(_ptr(parts), n_parts, B, H_q, head_dim, num_splits,
                                           _ptr(signs_v), _ptr(out), out_dtype, _stream(stream)))


def kvq_decode_attn(q, kc: kvq_codec, vc: kvq_codec, signs_k, signs_v, K: kvq_plane,
                    V: kvq_plane, ctx_len, B: int, H_q: int, H_kv: int, max_ctx: int,
                    softmax_scale: float, num_splits: int, workspace, ws_bytes: int, err_word,
                    out, out_dtype: int, stream=None):
    _check(lib().kvq_decode_attn(_ptr(q), C.byref(kc), C.byref(vc), _ptr(signs_k),
                                 _ptr(signs_v), C.byref(K), C.byref(V), _ptr(ctx_len), B, H_q,
                                 H_kv, max_ctx, softmax_scale, num_splits, _ptr(workspace),
                                 ws_bytes, _ptr(err_word), _ptr(out), out_dtype,
                                 _stream(stream)))


def kvq_decode_attn_noalloc(q, kc: kvq_codec, vc: kvq_codec, signs_k, signs_v, K: kvq_plane,
                            V: kvq_plane, ctx_len, B: int, H_q: int, H_kv: int, max_ctx: int,
                            softmax_scale: float, num_splits: int, err_word, out, out_dtype: int,
                            stream=None):
    """kvq_decode_attn with the library's built-in scratch instead of a
    caller workspace (for callers that cannot allocate device memory)."""
    _check(lib().kvq_decode_attn_noalloc(_ptr(q), C.byref(kc), C.byref(vc), _ptr(signs_k),
                                         _ptr(signs_v), C.byref(K), C.byref(V), _ptr(ctx_len), B,
                                         H_q, H_kv, max_ctx, softmax_scale, num_splits,
                                         _ptr(err_word), _ptr(out), out_dtype, _stream(stream)))


# ------------------------------------------------------ torch-side helpers --

def codec(head_dim: int, L: int, norm_mode: int) -> kvq_codec:
    return kvq_codec(head_dim, L, norm_mode)


@dataclass
class Plane:
    """Caller-owned device arrays of one compressed plane [B][H_kv][capacity][row]."""
    codec: kvq_codec
    B: int
    H_kv: int
    capacity: int
    angles: object
    norms: object
    params: object

    def c(self) -> kvq_plane:
        return kvq_plane(self.angles.data_ptr(), self.norms.data_ptr(), self.params.data_ptr(),
                         self.capacity)

    def rows(self, which: int):
        """uint8 view [B, H_kv, capacity, row_bytes] of one array."""
        t = (self.angles, self.norms, self.params)[which]
        return t.view(self.B, self.H_kv, self.capacity, -1)


def alloc_plane(c: kvq_codec, B: int, H_kv: int, capacity: int, device="cuda") -> Plane:
    import torch
    if capacity % 16:
        raise ValueError("capacity must be a multiple of 16")
    n = B * H_kv * capacity
    arrs = [torch.zeros(max(1, n * kvq_row_bytes(c, w)), dtype=torch.uint8, device=device)
            for w in range(3)]
    return Plane(c, B, H_kv, capacity, *arrs)


def encode(c: kvq_codec, signs, x, plane: Plane, pos0: int = 0, stream=None):
    """Encode x [B, H_kv, T, d] (fp16, contiguous) into plane tokens pos0.."""
    B, H, T, d = x.shape
    kvq_encode(c, signs, x, B, H, T, pos0, plane.c(), stream)


def encode_kv(kc: kvq_codec, signs_k, k, K: Plane, vc: kvq_codec, signs_v, v, V: Plane,
              pos0: int = 0, stream=None):
    """Encode k and v [B, H_kv, T, d] (fp16, contiguous) into K and V tokens
    pos0.. in one launch."""
    if tuple(k.shape) != tuple(v.shape):
        raise ValueError("k and v must have the same shape")
    B, H, T, d = k.shape
    kvq_encode_kv(kc, signs_k, k, K.c(), vc, signs_v, v, V.c(), B, H, T, pos0, stream)


def dequant(c: kvq_codec, signs, plane: Plane, T: int, pos0: int = 0, out=None, stream=None):
    import torch
    if out is None:
        out = torch.empty((plane.B, plane.H_kv, T, c.head_dim), dtype=torch.float16,
                          device=plane.angles.device)
    kvq_dequant(c, signs, plane.c(), plane.B, plane.H_kv, T, pos0, out, stream)
    return out


class DecodeWorkspace:
    """Scratch for kvq_decode_attn sized for (B, H_q, d, num_splits); zero-filled
    once, as the C ABI requires before first use."""

    def __init__(self, B, H_q, d, num_splits, device="cuda"):
        import torch
        self.num_splits = num_splits
        self.nbytes = kvq_decode_workspace_bytes(B, H_q, d, num_splits)
        self.buf = torch.zeros(max(16, self.nbytes), dtype=torch.uint8, device=device)


def decode_attn(q, kc: kvq_codec, vc: kvq_codec, signs_k, signs_v, K: Plane, V: Plane,
                ctx_len, max_ctx: int, softmax_scale: float | None = None, num_splits=None,
                workspace: DecodeWorkspace | None = None, err_word=None, out=None,
                out_dtype: int = OUT_FP32, stream=None):
    import torch
    B, H_q, d = q.shape
    if softmax_scale is None:
        softmax_scale = d ** -0.5
    if num_splits is None:
        sm = torch.cuda.get_device_properties(q.device).multi_processor_count
        num_splits = kvq_decode_num_splits(B, K.H_kv, max_ctx, sm)
    if workspace is None or workspace.num_splits != num_splits:
        workspace = DecodeWorkspace(B, H_q, d, num_splits, q.device)
    if out is None:
        out = torch.empty((B, H_q, d), dtype=torch.float16 if out_dtype == OUT_FP16
                          else torch.float32, device=q.device)
    kvq_decode_attn(q, kc, vc, signs_k, signs_v, K.c(), V.c(), ctx_len, B, H_q, K.H_kv, max_ctx,
                    softmax_scale, num_splits, workspace.buf, workspace.nbytes, err_word, out,
                    out_dtype, stream)
    return out


def decode_step(q, k_new, v_new, kc: kvq_codec, vc: kvq_codec, signs_k, signs_v, K: Plane,
                V: Plane, ctx_len, max_ctx: int, softmax_scale: float | None = None,
                num_splits=None, workspace: DecodeWorkspace | None = None, err_word=None, out=None,
                out_dtype: int = OUT_FP32, stream=None):
    """Append k_new / v_new [B, H_kv, d] at position ctx_len[b] - 1 and attend
    q over positions 0 .. ctx_len[b] - 1: one kernel, or an append launch
    followed by the decode where the decode instance carries no append code
    (the two-CTAs-per-SM and runtime-width kernels)."""
    import torch
    B, H_q, d = q.shape
    if softmax_scale is None:
        softmax_scale = d ** -0.5
    if num_splits is None:
        sm = torch.cuda.get_device_properties(q.device).multi_processor_count
        num_splits = kvq_decode_num_splits(B, K.H_kv, max_ctx, sm)
    if workspace is None or workspace.num_splits != num_splits:
        workspace = DecodeWorkspace(B, H_q, d, num_splits, q.device)
    if out is None:
        out = torch.empty((B, H_q, d), dtype=torch.float16 if out_dtype == OUT_FP16
                          else torch.float32, device=q.device)
    kvq_decode_step(q, k_new, v_new, kc, vc, signs_k, signs_v, K.c(), V.c(), ctx_len, B, H_q,
                    K.H_kv, max_ctx, softmax_scale, num_splits, workspace.buf, workspace.nbytes,
                    err_word, out, out_dtype, stream)
    return out


@dataclass
class PagedPlane:
    """Caller-owned pools [num_pages][H_kv][page_tokens][row] of one paged plane
    and its page table [B][max_pages] (int32, device)."""
    codec: kvq_codec
    H_kv: int
    page_tokens: int
    num_pages: int
    pages: object
    angles: object
    norms: object
    params: object

    @property
    def max_pages(self) -> int:
        return self.pages.shape[1]

    def c(self) -> kvq_paged_plane:
        return kvq_paged_plane(self.angles.data_ptr(), self.norms.data_ptr(),
                               self.params.data_ptr(), self.pages.data_ptr(), self.page_tokens,
                               self.max_pages, self.num_pages)

    def rows(self, which: int):
        """uint8 view [num_pages, H_kv, page_tokens, row_bytes] of one pool."""
        t = (self.angles, self.norms, self.params)[which]
        return t.view(self.num_pages, self.H_kv, self.page_tokens, -1)


def alloc_paged_plane(c: kvq_codec, H_kv: int, page_tokens: int, num_pages: int, pages,
                      device="cuda") -> PagedPlane:
    """Zeroed pools for `num_pages` pages; `pages` is the [B][max_pages] table."""
    import torch
    n = num_pages * H_kv * page_tokens
    arrs = [torch.zeros(max(1, n * kvq_row_bytes(c, w)), dtype=torch.uint8, device=device)
            for w in range(3)]
    pages = torch.as_tensor(pages, dtype=torch.int32, device=device).contiguous()
    return PagedPlane(c, H_kv, page_tokens, num_pages, pages, *arrs)
