"""Test infrastructure: the fp64 CPU oracle of the rotated-angle KV codec.

NOT part of the product.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It wraps the plain C
library ``kvq_oracle.c`` (built by :func:`build`) with ctypes and spreads
batches over host threads (ctypes releases the GIL during each C call).

The method it follows is "TurboAngle: Near-Lossless KV Cache Compression via
Uniform Angle Quantization", Abstract; the formulas are stated at the top of
``kvq_oracle.c``.
"""
from .oracle import (  # noqa: F401
    FLAG_ANGLE,
    FLAG_NORM,
    FLAG_PARAM,
    MODE_EXACT,
    MODE_LIN8,
    MODE_LOG4,
    Codes,
    angle_bits,
    attend,
    attend_rotated,
    build,
    default_threads,
    dequant,
    dequant_rotated,
    double_to_half_bits,
    encode,
    half_bits_to_double,
    lib,
    rotate,
    row_bytes,
    theta_hat,
    unpack,
    unrotate,
)
