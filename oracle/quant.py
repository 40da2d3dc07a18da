"""Group-wise asymmetric min-max 4-bit compression: the oracle's quantizer (test
infrastructure only).

Every value here is computed by the C++ oracle (``fg_oracle.cpp``: ``quantize_group``,
``code_value`` and the packing loops); this module only shapes numpy buffers for it.

What the pages fix: weights and the attention (KV) cache are compressed to 4 bits
("FlexGen" README mirror, key features, "Extreme Compression"; arXiv 2303.06865 record,
abstract; Manning concept page, first bullet list).  The README's out-of-memory section
says weight compression cuts weight memory by about 70 %; with 4-bit codes plus two fp16
numbers per group of 64 the cost is 4.5 bits per element, a 71.9 % cut.

Readings where the pages are silent (the C++ file states them as Q1-Q7):

1. A group is ``g`` consecutive elements along one axis of a 2-D fp16 tensor
   (default g = 64; ``axis=1`` groups along a row, ``axis=0`` down a column).
2. ``mn = min(group)``, ``mx = max(group)``; a zero extreme is taken as +0.
3. ``s = fp16(fp32(mx - mn) / 15)``: fp32 subtraction, fp32 division, one round to
   nearest even.  The stored scale is that fp16 ``s``.
4. ``code = clamp(rint(fp32(x - mn) / s), 0, 15)`` with fp32 subtraction and fp32
   division by the stored scale, ``rint`` half to even; ``s == 0`` gives code 0.
5. Byte j of a row holds column 2j in its low nibble and column 2j+1 in its high nibble.
6. Params are {min, scale} fp16 pairs: [rows][cols/g] for axis=1, [rows/g][cols] for axis=0.
7. Dequantization is ``fp16(mn + code*s)`` with a single rounding of the exact value.
"""
from __future__ import annotations

import numpy as np

from ._lib import f16, lib, p


def quantize_groups(x16: np.ndarray):
    """Quantize rows of ``x16`` ([ngroups, g] float16), one row per group.

    Returns (codes uint8 [ngroups, g] in 0..15, mn float16 [ngroups], s float16 [ngroups])."""
    x = f16(x16)
    n, g = x.shape
    q = np.empty((n, g), np.uint8)
    mn = np.empty(n, np.float16)
    s = np.empty(n, np.float16)
    lib().orc_quantize_groups(p(x), n, g, p(q), p(mn), p(s))
    return q, mn, s


def dequantize_groups(codes: np.ndarray, mn: np.ndarray, s: np.ndarray) -> np.ndarray:
    """fp16(mn + code*s), one rounding of the exact value (reading 7)."""
    q = np.ascontiguousarray(codes, np.uint8)
    n, g = q.shape
    out = np.empty((n, g), np.float16)
    lib().orc_dequantize_groups(p(q), p(f16(mn)), p(f16(s)), n, g, p(out))
    return out


def pack_nibbles(codes2d: np.ndarray) -> np.ndarray:
    """[rows, cols] codes -> [rows, cols/2] bytes; even column in the low nibble (reading 5)."""
    q = np.ascontiguousarray(codes2d, np.uint8)
    rows, cols = q.shape
    out = np.empty((rows, cols // 2), np.uint8)
    lib().orc_pack_nibbles(p(q), rows, cols, p(out))
    return out


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(packed, np.uint8)
    rows, half = b.shape
    out = np.empty((rows, 2 * half), np.uint8)
    lib().orc_unpack_nibbles(p(b), rows, 2 * half, p(out))
    return out


def _check(rows: int, cols: int, group: int, axis: int):
    if group < 2 or group % 2:
        raise ValueError("group must be an even number >= 2")
    if cols % 2:
        raise ValueError("cols must be even (two codes per byte along a row)")
    if axis not in (0, 1):
        raise ValueError("axis must be 0 or 1")
    if axis == 1 and cols % group:
        raise ValueError("cols must be a multiple of the group size")
    if axis == 0 and rows % group:
        raise ValueError("rows must be a multiple of the group size")


def quantize_pack(x: np.ndarray, group: int = 64, axis: int = 1):
    """fp16 [rows, cols] -> (codes uint8 [rows, cols/2], params float16 [..., 2] {min, scale}).

    params shape: [rows, cols/group, 2] for axis=1, [rows/group, cols, 2] for axis=0.
    """
    x = f16(x)
    rows, cols = x.shape
    _check(rows, cols, group, axis)
    codes = np.empty((rows, cols // 2), np.uint8)
    pshape = (rows, cols // group, 2) if axis == 1 else (rows // group, cols, 2)
    params = np.empty(pshape, np.float16)
    assert lib().orc_quantize_pack(p(x), rows, cols, group, axis, p(codes), p(params)) == 0
    return codes, params


def dequantize(codes: np.ndarray, params: np.ndarray, rows: int, cols: int, group: int = 64,
               axis: int = 1) -> np.ndarray:
    """Inverse map of ``quantize_pack`` (codes + params -> fp16 [rows, cols])."""
    _check(rows, cols, group, axis)
    c = np.ascontiguousarray(codes, np.uint8).reshape(rows, cols // 2)
    pr = f16(params)
    assert pr.size == 2 * rows * cols // group
    out = np.empty((rows, cols), np.float16)
    assert lib().orc_dequantize(p(c), p(pr), rows, cols, group, axis, p(out)) == 0
    return out


def storage_bytes(n_elems: int, group: int = 64) -> int:
    """Bytes of the compressed form: n/2 code bytes plus 4 bytes ({min, scale}) per group."""
    return n_elems // 2 + (n_elems // group) * 4
