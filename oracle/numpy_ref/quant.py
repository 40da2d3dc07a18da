"""Oracle for group-wise asymmetric min-max 4-bit compression (test infrastructure only).

What the pages fix: weights and the attention (KV) cache are compressed to 4 bits
("FlexGen" README mirror, key features, "Extreme Compression"; arXiv 2303.06865 record,
abstract; Manning concept page, first bullet list).  The README's out-of-memory section
says weight compression cuts weight memory by about 70 %; with 4-bit codes plus two fp16
numbers per group of 64 the cost is 4.5 bits per element, a 71.9 % cut.

Everything below that level is a reading (the pages are silent), chosen as the plainest
one consistent with the rest:

1. A group is ``g`` consecutive elements along one axis of a 2-D fp16 tensor
   (default g = 64; ``axis=1`` groups along a row, ``axis=0`` down a column).
2. ``mn = min(group)``, ``mx = max(group)``; a zero extreme is taken as +0.
3. ``d = mx - mn`` and ``s = fp16(d / 15)``: fp32 subtraction, fp32 division, then one
   round-to-nearest-even to fp16.  The stored scale is that fp16 ``s``.
4. ``code = clamp(rint((x - mn) / s), 0, 15)`` with fp32 subtraction and fp32 division
   by the *stored* fp16 scale, ``rint`` rounding half to even.  When ``s == 0`` (constant
   group, or d/15 below half the smallest fp16 subnormal) every code is 0.
5. Two codes per byte along the contiguous (column) axis: byte j of a row holds column
   2j in its low nibble and column 2j+1 in its high nibble.
6. Params are {min, scale} fp16 pairs (min first); for axis=1 they are laid out
   [rows][cols/g], for axis=0 [rows/g][cols].
7. Dequantization is ``fp16(mn + code*s)`` with a single rounding of the exact value
   (the product and sum are exact in float64: at most 41 significant bits).
"""
from __future__ import annotations

import numpy as np


def quantize_groups(x16: np.ndarray):
    """Quantize rows of ``x16`` ([ngroups, g] float16), one row per group.

    Returns (codes uint8 [ngroups, g] in 0..15, mn float16 [ngroups], s float16 [ngroups]).
    Steps 2-4 of the module docstring, in that order.
    """
    x16 = np.asarray(x16, dtype=np.float16)
    xf = x16.astype(np.float32)
    mn = xf.min(axis=1) + np.float32(0.0)          # -0 + 0 = +0 (zero extreme as +0)
    mx = xf.max(axis=1) + np.float32(0.0)
    d = mx - mn                                     # fp32, round to nearest
    s32 = d / np.float32(15.0)                      # fp32 IEEE division
    s16 = s32.astype(np.float16)                    # one RNE rounding to fp16
    sf = s16.astype(np.float32)
    zero = sf == np.float32(0.0)
    safe = np.where(zero, np.float32(1.0), sf)
    r = (xf - mn[:, None]) / safe[:, None]          # fp32 sub then fp32 div, no FMA
    q = np.clip(np.rint(r), 0.0, 15.0)              # rint: half to even
    q[zero] = 0.0
    return q.astype(np.uint8), mn.astype(np.float16), s16


def dequantize_groups(codes: np.ndarray, mn: np.ndarray, s: np.ndarray) -> np.ndarray:
    """fp16(mn + code*s), one rounding of the exact value (step 7)."""
    exact = (np.asarray(codes, dtype=np.float64) * np.asarray(s, np.float16).astype(np.float64)[:, None]
             + np.asarray(mn, np.float16).astype(np.float64)[:, None])
    return exact.astype(np.float16)


def pack_nibbles(codes2d: np.ndarray) -> np.ndarray:
    """[rows, cols] codes -> [rows, cols/2] bytes; even column in the low nibble (step 5)."""
    c = np.asarray(codes2d, dtype=np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = p & 0x0F
    out[:, 1::2] = p >> 4
    return out


def _groups_view(x: np.ndarray, group: int, axis: int) -> np.ndarray:
    rows, cols = x.shape
    if axis == 1:
        return x.reshape(rows * cols // group, group)
    # axis 0: group = `group` consecutive rows of one column
    return x.reshape(rows // group, group, cols).transpose(0, 2, 1).reshape(-1, group)


def _ungroup(g2d: np.ndarray, rows: int, cols: int, group: int, axis: int) -> np.ndarray:
    if axis == 1:
        return g2d.reshape(rows, cols)
    return g2d.reshape(rows // group, cols, group).transpose(0, 2, 1).reshape(rows, cols)


def _check(rows: int, cols: int, group: int, axis: int):
    if group < 2 or group % 2:
        raise ValueError("group must be an even number >= 2")
    if cols % 2:
        raise ValueError("cols must be even (two codes per byte along a row)")
    if axis == 1 and cols % group:
        raise ValueError("cols must be a multiple of the group size")
    if axis == 0 and rows % group:
        raise ValueError("rows must be a multiple of the group size")
    if axis not in (0, 1):
        raise ValueError("axis must be 0 or 1")


def quantize_pack(x: np.ndarray, group: int = 64, axis: int = 1):
    """fp16 [rows, cols] -> (codes uint8 [rows, cols/2], params float16 [..., 2] {min, scale}).

    params shape: [rows, cols/group, 2] for axis=1, [rows/group, cols, 2] for axis=0.
    """
    x = np.asarray(x, dtype=np.float16)
    rows, cols = x.shape
    _check(rows, cols, group, axis)
    q, mn, s = quantize_groups(_groups_view(x, group, axis))
    codes = pack_nibbles(_ungroup(q, rows, cols, group, axis))
    if axis == 1:
        params = np.stack([mn, s], axis=-1).reshape(rows, cols // group, 2)
    else:
        params = np.stack([mn, s], axis=-1).reshape(rows // group, cols, 2)
    return codes, params.astype(np.float16)


def dequantize(codes: np.ndarray, params: np.ndarray, rows: int, cols: int, group: int = 64,
               axis: int = 1) -> np.ndarray:
    """Inverse map of ``quantize_pack`` (codes + params -> fp16 [rows, cols])."""
    _check(rows, cols, group, axis)
    q = unpack_nibbles(np.asarray(codes, np.uint8).reshape(rows, cols // 2))
    p = np.asarray(params, np.float16).reshape(-1, 2)
    qg = _groups_view(q, group, axis)
    return _ungroup(dequantize_groups(qg, p[:, 0], p[:, 1]), rows, cols, group, axis)


def storage_bytes(n_elems: int, group: int = 64) -> int:
    """Bytes of the compressed form: n/2 code bytes plus 4 bytes per group."""
    return n_elems // 2 + (n_elems // group) * 4
