"""Seeded synthetic inputs shared by the tests, the oracle's callers and the bench.

This module holds no arithmetic of the compression method or of the decoder; it only
turns (seed, stream, element index) into input values.  Every element is computable on
its own (counter-based), so a test can regenerate any slice of a multi-gigabyte tensor on
the CPU, and the CUDA twin in ``gen.cu`` (built into ``libfgsynth.so``) produces the same
bits on the GPU for full-size workloads.

Generator definition (both sides implement exactly this):

* ``mix64`` is the SplitMix64 output function (Steele, Lea & Flood, "Fast splittable
  pseudorandom number generators", OOPSLA 2014).
* ``key(seed, stream) = mix64(seed*GAMMA + stream*DELTA)`` (all mod 2**64).
* ``bits(seed, stream, i) = mix64(key + (i+1)*GAMMA)``: 64 random bits for counter i.

Distributions (all exact integer work followed by IEEE-rounded float64 operations):

* normal(sigma): element i uses counters 3i..3i+2, i.e. twelve 16-bit fields v_j.
  S = sum v_j; z = (S - 393210) / 65536 (Irwin-Hall of 12 uniforms (v_j+1/2)/65536,
  mean 0, variance 1); value = fp16(z * sigma), one round-to-nearest-even.
* uniform(lo, hi): u = (bits >> 11) * 2**-53; value = fp16(lo + (hi-lo)*u).
* t3: z0..z3 are normals at element indices 4i..4i+3; chi = z1^2+z2^2+z3^2;
  value = fp16(clip(scale * z0 / sqrt(chi/3), -65504, 65504)) (0 when chi == 0).
* outlier columns: a 2-D [rows, cols] normal(1) tensor whose column j is multiplied by
  50 when ``bits(seed, stream ^ OUTLIER_TAG, j) >> 40`` is divisible by 100 (about 1 %).
* token ids: ``(bits >> 32) % vocab``.
"""
from __future__ import annotations

import numpy as np

MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
DELTA = 0xD1B54A32D192ED03
OUTLIER_TAG = 0x5A5A
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

DIST_NORMAL = 0
DIST_UNIFORM = 1
DIST_T3 = 2
DIST_OUTLIER = 3
DISTS = {"normal": DIST_NORMAL, "uniform": DIST_UNIFORM, "t3": DIST_T3, "outlier": DIST_OUTLIER}


def _mix64(z: np.ndarray) -> np.ndarray:
    z = z.astype(np.uint64, copy=True)
    z ^= z >> np.uint64(30)
    z *= _M1
    z ^= z >> np.uint64(27)
    z *= _M2
    z ^= z >> np.uint64(31)
    return z


def mix64_int(z: int) -> int:
    z &= MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def key(seed: int, stream: int) -> int:
    return mix64_int((seed * GAMMA + stream * DELTA) & MASK64)


def bits(seed: int, stream: int, idx) -> np.ndarray:
    """64 random bits for each counter in ``idx`` (int64/uint64 array)."""
    k = np.uint64(key(seed, stream))
    i = np.asarray(idx, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix64(k + (i + np.uint64(1)) * np.uint64(GAMMA))


def _normal_z(seed: int, stream: int, idx: np.ndarray) -> np.ndarray:
    """Irwin-Hall(12) standard normal as exact float64 multiples of 2**-16."""
    idx = np.asarray(idx, dtype=np.uint64)
    s = np.zeros(idx.shape, dtype=np.int64)
    for c in range(3):
        b = bits(seed, stream, idx * np.uint64(3) + np.uint64(c))
        for f in range(4):
            s += ((b >> np.uint64(16 * f)) & np.uint64(0xFFFF)).astype(np.int64)
    return (s - 393210).astype(np.float64) / 65536.0


def values(seed: int, stream: int, idx, dist: str = "normal", scale: float = 1.0,
           cols: int = 0) -> np.ndarray:
    """fp16 values of the flat element indices ``idx`` (see module docstring).

    ``scale`` is sigma for 'normal', the half-width for 'uniform' (U(-scale, scale)),
    a multiplier for 't3'; ``cols`` is the row length for 'outlier'.
    """
    idx = np.asarray(idx, dtype=np.int64)
    if dist == "normal":
        v = _normal_z(seed, stream, idx) * np.float64(scale)
    elif dist == "uniform":
        u = (bits(seed, stream, idx) >> np.uint64(11)).astype(np.float64) * 2.0 ** -53
        v = -np.float64(scale) + (2.0 * np.float64(scale)) * u
    elif dist == "t3":
        i4 = idx.astype(np.uint64) * np.uint64(4)
        z0 = _normal_z(seed, stream, i4)
        z1 = _normal_z(seed, stream, i4 + np.uint64(1))
        z2 = _normal_z(seed, stream, i4 + np.uint64(2))
        z3 = _normal_z(seed, stream, i4 + np.uint64(3))
        chi = z1 * z1 + z2 * z2
        chi = chi + z3 * z3
        den = np.sqrt(chi / 3.0)
        with np.errstate(divide="ignore", invalid="ignore"):
            v = np.where(chi == 0.0, 0.0, z0 / np.where(den == 0.0, 1.0, den))
        v = np.clip(v * np.float64(scale), -65504.0, 65504.0)   # keep every value finite in fp16
    elif dist == "outlier":
        if cols <= 0:
            raise ValueError("outlier distribution needs cols > 0")
        col = idx % cols
        tag = bits(seed, stream ^ OUTLIER_TAG, col) >> np.uint64(40)
        mult = np.where(tag % np.uint64(100) == 0, 50.0, 1.0)
        v = _normal_z(seed, stream, idx) * mult * np.float64(scale)
    else:
        raise ValueError(f"unknown distribution {dist!r}")
    return v.astype(np.float16)


def tensor(seed: int, stream: int, shape, dist: str = "normal", scale: float = 1.0,
           offset: int = 0) -> np.ndarray:
    """A whole fp16 tensor whose flat element i is ``values(..., offset + i)``."""
    n = int(np.prod(shape))
    cols = int(shape[-1]) if len(shape) else 1
    return values(seed, stream, np.arange(offset, offset + n, dtype=np.int64), dist, scale,
                  cols).reshape(shape)


def token_ids(seed: int, stream: int, shape, vocab: int) -> np.ndarray:
    n = int(np.prod(shape))
    b = bits(seed, stream, np.arange(n, dtype=np.int64))
    return ((b >> np.uint64(32)) % np.uint64(vocab)).astype(np.int32).reshape(shape)


# Stream ids of the decoder's tensors: layer l uses 64*l + kind.
S_LN1_G, S_LN1_B, S_LN2_G, S_LN2_B = 0, 1, 2, 3
S_WQKV, S_BQKV, S_WO, S_BO, S_W1, S_B1, S_W2, S_B2 = 4, 5, 6, 7, 8, 9, 10, 11
S_EMBED, S_POS, S_LNF_G, S_LNF_B = 1 << 20, (1 << 20) + 1, (1 << 20) + 2, (1 << 20) + 3
S_IDS, S_HIDDEN, S_DECODE_X = (1 << 20) + 4, (1 << 20) + 5, (1 << 20) + 6


def layer_stream(layer: int, kind: int) -> int:
    return 64 * layer + kind
