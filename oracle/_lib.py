"""Loader of the C++ oracle (``fg_oracle.cpp`` -> ``liboracle.so``, built here with g++).

TEST INFRASTRUCTURE ONLY.  This module does argument marshalling (numpy buffers to plain
pointers) and nothing else: every step of what the oracle computes runs in the C++ file.
The library is compiled on first use when it is missing or older than its source, with
``-O2 -ffp-contract=off -fno-fast-math`` (IEEE float and double arithmetic, no FMA
contraction, no reassociation) and OpenMP over independent rows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from ctypes import c_double, c_int, c_int32, c_int64, c_uint16, c_void_p, POINTER

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "fg_oracle.cpp")
LIB = os.path.join(HERE, "liboracle.so")
FLAGS = ["-std=c++17", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-shared", "-fPIC"]

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile liboracle.so when it is missing or older than fg_oracle.cpp."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = f"{LIB}.{os.getpid()}.tmp"
        r = subprocess.run(["g++"] + FLAGS + ["-o", tmp, SRC], capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"g++ failed for the oracle:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, LIB)
    return LIB


class LinearW(ctypes.Structure):
    _fields_ = [("w", c_void_p), ("bias", c_void_p), ("K", c_int), ("N", c_int)]


class Layer(ctypes.Structure):
    _fields_ = [("ln1_g", c_void_p), ("ln1_b", c_void_p), ("ln2_g", c_void_p), ("ln2_b", c_void_p),
                ("qkv", LinearW), ("out", LinearW), ("fc1", LinearW), ("fc2", LinearW)]


class Cache(ctypes.Structure):
    _fields_ = [("k_codes", c_void_p), ("v_codes", c_void_p), ("k_params", c_void_p), ("v_params", c_void_p),
                ("B", c_int), ("n_heads", c_int), ("head_dim", c_int), ("group", c_int), ("capacity", c_int),
                ("len", c_int)]


class Model(ctypes.Structure):
    _fields_ = [("n_layers", c_int), ("hidden", c_int), ("n_heads", c_int), ("head_dim", c_int), ("ffn", c_int),
                ("vocab", c_int), ("max_pos", c_int), ("group", c_int), ("embed", c_void_p),
                ("pos_embed", c_void_p), ("lnf_g", c_void_p), ("lnf_b", c_void_p), ("layers", POINTER(Layer))]


_SIGS = {
    "orc_threads": (c_int, [c_int]),
    "orc_d2h": (c_uint16, [c_double]),
    "orc_h2d": (c_double, [c_uint16]),
    "orc_d2h_array": (None, [c_void_p, c_int64, c_void_p]),
    "orc_quantize_groups": (None, [c_void_p, c_int64, c_int, c_void_p, c_void_p, c_void_p]),
    "orc_dequantize_groups": (None, [c_void_p, c_void_p, c_void_p, c_int64, c_int, c_void_p]),
    "orc_pack_nibbles": (None, [c_void_p, c_int64, c_int64, c_void_p]),
    "orc_unpack_nibbles": (None, [c_void_p, c_int64, c_int64, c_void_p]),
    "orc_quantize_pack": (c_int, [c_void_p, c_int64, c_int64, c_int, c_int, c_void_p, c_void_p]),
    "orc_dequantize": (c_int, [c_void_p, c_void_p, c_int64, c_int64, c_int, c_int, c_void_p]),
    "orc_code_values": (None, [c_void_p, c_void_p, c_int64, c_int64, c_int, c_void_p]),
    "orc_layernorm": (None, [c_void_p, c_int64, c_int, c_void_p, c_void_p, c_double, c_void_p]),
    "orc_linear": (None, [c_void_p, c_int64, c_int64, c_void_p, c_int, c_int, c_void_p, c_int, c_void_p,
                          c_void_p]),
    "orc_linear_nk": (None, [c_void_p, c_int64, c_void_p, c_int, c_int, c_void_p]),
    "orc_argmax": (None, [c_void_p, c_int64, c_int, c_void_p]),
    "orc_prefill_attention": (None, [c_void_p, c_int, c_int, c_int, c_int, c_void_p]),
    "orc_kv_append": (c_int, [POINTER(Cache), c_void_p, c_void_p, c_int64, c_int, c_int]),
    "orc_decode_attention": (None, [c_void_p, c_int64, POINTER(Cache), c_int, c_void_p]),
    "orc_prefill_layer": (c_int, [POINTER(Layer), POINTER(Cache), c_void_p, c_int, c_int]),
    "orc_decode_layer": (c_int, [POINTER(Layer), POINTER(Cache), c_void_p, c_void_p, c_int]),
    "orc_embed": (None, [POINTER(Model), c_void_p, c_int, c_int, c_int, c_void_p]),
    "orc_lm_head_argmax": (None, [POINTER(Model), c_void_p, c_int, c_void_p, c_void_p]),
    "orc_generate": (c_int, [POINTER(Model), c_void_p, c_int, c_int, c_int, c_void_p, POINTER(Cache),
                             c_void_p]),
}


def lib():
    """The loaded oracle library (built first if needed).  FG_ORACLE_LIB names another build
    of fg_oracle.cpp to load instead: the mutation test uses it to run the pins against
    copies of the oracle with planted mistakes."""
    global _lib
    with _lock:
        if _lib is None:
            path = os.environ.get("FG_ORACLE_LIB") or build()
            L = ctypes.CDLL(path)
            for name, (res, args) in _SIGS.items():
                f = getattr(L, name)
                f.restype = res
                f.argtypes = args
            _lib = L
    return _lib


def threads(n: int = 0) -> int:
    """Set the oracle's OpenMP thread count (n > 0) and return the count in use."""
    return int(lib().orc_threads(int(n)))


def p(a):
    """Plain pointer to a C-contiguous numpy buffer (None -> NULL)."""
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle buffers must be C-contiguous"
    return a.ctypes.data_as(c_void_p)


def f16(a):
    return np.ascontiguousarray(a, dtype=np.float16)
