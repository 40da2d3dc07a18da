"""GPU twin of the seeded input generator (build + ctypes wrapper over gen.cu).

Produces on the device exactly the bits ``fg_synth.values`` produces on the host, so
full-size workloads are generated in HBM while tests regenerate any slice on the CPU.
"""
from __future__ import annotations

import ctypes
import os
import shutil
import subprocess

from . import DISTS

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "gen.cu")
LIB = os.path.join(HERE, "libfgsynth.so")
_lib = None


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    nvcc = "/usr/local/cuda/bin/nvcc" if os.path.exists("/usr/local/cuda/bin/nvcc") else shutil.which("nvcc")
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-Xcompiler", "-fPIC",
           "-shared", "-cudart", "static", SRC, "-o", LIB + ".tmp"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for gen.cu:\n{r.stdout}\n{r.stderr}")
    os.replace(LIB + ".tmp", LIB)
    return LIB


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            build()
        _lib = ctypes.CDLL(LIB)
        _lib.fgsynth_fill.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int, ctypes.c_double,
                                      ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                      ctypes.c_void_p]
        _lib.fgsynth_ids.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64, ctypes.c_int,
                                     ctypes.c_void_p, ctypes.c_void_p]
    return _lib


def fill(out, seed: int, stream: int, dist: str = "normal", scale: float = 1.0, offset: int = 0,
         cols: int = 0, cuda_stream=None) -> None:
    """Fill a contiguous fp16 torch tensor on the GPU with fg_synth values."""
    import torch
    assert out.dtype == torch.float16 and out.is_cuda and out.is_contiguous()
    if cols <= 0:
        cols = int(out.shape[-1]) if out.dim() else 1
    s = cuda_stream if cuda_stream is not None else torch.cuda.current_stream().cuda_stream
    rc = lib().fgsynth_fill(seed, stream, DISTS[dist], float(scale), cols, offset, out.numel(),
                            out.data_ptr(), s)
    if rc != 0:
        raise RuntimeError(f"fgsynth_fill failed ({rc})")


def fill_ids(out, seed: int, stream: int, vocab: int, cuda_stream=None) -> None:
    import torch
    assert out.dtype == torch.int32 and out.is_cuda and out.is_contiguous()
    s = cuda_stream if cuda_stream is not None else torch.cuda.current_stream().cuda_stream
    rc = lib().fgsynth_ids(seed, stream, out.numel(), vocab, out.data_ptr(), s)
    if rc != 0:
        raise RuntimeError(f"fgsynth_ids failed ({rc})")
