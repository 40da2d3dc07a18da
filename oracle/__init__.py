"""CPU oracle for the 4-bit group-wise compression path and the OPT-shaped decoder.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, calls or links this
package; only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it.  It shares no code with the CUDA
library.

The oracle is a plain, slow C++17 program, ``fg_oracle.cpp`` (built with g++ into
``liboracle.so``, ``-O2 -ffp-contract=off -fno-fast-math``, OpenMP over independent
rows): its own fp16 rounding, the quantizer in IEEE single precision, the decoder in
double precision with fp16 at the storage points.  The Python modules ``quant.py`` and
``decoder.py`` only marshal numpy buffers into it.  ``numpy_ref/`` holds a second,
independent restatement in numpy, kept only as a cross-check of the C++ one.

Sources (pages of the subject, cited by page title and section):

* "FlexGen (giters.com mirror of the FlexGen README)", key-features list ("Extreme
  Compression": weights and attention cache compressed to 4 bits) and the benchmark
  section (workload: input length 512, output length 32; metric: generated tokens /
  (prompt time + generation time)).
* "FlexGen: High-Throughput Generative Inference of Large Language Models with a Single
  GPU" (pith.science record of arXiv 2303.06865), abstract: weights and attention cache
  compressed to 4 bits.
* "Domain-Specific Small Language Models" (Manning liveBook concept page), bullet on
  compressing weights and the attention cache to 4 bits.

The pages give no formula, group size, rounding mode or layout; the readings this
oracle takes where they are silent are listed at the top of ``fg_oracle.cpp`` and in
the module docstrings of ``quant.py`` and ``decoder.py``.
"""
from ._lib import build, threads
from .quant import (quantize_groups, dequantize_groups, pack_nibbles, unpack_nibbles,
                    quantize_pack, dequantize, storage_bytes)
from .decoder import (layernorm, qlinear, linear_fp16, prefill_attention, decode_attention,
                      kv_append, cache_dequant, cache_values, decode_layer, prefill_layer, generate, embed,
                      lm_head_argmax, QLinear, Linear16, QLayer, KVCache, Model)

__all__ = [
    "build", "threads",
    "quantize_groups", "dequantize_groups", "pack_nibbles", "unpack_nibbles",
    "quantize_pack", "dequantize", "storage_bytes", "layernorm", "qlinear", "linear_fp16",
    "prefill_attention", "decode_attention", "kv_append", "cache_dequant", "cache_values", "decode_layer",
    "prefill_layer", "generate", "embed", "lm_head_argmax", "QLinear", "Linear16", "QLayer", "KVCache", "Model",
]
