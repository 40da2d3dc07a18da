"""Second, independent restatement of the oracle in numpy (float32 where the definition
fixes IEEE single precision, float64 elsewhere).  TEST INFRASTRUCTURE ONLY.

The oracle proper is the plain C++ program ``oracle/fg_oracle.cpp``; this numpy version
is kept only as a cross-check that the C++ oracle must match (``tests/test_oracle_crosscheck.py``):
two restatements written in different languages that agree bit for bit on the quantizer
and within float64 summation-order differences on the decoder.
"""
from .quant import (quantize_groups, dequantize_groups, pack_nibbles, unpack_nibbles,
                    quantize_pack, dequantize, storage_bytes)
from .decoder import (layernorm, qlinear, linear_fp16, prefill_attention, decode_attention,
                      kv_append, cache_dequant, cache_values, decode_layer, prefill_layer, generate, embed,
                      lm_head_argmax, QLinear, Linear16, QLayer, KVCache, Model)
