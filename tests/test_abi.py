"""CPU checks of the C ABI: the library builds/loads, exports every call include/fg.h
declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    src = open(os.path.join(ROOT, "include", "fg.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(fg_[a-z0-9_]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def fg():
    from bit_group_quantized_fg_b200 import build
    build.build()
    import bit_group_quantized_fg_b200 as m
    return m


def test_header_declares_the_boundary_calls():
    names = header_functions()
    for required in ("fg_quantize_pack", "fg_dequantize", "fg_decode_layer", "fg_generate", "fg_workspace_bytes"):
        assert required in names


def test_library_exports_every_declared_symbol(fg):
    lib = fg.lib()
    missing = [n for n in header_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(header_functions()) == set(fg._SIGS), "binding signature table out of sync with fg.h"


def test_status_strings(fg):
    lib = fg.lib()
    assert lib.fg_status_string(0) == b"ok"
    assert lib.fg_status_string(-4) == b"KV cache capacity exceeded"
    assert lib.fg_version() > 0


def test_host_validation_rejects_without_launch(fg):
    lib = fg.lib()
    fake = 0x10000  # aligned, never dereferenced: validation fails first
    assert lib.fg_quantize_pack(None, 64, 64, 64, 1, fake, fake, None) == -1
    assert lib.fg_quantize_pack(None, 0, 64, 64, 1, None, None, None) == 0       # empty: nothing touched
    assert lib.fg_quantize_pack(fake, 64, 64, 48, 1, fake, fake, None) == -2      # group 48
    assert lib.fg_quantize_pack(fake, 64, 96, 64, 1, fake, fake, None) == -2      # cols % group
    assert lib.fg_quantize_pack(fake, 96, 64, 64, 0, fake, fake, None) == -2      # rows % group (axis 0)
    assert lib.fg_quantize_pack(fake + 8, 64, 64, 64, 1, fake, fake, None) == -3  # misaligned
    assert lib.fg_dequantize(fake, fake, 64, 60, 32, 1, fake, None) == -2         # cols % 8
    assert b"group" in lib.fg_last_error() or b"cols" in lib.fg_last_error()


def test_kv_append_capacity_overflow_is_reported(fg):
    lib = fg.lib()
    fake = 0x10000
    c = fg.KVCache(fake, fake, fake, fake, 2, 4, 64, 64, 8, 7)
    assert lib.fg_kv_append(ctypes.byref(c), fake, fake, 256, 2, None) == -4
    assert c.len == 7
    c2 = fg.KVCache(fake, fake, fake, fake, 2, 4, 64, 48, 8, 0)   # group does not divide head_dim
    assert lib.fg_kv_append(ctypes.byref(c2), fake, fake, 256, 1, None) == -2


def test_gemm_shape_checks(fg):
    lib = fg.lib()
    fake = 0x10000
    w = fg.QLinear(fake, fake, None, 100, 256, 64)       # K not a multiple of 64
    assert lib.fg_qgemm(fake, 4, ctypes.byref(w), None, 0, fake, None, 0, None) == -2
    w = fg.QLinear(fake, fake, None, 128, 200, 64)       # N not a multiple of 256
    assert lib.fg_qgemm(fake, 4, ctypes.byref(w), None, 0, fake, None, 0, None) == -2


def test_workspace_size_queries(fg):
    lib = fg.lib()
    assert lib.fg_decode_layer_workspace_bytes(4096, 16384, 32, 64, 544) > 0
    assert lib.fg_prefill_layer_workspace_bytes(768, 3072, 4, 32) > 0
    assert lib.fg_lm_head_workspace_bytes(64, 50272) >= 64 * 50272 * 4


def test_prefill_attention_and_layernorm_checks(fg):
    lib = fg.lib()
    fake = 0x10000
    assert lib.fg_prefill_attention(None, 2, 64, 4, 128, fake, None) == -1
    assert lib.fg_prefill_attention(fake, 0, 64, 4, 128, fake, None) == -2
    assert lib.fg_prefill_attention(fake, 2, 64, 4, 96, fake, None) == -6          # head_dim 96
    assert lib.fg_prefill_attention(fake, 1 << 16, 1 << 15, 4, 128, fake, None) == -2  # B*L >= 2^31
    assert lib.fg_prefill_attention(fake + 8, 2, 64, 4, 128, fake, None) == -3
    assert lib.fg_layernorm(fake, 4, 100, fake, fake, fake, None) == -2            # cols % 8
    assert lib.fg_layernorm(fake, 4, 16384, fake, fake, fake, None) == -6          # above 12288
    assert lib.fg_layernorm(fake + 4, 4, 4096, fake, fake, fake, None) == -3
    assert lib.fg_layernorm(fake, 0, 4096, fake, fake, fake, None) == 0             # no rows: no launch
