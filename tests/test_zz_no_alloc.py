"""The no-allocation decode attention (fg_decode_attention_noalloc) against the regular entry
point that takes a caller workspace.

The variant exists for callers that cannot call cudaMalloc (a host program owning all device
memory through its own pool, or a decode loop that must not allocate); its split-context
scratch is a fixed array inside the library.  This file is collected last so that a failure
here leaves every other test already run; it also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest

import fg_synth
from gpu_util import assert_close_rms, to_dev, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fg():
    import torch
    assert torch.cuda.is_available(), "GPU test"
    import bit_group_quantized_fg_b200 as m
    m.lib()
    return m


def _cache(fg, B, nh, hd, S, seed):
    h = nh * hd
    k = fg_synth.tensor(seed, 1, (B * S, h), "normal", 1.0)
    v = fg_synth.tensor(seed, 2, (B * S, h), "t3", 1.0)
    q = fg_synth.tensor(seed, 3, (B, 3 * h), "normal", 1.0)
    cache = fg.DeviceKVCache(B, nh, hd, S, 64)
    fg.fg_kv_append(cache, to_dev(k), to_dev(v), h, S)
    return to_dev(q), cache


def test_noalloc_matches_workspace_entry_point_twice(fg):
    import torch
    # two calls in a row with different shapes and inputs; both split the context, so the
    # fixed scratch array is really used (and reused) by the second call
    for (B, nh, hd, S, seed) in [(1, 2, 64, 5000, 41), (2, 3, 128, 3000, 42)]:
        assert fg.lib().fg_decode_attention_workspace_bytes(B, nh, hd, S) > 0
        q, cache = _cache(fg, B, nh, hd, S, seed)
        ref = fg.fg_decode_attention(q, 3 * nh * hd, cache)
        out = torch.full((B, nh * hd), float("nan"), dtype=torch.float16, device="cuda")
        st = fg.lib().fg_decode_attention_noalloc(q.data_ptr(), 3 * nh * hd, ctypes.byref(cache.c),
                                                  out.data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert st == 0, fg.lib().fg_last_error()
        torch.cuda.synchronize()
        # the same kernels with the same context split: bit-identical results (an offset into
        # the scratch array that is slightly off would show here)
        assert torch.equal(out, ref), f"no-alloc differs from the workspace entry point (B={B}, S={S})"
        assert_close_rms(to_np(out), to_np(ref), what=f"no-alloc vs workspace (B={B}, S={S})")


def test_noalloc_rejects_shapes_beyond_its_array(fg):
    # every pointer NULL: if a launch path were ever reached before the size check, the host
    # would reject the null pointers (FG_ERR_INVALID_ARG) and nothing would run on the GPU
    c = fg.KVCache(None, None, None, None, 256, 96, 128, 64, 8192, 8192)
    need = fg.lib().fg_decode_attention_workspace_bytes(256, 96, 128, 8192)
    assert need > (4 << 20)
    st = fg.lib().fg_decode_attention_noalloc(None, 3 * 96 * 128, ctypes.byref(c), None, None)
    assert st == -7 and b"no-allocation" in fg.lib().fg_last_error()
