"""Generation with the layers' 4-bit weights in pinned host memory, streamed layer by layer into
two device slots while the previous layer computes (fg_generate_offload; "FlexGen" README
mirror: weights offloaded to CPU memory, pinned, with the block schedule overlapping weight
loading and computation).  The same kernels run on the same values as the resident path, so
the tokens must be identical to fg_generate's, and they are checked against the oracle."""
import ctypes

import numpy as np
import pytest

import fg_synth
import oracle
from gpu_util import compare_free_running, to_dev, to_np
from test_gpu_layer import small_model

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fg():
    import torch
    assert torch.cuda.is_available()
    import bit_group_quantized_fg_b200 as m
    m.lib()
    return m


def offloaded(fg, md):
    """The same model with every layer's tensors copied to pinned host memory."""
    E, P, g1, b1 = md.tensors
    c = md.c
    return fg.DeviceModel(c.n_layers, c.hidden, c.n_heads, c.head_dim, c.ffn, c.vocab, c.max_pos, c.group, E, P,
                          g1, b1, [fg.pinned_layer(l) for l in md.layers])


@pytest.mark.parametrize("n_layers,uncompressed", [(3, False), (1, False), (2, True)])
def test_offloaded_generation_matches_resident_and_oracle(fg, n_layers, uncompressed):
    import torch
    mo, md = small_model(fg, seed=40 + n_layers, n_layers=n_layers, uncompressed=uncompressed)
    mh = offloaded(fg, md)
    B, L, T = 3, 20, 7
    ids = fg_synth.token_ids(40, fg_synth.S_IDS, (B, L), mo.vocab)
    ids_d = to_dev(ids)
    caches = [fg.DeviceKVCache(B, mo.n_heads, mo.head_dim, L + T, 64) for _ in range(n_layers)]
    ref, _ = fg.fg_generate(md, ids_d, T, caches)
    torch.cuda.synchronize()
    ref = to_np(ref)
    caches2 = [fg.DeviceKVCache(B, mo.n_heads, mo.head_dim, L + T, 64) for _ in range(n_layers)]
    for _ in range(2):   # the library's copy stream and slots are reused by a second call
        out, timing, h2d = fg.fg_generate_offload(mh, ids_d, T, caches2)
        torch.cuda.synchronize()
        assert np.array_equal(to_np(out), ref)
        assert all(c.length == L + T - 1 for c in caches2)
        assert timing.tokens == B * T and timing.tok_per_s > 0
    # every layer's tensors crossed once per pass: the prompt pass and T-1 decode steps
    lay = mh.layers[0]
    per_layer = sum(t.numel() * t.element_size() for t in lay.t)
    for q in (lay.qkv, lay.out, lay.fc1, lay.fc2):
        per_layer += sum(t.numel() * t.element_size() for t in (q.codes, q.params, q.bias, q.w16) if t is not None)
    assert h2d == per_layer * n_layers * T
    exp, logits = oracle.generate(mo, ids, T, return_logits=True)
    compare_free_running(to_np(out), exp, logits)


def test_offload_rejects_device_weights(fg):
    """Layer tensors that are not pinned host memory are refused before anything runs."""
    import torch
    mo, md = small_model(fg, seed=50, n_layers=1)
    B, L, T = 2, 8, 3
    ids = to_dev(fg_synth.token_ids(50, fg_synth.S_IDS, (B, L), mo.vocab))
    caches = [fg.DeviceKVCache(B, mo.n_heads, mo.head_dim, L + T, 64)]
    with pytest.raises(fg.FGError) as e:
        fg.fg_generate_offload(md, ids, T, caches)    # weights still in device memory
    assert e.value.status == -1 and "pinned host memory" in str(e.value)
