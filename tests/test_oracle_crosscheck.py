"""The C++ oracle against the second, independent numpy restatement (``oracle.numpy_ref``).

Both restate the same definition in different languages and share nothing but the seeded
inputs.  The quantizer, dequantizer, packing, KV append and embedding are bit-exact (both
take every rounding in the same precision); LayerNorm, the linear layer, both attentions
and the layers accumulate float64 sums in different orders (loops here, BLAS and pairwise
sums there), so their fp16 results may differ by one unit in the last place, rarely.
"""
import numpy as np
import pytest

import fg_synth
import oracle
from oracle import numpy_ref as ref


def ulp_diff(a, b):
    """Largest distance in fp16 units in the last place (same-sign finite values)."""
    ia = np.asarray(a, np.float16).view(np.int16).astype(np.int64)
    ib = np.asarray(b, np.float16).view(np.int16).astype(np.int64)
    ia = np.where(ia < 0, -(ia & 0x7FFF), ia)
    ib = np.where(ib < 0, -(ib & 0x7FFF), ib)
    return int(np.max(np.abs(ia - ib))) if ia.size else 0


def close16(a, b, frac=0.99):
    a = np.asarray(a, np.float16)
    b = np.asarray(b, np.float16)
    assert a.shape == b.shape
    assert ulp_diff(a, b) <= 1
    assert np.mean(a.view(np.uint16) == b.view(np.uint16)) >= frac


@pytest.mark.parametrize("dist,scale", [("normal", 0.02), ("uniform", 1.0), ("t3", 1.0), ("outlier", 1.0)])
@pytest.mark.parametrize("g,axis", [(32, 1), (64, 1), (128, 1), (64, 0)])
def test_quantizer_bit_exact(dist, scale, g, axis):
    x = fg_synth.tensor(g + axis, 5, (256, 384), dist, scale)
    c1, p1 = oracle.quantize_pack(x, g, axis)
    c2, p2 = ref.quantize_pack(x, g, axis)
    assert np.array_equal(c1, c2)
    assert np.array_equal(p1.view(np.uint16), p2.view(np.uint16))
    d1 = oracle.dequantize(c1, p1, 256, 384, g, axis)
    d2 = ref.dequantize(c2, p2, 256, 384, g, axis)
    assert np.array_equal(d1.view(np.uint16), d2.view(np.uint16))


def test_edge_groups_bit_exact():
    vals = [0.0, -0.0, 65504.0, -65504.0, 2.0 ** -24, -(2.0 ** -24), 6.1e-5, 1.0, -1.0, 0.5]
    rng = np.random.default_rng(1)
    rows = [np.full(64, v, np.float16) for v in vals]
    rows += [rng.choice(np.array(vals, np.float16), 64) for _ in range(40)]
    x = np.stack(rows)
    a = oracle.quantize_groups(x)
    b = ref.quantize_groups(x)
    for u, v in zip(a, b):
        assert np.array_equal(np.asarray(u).view(np.uint8 if u.dtype == np.uint8 else np.uint16),
                              np.asarray(v).view(np.uint8 if v.dtype == np.uint8 else np.uint16))
    assert np.array_equal(oracle.dequantize_groups(*a).view(np.uint16), ref.dequantize_groups(*b).view(np.uint16))


def test_layernorm_and_linear():
    x = fg_synth.tensor(2, 1, (40, 512), "t3", 1.0)
    g = fg_synth.tensor(2, 2, (512,), "normal", 0.5)
    b = fg_synth.tensor(2, 3, (512,), "normal", 0.5)
    close16(oracle.layernorm(x, g, b), ref.layernorm(x, g, b))
    w = fg_synth.tensor(2, 4, (512, 384), "normal", 0.05)
    bias = fg_synth.tensor(2, 5, (384,), "normal", 0.2)
    r = fg_synth.tensor(2, 6, (40, 384), "normal", 1.0)
    l1 = oracle.QLinear.from_fp16(w, bias, 64)
    l2 = ref.QLinear.from_fp16(w, bias, 64)
    for relu, res in ((False, None), (True, r)):
        close16(oracle.qlinear(x, l1, relu=relu, residual16=res), ref.qlinear(x, l2, relu=relu, residual16=res))
    close16(oracle.qlinear(x, oracle.Linear16(w, bias)), ref.qlinear(x, ref.Linear16(w, bias)))
    E = fg_synth.tensor(2, 7, (100, 512), "normal", 0.5)
    la, lb = oracle.linear_fp16(x, E), ref.linear_fp16(x, E)
    assert np.max(np.abs(la - lb)) <= 1e-12 * np.max(np.abs(lb))


def test_attention_and_cache():
    B, L, nh, hd, g = 2, 33, 2, 64, 32
    h = nh * hd
    qkv = fg_synth.tensor(3, 1, (B, L, 3 * h), "normal", 1.0)
    close16(oracle.prefill_attention(qkv, nh, hd), ref.prefill_attention(qkv, nh, hd))
    c1 = oracle.KVCache(B, nh, hd, g, L + 2)
    c2 = ref.KVCache(B, nh, hd, g, L + 2)
    oracle.kv_append(c1, qkv[:, :, h:2 * h], qkv[:, :, 2 * h:], 1)
    ref.kv_append(c2, qkv[:, :, h:2 * h], qkv[:, :, 2 * h:], 1)
    for a, b in ((c1.k_codes, c2.k_codes), (c1.v_codes, c2.v_codes)):
        assert np.array_equal(a, b)
    for a, b in ((c1.k_params, c2.k_params), (c1.v_params, c2.v_params)):
        assert np.array_equal(a.view(np.uint16), b.view(np.uint16))
    assert np.array_equal(oracle.cache_values(c1, "v", 1, 1, L + 1), ref.cache_values(c2, "v", 1, 1, L + 1))
    q = fg_synth.tensor(3, 2, (B, 3 * h), "normal", 1.0)
    close16(oracle.decode_attention(q, c1, L + 1), ref.decode_attention(q[:, :h], c2, L + 1))


def _models(seed=4, n_layers=2, h=128, nh=2, F=256, V=300, max_pos=40, g=64):
    mods = []
    for lib in (oracle, ref):
        layers = []
        for l in range(n_layers):
            ws = [fg_synth.tensor(seed, 10 * l + i, s, "normal", 0.05)
                  for i, s in enumerate([(h, 3 * h), (h, h), (h, F), (F, h)])]
            bs = [fg_synth.tensor(seed, 10 * l + 5 + i, (w.shape[1],), "normal", 0.02) for i, w in enumerate(ws)]
            ln = [fg_synth.tensor(seed, 100 + 4 * l + i, (h,), "normal", 0.1) + np.float16(1.0 if i % 2 == 0 else 0.0)
                  for i in range(4)]
            layers.append(lib.QLayer(*ln, *[lib.QLinear.from_fp16(w, b, g) for w, b in zip(ws, bs)]))
        E = fg_synth.tensor(seed, 200, (V, h), "normal", 0.5)
        P = fg_synth.tensor(seed, 201, (max_pos, h), "normal", 0.1)
        mods.append(lib.Model(n_layers, h, nh, h // nh, F, V, max_pos, g, E, P,
                              np.ones(h, np.float16), np.zeros(h, np.float16), layers))
    return mods


def test_layers_embedding_and_generation():
    mo, mr = _models()
    B, L, T = 3, 12, 6
    ids = fg_synth.token_ids(4, 9, (B, L), mo.vocab)
    assert np.array_equal(oracle.embed(mo, ids, 2).view(np.uint16), ref.embed(mr, ids, 2).view(np.uint16))
    x = fg_synth.tensor(4, 300, (B, L, mo.hidden), "normal", 1.0)
    c1 = oracle.KVCache(B, mo.n_heads, mo.head_dim, mo.group, L + 1)
    c2 = ref.KVCache(B, mr.n_heads, mr.head_dim, mr.group, L + 1)
    close16(oracle.prefill_layer(mo.layers[0], c1, x), ref.prefill_layer(mr.layers[0], c2, x))
    xd = fg_synth.tensor(4, 301, (B, mo.hidden), "normal", 1.0)
    close16(oracle.decode_layer(mo.layers[0], c1, xd), ref.decode_layer(mr.layers[0], c2, xd))
    t1, lg1 = oracle.generate(mo, ids, T, return_logits=True)
    t2, lg2 = ref.generate(mr, ids, T, return_logits=True)
    assert np.array_equal(t1, t2)
    assert np.max(np.abs(lg1 - lg2)) <= 1e-2 * np.sqrt(np.mean(lg2 ** 2))
