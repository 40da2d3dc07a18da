"""Pins of the decoder oracle (LayerNorm, quantized linear, attention, layer, generate).

Each check is a closed form, an invariant or a special case that reduces to something
known without the oracle's own formula: LayerNorm statistics and affine behaviour,
linear layers with weights exactly on the 4-bit grid, attention with one position /
equal keys / a dominant key / causal independence / permutation invariance, a layer with
zero weights (output = input + out bias + fc2 bias), the generate loop's position
schedule with zero layers and a hand-built embedding, argmax ties, batch-row
independence, the tied LM head on one-hot inputs, and the KV cache layout on grid values.  The readings are those of the OPT decoder block named by the FlexGen
README mirror's benchmark table (OPT-6.7B/30B/175B, input 512, output 32).
"""
import numpy as np
import pytest

import fg_synth
import oracle
from oracle.decoder import QLinear, QLayer, KVCache, Model


def f16(a):
    return np.asarray(a, dtype=np.float16)


# ---------------------------------------------------------------- LayerNorm
def test_layernorm_standardizes():
    x = fg_synth.tensor(1, 2, (16, 768), "normal", 3.0) + f16(5.0)
    y = oracle.layernorm(x, np.ones(768, np.float16), np.zeros(768, np.float16)).astype(np.float64)
    assert np.all(np.abs(y.mean(axis=1)) < 2e-3)
    assert np.all(np.abs(y.var(axis=1) - 1.0) < 2e-3)


def test_layernorm_affine_and_constant_row():
    x = fg_synth.tensor(1, 3, (4, 64), "uniform", 2.0)
    g = np.full(64, 2.0, np.float16)
    b = np.full(64, 1.0, np.float16)
    y1 = oracle.layernorm(x, np.ones(64, np.float16), np.zeros(64, np.float16)).astype(np.float64)
    y2 = oracle.layernorm(x, g, b).astype(np.float64)
    assert np.allclose(y2, 2 * y1 + 1, atol=4e-3)
    c = np.full((1, 64), 7.0, np.float16)
    beta = fg_synth.tensor(1, 4, (64,), "normal", 1.0)
    assert np.array_equal(oracle.layernorm(c, g, beta), beta[None, :])


# ---------------------------------------------------------------- quantized linear
def _grid_linear(K, N, g=64, seed=0):
    """A QLinear built from chosen codes/params, so its weight is known exactly."""
    rng = np.random.default_rng(seed)
    q = rng.integers(0, 16, size=(K, N)).astype(np.uint8)
    mn = f16(rng.integers(-8, 8, size=(K, N // g)) * 0.25)
    s = f16(rng.integers(1, 4, size=(K, N // g)) * 0.125)
    W = q.astype(np.float64) * np.repeat(s.astype(np.float64), g, 1) + np.repeat(mn.astype(np.float64), g, 1)
    codes = oracle.pack_nibbles(q)
    params = np.stack([mn, s], -1)
    b = f16(rng.integers(-4, 4, size=N) * 0.5)
    return QLinear(codes, params, b, K, N, g), W, b.astype(np.float64)


def test_qlinear_picks_rows_and_applies_bias_relu_residual():
    K, N = 64, 128
    lin, W, b = _grid_linear(K, N)
    assert np.array_equal(lin.weight(), W)          # all weights exactly representable
    eye = np.eye(K, dtype=np.float16)
    y = oracle.qlinear(eye, lin).astype(np.float64)
    assert np.array_equal(y, W + b)                  # e_i @ W = row i (catches a transpose)
    yr = oracle.qlinear(eye, lin, relu=True).astype(np.float64)
    assert np.array_equal(yr, np.maximum(W + b, 0))
    res = np.full((K, N), 0.5, np.float16)
    yres = oracle.qlinear(eye, lin, residual16=res).astype(np.float64)
    assert np.array_equal(yres, W + b + 0.5)
    # ReLU applies to X W + b, before the residual is added
    yrr = oracle.qlinear(eye, lin, relu=True, residual16=res).astype(np.float64)
    assert np.array_equal(yrr, np.maximum(W + b, 0) + 0.5)
    assert np.any((W + b < 0) & (W + b > -0.5))       # where the other order would differ
    cols = np.array([0, 1, 63, 64, 127])
    assert np.array_equal(lin.columns(cols), W[:, cols])


def test_qlinear_from_fp16_round_trips_grid_weights():
    K, N = 32, 128
    lin, W, b = _grid_linear(K, N, seed=3)
    lin2 = QLinear.from_fp16(W.astype(np.float16), lin.bias)
    x = fg_synth.tensor(2, 2, (5, K), "normal", 1.0)
    # a grid weight re-quantizes to a weight within s/2 of itself; values compared loosely
    assert np.max(np.abs(lin2.weight() - W)) <= 0.125 / 2 + 1e-9
    y = oracle.qlinear(x, lin2).astype(np.float64)
    assert np.allclose(y, x.astype(np.float64) @ lin2.weight() + b, rtol=1e-3, atol=1e-3)


# ---------------------------------------------------------------- attention
def _cache_with(kv_k, kv_v, nh, hd, g=64):
    B, S, h = kv_k.shape
    c = KVCache(B, nh, hd, g, S + 4)
    oracle.kv_append(c, kv_k, kv_v, 0)
    c.length = S
    return c


def test_decode_attention_single_position_returns_v():
    B, nh, hd = 2, 2, 64
    k = fg_synth.tensor(4, 1, (B, 1, nh * hd), "normal", 1.0)
    v = fg_synth.tensor(4, 2, (B, 1, nh * hd), "normal", 1.0)
    c = _cache_with(k, v, nh, hd)
    q = fg_synth.tensor(4, 3, (B, nh * hd), "normal", 1.0)
    out = oracle.decode_attention(q, c, 1)
    vhat = np.stack([np.concatenate([oracle.cache_values(c, "v", b, j, 1)[0] for j in range(nh)])
                     for b in range(B)])
    assert np.array_equal(out, vhat.astype(np.float16))
    # the exact code values round to the fp16 storage form fg_dequantize writes
    assert np.array_equal(oracle.cache_values(c, "k", 1, 1, 1).astype(np.float16),
                          oracle.cache_dequant(c, "k", 1, 1, 1))


def test_decode_attention_equal_keys_gives_mean_and_dominant_key_selects():
    B, nh, hd, S = 1, 1, 64, 8
    k = np.zeros((B, S, hd), np.float16)
    v = fg_synth.tensor(5, 1, (B, S, hd), "uniform", 1.0)
    c = _cache_with(k, v, nh, hd)
    q = fg_synth.tensor(5, 2, (B, hd), "normal", 1.0)
    out = oracle.decode_attention(q, c, S).astype(np.float64)
    vhat = oracle.cache_values(c, "v", 0, 0, S)
    assert np.allclose(out[0], vhat.mean(axis=0), atol=1e-3)
    # one key aligned with a large query dominates: output = that position's V
    k2 = np.zeros((B, S, hd), np.float16)
    k2[0, 5, :] = 8.0
    c2 = _cache_with(k2, v, nh, hd)
    q2 = np.full((B, hd), 8.0, np.float16)
    out2 = oracle.decode_attention(q2, c2, S).astype(np.float64)
    assert np.allclose(out2[0], oracle.cache_values(c2, "v", 0, 0, S)[5], atol=1e-3)


def test_decode_attention_permutation_invariant():
    B, nh, hd, S = 2, 3, 64, 9
    k = fg_synth.tensor(6, 1, (B, S, nh * hd), "normal", 1.0)
    v = fg_synth.tensor(6, 2, (B, S, nh * hd), "normal", 1.0)
    q = fg_synth.tensor(6, 3, (B, nh * hd), "normal", 1.0)
    perm = np.random.default_rng(0).permutation(S)
    a = oracle.decode_attention(q, _cache_with(k, v, nh, hd), S).astype(np.float64)
    b = oracle.decode_attention(q, _cache_with(k[:, perm], v[:, perm], nh, hd), S).astype(np.float64)
    assert np.allclose(a, b, atol=2e-3)


def test_prefill_attention_causal():
    B, L, nh, hd = 2, 7, 2, 64
    h = nh * hd
    qkv = fg_synth.tensor(7, 1, (B, L, 3 * h), "normal", 1.0)
    out = oracle.prefill_attention(qkv, nh, hd)
    # position 0 sees only itself: output = its own V (fp16 values, one rounding)
    assert np.array_equal(out[:, 0, :], qkv[:, 0, 2 * h:])
    # changing the last token's K and V leaves every earlier position unchanged
    qkv2 = qkv.copy()
    qkv2[:, -1, h:] = f16(3.0)
    out2 = oracle.prefill_attention(qkv2, nh, hd)
    assert np.array_equal(out[:, :-1], out2[:, :-1])
    assert not np.array_equal(out[:, -1], out2[:, -1])
    # heads are independent: zeroing head 1's K/V leaves head 0 alone
    qkv3 = qkv.copy()
    qkv3[:, :, h + hd:2 * h] = 0
    out3 = oracle.prefill_attention(qkv3, nh, hd)
    assert np.array_equal(out[:, :, :hd], out3[:, :, :hd])


# ---------------------------------------------------------------- a whole layer
def _zero_layer(h, F, g=64, bo=0.25, b2=-0.5, b1=1.0):
    def zl(K, N, bval):
        return QLinear.from_fp16(np.zeros((K, N), np.float16), np.full(N, bval, np.float16), g)
    ones, zeros = np.ones(h, np.float16), np.zeros(h, np.float16)
    return QLayer(ones, zeros, ones, zeros, zl(h, 3 * h, 0.0), zl(h, h, bo), zl(h, F, b1), zl(F, h, b2))


def test_zero_weight_layer_is_residual_plus_biases():
    h, F, B = 128, 512, 3
    layer = _zero_layer(h, F)
    x = fg_synth.tensor(8, 1, (B, h), "normal", 1.0)
    cache = KVCache(B, 2, 64, 64, 4)
    y = oracle.decode_layer(layer, cache, x)
    expect = ((x.astype(np.float64) + 0.25).astype(np.float16).astype(np.float64) - 0.5).astype(np.float16)
    assert np.array_equal(y, expect)
    assert cache.length == 1
    xp = fg_synth.tensor(8, 2, (B, 5, h), "normal", 1.0)
    cache2 = KVCache(B, 2, 64, 64, 8)
    yp = oracle.prefill_layer(layer, cache2, xp)
    expect_p = ((xp.astype(np.float64) + 0.25).astype(np.float16).astype(np.float64) - 0.5).astype(np.float16)
    assert np.array_equal(yp, expect_p) and cache2.length == 5


# ---------------------------------------------------------------- generate loop
def _toy_model(n_layers=0, h=16, V=16, max_pos=64):
    E = (4.0 * np.eye(V, h)).astype(np.float16)
    P = np.zeros((max_pos, h), np.float16)
    for pos in range(max_pos):
        P[pos, (3 * pos) % h] = 8.0
    return Model(n_layers, h, 1, h, 4 * h, V, max_pos, 16 if h % 16 == 0 else 2, E, P,
                 np.ones(h, np.float16), np.zeros(h, np.float16), [])


def test_generate_position_schedule_closed_form():
    m = _toy_model()
    B, L, T = 3, 5, 6
    ids = np.array([[1, 2, 3, 4, 5], [0, 0, 0, 0, 0], [9, 8, 7, 6, 5]], np.int32)
    toks = oracle.generate(m, ids, T)
    # token j is produced at position L-1+j, whose positional vector points at 3*pos mod 16
    expect = np.array([[(3 * (L - 1 + j)) % 16 for j in range(T)]] * B)
    assert np.array_equal(toks, expect)


def test_argmax_ties_pick_lowest_id():
    m = _toy_model()
    m.embed = m.embed.copy()
    m.embed[7] = m.embed[2]
    x = np.zeros((1, 16), np.float16)
    x[0, 2] = 5.0
    tok, logits = oracle.lm_head_argmax(m, x)
    assert logits[0, 2] == logits[0, 7] and tok[0] == 2


def test_batch_rows_are_independent():
    rng = np.random.default_rng(0)
    h, nh, F, V, g = 128, 2, 256, 97, 64

    def lin(K, N, s):
        return QLinear.from_fp16(fg_synth.tensor(9, s, (K, N), "normal", 0.05),
                                 fg_synth.tensor(9, s + 100, (N,), "normal", 0.02), g)
    ones, zeros = np.ones(h, np.float16), np.zeros(h, np.float16)
    layers = [QLayer(ones, zeros, ones, zeros, lin(h, 3 * h, 1), lin(h, h, 2), lin(h, F, 3), lin(F, h, 4))]
    m = Model(1, h, nh, h // nh, F, V, 32, g, fg_synth.tensor(9, 50, (V, h), "normal", 0.5),
              fg_synth.tensor(9, 51, (32, h), "normal", 0.1), ones, zeros, layers)
    ids = rng.integers(0, V, size=(4, 6)).astype(np.int32)
    full = oracle.generate(m, ids, 4)
    sub = oracle.generate(m, ids[[3, 1]], 4)
    assert np.array_equal(full[[3, 1]], sub)
    assert full.min() >= 0 and full.max() < V


def test_two_position_attention_is_logistic_of_scaled_score():
    # keys 0 and c*e0, values 0 and 1: output = 1 / (1 + exp(-q.k1 / sqrt(hd)))
    import math
    hd = 64
    k = np.zeros((1, 2, hd), np.float16)
    k[0, 1, 0] = 4.0
    v = np.zeros((1, 2, hd), np.float16)
    v[0, 1, :] = 1.0
    q = np.zeros((1, hd), np.float16)
    q[0, 0] = 2.5
    c = _cache_with(k, v, 1, hd)
    out = oracle.decode_attention(q, c, 2).astype(np.float64)
    expect = 1.0 / (1.0 + math.exp(-2.5 * 4.0 / math.sqrt(hd)))
    assert np.all(np.abs(out - expect) <= 2 ** -11)
    # prefill: query at position 1 sees keys 0 and 1 the same way
    qkv = np.zeros((1, 2, 3 * hd), np.float16)
    qkv[0, 1, 0] = 2.5
    qkv[0, 1, hd] = 4.0
    qkv[0, 1, 2 * hd:] = 1.0
    outp = oracle.prefill_attention(qkv, 1, hd).astype(np.float64)
    assert np.all(np.abs(outp[0, 1] - expect) <= 2 ** -11)


def test_linear16_is_the_plain_product():
    """The uncompressed layer uses the fp16 weight itself: an identity weight returns
    x + b exactly, and a weight on the fp16 grid gives the exact product rounded once."""
    h = 64
    x = fg_synth.tensor(3, 1, (5, h), "normal", 1.0)
    b = fg_synth.tensor(3, 2, (h,), "normal", 0.5)
    eye = np.eye(h, dtype=np.float16)
    y = oracle.qlinear(x, oracle.Linear16(eye, b))
    assert np.array_equal(y, (x.astype(np.float64) + b.astype(np.float64)).astype(np.float16))
    w = (np.arange(h * 8).reshape(h, 8) % 7 - 3).astype(np.float16)   # small integers
    xi = (np.arange(5 * h).reshape(5, h) % 5 - 2).astype(np.float16)
    y2 = oracle.qlinear(xi, oracle.Linear16(w, np.zeros(8, np.float16)), relu=True)
    ref = np.maximum(xi.astype(np.int64) @ w.astype(np.int64), 0).astype(np.float16)
    assert np.array_equal(y2, ref)


# ---------------------------------------------------------------- LM head and cache layout
def test_tied_lm_head_reads_embedding_rows():
    """logits = x E^T over an [V][h] embedding: a one-hot x at feature i returns column i
    of E, one logit per vocabulary row (a transposed operand cannot produce [V] logits from
    a non-square E, nor these values)."""
    V, h = 7, 4
    E = f16(np.arange(V * h).reshape(V, h) * 0.25 - 3.0)
    for i in range(h):
        x = np.zeros((1, h), np.float16)
        x[0, i] = 1.0
        logits = oracle.linear_fp16(x, E)
        assert logits.shape == (1, V)
        assert np.array_equal(logits[0], E[:, i].astype(np.float64))
    x = f16([[1.0, -2.0, 0.5, 4.0]])
    assert np.array_equal(oracle.linear_fp16(x, E)[0],
                          np.array([sum(float(x[0, k]) * float(E[n, k]) for k in range(h)) for n in range(V)]))


def test_kv_append_places_heads_and_positions():
    """Tokens appended at positions pos..pos+T-1 land, head by head, at those positions of
    their (sequence, head) rows; values on the 4-bit grid (min + code * 2^-3 with codes 0..15
    in every group) come back exactly; other positions stay empty."""
    B, nh, hd, g, cap, T, pos = 2, 3, 64, 32, 9, 3, 4
    h = nh * hd
    rng = np.random.default_rng(5)
    codes = np.tile(np.arange(16), h // 16 * B * T).reshape(B, T, h)
    codes = rng.permuted(codes.reshape(-1, g), axis=1).reshape(B, T, h)   # 0..15 in each group
    mins = rng.integers(-8, 8, size=(B, T, h // g)).repeat(g, axis=2) * 0.5
    k = f16(mins + codes * 0.125)
    v = f16(-mins + codes * 0.25)
    cache = KVCache(B, nh, hd, g, cap)
    oracle.kv_append(cache, k, v, pos)
    for b in range(B):
        for j in range(nh):
            kk = oracle.cache_values(cache, "k", b, j, cap)
            vv = oracle.cache_values(cache, "v", b, j, cap)
            for t in range(T):
                assert np.array_equal(kk[pos + t], k[b, t, j * hd:(j + 1) * hd].astype(np.float64))
                assert np.array_equal(vv[pos + t], v[b, t, j * hd:(j + 1) * hd].astype(np.float64))
            untouched = [p for p in range(cap) if not pos <= p < pos + T]
            assert not cache.k_codes[b, j, untouched].any() and not cache.v_params[b, j, untouched].any()


# ---------------------------------------------------------------- LayerNorm epsilon and LN2's input
def test_layernorm_epsilon_inside_the_square_root():
    """A near-constant row 1 +- 2^-8 has variance 2^-16 (the same order as eps = 1e-5), so
    where eps sits shows: y = +-1/sqrt(1 + eps/2^-16) with eps inside the square root,
    +-1/(1 + eps/2^-8) with eps added to the standard deviation, +-1 without it."""
    import math
    d = 2.0 ** -8
    x = np.array([[1.0 + d, 1.0 - d] * 32], np.float16)
    y = oracle.layernorm(x, np.ones(64, np.float16), np.zeros(64, np.float16)).astype(np.float64)
    inside = 1.0 / math.sqrt(1.0 + 1e-5 / d ** 2)
    assert np.all(np.abs(y[0, 0::2] - inside) <= 2.0 ** -11)
    assert np.all(np.abs(y[0, 1::2] + inside) <= 2.0 ** -11)
    for wrong in (1.0, 1.0 / (1.0 + 1e-5 / d)):
        assert np.all(np.abs(y[0, 0::2] - wrong) > 1e-2)


def test_second_layernorm_reads_the_attention_residual():
    """A block with V = 0 (attention output 0), an out-projection bias bo that varies by
    feature, and identity FFN weights: x1 = fp16(x + bo), and the output must be
    fp16(x1 + relu(LN2(x1))).  Feeding LN2 the block input x instead (LayerNorm is not
    shift-invariant for a non-constant bo) gives a different result, which is asserted too."""
    h, F, B, nh = 64, 256, 3, 1
    zeros_h, ones_h = np.zeros(h, np.float16), np.ones(h, np.float16)
    bo = f16(np.linspace(-2.0, 2.0, h))
    w1 = np.zeros((h, F), np.float16)
    w1[np.arange(h), np.arange(h)] = 1.0
    w2 = np.zeros((F, h), np.float16)
    w2[np.arange(h), np.arange(h)] = 1.0
    layer = QLayer(ones_h, zeros_h, ones_h, zeros_h,
                   oracle.Linear16(np.zeros((h, 3 * h), np.float16), np.zeros(3 * h, np.float16)),
                   oracle.Linear16(np.zeros((h, h), np.float16), bo),
                   oracle.Linear16(w1, np.zeros(F, np.float16)),
                   oracle.Linear16(w2, np.zeros(h, np.float16)))
    x = fg_synth.tensor(12, 1, (B, h), "normal", 1.0)
    x1 = (x.astype(np.float64) + bo.astype(np.float64)).astype(np.float16)

    def block_out(ln_in):
        ln = oracle.layernorm(ln_in, ones_h, zeros_h).astype(np.float64)
        return (x1.astype(np.float64) + np.maximum(ln, 0.0)).astype(np.float16)
    expect, wrong = block_out(x1), block_out(x)
    assert not np.array_equal(expect, wrong)
    y = oracle.decode_layer(layer, KVCache(B, nh, h, 64, 2), x)
    assert np.array_equal(y, expect)
    xp = fg_synth.tensor(12, 2, (B, 4, h), "normal", 1.0)
    x1p = (xp.astype(np.float64) + bo.astype(np.float64)).astype(np.float16)
    lnp = oracle.layernorm(x1p, ones_h, zeros_h).astype(np.float64)
    yp = oracle.prefill_layer(layer, KVCache(B, nh, h, 64, 4), xp)
    assert np.array_equal(yp, (x1p.astype(np.float64) + np.maximum(lnp, 0.0)).astype(np.float16))


def test_decode_step_attends_over_the_new_token():
    """All keys zero (uniform attention), V = LN1(x), identity out-projection, zero FFN: a
    decode step after a 3-token prompt outputs fp16(x + fp16(mean of the 4 cached V)), the
    new token's V included; the mean over the 3 prompt positions alone is far from it."""
    h, B, L = 64, 2, 3
    z = np.zeros
    wqkv = z((h, 3 * h), np.float16)
    wqkv[np.arange(h), 2 * h + np.arange(h)] = 1.0          # v = LN1(x); q = k = 0
    ones_h, zeros_h = np.ones(h, np.float16), z(h, np.float16)
    layer = QLayer(ones_h, zeros_h, ones_h, zeros_h,
                   oracle.Linear16(wqkv, z(3 * h, np.float16)),
                   oracle.Linear16(np.eye(h, dtype=np.float16), zeros_h),
                   oracle.Linear16(z((h, 128), np.float16), z(128, np.float16)),
                   oracle.Linear16(z((128, h), np.float16), zeros_h))
    cache = KVCache(B, 1, h, 64, L + 1)
    oracle.prefill_layer(layer, cache, fg_synth.tensor(13, 1, (B, L, h), "normal", 1.0))
    x = fg_synth.tensor(13, 2, (B, h), "normal", 1.0)
    y = oracle.decode_layer(layer, cache, x).astype(np.float64)
    assert cache.length == L + 1
    for b in range(B):
        V = oracle.cache_values(cache, "v", b, 0, L + 1)
        with_new = (x[b].astype(np.float64) + V.mean(axis=0).astype(np.float16)).astype(np.float16)
        without = (x[b].astype(np.float64) + V[:L].mean(axis=0).astype(np.float16)).astype(np.float16)
        assert np.max(np.abs(y[b] - with_new.astype(np.float64))) <= 2.0 ** -9
        assert np.max(np.abs(y[b] - without.astype(np.float64))) > 0.05
