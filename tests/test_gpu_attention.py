"""GPU parity of decode attention over the 4-bit cache (K4 + split combine) and of the
causal prefill attention (K5) against the oracle; tolerance max|err| <= 1e-2 * RMS."""
import numpy as np
import pytest

import fg_synth
import oracle
from gpu_util import assert_close_rms, to_dev, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fg():
    import torch
    assert torch.cuda.is_available()
    import bit_group_quantized_fg_b200 as m
    m.lib()
    return m


def _build(fg, B, nh, hd, g, S, seed, dist="normal"):
    """Cache filled by the GPU append from seeded K/V; the oracle cache from the same values."""
    import torch
    h = nh * hd
    k = fg_synth.tensor(seed, 1, (B, S, h), dist, 1.0)
    v = fg_synth.tensor(seed, 2, (B, S, h), dist, 1.0)
    q = fg_synth.tensor(seed, 3, (B, 3 * h), "normal", 1.0)   # q in the first h columns (QKV row)
    cache = fg.DeviceKVCache(B, nh, hd, S + 3, g)
    fg.fg_kv_append(cache, to_dev(k.reshape(B * S, h)), to_dev(v.reshape(B * S, h)), h, S)
    ref = oracle.KVCache(B, nh, hd, g, S + 3)
    oracle.kv_append(ref, k, v, 0)
    ref.length = S
    torch.cuda.synchronize()
    return q, cache, ref


@pytest.mark.parametrize("B,nh,hd,g,S", [
    (4, 12, 64, 64, 36),      # config-1 shape (h 768), a few positions
    (2, 4, 128, 64, 1),       # a single position: output = V
    (3, 2, 128, 32, 300),     # several groups per head
    (2, 3, 128, 128, 77),
    (1, 2, 64, 32, 5000),     # long context, few heads: split over many chunks
    (1, 1, 128, 64, 8192),    # the sweep's longest context
])
def test_decode_attention_matches_oracle(fg, B, nh, hd, g, S):
    q, cache, ref = _build(fg, B, nh, hd, g, S, seed=S + nh)
    import torch
    out = fg.fg_decode_attention(to_dev(q), 3 * nh * hd, cache)
    torch.cuda.synchronize()
    exp = oracle.decode_attention(q[:, :nh * hd], ref, S)
    assert_close_rms(to_np(out), exp, what="decode attention")


def test_decode_attention_t3_and_outliers(fg):
    import torch
    for dist in ("t3", "outlier"):
        q, cache, ref = _build(fg, 2, 4, 128, 64, 129, seed=99, dist=dist)
        out = fg.fg_decode_attention(to_dev(q), 3 * 512, cache)
        torch.cuda.synchronize()
        assert_close_rms(to_np(out), oracle.decode_attention(q[:, :512], ref, 129), what=dist)


@pytest.mark.parametrize("B,nh,S", [
    (64, 32, 543),    # OPT-6.7B shape, batch 64, last decode step
    (256, 56, 543),   # OPT-30B shape, batch 256
    (144, 96, 543),   # OPT-175B shape, batch 144
    (64, 32, 2048),   # a long context with enough sequences x heads for one chunk each
    (64, 32, 8192),   # the sweep's longest context at batch 64: the offset-code cancellation
                      # (64 + c summed over the context, 64 * sum(w) subtracted) at its largest
])
def test_decode_attention_sampled_full_size(fg, B, nh, S):
    """Decode attention at the configurations' full shapes (head dim 128, group 64, context
    543) and at long contexts: sampled sequences checked against the oracle, the rest for
    finiteness."""
    import torch
    hd, g = 128, 64
    h = nh * hd
    from fg_synth import gpu as sg
    kv = torch.empty((B * S, 2 * h), dtype=torch.float16, device="cuda")
    sg.fill(kv, 77, 1, "normal", 1.0)
    q = torch.empty((B, 3 * h), dtype=torch.float16, device="cuda")
    sg.fill(q, 77, 2, "normal", 1.0)
    cache = fg.DeviceKVCache(B, nh, hd, S + 1, g)
    fg.fg_kv_append(cache, kv, kv[:, h:], 2 * h, S)
    out = fg.fg_decode_attention(q, 3 * h, cache)
    torch.cuda.synchronize()
    assert bool(torch.isfinite(out.float()).all())
    for b in (0, B // 2 - 1, B - 1):
        qb = fg_synth.values(77, 2, np.arange(b * 3 * h, b * 3 * h + h), "normal", 1.0, 3 * h).reshape(1, h)
        rows = fg_synth.values(77, 1, np.arange(b * S * 2 * h, (b + 1) * S * 2 * h), "normal", 1.0, 2 * h)
        rows = rows.reshape(1, S, 2 * h)
        ref = oracle.KVCache(1, nh, hd, g, S)
        oracle.kv_append(ref, rows[:, :, :h], rows[:, :, h:], 0)
        exp = oracle.decode_attention(qb, ref, S)
        err, rms = assert_close_rms(to_np(out[b:b + 1]), exp, what=f"row {b}")
        print(f"B {B} nh {nh} S {S} row {b}: max|err| / RMS = {err / rms:.2e}")


@pytest.mark.parametrize("B,L,nh,hd,scale", [
    (4, 32, 12, 64, 1.0), (2, 100, 2, 128, 1.0), (1, 200, 3, 64, 1.0), (2, 64, 1, 128, 1.0),
    (3, 129, 1, 128, 1.0),   # one query past a tile edge
    (2, 300, 2, 128, 1.0),   # three query tiles, ragged tail
    (1, 512, 2, 128, 3.0),   # wide scores: the running maximum is raised from tile to tile
    (2, 257, 2, 64, 3.0),
])
def test_prefill_attention_matches_oracle(fg, B, L, nh, hd, scale):
    import torch
    h = nh * hd
    qkv = fg_synth.tensor(L, nh, (B, L, 3 * h), "normal", scale)
    out = fg.fg_prefill_attention(to_dev(qkv.reshape(B * L, 3 * h)), B, L, nh, hd)
    torch.cuda.synchronize()
    exp = oracle.prefill_attention(qkv, nh, hd)
    err, rms = assert_close_rms(to_np(out).reshape(B, L, h), exp, what="prefill attention")
    print(f"B {B} L {L} nh {nh} hd {hd} scale {scale}: max|err| / RMS = {err / rms:.2e}")


def test_prefill_attention_spike_in_late_tile(fg):
    """A key far later than the first tile that matches every query much better than the
    rest: each row's maximum jumps at that tile and earlier contributions must vanish."""
    import torch
    B, L, nh, hd = 1, 400, 1, 128
    qkv = fg_synth.tensor(5, 5, (B, L, 3 * hd), "normal", 0.5).astype(np.float64)
    qkv[0, :, :hd] = np.abs(qkv[0, :, :hd]) + 0.5          # queries in the positive orthant
    qkv[0, 300, hd:2 * hd] = 4.0                            # key 300: score ~ 4 * sum(q) / sqrt(hd)
    qkv = qkv.astype(np.float16)
    out = fg.fg_prefill_attention(to_dev(qkv.reshape(L, 3 * hd)), B, L, nh, hd)
    torch.cuda.synchronize()
    exp = oracle.prefill_attention(qkv, nh, hd)
    assert_close_rms(to_np(out).reshape(B, L, hd), exp, what="late spike")


def test_prefill_attention_sampled_full_size(fg):
    """The prompt pass of the OPT-6.7B-shaped workload (B 64, L 512, 32 heads x 128): the
    projections are drawn on the device, sampled (sequence, head) pairs are recomputed by
    the oracle from the same seeded values, every output is checked for finiteness."""
    import torch
    from fg_synth import gpu as sg
    B, L, nh, hd = 64, 512, 32, 128
    h = nh * hd
    qkv = torch.empty((B * L, 3 * h), dtype=torch.float16, device="cuda")
    sg.fill(qkv, 91, 4, "normal", 1.0)
    out = fg.fg_prefill_attention(qkv, B, L, nh, hd)
    torch.cuda.synchronize()
    assert bool(torch.isfinite(out.float()).all())
    cols = np.arange(hd)
    for b, j in ((0, 0), (37, 11), (63, 31)):
        rows = np.arange(b * L, (b + 1) * L, dtype=np.int64)[:, None]
        idx = np.concatenate([rows * 3 * h + j * hd + cols, rows * 3 * h + h + j * hd + cols,
                              rows * 3 * h + 2 * h + j * hd + cols], axis=1)
        part = fg_synth.values(91, 4, idx.reshape(-1), "normal", 1.0).reshape(1, L, 3 * hd)
        exp = oracle.prefill_attention(part, 1, hd)
        got = to_np(out[b * L:(b + 1) * L, j * hd:(j + 1) * hd]).reshape(1, L, hd)
        err, rms = assert_close_rms(got, exp, what=f"sequence {b} head {j}")
        print(f"B {B} L {L} sequence {b} head {j}: max|err| / RMS = {err / rms:.2e}")
