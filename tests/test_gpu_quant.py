"""GPU parity of quantize/pack (K1), dequantize (K2) and KV append against the oracle.
Codes and params must be bit-exact; dequantized values bit-exact."""
import numpy as np
import pytest

import fg_synth
import oracle
from gpu_util import to_dev, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fg():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_group_quantized_fg_b200 as m
    m.lib()
    return m


def _check_pack(fg, x, g, axis):
    import torch
    codes, params = fg.fg_quantize_pack(to_dev(x), g, axis)
    torch.cuda.synchronize()
    c_ref, p_ref = oracle.quantize_pack(x, g, axis)
    c_got, p_got = to_np(codes), to_np(params)
    assert np.array_equal(c_got, c_ref)
    assert np.array_equal(p_got.view(np.uint16), p_ref.view(np.uint16))
    d = fg.fg_dequantize(codes, params, x.shape[0], x.shape[1], g, axis)
    torch.cuda.synchronize()
    d_ref = oracle.dequantize(c_ref, p_ref, x.shape[0], x.shape[1], g, axis)
    assert np.array_equal(to_np(d).view(np.uint16), d_ref.view(np.uint16))


@pytest.mark.parametrize("dist,scale", [("normal", 0.02), ("normal", 1.0), ("uniform", 1.0), ("t3", 1.0),
                                        ("outlier", 1.0)])
@pytest.mark.parametrize("g", [32, 64, 128])
def test_pack_bit_exact_axis1(fg, dist, scale, g):
    # 37 rows x 1536 cols: several CTAs' tiles plus a ragged last tile
    x = fg_synth.tensor(21, 7, (37, 1536), dist, scale)
    _check_pack(fg, x, g, 1)


@pytest.mark.parametrize("g", [32, 64, 128])
def test_pack_bit_exact_axis0(fg, g):
    x = fg_synth.tensor(22, 8, (2 * g, 520), "t3", 1.0)
    _check_pack(fg, x, g, 0)


def test_pack_edge_values(fg):
    rows = []
    for v in [0.0, -0.0, 1.0, -3.5, 65504.0, -65504.0, 2.0 ** -24, -(2.0 ** -20)]:
        rows.append(np.full(128, v))                      # constant groups
    r = np.linspace(-65504, 65504, 128)                   # full fp16 range in one group
    rows.append(r)
    rows.append(np.concatenate([np.zeros(127), [2.0 ** -24]]))   # underflowing scale
    t = np.zeros(128)
    t[::2] = 15.0
    t[1::4] = 2.5
    t[3::4] = 3.5                                          # exact half ties
    rows.append(t)
    x = np.array(rows, dtype=np.float16)
    for g in (32, 64, 128):
        _check_pack(fg, x, g, 1)


def test_pack_empty_and_tiny(fg):
    import torch
    x = np.zeros((0, 64), np.float16)
    codes, params = fg.fg_quantize_pack(torch.zeros((0, 64), dtype=torch.float16, device="cuda"), 64, 1)
    assert codes.numel() == 0 and params.numel() == 0
    _check_pack(fg, fg_synth.tensor(1, 1, (1, 64), "normal", 1.0), 64, 1)
    _check_pack(fg, fg_synth.tensor(1, 2, (1, 32), "uniform", 1.0), 32, 1)


@pytest.mark.slow
def test_pack_large_sampled(fg):
    """A 1 GiB fp16 tensor (2^29 elements) generated on the GPU; sampled rows vs the oracle,
    and a whole-tensor invariant: dequantized error within s/2 + half an fp16 ulp."""
    import torch
    from fg_synth import gpu as sg
    rows, cols = 131072, 4096
    x = torch.empty((rows, cols), dtype=torch.float16, device="cuda")
    sg.fill(x, 5, 3, "outlier")
    codes, params = fg.fg_quantize_pack(x, 64, 1)
    torch.cuda.synchronize()
    for r in [0, 1, 4097, rows // 2 + 3, rows - 1]:
        xr = fg_synth.values(5, 3, np.arange(r * cols, (r + 1) * cols), "outlier", 1.0, cols)[None, :]
        assert np.array_equal(to_np(x[r:r + 1]).view(np.uint16), xr.view(np.uint16))
        c_ref, p_ref = oracle.quantize_pack(xr, 64, 1)
        assert np.array_equal(to_np(codes[r:r + 1]), c_ref)
        assert np.array_equal(to_np(params[r:r + 1]).view(np.uint16), p_ref.view(np.uint16))
    d = fg.fg_dequantize(codes, params, rows, cols, 64, 1)
    s = params[..., 1].float().repeat_interleave(64, dim=1)
    err = (d.float() - x.float()).abs()
    ulp = torch.exp2(torch.floor(torch.log2(torch.clamp(d.float().abs(), min=2.0 ** -14))) - 10)
    assert bool((err <= s * 0.5 * (1 + 2.0 ** -20) + 0.5 * ulp).all())


def test_synth_gpu_twin_matches_cpu(fg):
    import torch
    from fg_synth import gpu as sg
    for dist, scale in [("normal", 0.02), ("uniform", 1.0), ("t3", 1.0), ("outlier", 1.0)]:
        x = torch.empty((33, 256), dtype=torch.float16, device="cuda")
        sg.fill(x, 9, 4, dist, scale, offset=1000)
        torch.cuda.synchronize()
        ref = fg_synth.values(9, 4, np.arange(1000, 1000 + x.numel()), dist, scale, 256).reshape(33, 256)
        assert np.array_equal(to_np(x).view(np.uint16), ref.view(np.uint16)), dist
    ids = torch.empty((4, 50), dtype=torch.int32, device="cuda")
    sg.fill_ids(ids, 3, 2, 50272)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(ids), fg_synth.token_ids(3, 2, (4, 50), 50272))


@pytest.mark.parametrize("hd,g", [(64, 64), (128, 64), (128, 32), (128, 128)])
def test_kv_append_bit_exact(fg, hd, g):
    import torch
    B, nh, T, cap = 3, 5, 7, 16
    h = nh * hd
    kv = fg_synth.tensor(31, hd + g, (B * T, 3 * h), "normal", 1.0)   # rows like a QKV output
    dev = to_dev(kv)
    cache = fg.DeviceKVCache(B, nh, hd, cap, g)
    cache.length = 2
    fg.fg_kv_append(cache, dev[:, h:], dev[:, 2 * h:], 3 * h, T)
    torch.cuda.synchronize()
    assert cache.length == 9
    ref = oracle.KVCache(B, nh, hd, g, cap)
    oracle.kv_append(ref, kv[:, h:2 * h].reshape(B, T, h), kv[:, 2 * h:].reshape(B, T, h), 2)
    assert np.array_equal(to_np(cache.k_codes)[:, :, 2:9], ref.k_codes[:, :, 2:9])
    assert np.array_equal(to_np(cache.v_codes)[:, :, 2:9], ref.v_codes[:, :, 2:9])
    assert np.array_equal(to_np(cache.k_params)[:, :, 2:9].view(np.uint16), ref.k_params[:, :, 2:9].view(np.uint16))
    assert np.array_equal(to_np(cache.v_params)[:, :, 2:9].view(np.uint16), ref.v_params[:, :, 2:9].view(np.uint16))
    # positions outside the appended range untouched
    assert not to_np(cache.k_codes)[:, :, :2].any() and not to_np(cache.k_codes)[:, :, 9:].any()
    with pytest.raises(fg.FGError):
        fg.fg_kv_append(cache, dev[:, h:], dev[:, 2 * h:], 3 * h, T + 1)   # 9 + 8 > 16 (rejected before launch)
    assert cache.length == 9


@pytest.mark.slow
def test_pack_beyond_2pow31_elements_sampled(fg):
    """A tensor of 2^31 + 2^18 fp16 elements (4 GiB + 512 KiB): rows on both sides of
    element 2^31 against the oracle, codes, params and dequantized values bit for bit."""
    import torch
    from fg_synth import gpu as sg
    rows, cols = 524288 + 64, 4096
    x = torch.empty((rows, cols), dtype=torch.float16, device="cuda")
    sg.fill(x, 6, 3, "normal", 0.02)
    codes, params = fg.fg_quantize_pack(x, 64, 1)
    d = fg.fg_dequantize(codes, params, rows, cols, 64, 1)
    torch.cuda.synchronize()
    for r in [0, 524287, 524288, rows - 1]:
        xr = fg_synth.values(6, 3, np.arange(r * cols, (r + 1) * cols), "normal", 0.02)[None, :]
        assert np.array_equal(to_np(x[r:r + 1]).view(np.uint16), xr.view(np.uint16))
        c_ref, p_ref = oracle.quantize_pack(xr, 64, 1)
        assert np.array_equal(to_np(codes[r:r + 1]), c_ref)
        assert np.array_equal(to_np(params[r:r + 1]).view(np.uint16), p_ref.view(np.uint16))
        d_ref = oracle.dequantize(c_ref, p_ref, 1, cols, 64, 1)
        assert np.array_equal(to_np(d[r:r + 1]).view(np.uint16), d_ref.view(np.uint16))


def _kv_rows(seed, stream, b, T, h, part):
    """K (part 1) or V (part 2) rows of sequence b of a [B*T][3h] projection tensor drawn
    with fg_synth (the CPU twin of the values the GPU generator wrote)."""
    rows = np.arange(b * T, (b + 1) * T, dtype=np.int64)[:, None]
    idx = rows * 3 * h + part * h + np.arange(h, dtype=np.int64)[None, :]
    return fg_synth.values(seed, stream, idx.reshape(-1), "normal", 1.0).reshape(T, h)


def test_kv_append_prompt_size_sampled(fg):
    """A prompt pass's append (16 sequences x 512 tokens x 32 heads of 128, 2.1 M chunks, the
    path the full-size prompt takes) at cache offset 3: sampled sequences bit-exact against
    the oracle, untouched positions still empty."""
    import torch
    from fg_synth import gpu as sg
    B, T, nh, hd, g, off = 16, 512, 32, 128, 64, 3
    h = nh * hd
    qkv = torch.empty((B * T, 3 * h), dtype=torch.float16, device="cuda")
    sg.fill(qkv, 44, 9, "normal", 1.0)
    cache = fg.DeviceKVCache(B, nh, hd, T + 8, g)
    cache.length = off
    fg.fg_kv_append(cache, qkv[:, h:], qkv[:, 2 * h:], 3 * h, T)
    torch.cuda.synchronize()
    assert cache.length == off + T
    for b in (0, 7, B - 1):
        k = _kv_rows(44, 9, b, T, h, 1)
        v = _kv_rows(44, 9, b, T, h, 2)
        ref = oracle.KVCache(1, nh, hd, g, T + 8)
        oracle.kv_append(ref, k[None], v[None], off)
        sl = slice(off, off + T)
        assert np.array_equal(to_np(cache.k_codes[b, :, sl]), ref.k_codes[0, :, sl])
        assert np.array_equal(to_np(cache.v_codes[b, :, sl]), ref.v_codes[0, :, sl])
        assert np.array_equal(to_np(cache.k_params[b, :, sl]).view(np.uint16), ref.k_params[0, :, sl].view(np.uint16))
        assert np.array_equal(to_np(cache.v_params[b, :, sl]).view(np.uint16), ref.v_params[0, :, sl].view(np.uint16))
        assert not to_np(cache.k_codes[b, :, :off]).any() and not to_np(cache.v_codes[b, :, off + T:]).any()
