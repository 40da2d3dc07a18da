"""GPU parity of the dequant-fused tcgen05 GEMM (K3) and the tied LM head against the
oracle's float64 product of the same fp16 operands; tolerance max|err| <= 1e-2 * RMS."""
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


def _case(fg, M, N, K, g, relu, resid, seed):
    import torch
    x = fg_synth.tensor(seed, 1, (M, K), "normal", 1.0)
    w = fg_synth.tensor(seed, 2, (K, N), "normal", 0.02)
    b = fg_synth.tensor(seed, 3, (N,), "normal", 0.5)
    r = fg_synth.tensor(seed, 4, (M, N), "normal", 1.0) if resid else None
    lin = fg.DeviceQLinear.from_fp16(to_dev(w), to_dev(b), g)
    y = fg.fg_qgemm(to_dev(x), lin, R=None if r is None else to_dev(r), relu=relu)
    torch.cuda.synchronize()
    ref_lin = oracle.QLinear.from_fp16(w, b, g)
    assert np.array_equal(to_np(lin.codes), ref_lin.codes)
    exp = oracle.qlinear(x, ref_lin, relu=relu, residual16=r)
    return to_np(y), exp


@pytest.mark.parametrize("M,N,K,g,relu,resid", [
    (4, 256, 64, 64, False, False),        # one k-block, tiny M
    (4, 2304, 768, 64, False, False),      # config-1 QKV at decode
    (128, 768, 768, 64, False, True),      # config-1 out-proj (prefill rows), residual
    (128, 3072, 768, 64, True, False),     # config-1 fc1 + ReLU
    (128, 768, 3072, 64, False, True),     # config-1 fc2 + residual
    (300, 512, 320, 32, True, True),       # ragged M over 3 tiles, g 32
    (64, 1024, 512, 128, False, False),    # g 128
    (1000, 768, 256, 64, False, False),    # 8 M-tiles, band raster
])
def test_qgemm_matches_oracle(fg, M, N, K, g, relu, resid):
    got, exp = _case(fg, M, N, K, g, relu, resid, seed=M + N + K)
    assert_close_rms(got, exp, what="qgemm")


def test_qgemm_decode_split_k(fg):
    """M = 64 rows with few output tiles: the K loop is split and the fp32 partials are
    reduced by the epilogue kernel."""
    got, exp = _case(fg, 64, 4096, 4096, 64, False, True, seed=7)
    assert_close_rms(got, exp, what="split-K")


@pytest.mark.parametrize("M,N,K,g,relu,resid", [
    (1, 256, 128, 64, False, True),        # one row
    (17, 512, 1024, 64, True, True),       # rows not a multiple of 16
    (144, 768, 512, 32, False, True),      # two row chunks (128 + 16), g 32
    (256, 512, 640, 128, True, False),     # two full row chunks, g 128
    (64, 256, 4096, 64, False, False),     # one tile, K split 8 ways
    (64, 3072, 4096, 64, False, False),    # 12 tiles x 8-way K split
    (256, 4096, 2048, 64, False, True),    # two row tiles, K split 4 ways
    (200, 20480, 2048, 64, True, True),    # 160 tiles: 148 whole + a wave tail of 12
])
def test_qgemm_decode_batches(fg, M, N, K, g, relu, resid):
    """Decode-size GEMMs (M <= 256): ragged rows, row tiles, group sizes, deep K splits, the
    wave tail."""
    got, exp = _case(fg, M, N, K, g, relu, resid, seed=3 * M + N + K)
    assert_close_rms(got, exp, what="decode qgemm")


def oracle_weight_groups(seed, stream, K, N, g, cols):
    """The oracle's QLinear over just the column groups that hold ``cols`` of a seeded
    N(0, 0.02) weight [K][N] (groups run along N, so each is quantized exactly as inside the
    full weight), with the N(0, 0.5) bias of those columns drawn from stream + 1; and the
    positions of ``cols`` in it."""
    cols = np.asarray(cols)
    groups = np.unique(cols // g)
    idx = (np.arange(K)[:, None] * N + (groups[:, None] * g + np.arange(g)[None, :]).reshape(1, -1)).ravel()
    w = fg_synth.values(seed, stream, idx, "normal", 0.02).reshape(K, len(groups) * g)
    bcols = (groups[:, None] * g + np.arange(g)[None, :]).ravel()
    b = fg_synth.values(seed, stream + 1, bcols, "normal", 0.5)
    pos = np.searchsorted(groups, cols // g) * g + cols % g
    return oracle.QLinear.from_fp16(w, b, g), pos


def _sampled_qgemm(fg, M, N, K, g, seed, rows, cols):
    """Y = X W_hat + b at full size on the GPU (inputs from the GPU twin of the generator);
    the oracle recomputes the sampled rows x columns from CPU-generated inputs."""
    import torch
    from fg_synth import gpu as sg
    x = torch.empty((M, K), dtype=torch.float16, device="cuda")
    sg.fill(x, seed, 1, "normal", 1.0)
    w = torch.empty((K, N), dtype=torch.float16, device="cuda")
    sg.fill(w, seed, 2, "normal", 0.02)
    b = torch.empty((N,), dtype=torch.float16, device="cuda")
    sg.fill(b, seed, 3, "normal", 0.5)
    lin = fg.DeviceQLinear.from_fp16(w, b, g)
    del w
    y = fg.fg_qgemm(x, lin)
    torch.cuda.synchronize()
    assert bool(torch.isfinite(y.float()).all())
    sub, pos = oracle_weight_groups(seed, 2, K, N, g, cols)
    xr = fg_synth.values(seed, 1, (rows[:, None] * K + np.arange(K)[None, :]).ravel(), "normal", 1.0).reshape(-1, K)
    exp = oracle.qlinear(xr, sub)[:, pos]
    return to_np(y)[rows][:, cols], exp


@pytest.mark.parametrize("M,N,K", [
    (256, 21504, 7168),    # OPT-30B-shaped QKV at batch 256
    (144, 49152, 12288),   # OPT-175B-shaped fc1 at batch 144
])
def test_qgemm_large_decode_sampled(fg, M, N, K):
    """Decode GEMMs at the larger configurations' shapes, on sampled outputs."""
    rng = np.random.default_rng(M)
    rows = np.concatenate([[0, M - 1], rng.integers(0, M, 6)])
    cols = np.concatenate([[0, N - 1], rng.integers(0, N, 14)])
    got, exp = _sampled_qgemm(fg, M, N, K, 64, M + 5, rows, cols)
    assert_close_rms(got, exp, what="sampled decode GEMM")


@pytest.mark.parametrize("M,N,K", [
    (256, 21504, 7168),    # wave tail over the pairs (84 tiles on 74 pairs)
    (256, 7168, 28672),    # K split in two
    (144, 12288, 12288),   # every tile's k-blocks spread over the pairs
])
def test_qgemm_pair_repeatable(fg, M, N, K):
    """From 129 to 256 rows each SM of a pair expands half of every weight tile and hands it
    to the pair's MMA through a barrier of the other SM.  A hand-off that let the MMA read a
    half-tile before it was written would make repeated launches differ: 16 launches must be
    bitwise identical, and sampled outputs match the oracle."""
    import torch
    from fg_synth import gpu as sg
    x = torch.empty((M, K), dtype=torch.float16, device="cuda")
    sg.fill(x, 9, 1, "normal", 1.0)
    w = torch.empty((K, N), dtype=torch.float16, device="cuda")
    sg.fill(w, 9, 2, "normal", 0.02)
    b = torch.empty((N,), dtype=torch.float16, device="cuda")
    sg.fill(b, 9, 3, "normal", 0.5)
    lin = fg.DeviceQLinear.from_fp16(w, b, 64)
    del w
    ws = torch.empty((max(fg.fg_qgemm_workspace_bytes(M, N, K), 16),), dtype=torch.uint8, device="cuda")
    y0 = fg.fg_qgemm(x, lin, workspace=ws)
    outs = [fg.fg_qgemm(x, lin, workspace=ws) for _ in range(15)]
    torch.cuda.synchronize()
    assert all(torch.equal(y0, y) for y in outs)
    rng = np.random.default_rng(N)
    rows = np.concatenate([[0, M - 1], rng.integers(0, M, 4)])
    cols = np.concatenate([[0, N - 1], rng.integers(0, N, 10)])
    sub, pos = oracle_weight_groups(9, 2, K, N, 64, cols)
    xr = fg_synth.values(9, 1, (rows[:, None] * K + np.arange(K)[None, :]).ravel(), "normal", 1.0).reshape(-1, K)
    exp = oracle.qlinear(xr, sub)[:, pos]
    assert_close_rms(to_np(y0)[rows][:, cols], exp, what="pair decode GEMM")


def test_qgemm_prefill_size_sampled(fg):
    """Config-2 prefill QKV shape (M 32768, N 12288, K 4096) on sampled outputs."""
    M, N, K = 32768, 12288, 4096
    rng = np.random.default_rng(0)
    rows = np.concatenate([[0, 127, 128, M - 1], rng.integers(0, M, 12)])
    cols = np.concatenate([[0, 255, 256, N - 1], rng.integers(0, N, 28)])
    got, exp = _sampled_qgemm(fg, M, N, K, 64, 11, rows, cols)
    assert_close_rms(got, exp, what="sampled prefill GEMM")


@pytest.mark.parametrize("M,N,K", [(4, 256, 64), (300, 768, 320), (64, 4096, 2048)])
def test_gemm_f16_matches_oracle(fg, M, N, K):
    """The uncompressed fp16-weight GEMM against the oracle's linear layer over the same fp16
    weight (the uncompressed side of the README mirror's with/without compression table)."""
    import torch
    x = fg_synth.tensor(M, 1, (M, K), "normal", 1.0)
    w = fg_synth.tensor(M, 2, (K, N), "normal", 0.02)
    b = fg_synth.tensor(M, 3, (N,), "normal", 0.5)
    r = fg_synth.tensor(M, 4, (M, N), "normal", 1.0)
    y = fg.fg_gemm_f16(to_dev(x), to_dev(w), bias=to_dev(b), R=to_dev(r), relu=True)
    torch.cuda.synchronize()
    exp = oracle.qlinear(x, oracle.Linear16(w, b), relu=True, residual16=r)
    assert_close_rms(to_np(y), exp, what="fp16 GEMM")


@pytest.mark.parametrize("M,N,K,relu,resid", [
    (1024, 256, 64, False, False),     # one k-block, one column tile, eight row tiles
    (1300, 768, 320, True, True),      # ragged rows: the last row tile is mostly past M
    (2176, 512, 2048, False, True),    # a second band with one row tile
    (4096, 1024, 1024, True, False),   # two rasterization bands of 16 row tiles
])
def test_gemm_f16_prompt_rows(fg, M, N, K, relu, resid):
    """fp16 GEMMs at prompt-pass row counts (ragged rows, several rasterization bands) against
    the oracle's linear layer over the same fp16 weight."""
    import torch
    x = fg_synth.tensor(M + 1, 1, (M, K), "normal", 1.0)
    w = fg_synth.tensor(M + 1, 2, (K, N), "normal", 0.02)
    b = fg_synth.tensor(M + 1, 3, (N,), "normal", 0.5)
    r = fg_synth.tensor(M + 1, 4, (M, N), "normal", 1.0) if resid else None
    y = fg.fg_gemm_f16(to_dev(x), to_dev(w), bias=to_dev(b), R=None if r is None else to_dev(r), relu=relu)
    torch.cuda.synchronize()
    exp = oracle.qlinear(x, oracle.Linear16(w, b), relu=relu, residual16=r)
    err, rms = assert_close_rms(to_np(y), exp, what="prompt-row GEMM")
    print(f"fp16 GEMM {M}x{N}x{K}: max|err| / RMS = {err / rms:.2e}")


@pytest.mark.parametrize("M,N,K,g,relu,resid", [
    (64, 4096, 4096, 64, False, True),    # decode batch with the K loop split
    (144, 768, 512, 32, True, False),     # G 32: two parameter rows per 64-deep k-block
    (256, 512, 1024, 128, False, True),   # G 128: one parameter row serves two k-blocks
    (1024, 512, 640, 64, True, True),     # prompt rows: expanded along K, then the pair GEMM
])
def test_qgemm_groups_along_k(fg, M, N, K, g, relu, resid):
    """Weights grouped along K (the input dimension, one group per column): quantized
    bit-exactly like the oracle's axis-0 quantizer, then the fused GEMM (decode rows) or the
    expanded fp16 weight (prompt rows) against the oracle's linear layer."""
    import torch
    x = fg_synth.tensor(K + g, 1, (M, K), "normal", 1.0)
    w = fg_synth.tensor(K + g, 2, (K, N), "outlier", 0.02)
    b = fg_synth.tensor(K + g, 3, (N,), "normal", 0.5)
    r = fg_synth.tensor(K + g, 4, (M, N), "normal", 1.0) if resid else None
    lin = fg.DeviceQLinear.from_fp16(to_dev(w), to_dev(b), g, along_k=True)
    ref = oracle.QLinear.from_fp16(w, b, g, axis=0)
    assert np.array_equal(to_np(lin.codes), ref.codes)
    assert np.array_equal(to_np(lin.params).view(np.uint16).reshape(-1), ref.params.view(np.uint16).reshape(-1))
    y = fg.fg_qgemm(to_dev(x), lin, R=None if r is None else to_dev(r), relu=relu)
    torch.cuda.synchronize()
    err, rms = assert_close_rms(to_np(y), oracle.qlinear(x, ref, relu=relu, residual16=r), what="groups along K")
    print(f"groups along K {M}x{N}x{K} g {g}: max|err| / RMS = {err / rms:.2e}")


def test_lm_head_argmax(fg):
    import torch
    B, h, V = 5, 256, 1000      # V not a multiple of the 256-wide tile
    x = fg_synth.tensor(3, 1, (B, h), "normal", 1.0)
    E = fg_synth.tensor(3, 2, (V, h), "normal", 0.5)
    logits = torch.empty((B, V), dtype=torch.float32, device="cuda")
    tok = fg.fg_lm_head_argmax(to_dev(x), to_dev(E), logits=logits)
    torch.cuda.synchronize()
    exp = oracle.linear_fp16(x, E)
    assert_close_rms(to_np(logits), exp, tol=1e-3, what="logits")
    top2 = np.sort(exp, axis=1)[:, -2:]
    for i in range(B):
        if top2[i, 1] - top2[i, 0] > 1e-3 * np.sqrt(np.mean(exp ** 2)):
            assert int(to_np(tok)[i]) == int(np.argmax(exp[i]))
    # ties go to the lowest id
    E2 = E.copy()
    E2[700] = E2[123] = np.float16(0)
    E2[123, :] = x[0] * np.float16(0.25)
    E2[700] = E2[123]
    tok2 = fg.fg_lm_head_argmax(to_dev(x[:1]), to_dev(E2))
    torch.cuda.synchronize()
    assert int(to_np(tok2)[0]) == 123


def test_two_devices_in_one_process(fg):
    """Launch state kept per device (shared-memory attributes, capture streams): a GEMM on
    device 0 and then on device 1 of the same process both match the oracle.  Skipped with a
    single visible GPU."""
    import torch
    if torch.cuda.device_count() < 2:
        pytest.skip("needs two visible GPUs")
    M, N, K, g = 64, 1024, 512, 64
    x = fg_synth.tensor(31, 1, (M, K), "normal", 1.0)
    w = fg_synth.tensor(31, 2, (K, N), "normal", 0.02)
    b = fg_synth.tensor(31, 3, (N,), "normal", 0.5)
    exp = oracle.qlinear(x, oracle.QLinear.from_fp16(w, b, g))
    for d in (0, 1):
        with torch.cuda.device(d):
            dev = torch.device("cuda", d)
            lin = fg.DeviceQLinear.from_fp16(torch.from_numpy(w).to(dev), torch.from_numpy(b).to(dev), g)
            y = fg.fg_qgemm(torch.from_numpy(x).to(dev), lin)
            torch.cuda.synchronize(d)
            assert_close_rms(to_np(y), exp, what=f"GEMM on device {d}")
