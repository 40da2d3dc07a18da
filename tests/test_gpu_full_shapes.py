"""GPU parity at the benchmarked shapes, composed: whole decoder layers and a generation whose
launch paths are the ones the benchmark times (the prompt pass over M = B*L >= 1024 rows
expands each 4-bit weight to fp16 once and runs the fp16 tensor-core GEMM; decode steps run
the fused 4-bit GEMM with split-K at batch 64 and without it at batch 256; fg_generate's third
call replays its recorded CUDA graphs).

Sequences are independent, so the oracle runs a subset of the batch: the same seeded inputs
(drawn by the generator's GPU twin, which produces the CPU generator's bits) for the sampled
sequences only.  Tolerances as everywhere: max|err| <= 1e-2 * RMS(oracle)."""
import numpy as np
import pytest

import fg_synth
import oracle
from fg_synth import layer_stream as ls
from gpu_util import assert_close_rms, check_logits_and_tokens, compare_free_running, stepwise_forced, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fg():
    import torch
    assert torch.cuda.is_available()
    import bit_group_quantized_fg_b200 as m
    m.lib()
    return m


def layer_pair(fg, seed, l, h, F, g=64):
    """One decoder layer with N(0, 0.02) weights and N(0, 0.02) biases drawn on the GPU and
    LayerNorm parameters near (1, 0): the device copy quantized by the library, the oracle
    copy quantized by the oracle from the same fp16 values."""
    import torch
    from fg_synth import gpu as sg
    ln = [fg_synth.tensor(seed, ls(l, k), (h,), "normal", 0.1) + np.float16(1.0 if k % 2 == 0 else 0.0)
          for k in range(4)]
    d_lins, o_lins = [], []
    for wk, bk, K, N in ((fg_synth.S_WQKV, fg_synth.S_BQKV, h, 3 * h), (fg_synth.S_WO, fg_synth.S_BO, h, h),
                         (fg_synth.S_W1, fg_synth.S_B1, h, F), (fg_synth.S_W2, fg_synth.S_B2, F, h)):
        w = torch.empty((K, N), dtype=torch.float16, device="cuda")
        sg.fill(w, seed, ls(l, wk), "normal", 0.02)
        b = torch.empty((N,), dtype=torch.float16, device="cuda")
        sg.fill(b, seed, ls(l, bk), "normal", 0.02)
        d_lins.append(fg.DeviceQLinear.from_fp16(w, b, g))
        o_lins.append(oracle.QLinear.from_fp16(w.cpu().numpy(), b.cpu().numpy(), g))
        del w
    dev_ln = [torch.from_numpy(a).cuda() for a in ln]
    return fg.DeviceLayer(*dev_ln, *d_lins), oracle.QLayer(*ln, *o_lins)


def run_layer_case(fg, seed, h, nh, F, B, L, seqs, steps):
    import torch
    from fg_synth import gpu as sg
    hd, g = h // nh, 64
    dl, ol = layer_pair(fg, seed, 0, h, F, g)
    x = torch.empty((B * L, h), dtype=torch.float16, device="cuda")
    sg.fill(x, seed, fg_synth.S_HIDDEN, "normal", 1.0)
    x_host = x.cpu().numpy().reshape(B, L, h)[seqs]
    cache = fg.DeviceKVCache(B, nh, hd, L + steps, g)
    fg.fg_prefill_layer(dl, cache, x, B, L)
    torch.cuda.synchronize()
    assert bool(torch.isfinite(x.float()).all())
    oc = oracle.KVCache(len(seqs), nh, hd, g, L + steps)
    xo = oracle.prefill_layer(ol, oc, x_host)
    err, rms = assert_close_rms(to_np(x).reshape(B, L, h)[seqs], xo, what="prompt pass")
    print(f"h {h} B {B} L {L} prompt pass: max|err| / RMS = {err / rms:.2e}")
    for s in range(steps):
        # each decode step starts from the oracle's 4-bit cache for the sampled sequences: a
        # code that the two sides round differently (their K/V an fp16 ulp apart after the
        # prompt pass) would otherwise move the step's attention by a whole quantization step
        for name in ("k_codes", "v_codes", "k_params", "v_params"):
            getattr(cache, name)[seqs] = torch.from_numpy(getattr(oc, name)).cuda()
        xin = torch.empty((B, h), dtype=torch.float16, device="cuda")
        sg.fill(xin, seed, fg_synth.S_DECODE_X, "normal", 1.0, offset=s * B * h)
        y = fg.fg_decode_layer(dl, cache, xin)
        torch.cuda.synchronize()
        assert bool(torch.isfinite(y.float()).all())
        yo = oracle.decode_layer(ol, oc, xin.cpu().numpy()[seqs])
        err, rms = assert_close_rms(to_np(y)[seqs], yo, what=f"decode step {s}")
        print(f"h {h} B {B} decode step {s}: max|err| / RMS = {err / rms:.2e}")
    assert cache.length == L + steps


def test_layer_opt6p7b_shape_prompt_and_decode(fg):
    """OPT-6.7B-shaped layer (h 4096, 32 x 128, F 16384) at batch 64, prompt 512, then two
    decode steps; sequences 0 and 63 against the oracle."""
    run_layer_case(fg, 2024, 4096, 32, 16384, 64, 512, [0, 63], 2)


def test_layer_opt30b_shape_prompt_and_decode(fg):
    """OPT-30B-shaped layer (h 7168, 56 x 128, F 28672) at batch 256, prompt 512, then one
    decode step (the M = 256 decode GEMMs); sequence 255 against the oracle."""
    run_layer_case(fg, 2030, 7168, 56, 28672, 256, 512, [255], 1)


def test_generate_two_layer_opt6p7b_shape_graph_replay(fg):
    """Two OPT-6.7B-shaped layers with the 50272-token vocabulary, batch 4, prompt 256
    (M = 1024 prompt rows: the expand-then-fp16-GEMM path), 6 tokens.  The third fg_generate
    call replays the recorded graphs; its tokens are compared with the oracle's generation,
    and every position is scored by teacher forcing through the layer calls."""
    import torch
    from fg_synth import gpu as sg
    seed, h, nh, F, V, P, g = 77, 4096, 32, 16384, 50272, 2048, 64
    B, L, T = 4, 256, 6
    pairs = [layer_pair(fg, seed, l, h, F, g) for l in range(2)]
    E = torch.empty((V, h), dtype=torch.float16, device="cuda")
    sg.fill(E, seed, fg_synth.S_EMBED, "normal", 0.02)
    Pm = torch.empty((P, h), dtype=torch.float16, device="cuda")
    sg.fill(Pm, seed, fg_synth.S_POS, "normal", 0.02)
    ones, zeros = np.ones(h, np.float16), np.zeros(h, np.float16)
    md = fg.DeviceModel(2, h, nh, h // nh, F, V, P, g, E, Pm, torch.from_numpy(ones).cuda(),
                        torch.from_numpy(zeros).cuda(), [p[0] for p in pairs])
    mo = oracle.Model(2, h, nh, h // nh, F, V, P, g, E.cpu().numpy(), Pm.cpu().numpy(), ones, zeros,
                      [p[1] for p in pairs])
    ids = fg_synth.token_ids(seed, fg_synth.S_IDS, (B, L), V)
    ids_d = torch.from_numpy(ids).cuda()
    caches = [fg.DeviceKVCache(B, nh, h // nh, L + T, g) for _ in range(2)]
    out = torch.empty((B, T), dtype=torch.int32, device="cuda")
    ws = torch.empty((fg.fg_workspace_bytes(md, B, L, T),), dtype=torch.uint8, device="cuda")
    calls = []
    for _ in range(3):   # eager, recorded, replayed
        out.fill_(-1)
        fg.fg_generate(md, ids_d, T, caches, out_ids=out, workspace=ws)
        torch.cuda.synchronize()
        calls.append(to_np(out).copy())
    assert np.array_equal(calls[0], calls[1]) and np.array_equal(calls[1], calls[2])
    exp, logits = oracle.generate(mo, ids, T, return_logits=True)
    agree, compared = compare_free_running(calls[2], exp, logits)
    print(f"free-running replay: {agree}/{compared} compared positions agree")
    g_lg, f_tok, f_lg = stepwise_forced(fg, md, mo, ids, T, g)
    assert np.array_equal(f_tok, exp)
    # logits after two full-width layers: each layer's fp16 storage points leave the two sides
    # up to ~3.5e-3 RMS apart (1 ulp of the largest values, measured at the OPT-30B layer shape),
    # two layers, the final LayerNorm and the LM head reach ~1.0e-2; the bound is 2e-2 here,
    # 1e-2 for every single layer and kernel
    frac = check_logits_and_tokens(g_lg, f_tok, f_lg, tol=2e-2)
    print(f"stepwise token agreement {frac:.3f}")
