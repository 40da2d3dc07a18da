"""Helpers shared by the GPU tests: device tensors from fg_synth inputs, oracle<->device
conversions and the float tolerance (max |err| <= 1e-2 * RMS(oracle output))."""
import numpy as np

import fg_synth
import oracle

TOL_RMS = 1e-2


def cuda():
    import torch
    return torch.device("cuda:0")


def to_dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).to(cuda())


def to_np(t):
    return t.detach().cpu().numpy()


def synth_dev(seed, stream, shape, dist="normal", scale=1.0):
    return to_dev(fg_synth.tensor(seed, stream, shape, dist, scale))


def assert_close_rms(got, ref, tol=TOL_RMS, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    rms = float(np.sqrt(np.mean(ref * ref)))
    err = float(np.max(np.abs(got - ref))) if got.size else 0.0
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert err <= tol * max(rms, 1e-30), f"{what}: max|err| {err:.3e} > {tol} * RMS {rms:.3e}"
    return err, rms


def near_tie(logits_row, tol=TOL_RMS):
    """The oracle's top-2 logit margin is within the float tolerance: either token is a
    correct greedy choice."""
    lg = np.asarray(logits_row, np.float64)
    top2 = np.sort(lg)[-2:]
    return top2[1] - top2[0] <= tol * np.sqrt(np.mean(lg * lg))


def compare_free_running(got, exp_tokens, exp_logits):
    """Free-running greedy generations, position by position: they must agree until the first
    position where the oracle's top-2 margin is a near tie (both tokens correct; from there
    the two continuations legitimately differ and are not compared).  A disagreement that is
    not a near tie fails.  Returns (agreeing positions, compared positions)."""
    B, T = exp_tokens.shape
    agree = compared = 0
    for b in range(B):
        for t in range(T):
            compared += 1
            if got[b, t] == exp_tokens[b, t]:
                agree += 1
                continue
            assert near_tie(exp_logits[t, b]), \
                f"seq {b} pos {t}: token {got[b, t]} vs oracle {exp_tokens[b, t]} (not a near tie)"
            break
    return agree, compared


def stepwise_forced(fg, md, mo, ids, T, group=64):
    """Every position scored from the same state on both sides.  The oracle generates greedily
    step by step (its layer calls); the GPU runs the prompt pass itself, and before each decode
    step j its caches are loaded with the oracle's 4-bit caches after step j-1 and it embeds
    the oracle's token j-1.  Within a step both sides run their own layers, so the comparison
    covers the embedding, every decode layer (KV append, attention over the cache, projections,
    FFN), the final LayerNorm and the LM head, while a 4-bit code that one side rounds
    differently (its K/V differ by an fp16 ulp) cannot carry over into later steps.
    Returns (GPU logits [T, B, V], oracle tokens [B, T], oracle logits [T, B, V])."""
    import torch
    E, P, lnf_g, lnf_b = md.tensors
    B, L = ids.shape
    V, h = E.shape
    nh, hd = md.c.n_heads, md.c.head_dim
    n_layers = len(md.layers)
    dc = [fg.DeviceKVCache(B, nh, hd, L + T, group) for _ in range(n_layers)]
    oc = [oracle.KVCache(B, nh, hd, group, L + T) for _ in range(n_layers)]
    g_logits = torch.empty((T, B, V), dtype=torch.float32, device=E.device)
    o_tok = np.empty((B, T), np.int32)
    o_logits = np.empty((T, B, V), np.float64)
    # prompt pass
    x = fg.fg_embed(to_dev(np.ascontiguousarray(ids, np.int32)), 0, E, P)
    for layer, c in zip(md.layers, dc):
        fg.fg_prefill_layer(layer, c, x, B, L)
    last = x.view(B, L, h)[:, L - 1, :].contiguous()
    fg.fg_lm_head_argmax(fg.fg_layernorm(last, lnf_g, lnf_b), E, logits=g_logits[0])
    xo = oracle.embed(mo, ids, 0)
    for layer, c in zip(mo.layers, oc):
        xo = oracle.prefill_layer(layer, c, xo)
    o_tok[:, 0], o_logits[0] = oracle.lm_head_argmax(mo, xo[:, -1, :])
    for j in range(1, T):
        for d, o in zip(dc, oc):   # the oracle's cache state after step j-1
            d.k_codes.copy_(torch.from_numpy(o.k_codes))
            d.v_codes.copy_(torch.from_numpy(o.v_codes))
            d.k_params.copy_(torch.from_numpy(o.k_params))
            d.v_params.copy_(torch.from_numpy(o.v_params))
            d.length = o.length
        tok = np.ascontiguousarray(o_tok[:, j - 1:j])
        xd = fg.fg_embed(to_dev(tok), L + j - 1, E, P)
        for layer, c in zip(md.layers, dc):
            xd = fg.fg_decode_layer(layer, c, xd)
        fg.fg_lm_head_argmax(fg.fg_layernorm(xd, lnf_g, lnf_b), E, logits=g_logits[j])
        xo = oracle.embed(mo, tok, L + j - 1)[:, 0, :]
        for layer, c in zip(mo.layers, oc):
            xo = oracle.decode_layer(layer, c, xo)
        o_tok[:, j], o_logits[j] = oracle.lm_head_argmax(mo, xo)
    torch.cuda.synchronize()
    return to_np(g_logits).astype(np.float64), o_tok, o_logits


def check_logits_and_tokens(gpu_logits, exp_tokens, exp_logits, min_agree=0.99, tol=TOL_RMS):
    """Logits within the float tolerance at every position, and the GPU's argmax equal to the
    oracle's token at >= 99 % of all positions, every disagreement a near tie."""
    T, B, _ = gpu_logits.shape
    agree = 0
    for t in range(T):
        err, rms = assert_close_rms(gpu_logits[t], exp_logits[t], tol=tol, what=f"logits at position {t}")
        print(f"logits at position {t}: max|err| / RMS = {err / rms:.2e}")
        for b in range(B):
            g = int(np.argmax(gpu_logits[t, b]))
            if g == exp_tokens[b, t]:
                agree += 1
            else:
                assert near_tie(exp_logits[t, b]), f"seq {b} pos {t}: {g} vs {exp_tokens[b, t]} (not a near tie)"
    assert agree / (T * B) >= min_agree, f"token agreement {agree}/{T * B}"
    return agree / (T * B)
