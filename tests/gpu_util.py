"""Helpers shared by the GPU tests: device tensors from fg_synth inputs, oracle<->device
conversions and the float tolerance (max |err| <= 1e-2 * RMS(oracle output))."""
import numpy as np

import fg_synth

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


def gpu_teacher_forced(fg, md, ids, forced, group=64):
    """GPU logits [T, B, V] at every position of a generation whose history is ``forced``
    (the oracle's tokens [B, T]), through the layer calls: prompt pass, then decode step j
    embeds forced[:, j-1] at position L + j - 1.  Every position is then scored on the same
    history on both sides."""
    import torch
    E, P, lnf_g, lnf_b = md.tensors
    B, L = ids.shape
    T = forced.shape[1]
    V, h = E.shape
    nh, hd = md.c.n_heads, md.c.head_dim
    caches = [fg.DeviceKVCache(B, nh, hd, L + T, group) for _ in md.layers]
    x = fg.fg_embed(to_dev(np.ascontiguousarray(ids, np.int32)), 0, E, P)
    for layer, c in zip(md.layers, caches):
        fg.fg_prefill_layer(layer, c, x, B, L)
    logits = torch.empty((T, B, V), dtype=torch.float32, device=E.device)
    last = x.view(B, L, h)[:, L - 1, :].contiguous()
    fg.fg_lm_head_argmax(fg.fg_layernorm(last, lnf_g, lnf_b), E, logits=logits[0])
    for j in range(1, T):
        xd = fg.fg_embed(to_dev(np.ascontiguousarray(forced[:, j - 1:j], np.int32)), L + j - 1, E, P)
        for layer, c in zip(md.layers, caches):
            xd = fg.fg_decode_layer(layer, c, xd)
        fg.fg_lm_head_argmax(fg.fg_layernorm(xd, lnf_g, lnf_b), E, logits=logits[j])
    torch.cuda.synchronize()
    return to_np(logits).astype(np.float64)


def check_teacher_forced(gpu_logits, exp_tokens, exp_logits, min_agree=0.99):
    """Logits within the float tolerance at every position, and the GPU's argmax equal to the
    oracle's token at >= 99 % of all positions, every disagreement a near tie."""
    T, B, _ = gpu_logits.shape
    agree = 0
    for t in range(T):
        assert_close_rms(gpu_logits[t], exp_logits[t], what=f"logits at position {t}")
        for b in range(B):
            g = int(np.argmax(gpu_logits[t, b]))
            if g == exp_tokens[b, t]:
                agree += 1
            else:
                assert near_tie(exp_logits[t, b]), f"seq {b} pos {t}: {g} vs {exp_tokens[b, t]} (not a near tie)"
    assert agree / (T * B) >= min_agree, f"token agreement {agree}/{T * B}"
    return agree / (T * B)
