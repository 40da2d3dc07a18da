"""Throughput benchmark: greedy generation over 4-bit weights and a 4-bit KV cache.

Workloads (one "step" = one whole generation; synthetic, seeded data, random-init weights
~ N(0, 0.02) compressed to 4 bits in groups of 64 along each weight's output channel; the
metric of the FlexGen README mirror's benchmark table: generated tokens / (prompt time +
generation time), input length 512, output length 32):

  c3 (default)  OPT-30B-shaped decoder: 48 layers, hidden 7168, 56 heads x 128, FFN 28672,
                vocab 50272, batch 256, prompt 512 uniform token ids, 32 generated tokens
                (1 from the prompt pass + 31 decode steps); all state resident in HBM.
  c2            OPT-6.7B-shaped decoder: 32 layers, hidden 4096, 32 x 128, FFN 16384,
                batch 64, otherwise as c3.
  c4            OPT-175B-shaped 12-layer slice: hidden 12288, 96 x 128, FFN 49152, batch
                144 (the arXiv 2303.06865 abstract's effective batch), prompt 512 hidden
                states ~ N(0, 1), 32 decode steps with N(0, 1) inputs; no embedding or LM
                head.  Timed through the layer calls; tokens/s of the slice are reported
                per layer and extrapolated to 96 layers (x 12/96).

    python bench.py [--config c2|c3|c4] [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs N independent replicas (one process per GPU, launched by torchrun): the batch
dimension shards with no exchange step, so each rank generates its own batch (weak
scaling) and the value is all ranks' tokens divided by the slowest rank's time.
`--impl reference` times the CPU oracle on a bounded sample of the same workload.
Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "generated tokens/s at 1 B200 (prefill+decode) vs roofline; quantizer GB/s"
CONFIGS = {
    "c2": dict(kind="generate", model="OPT-6.7B-shaped 32-layer decoder", n_layers=32, hidden=4096, n_heads=32,
               head_dim=128, ffn=16384, vocab=50272, max_pos=2048, group=64, batch=64, prompt_len=512,
               gen_len=32),
    "c3": dict(kind="generate", model="OPT-30B-shaped 48-layer decoder", n_layers=48, hidden=7168, n_heads=56,
               head_dim=128, ffn=28672, vocab=50272, max_pos=2048, group=64, batch=256, prompt_len=512,
               gen_len=32),
    "c4": dict(kind="slice", model="OPT-175B-shaped 12-layer slice", n_layers=12, full_layers=96, hidden=12288,
               n_heads=96, head_dim=128, ffn=49152, vocab=0, max_pos=0, group=64, batch=144, prompt_len=512,
               gen_len=32),
}
DEFAULT_CONFIG = "c3"
CFG = CONFIGS[DEFAULT_CONFIG]
SEED = 1234


def use_config(name):
    """Select the workload the module-level helpers use."""
    global CFG
    CFG = CONFIGS[name]
    return CFG


def tokens_per_step(c):
    """Generated tokens of one step: B x gen_len (for the slice: one per sequence and decode step)."""
    return c["batch"] * c["gen_len"]


def weight_bytes_4bit(c):
    h, F = c["hidden"], c["ffn"]
    return c["n_layers"] * (h * 3 * h + h * h + 2 * h * F) * (0.5 + 4.0 / c["group"])


def describe(c, wdesc):
    if c["kind"] == "slice":
        return (f"{c['model']} ({c['n_layers']} of {c['full_layers']} layers), {wdesc} + 4-bit KV (group "
                f"{c['group']}), batch {c['batch']} per GPU, prompt {c['prompt_len']}, {c['gen_len']} decode steps; "
                f"value extrapolated to {c['full_layers']} layers (no embedding / LM head)")
    return (f"{c['model']}, {wdesc} + 4-bit KV (group {c['group']}), batch {c['batch']} per GPU, "
            f"prompt {c['prompt_len']}, generate {c['gen_len']}")


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], tf=d["bf16_tflops"], tf_sust=d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                    src="measured")
    return dict(hbm=6650.0, tf=1590.0, tf_sust=1400.0, src="fallback")


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.f = None

    def __enter__(self):
        try:
            self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.index)], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.f is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.f.flush()
        rows = [l.split(",") for l in open(self.f.name).read().strip().splitlines() if l.count(",") >= 8]
        os.unlink(self.f.name)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for name, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------- model
def build_model(fg, torch, dev, weights="4bit"):
    from fg_synth import gpu as sg
    from fg_synth import layer_stream as ls
    import fg_synth
    c = CFG
    h, F, g = c["hidden"], c["ffn"], c["group"]
    ones = torch.ones(h, dtype=torch.float16, device=dev)
    zeros = torch.zeros(h, dtype=torch.float16, device=dev)
    layers = []
    for l in range(c["n_layers"]):
        lins = []
        for kind, K, N in ((fg_synth.S_WQKV, h, 3 * h), (fg_synth.S_WO, h, h), (fg_synth.S_W1, h, F),
                           (fg_synth.S_W2, F, h)):
            w = torch.empty((K, N), dtype=torch.float16, device=dev)
            sg.fill(w, SEED, ls(l, kind), "normal", 0.02)
            b = torch.zeros(N, dtype=torch.float16, device=dev)
            if weights == "fp16":   # the uncompressed side of the compression contrast
                lins.append(fg.DeviceQLinear.uncompressed(w, b))
            else:
                lins.append(fg.DeviceQLinear.from_fp16(w, b, g))
            del w
        layers.append(fg.DeviceLayer(ones, zeros, ones, zeros, *lins))
    caches = [fg.DeviceKVCache(c["batch"], c["n_heads"], c["head_dim"], c["prompt_len"] + c["gen_len"], g, dev)
              for _ in range(c["n_layers"])]
    if c["kind"] == "slice":   # a stack of layers, no embedding or LM head
        return layers, caches
    E = torch.empty((c["vocab"], h), dtype=torch.float16, device=dev)
    sg.fill(E, SEED, fg_synth.S_EMBED, "normal", 0.02)
    P = torch.empty((c["max_pos"], h), dtype=torch.float16, device=dev)
    sg.fill(P, SEED, fg_synth.S_POS, "normal", 0.02)
    model = fg.DeviceModel(c["n_layers"], h, c["n_heads"], c["head_dim"], F, c["vocab"], c["max_pos"], g, E, P,
                           ones, zeros, layers)
    return model, caches


# ---------------------------------------------------------------------------- oracle baseline
def synth_host(stream, shape, dist="normal", scale=1.0):
    """fg_synth values as a host numpy array; generated by the generator's GPU twin when a
    GPU is present (same bits, much faster than the numpy generator for 10^8 elements)."""
    import fg_synth
    try:
        import torch
        if torch.cuda.is_available():
            from fg_synth import gpu as sg
            t = torch.empty(shape, dtype=torch.float16, device="cuda")
            sg.fill(t, SEED, stream, dist, scale)
            return t.cpu().numpy()
    except Exception:
        pass
    return fg_synth.tensor(SEED, stream, shape, dist, scale)


def params_per_layer(c):
    h, F = c["hidden"], c["ffn"]
    return h * 3 * h + h * h + 2 * h * F


def oracle_sample():
    """The C++ CPU oracle on a bounded sample of the workload: one sequence through one
    decoder layer's prompt pass over its first `n_prompt` tokens, one decode step of that
    layer at context L + T/2 (the middle of the decode steps) and, for a full decoder, one
    LM-head token.  Weights are generated and quantized by the oracle before the clock
    starts.  Returns run(n_prompt) -> seconds of (prompt sample, decode step, LM head)."""
    import numpy as np
    import fg_synth
    import oracle
    from fg_synth import layer_stream as ls
    c = CFG
    h, F, g, L, T = c["hidden"], c["ffn"], c["group"], c["prompt_len"], c["gen_len"]
    nh, hd = c["n_heads"], c["head_dim"]
    lins = []
    for kind, K, N in ((fg_synth.S_WQKV, h, 3 * h), (fg_synth.S_WO, h, h), (fg_synth.S_W1, h, F),
                       (fg_synth.S_W2, F, h)):
        w = synth_host(ls(0, kind), (K, N), "normal", 0.02)
        lin = oracle.QLinear.from_fp16(w, np.zeros(N, np.float16), g)
        lin.weight16()
        lins.append(lin)
        del w
    ones, zeros = np.ones(h, np.float16), np.zeros(h, np.float16)
    layer = oracle.QLayer(ones, zeros, ones, zeros, *lins)
    model = None
    if c["kind"] == "generate":
        E = synth_host(fg_synth.S_EMBED, (c["vocab"], h), "normal", 0.02)
        P = synth_host(fg_synth.S_POS, (c["max_pos"], h), "normal", 0.02)
        model = oracle.Model(1, h, nh, hd, F, c["vocab"], c["max_pos"], g, E, P, ones, zeros, [layer])
    x_prompt = fg_synth.tensor(SEED, fg_synth.S_HIDDEN, (1, L, h), "normal", 1.0)
    x_dec = fg_synth.tensor(SEED, fg_synth.S_DECODE_X, (1, h), "normal", 1.0)
    ctx = L + T // 2

    def run(n_prompt):
        cache = oracle.KVCache(1, nh, hd, g, max(ctx, n_prompt) + 1)
        t0 = time.perf_counter()
        oracle.prefill_layer(layer, cache, x_prompt[:, :n_prompt])
        t1 = time.perf_counter()
        cache.length = ctx - 1           # attend over ctx positions (the cache holds valid codes)
        xd = oracle.decode_layer(layer, cache, x_dec)
        t2 = time.perf_counter()
        if model is not None:
            oracle.lm_head_argmax(model, xd)
        t3 = time.perf_counter()
        return t1 - t0, t2 - t1, t3 - t2
    return run


def oracle_rate(t_pf, t_dec, t_lm):
    """Extrapolated tokens/s of the whole workload from one sample (sequences independent,
    so B sequences take B times one sequence's time for B times its tokens): a full decoder
    runs n_layers x (prompt pass + T-1 decode steps) + T LM-head tokens per sequence; the
    slice runs full_layers x (prompt pass + T decode steps), its value extrapolated to the
    full depth like the GPU's."""
    c = CFG
    if c["kind"] == "slice":
        per_seq = c["full_layers"] * (t_pf + c["gen_len"] * t_dec)
    else:
        per_seq = c["n_layers"] * (t_pf + (c["gen_len"] - 1) * t_dec) + c["gen_len"] * t_lm
    return c["gen_len"] / per_seq


def oracle_measure(run, n_prompt, steps, warmup):
    """Median seconds of the sample parts; the prompt-pass sample scaled to the full prompt
    (linear in tokens: the projections and FFN, ~99 % of a prompt pass's arithmetic at
    L = 512, are per token; attention's share is undercounted by this scaling)."""
    for _ in range(warmup):
        run(n_prompt)
    ts = [run(n_prompt) for _ in range(steps)]
    scale = CFG["prompt_len"] / n_prompt
    return (statistics.median(t[0] for t in ts) * scale, statistics.median(t[1] for t in ts),
            statistics.median(t[2] for t in ts), ts)


def cpu_baseline_line(args, steps, warmup, single_thread=True):
    """cpu_baseline of the bench line: the C++ oracle with OpenMP over rows on every host core
    (the value), and single-threaded (reported beside it)."""
    import oracle
    c = CFG
    P = params_per_layer(c)
    n_omp = max(4, min(64, int(40e9 / P)))     # ~40 GMAC of prompt-pass sample with all cores
    n_one = max(2, min(64, int(5e9 / P)))      # ~5 GMAC single-threaded
    run = oracle_sample()
    cores = oracle.threads(os.cpu_count() or 1)
    t_pf, t_dec, t_lm, ts = oracle_measure(run, n_omp, steps, warmup)
    rate = oracle_rate(t_pf, t_dec, t_lm)
    seconds = sum(sum(t) for t in ts)
    lm = f", one LM-head token ({t_lm:.2f} s)" if c["kind"] == "generate" else ""
    sample = (f"C++ oracle (OpenMP over rows, {cores} threads) on 1 sequence x 1 layer: prompt pass over "
              f"{n_omp} of {c['prompt_len']} tokens scaled to {c['prompt_len']} ({t_pf:.2f} s), one decode step "
              f"at context {c['prompt_len'] + c['gen_len'] // 2} ({t_dec:.2f} s){lm}; extrapolated to "
              f"{c['batch']} sequences x {c.get('full_layers', c['n_layers'])} layers")
    out = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample,
           "sample_seconds": seconds}
    if single_thread:
        oracle.threads(1)
        s_pf, s_dec, s_lm, ts1 = oracle_measure(run, n_one, 1, 0)
        out["single_thread"] = {"value": oracle_rate(s_pf, s_dec, s_lm), "cores": 1,
                                "sample": f"prompt pass over {n_one} tokens scaled to {c['prompt_len']} "
                                          f"({s_pf:.2f} s), decode step ({s_dec:.2f} s)"
                                          + (f", LM head ({s_lm:.2f} s)" if c["kind"] == "generate" else "")}
        out["sample_seconds"] += sum(sum(t) for t in ts1)
        oracle.threads(cores)
    return out


# ---------------------------------------------------------------------------- kernel-only cases
def time_launches(run, steps, warmup):
    """(ms per launch from a replayed CUDA graph of `steps` launches, ms per eager launch)."""
    import torch
    for _ in range(warmup):
        run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        run()
    e1.record()
    torch.cuda.synchronize()
    ms_eager = e0.elapsed_time(e1) / max(steps, 1)
    # device time per launch: the same launches recorded into a CUDA graph and replayed, so
    # the host's per-call cost (Python, argument checks) cannot leave the GPU idle in between
    graph = torch.cuda.CUDAGraph()
    cs = torch.cuda.Stream()
    cs.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(graph, stream=cs, capture_error_mode="thread_local"):
        for _ in range(steps):
            run()
    graph.replay()
    torch.cuda.synchronize()
    e0.record()
    graph.replay()
    e1.record()
    torch.cuda.synchronize()
    del graph
    return e0.elapsed_time(e1) / max(steps, 1), ms_eager


def sweep_case(args):
    """The measurement sweep of the quantizer, the dequantizer, decode attention and the
    4-bit GEMM over sizes, group sizes, value distributions, batches and contexts (one JSON
    line per point; each point is `--steps` launches replayed from a CUDA graph after
    `--warmup` eager ones).  Points whose bytes fit in L2 (126 MB) say so: their rate is an
    L2 rate, not an HBM one."""
    import torch
    import bit_group_quantized_fg_b200 as fg
    from fg_synth import gpu as sg
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    L2 = 126e6

    def emit(kind, point, ms, work):
        res = {"sweep": kind, **point, "ms_per_launch": round(ms, 5)}
        if "bytes" in work:
            res["GB/s"] = round(work["bytes"] / (ms * 1e-3) / 1e9, 1)
            res["l2_resident"] = work["bytes"] < L2 and not work.get("streamed", False)
        if "flops" in work:
            res["TFLOP/s"] = round(work["flops"] / (ms * 1e-3) / 1e12, 1)
        print(json.dumps(res), flush=True)

    # quantize / dequantize: rows of 4096 (grouped along the row), fp16 in
    cols = 4096
    points = [(mb, 64, "normal", 0.02) for mb in (1, 16, 256, 1024, 4096)]
    points += [(1024, g, "normal", 0.02) for g in (32, 128)]
    points += [(1024, 64, d, sc) for d, sc in (("uniform", 1.0), ("t3", 1.0), ("outlier", 1.0))]
    for mb, g, dist, sc in points:
        rows = mb * (1 << 20) // (2 * cols)
        x = torch.empty((rows, cols), dtype=torch.float16, device=dev)
        sg.fill(x, SEED, 30, dist, sc)
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
        params = torch.empty((rows, cols // g, 2), dtype=torch.float16, device=dev)
        y = torch.empty_like(x)
        n = x.numel()
        bytes_ = n * (2 + 0.5 + 4.0 / g)
        pt = {"MB": mb, "group": g, "dist": dist}
        ms, _ = time_launches(lambda: fg.fg_quantize_pack(x, g, 1, codes, params), args.steps, args.warmup)
        emit("quantize", pt, ms, {"bytes": bytes_})
        ms, _ = time_launches(lambda: fg.fg_dequantize(codes, params, rows, cols, g, 1, y), args.steps, args.warmup)
        emit("dequantize", pt, ms, {"bytes": bytes_})
        del x, codes, params, y
        torch.cuda.empty_cache()

    # decode attention over a 4-bit cache (head dim 128, group 64); the codes and params are
    # drawn directly (every byte is a valid pair of codes), so no fp16 cache is ever built
    hd, g = 128, 64
    att = [(B, S, 32) for B in (1, 8, 64, 144, 256) for S in (128, 512, 2048, 8192)]
    att += [(256, 543, 56), (144, 543, 96), (256, 8192, 96)]
    for B, S, nh in att:
        h = nh * hd
        cache = fg.DeviceKVCache(B, nh, hd, S, g, dev)
        for t, st in ((cache.k_codes, 40), (cache.v_codes, 41)):
            sg.fill(t.view(torch.float16), SEED, st, "uniform", 1.0)
        for t, st in ((cache.k_params, 42), (cache.v_params, 43)):
            sg.fill(t, SEED, st, "uniform", 0.1)
        cache.c.len = S
        q = torch.empty((B, 3 * h), dtype=torch.float16, device=dev)
        sg.fill(q, SEED, 44, "normal", 1.0)
        out = torch.empty((B, h), dtype=torch.float16, device=dev)
        wsb = fg.lib().fg_decode_attention_workspace_bytes(B, nh, hd, S)
        ws = torch.empty((max(wsb, 16),), dtype=torch.uint8, device=dev)
        ms, _ = time_launches(lambda: fg.fg_decode_attention(q, 3 * h, cache, out=out, workspace=ws),
                              args.steps, args.warmup)
        emit("decode_attention", {"B": B, "S": S, "heads": nh},
             ms, {"bytes": B * nh * S * 2.0 * (hd / 2 + 4.0 * hd / g) + 4.0 * B * h})
        del cache, q, out, ws
        torch.cuda.empty_cache()

    # 4-bit GEMM (group 64): the OPT-6.7B projections at decode batches and the prompt pass,
    # and the OPT-30B / OPT-175B decode shapes.  Weight copies used in turn exceed the L2,
    # so every launch streams its weight from HBM as a decode step does (one weight re-read
    # launch after launch runs slower at the larger shapes: 0.26 vs 0.14 ms at 256 x 21504
    # x 7168, where 87 MB of codes only partly stay in the L2)
    h = 4096
    shapes = [(M, N, K) for M in (64, 144, 256, 32768)
              for N, K in ((3 * h, h), (h, h), (4 * h, h), (h, 4 * h))]
    shapes += [(256, 3 * 7168, 7168), (144, 4 * 12288, 12288)]
    lins = {}
    for M, N, K in shapes:
        if (N, K) not in lins:
            lins.clear()
            torch.cuda.empty_cache()
            copies = max(2, int(-(-256e6 // (N * K * (0.5 + 4 / 64)))))
            w = torch.empty((K, N), dtype=torch.float16, device=dev)
            lins[(N, K)] = []
            for i in range(copies):
                sg.fill(w, SEED, 50 + i, "normal", 0.02)
                lins[(N, K)].append(
                    fg.DeviceQLinear.from_fp16(w, torch.zeros(N, dtype=torch.float16, device=dev), 64))
            del w
        ring = lins[(N, K)]
        x = torch.empty((M, K), dtype=torch.float16, device=dev)
        sg.fill(x, SEED, 51, "normal", 1.0)
        y = torch.empty((M, N), dtype=torch.float16, device=dev)
        wsb = fg.fg_qgemm_workspace_bytes(M, N, K)
        ws = torch.empty((max(wsb, 16),), dtype=torch.uint8, device=dev)
        it = [0]

        def run_gemm():
            fg.fg_qgemm(x, ring[it[0] % len(ring)], Y=y, workspace=ws)
            it[0] += 1
        ms, _ = time_launches(run_gemm, args.steps, args.warmup)
        emit("qgemm", {"M": M, "N": N, "K": K}, ms,
             {"flops": 2.0 * M * N * K, "bytes": N * K * (0.5 + 4.0 / 64) + 2.0 * M * (K + N),
              "streamed": True})
        del x, y, ws


def kernel_case(args):
    """One kernel class on its own (for ncu captures and micro-measurements):
    qgemm            prompt-pass QKV slice: M 16384, N 12288, K 4096, group 64 (X 134 MB)
    qgemm_decode     a decode step's QKV projection: M 64, N 12288, K 4096 (or --mnk M,N,K)
    gemm_f16         the QKV slice over an fp16 weight; lm_head: [N][K] weight, fp32 logits
    gemm_prefill     one layer's four prompt-pass GEMMs at M = B*L of --config over fp16 weights
    decode_attention config-2 decode step: B 64, 32 heads x 128, context 543 (160 MB of cache)
    prefill_attention the prompt pass's causal attention of one layer: B 64, L 512, 32 x 128
                     (805 MB of projections, 268 MB out)
    quantize         1 GiB fp16 tensor [131072 x 4096], group 64
    Runs `--warmup` untimed and `--steps` timed launches and prints their mean time."""
    import torch
    import bit_group_quantized_fg_b200 as fg
    from fg_synth import gpu as sg
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if args.case == "qgemm":
        M, N, K = 16384, 12288, 4096
        x = torch.empty((M, K), dtype=torch.float16, device=dev)
        sg.fill(x, SEED, 1, "normal", 1.0)
        w = torch.empty((K, N), dtype=torch.float16, device=dev)
        sg.fill(w, SEED, 2, "normal", 0.02)
        lin = fg.DeviceQLinear.from_fp16(w, torch.zeros(N, dtype=torch.float16, device=dev), 64)
        del w
        y = torch.empty((M, N), dtype=torch.float16, device=dev)
        run = lambda: fg.fg_qgemm(x, lin, Y=y)
        work = {"flops": 2.0 * M * N * K}
    elif args.case == "qgemm_decode":
        # one decode step's QKV projection: 64 rows, 4-bit weight [4096][12288] (or --mnk)
        # (several weight copies, used in turn, so that each launch reads its weight from HBM
        # as a decode step does: together they exceed the 126 MB L2)
        M, N, K = (int(v) for v in args.mnk.split(",")) if args.mnk else (64, 12288, 4096)
        x = torch.empty((M, K), dtype=torch.float16, device=dev)
        sg.fill(x, SEED, 1, "normal", 1.0)
        n_copies = max(2, int(-(-256e6 // (N * K * (0.5 + 4 / 64)))))
        lins = []
        for i in range(n_copies):
            w = torch.empty((K, N), dtype=torch.float16, device=dev)
            sg.fill(w, SEED, 2 + i, "normal", 0.02)
            lins.append(fg.DeviceQLinear.from_fp16(w, torch.zeros(N, dtype=torch.float16, device=dev), 64))
            del w
        y = torch.empty((M, N), dtype=torch.float16, device=dev)
        wsd = torch.empty((max(fg.fg_qgemm_workspace_bytes(M, N, K), 16),), dtype=torch.uint8, device=dev)
        it = [0]

        def run():
            fg.fg_qgemm(x, lins[it[0] % n_copies], Y=y, workspace=wsd)
            it[0] += 1
        work = {"flops": 2.0 * M * N * K, "bytes": N * K * (0.5 + 4 / 64) + M * K * 2 + M * N * 2}
    elif args.case in ("gemm_f16", "lm_head"):
        # the same prompt-pass shape with an uncompressed fp16 weight: [K][N] (MN-major
        # operand) for gemm_f16, [N][K] (K-major, fp32 logits + argmax) for lm_head
        M, N, K = 16384, 12288, 4096
        x = torch.empty((M, K), dtype=torch.float16, device=dev)
        sg.fill(x, SEED, 1, "normal", 1.0)
        shape = (K, N) if args.case == "gemm_f16" else (N, K)
        w = torch.empty(shape, dtype=torch.float16, device=dev)
        sg.fill(w, SEED, 2, "normal", 0.02)
        if args.case == "gemm_f16":
            y = torch.empty((M, N), dtype=torch.float16, device=dev)
            run = lambda: fg.fg_gemm_f16(x, w, Y=y)
        else:
            logits = torch.empty((M, N), dtype=torch.float32, device=dev)
            run = lambda: fg.fg_lm_head_argmax(x, w, logits=logits)
        work = {"flops": 2.0 * M * N * K}
    elif args.case == "gemm_prefill":
        # the prompt pass's four GEMMs of one layer at B*L rows of the --config workload, over
        # the fp16 weights the 4-bit ones expand to: QKV (+bias), out (+bias +residual), fc1
        # (+bias, relu), fc2 (+bias +residual); one launch each per step (c2: M 32768, 2.8 GB
        # on the device; c3: M 131072, 14 GB)
        c = use_config(args.config)
        M, h, F = c["batch"] * c["prompt_len"], c["hidden"], c["ffn"]
        if args.rows:   # fewer rows of the same shapes (a capture small enough for ncu)
            M = args.rows
        x = torch.empty((M, h), dtype=torch.float16, device=dev)
        sg.fill(x, SEED, 1, "normal", 1.0)
        ws_ = {}
        for i, (K, N) in enumerate([(h, 3 * h), (h, h), (h, F), (F, h)]):
            w = torch.empty((K, N), dtype=torch.float16, device=dev)
            sg.fill(w, SEED, 10 + i, "normal", 0.02)
            b = torch.empty((N,), dtype=torch.float16, device=dev)
            sg.fill(b, SEED, 20 + i, "normal", 0.02)
            ws_[i] = (w, b)
        yqkv = torch.empty((M, 3 * h), dtype=torch.float16, device=dev)
        yo = torch.empty((M, h), dtype=torch.float16, device=dev)
        yf = torch.empty((M, F), dtype=torch.float16, device=dev)

        def run():
            fg.fg_gemm_f16(x, ws_[0][0], bias=ws_[0][1], Y=yqkv)
            fg.fg_gemm_f16(x, ws_[1][0], bias=ws_[1][1], R=x, Y=yo)
            fg.fg_gemm_f16(x, ws_[2][0], bias=ws_[2][1], relu=True, Y=yf)
            fg.fg_gemm_f16(yf, ws_[3][0], bias=ws_[3][1], R=x, Y=yo)
        work = {"flops": 2.0 * M * h * (3 * h + h + F + F)}
    elif args.case == "decode_attention":
        B, nh, hd, S = 64, 32, 128, 543
        h = nh * hd
        kv = torch.empty((B * S, 2 * h), dtype=torch.float16, device=dev)
        sg.fill(kv, SEED, 3, "normal", 1.0)
        q = torch.empty((B, 3 * h), dtype=torch.float16, device=dev)
        sg.fill(q, SEED, 4, "normal", 1.0)
        cache = fg.DeviceKVCache(B, nh, hd, S + 1, 64, dev)
        fg.fg_kv_append(cache, kv, kv[:, h:], 2 * h, S)
        del kv
        out = torch.empty((B, h), dtype=torch.float16, device=dev)
        run = lambda: fg.fg_decode_attention(q, 3 * h, cache, out=out)
        work = {"bytes": B * nh * S * 2.0 * (hd / 2 + 4.0 * hd / 64) + 4.0 * B * h}
    elif args.case == "prefill_attention":
        B, L, nh, hd = 64, 512, 32, 128
        h = nh * hd
        qkv = torch.empty((B * L, 3 * h), dtype=torch.float16, device=dev)
        sg.fill(qkv, SEED, 5, "normal", 1.0)
        out = torch.empty((B * L, h), dtype=torch.float16, device=dev)
        run = lambda: fg.fg_prefill_attention(qkv, B, L, nh, hd, out=out)
        # projections read once, output written once: 1.07 GB; 137 GFLOP (causal)
        work = {"flops": 4.0 * B * nh * L * (L + 1) / 2.0 * hd, "bytes": 2.0 * B * L * 4 * h}
    else:
        x = torch.empty((131072, 4096), dtype=torch.float16, device=dev)
        sg.fill(x, SEED, 7, "normal", 0.02)
        codes = torch.empty((131072, 2048), dtype=torch.uint8, device=dev)
        params = torch.empty((131072, 64, 2), dtype=torch.float16, device=dev)
        run = lambda: fg.fg_quantize_pack(x, 64, 1, codes, params)
        work = {"bytes": x.numel() * (2 + 0.5 + 4 / 64)}
    ms, ms_eager = time_launches(run, args.steps, args.warmup)
    res = {"case": args.case, "ms_per_launch": ms, "ms_per_launch_eager": ms_eager}
    if "flops" in work:
        res["TFLOP/s"] = work["flops"] / (ms * 1e-3) / 1e12
    if "bytes" in work:
        res["GB/s"] = work["bytes"] / (ms * 1e-3) / 1e9
    print(json.dumps(res))


# ---------------------------------------------------------------------------- replicas
# N > 1: N independent replicas, one process per GPU; each generates its own batch (seeded by
# its rank) and the only cross-rank traffic is the barrier and the max of the timings.
def replica_env():
    """(world, rank, local_rank) from the torchrun environment (1, 0, 0 without it)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def replica_seed(rank):
    """Seed of a replica's prompt ids: every rank generates a different batch."""
    return SEED + rank


def max_over_ranks(x, device):
    """The largest per-rank value (the slowest rank's time) over the process group, if any."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank_step, world, steps, ms_max):
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank_step * world * steps / (ms_max / 1000.0)


# ---------------------------------------------------------------------------- main
def run_generate(args, fg, torch, dev, stream, world, rank, barrier):
    """The timed generations of a full decoder (c2, c3) through fg_generate."""
    from fg_synth import gpu as sg
    import fg_synth
    c = CFG
    offload = args.weights == "offload"
    model, caches = build_model(fg, torch, dev, "4bit" if offload else args.weights)
    B, L, T = c["batch"], c["prompt_len"], c["gen_len"]
    ids = torch.empty((B, L), dtype=torch.int32, device=dev)
    sg.fill_ids(ids, replica_seed(rank), fg_synth.S_IDS, c["vocab"])
    out = torch.empty((B, T), dtype=torch.int32, device=dev)
    h2d_weights = [0.0]
    if offload:
        # every layer's 4-bit weights to pinned host memory; the device copies are freed
        mc = model.c
        host_layers = []
        for i in range(len(model.layers)):
            host_layers.append(fg.pinned_layer(model.layers[i]))
            model.layers[i] = None
        E, P, g1, b1 = model.tensors
        model = fg.DeviceModel(mc.n_layers, mc.hidden, mc.n_heads, mc.head_dim, mc.ffn, mc.vocab, mc.max_pos,
                               mc.group, E, P, g1, b1, host_layers)
        torch.cuda.empty_cache()
        ws = torch.empty((fg.fg_offload_workspace_bytes(model, B, L, T),), dtype=torch.uint8, device=dev)

        def generate():
            o, tm, hb = fg.fg_generate_offload(model, ids, T, caches, out_ids=out, workspace=ws)
            h2d_weights[0] = hb
            return o, tm
    else:
        ws = torch.empty((fg.fg_workspace_bytes(model, B, L, T),), dtype=torch.uint8, device=dev)

        def generate():
            return fg.fg_generate(model, ids, T, caches, out_ids=out, workspace=ws)
    torch.cuda.synchronize()

    # The roofline kernel (the prompt-pass GEMM) is timed by CUDA events from the warm-up on:
    # the library records them as nodes of its CUDA graphs (first call eager, second
    # captured, later ones replayed), so the timed steps replay graphs that carry them.
    # Only that kernel class is timed here; the per-kernel breakdown comes from one more,
    # separately profiled step after the timed regions.
    fg.fg_profile_select([0])
    fg.fg_profile_enable(True)
    for _ in range(args.warmup):
        generate()
    # ---- timed region: device-resident inputs
    fg.fg_profile_reset()
    launches0 = fg.fg_launch_count()
    timings = []
    barrier()
    with ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ else 0) as clk:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            _, tm = generate()
            timings.append((tm.prefill_ms, tm.decode_ms))
        e1.record(stream)
        barrier()
    launches = fg.fg_launch_count() - launches0
    ms_total = max_over_ranks(e0.elapsed_time(e1), dev)
    prof = fg.fg_profile_read(0)
    clocks = clk.summary()

    # ---- e2e: host buffers through the public API, copies inside the timed region (the
    # prompt ids go host -> the same device buffer, so the recorded graphs stay valid)
    ids_host = ids.cpu().pin_memory()
    out_host = torch.empty((B, T), dtype=torch.int32).pin_memory()
    e2e_steps = max(1, min(args.steps, 5))
    barrier()
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    for _ in range(e2e_steps):
        ids.copy_(ids_host, non_blocking=True)
        generate()
        out_host.copy_(out, non_blocking=True)
    e3.record(stream)
    barrier()
    ms_e2e = max_over_ranks(e2.elapsed_time(e3), dev)

    # ---- per-kernel breakdown: every kernel class timed, one replayed step (not timed above)
    fg.fg_profile_select(None)
    for _ in range(2):   # eager, then captured with the new timing nodes
        generate()
    fg.fg_profile_reset()
    generate()
    breakdown = {fg.PROF_NAMES[k]: fg.fg_profile_read(k) for k in range(7)}
    fg.fg_profile_enable(False)
    del model, caches, ws
    torch.cuda.empty_cache()
    return dict(ms_total=ms_total, ms_e2e=ms_e2e, e2e_steps=e2e_steps, timings=timings, prof=prof,
                breakdown=breakdown, clocks=clocks, launches=launches,
                h2d=B * L * 4, d2h=B * T * 4, h2d_weights=h2d_weights[0])


def run_slice(args, fg, torch, dev, stream, world, rank, barrier):
    """The timed steps of a layer slice (c4) through fg_prefill_layer / fg_decode_layer: the
    prompt pass over B x L hidden states, then gen_len decode steps of one new token per
    sequence, every layer in turn.  Launched eagerly (the host issues ~120 launches per
    decode step, far ahead of the GPU's ~10 ms of work per step)."""
    from fg_synth import gpu as sg
    import fg_synth
    c = CFG
    layers, caches = build_model(fg, torch, dev, args.weights)
    B, L, T, h, F = c["batch"], c["prompt_len"], c["gen_len"], c["hidden"], c["ffn"]
    x0 = torch.empty((B * L, h), dtype=torch.float16, device=dev)
    sg.fill(x0, replica_seed(rank), fg_synth.S_HIDDEN, "normal", 1.0)
    xdec = torch.empty((T, B, h), dtype=torch.float16, device=dev)
    sg.fill(xdec, replica_seed(rank), fg_synth.S_DECODE_X, "normal", 1.0)
    x = torch.empty_like(x0)
    xa = torch.empty((B, h), dtype=torch.float16, device=dev)
    wsb = max(fg.lib().fg_prefill_layer_workspace_bytes(h, F, B, L),
              fg.lib().fg_decode_layer_workspace_bytes(h, F, c["n_heads"], B, L + T))
    ws = torch.empty((wsb,), dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()

    def step(prompt, dec_inputs, marks=None):
        x.copy_(prompt, non_blocking=True)
        for cache in caches:
            cache.length = 0
        for layer, cache in zip(layers, caches):
            fg.fg_prefill_layer(layer, cache, x, B, L, workspace=ws)
        if marks is not None:
            marks.record(stream)
        for j in range(T):
            cur = dec_inputs[j]
            for layer, cache in zip(layers, caches):
                fg.fg_decode_layer(layer, cache, cur, x_out=xa, workspace=ws)
                cur = xa
        return xa

    fg.fg_profile_select([0])
    fg.fg_profile_enable(True)
    for _ in range(args.warmup):
        step(x0, xdec)
    fg.fg_profile_reset()
    launches0 = fg.fg_launch_count()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier()
    with ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ else 0) as clk:
        for a, m, b in ev:
            a.record(stream)
            step(x0, xdec, m)
            b.record(stream)
        barrier()
    launches = fg.fg_launch_count() - launches0
    ms_total = max_over_ranks(ev[0][0].elapsed_time(ev[-1][2]), dev)
    timings = [(a.elapsed_time(m), m.elapsed_time(b)) for a, m, b in ev]
    prof = fg.fg_profile_read(0)
    clocks = clk.summary()

    # ---- e2e: the prompt's hidden states and the decode inputs from pinned host memory, the
    # last hidden states back to the host, every step inside the timed region
    x0_host = x0.cpu().pin_memory()
    xdec_host = xdec.cpu().pin_memory()
    xdec_dev = torch.empty_like(xdec)
    out_host = torch.empty((B, h), dtype=torch.float16).pin_memory()
    e2e_steps = max(1, min(args.steps, 5))
    barrier()
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    for _ in range(e2e_steps):
        xdec_dev.copy_(xdec_host, non_blocking=True)
        y = step(x0_host, xdec_dev)
        out_host.copy_(y, non_blocking=True)
    e3.record(stream)
    barrier()
    ms_e2e = max_over_ranks(e2.elapsed_time(e3), dev)

    fg.fg_profile_select(None)
    fg.fg_profile_reset()
    step(x0, xdec)
    breakdown = {fg.PROF_NAMES[k]: fg.fg_profile_read(k) for k in range(7)}
    fg.fg_profile_enable(False)
    del layers, caches, ws, x, x0, xdec, xdec_dev
    torch.cuda.empty_cache()
    return dict(ms_total=ms_total, ms_e2e=ms_e2e, e2e_steps=e2e_steps, timings=timings, prof=prof,
                breakdown=breakdown, clocks=clocks, launches=launches,
                h2d=(B * L + T * B) * h * 2, d2h=B * h * 2)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", choices=sorted(CONFIGS), default=DEFAULT_CONFIG,
                    help="c3: OPT-30B batch 256 (default); c2: OPT-6.7B batch 64; c4: OPT-175B 12-layer slice, batch 144")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--case", choices=["generate", "qgemm", "qgemm_decode", "gemm_f16", "gemm_prefill", "lm_head",
                                       "decode_attention", "prefill_attention", "quantize", "sweep"],
                    default="generate",
                    help="kernel-only cases sized for ncu captures (inputs larger than L2, a few GB at most)")
    ap.add_argument("--mnk", default="", help="M,N,K of the qgemm_decode case")
    ap.add_argument("--rows", type=int, default=0, help="rows M of the gemm_prefill case (default B*L)")
    ap.add_argument("--batch", type=int, default=0,
                    help="sequences per GPU instead of the configuration's (small batches: the latency side)")
    ap.add_argument("--weights", choices=["4bit", "fp16", "offload"], default="4bit",
                    help="fp16: the same generation over uncompressed weights (compression contrast); "
                         "offload: 4-bit weights in pinned host memory, streamed layer by layer")
    args = ap.parse_args()
    if args.case == "sweep":
        return sweep_case(args)
    if args.case != "generate":
        return kernel_case(args)
    c = use_config(args.config)
    if args.batch:
        c["batch"] = args.batch
    world, rank, local = replica_env()
    wdesc = {"4bit": "4-bit weights", "fp16": "fp16 (uncompressed) weights",
             "offload": "4-bit weights in pinned host memory (streamed per layer)"}[args.weights]
    config = {"workload": describe(c, wdesc), "name": args.config, "layers": c["n_layers"], "hidden": c["hidden"],
              "heads": f"{c['n_heads']}x{c['head_dim']}", "ffn": c["ffn"], "vocab": c["vocab"] or None,
              "global_batch": c["batch"] * max(world, args.gpus if world == 1 else world),
              "prompt_len": c["prompt_len"], "gen_len": c["gen_len"], "group": c["group"],
              "parallelism": f"replicas x{max(world, 1)} (batch-sharded, no exchange)",
              "l2": f"inputs larger than L2 ({weight_bytes_4bit(c) / 1e9:.1f} GB of 4-bit weights and the KV "
                    f"cache read every decode step)"}
    if c["kind"] == "slice":
        config["full_layers"] = c["full_layers"]

    if args.impl == "reference":
        if rank != 0:
            return
        steps, warmup = args.steps, args.warmup
        cb = cpu_baseline_line(args, steps, warmup, single_thread=False)
        line = {"metric": METRIC, "value": cb["value"], "unit": "tokens/s", "n_gpus": world, "steps": steps,
                "warmup": warmup, "ms_per_step": 1000.0 * tokens_per_step(c) / cb["value"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": config, "impl": "reference",
                "cpu_baseline": {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")},
                "e2e": {"value": cb["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    import torch
    import bit_group_quantized_fg_b200 as fg
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()

    if c["kind"] == "slice" and args.weights == "offload":
        raise SystemExit("--weights offload runs a full decoder (c2 or c3)")
    runner = run_slice if c["kind"] == "slice" else run_generate
    r = runner(args, fg, torch, dev, stream, world, rank, barrier)
    B, L, T = c["batch"], c["prompt_len"], c["gen_len"]
    scale = c["n_layers"] / c["full_layers"] if c["kind"] == "slice" else 1.0
    ms_step = r["ms_total"] / args.steps
    slice_value = job_throughput(tokens_per_step(c), world, args.steps, r["ms_total"])
    value = slice_value * scale
    e2e_value = job_throughput(tokens_per_step(c), world, r["e2e_steps"], r["ms_e2e"]) * scale

    # ---- quantizer GB/s on a 1 GiB fp16 tensor (group 64), bytes = 2 + 0.5 + 4/64 per element
    from fg_synth import gpu as sg
    xq = torch.empty((131072, 4096), dtype=torch.float16, device=dev)
    sg.fill(xq, SEED, 7, "normal", 0.02)
    codes = torch.empty((131072, 2048), dtype=torch.uint8, device=dev)
    params = torch.empty((131072, 64, 2), dtype=torch.float16, device=dev)
    for _ in range(3):
        fg.fg_quantize_pack(xq, 64, 1, codes, params)
    e4, e5 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 10
    e4.record(stream)
    for _ in range(reps):
        fg.fg_quantize_pack(xq, 64, 1, codes, params)
    e5.record(stream)
    torch.cuda.synchronize()
    q_ms = e4.elapsed_time(e5) / reps
    q_gbs = xq.numel() * (2 + 0.5 + 4 / 64) / (q_ms * 1e-3) / 1e9
    del xq, codes, params

    # ---- decode attention GB/s at the last decode step's shape of this workload (larger
    # than L2), timed on its own
    S_att = L + T - 1
    h, nh, hd, g = c["hidden"], c["n_heads"], c["head_dim"], c["group"]
    acache = fg.DeviceKVCache(B, nh, hd, S_att, g, dev)
    qa = torch.empty((B, 3 * h), dtype=torch.float16, device=dev)
    sg.fill(qa, SEED, 4, "normal", 1.0)
    kvsrc = torch.empty((B * S_att, 2 * h), dtype=torch.float16, device=dev)   # 4 GB at c3
    sg.fill(kvsrc, SEED, 3, "normal", 1.0)
    fg.fg_kv_append(acache, kvsrc, kvsrc[:, h:], 2 * h, S_att)
    del kvsrc
    torch.cuda.empty_cache()
    aout = torch.empty((B, h), dtype=torch.float16, device=dev)
    for _ in range(3):
        fg.fg_decode_attention(qa, 3 * h, acache, out=aout)
    e4.record(stream)
    for _ in range(reps):
        fg.fg_decode_attention(qa, 3 * h, acache, out=aout)
    e5.record(stream)
    torch.cuda.synchronize()
    att_ms = e4.elapsed_time(e5) / reps
    att_bytes = B * nh * S_att * 2.0 * (hd / 2 + 4.0 * hd / g) + 4.0 * B * h
    att_gbs = att_bytes / (att_ms * 1e-3) / 1e9
    del acache, qa, aout

    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    pk = peaks()
    prof, breakdown = r["prof"], r["breakdown"]
    g_ms = prof["ms"] / max(prof["launches"], 1)
    g_flops = prof["flops"] / max(prof["launches"], 1)
    achieved_tf = g_flops / (g_ms * 1e-3) / 1e12 if g_ms > 0 else 0.0
    traffic = None
    tfile = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tfile):
        traffic = json.load(open(tfile)).get(f"gemm_prefill_bytes_per_launch_{args.config}")
    da = breakdown["decode_attention"]
    kernels = {}
    for name, p in breakdown.items():
        if p["launches"]:
            d = {"launches_per_step": p["launches"], "ms_per_step": p["ms"]}
            if p["flops"] and p["ms"]:
                d["TFLOP/s"] = p["flops"] / (p["ms"] * 1e-3) / 1e12
            if p["bytes"] and p["ms"]:
                d["GB/s"] = p["bytes"] / (p["ms"] * 1e-3) / 1e9
            kernels[name] = d
    M_pf = B * L
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16", "data": "synthetic", "config": config,
        "prefill_ms": statistics.median(t[0] for t in r["timings"]),
        "decode_ms": statistics.median(t[1] for t in r["timings"]),
        "roofline": {"kernel": f"tcgen05 GEMM of the prompt pass on CTA pairs (M = {M_pf}; " +
                               ("4-bit weights expanded to fp16 once per layer)" if args.weights != "fp16"
                                else "uncompressed fp16 weights)"), "bound": "tensor",
                     "achieved": achieved_tf, "peak": pk["tf_sust"], "unit": "TFLOP/s",
                     "frac": achieved_tf / pk["tf_sust"], "traffic": traffic,
                     "flop_per_launch": g_flops, "ms_per_launch": g_ms,
                     "peak_source": f"bf16_tflops_sustained of {pk['src']} peaks (fp16 and bf16 dense rates are equal)"},
        "quantizer": {"GB/s": q_gbs, "frac": q_gbs / pk["hbm"], "peak_GB/s": pk["hbm"],
                      "tensor": "1 GiB fp16 (131072 x 4096), group 64"},
        "decode_attention": {"GB/s": att_gbs, "frac": att_gbs / pk["hbm"], "peak_GB/s": pk["hbm"],
                             "shape": f"B {B}, {nh} x {hd}, context {S_att}, group {g}",
                             "in_step_GB/s": da["bytes"] / (da["ms"] * 1e-3) / 1e9 if da["ms"] else None},
        "kernels": kernels,
        "kernels_note": "one extra step with every kernel class timed (outside the timed region)",
        "clocks": r["clocks"],
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": r["h2d"],
                "d2h_bytes_per_step": r["d2h"], "steps": r["e2e_steps"]},
        "gpu_launches": r["launches"],
    }
    if r.get("h2d_weights"):
        per_step_s = ms_step * 1e-3
        line["offload"] = {"weight_bytes_h2d_per_step": r["h2d_weights"],
                           "host_link_GB/s": r["h2d_weights"] / per_step_s / 1e9,
                           "note": "weights cross the host link once per pass (prompt pass + each decode step)"}
    if c["kind"] == "slice":
        line["slice"] = {"tokens_per_s_12_layers": slice_value, "per_layer_tokens_per_s": slice_value * c["n_layers"],
                         "extrapolation": f"value = slice tokens/s x {c['n_layers']}/{c['full_layers']} "
                                          "(per-layer time constant; embedding and LM head excluded)"}
    if world == 1 and not args.no_cpu_baseline:
        try:
            cb = cpu_baseline_line(args, 1, 0)
            line["cpu_baseline"] = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample", "single_thread")}
        except Exception as ex:  # the baseline is informative only
            line["cpu_baseline"] = {"value": None, "unit": "tokens/s", "cores": os.cpu_count(), "kind": "oracle",
                                    "sample": f"failed: {ex}"}
    print(json.dumps(line))


if __name__ == "__main__":
    main()
