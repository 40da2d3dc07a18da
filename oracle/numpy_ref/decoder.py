"""Oracle for the OPT-shaped decoder over 4-bit weights and a 4-bit KV cache
(test infrastructure only).

The pages name the model family and workload only: OPT-6.7B/30B/175B generation with
input length 512 and output length 32, throughput = generated tokens / (prompt time +
generation time) ("FlexGen" README mirror, benchmark table and its workload/metric
notes), with weights and attention cache compressed to 4 bits (same page, key features;
arXiv 2303.06865 record, abstract).  The block structure is the standard OPT decoder
block (pre-LayerNorm, multi-head causal attention, ReLU FFN, learned positions, tied
LM head).  Readings taken where the pages are silent:

* Math convention Y = X @ W + b with W stored [in][out] (out contiguous) and quantized
  in groups along `out` (see ``quant.py``); Q, K and V come from one [h, 3h] projection,
  columns ordered q | k | v, head j owning columns j*hd .. (j+1)*hd-1 of each part.
* Storage precision points (the values the GPU path keeps in memory) are fp16: the
  residual stream, LayerNorm outputs, projection outputs, attention outputs, the
  dequantized weights and K/V.  Between those points this oracle computes in float64.
* LayerNorm eps = 1e-5, statistics over the hidden dimension.
* Attention scale 1/sqrt(hd).  Prefill attention uses this pass's unquantized fp16 K/V;
  every token's K and V is then appended to the 4-bit cache in groups of g along the
  hidden dimension (g divides hd).  A decode step appends the new token first and then
  attends over all cached positions 0..len (the new one included).  Decode attention
  consumes the value each code stands for, mn + code*s, exactly (no second rounding to
  fp16); the softmax and the weighted sum are float64 here, fp32 on the GPU.
* Embedding x = fp16(E[id] + P[pos]) (one rounding), positions 0..L-1 for the prompt and
  L+j-1 for the j-th generated token; no position offset.
* LM head logits = LN_f(x) @ E^T with the tied fp16 embedding (not quantized); greedy
  token = argmax, ties to the lowest id.
* Output length T counts the token produced by the prefill: T tokens = 1 from the
  prefill + T-1 decode steps.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

from .quant import quantize_pack, dequantize

LN_EPS = 1e-5


def _f64(a):
    return np.asarray(a).astype(np.float64)


def layernorm(x16: np.ndarray, g16: np.ndarray, b16: np.ndarray, eps: float = LN_EPS) -> np.ndarray:
    """y = (x - mean) / sqrt(var + eps) * gamma + beta over the last axis -> fp16."""
    x = _f64(x16)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    y = (x - mu) / np.sqrt(var + eps) * _f64(g16) + _f64(b16)
    return y.astype(np.float16)


@dataclass
class QLinear:
    """A linear layer whose [K][N] weight is stored as 4-bit codes + {min, scale} params."""
    codes: np.ndarray           # uint8 [K, N/2]
    params: np.ndarray          # fp16 [K, N/group, 2]
    bias: np.ndarray            # fp16 [N]
    K: int
    N: int
    group: int = 64
    _w: Optional[np.ndarray] = field(default=None, repr=False)

    @staticmethod
    def from_fp16(w16: np.ndarray, b16: np.ndarray, group: int = 64) -> "QLinear":
        K, N = w16.shape
        codes, params = quantize_pack(w16, group, axis=1)
        return QLinear(codes, params, np.asarray(b16, np.float16), K, N, group)

    def weight(self) -> np.ndarray:
        """Dequantized weight as float64 [K, N] (the exact fp16 values)."""
        if self._w is None:
            self._w = dequantize(self.codes, self.params, self.K, self.N, self.group, 1).astype(np.float64)
        return self._w

    def columns(self, cols) -> np.ndarray:
        """Dequantized columns ``cols`` only, float64 [K, len(cols)] (for sampled checks)."""
        cols = np.asarray(cols)
        p = np.asarray(self.params, np.float16)
        q_lo_hi = self.codes[:, cols // 2]
        q = np.where(cols % 2 == 0, q_lo_hi & 0x0F, q_lo_hi >> 4).astype(np.float64)
        grp = p[:, cols // self.group, :]
        exact = q * grp[..., 1].astype(np.float64) + grp[..., 0].astype(np.float64)
        return exact.astype(np.float16).astype(np.float64)


@dataclass
class Linear16:
    """An uncompressed linear layer: the fp16 weight [K][N] itself stands where W_hat does
    ("FlexGen" README mirror, benchmark table: FlexGen without compression)."""
    w16: np.ndarray             # fp16 [K, N]
    bias: np.ndarray            # fp16 [N]

    @property
    def K(self) -> int:
        return self.w16.shape[0]

    @property
    def N(self) -> int:
        return self.w16.shape[1]

    def weight(self) -> np.ndarray:
        return np.asarray(self.w16, np.float16).astype(np.float64)


def qlinear(a16: np.ndarray, lin: QLinear, relu: bool = False,
            residual16: Optional[np.ndarray] = None) -> np.ndarray:
    """fp16( [relu](a @ W_hat + b) [+ residual] ), float64 in between."""
    acc = _f64(a16) @ lin.weight() + _f64(lin.bias)
    if relu:
        acc = np.maximum(acc, 0.0)
    if residual16 is not None:
        acc = acc + _f64(residual16)
    return acc.astype(np.float16)


def linear_fp16(a16: np.ndarray, w_nk16: np.ndarray) -> np.ndarray:
    """a @ W^T for an fp16 weight stored [N][K]; float64 result (logits)."""
    return _f64(a16) @ _f64(w_nk16).T


@dataclass
class QLayer:
    ln1_g: np.ndarray
    ln1_b: np.ndarray
    ln2_g: np.ndarray
    ln2_b: np.ndarray
    qkv: QLinear
    out: QLinear
    fc1: QLinear
    fc2: QLinear


@dataclass
class KVCache:
    """4-bit cache of one layer: codes [B][nh][cap][hd/2], params [B][nh][cap][hd/g][2]."""
    B: int
    n_heads: int
    head_dim: int
    group: int
    capacity: int
    length: int = 0
    k_codes: np.ndarray = None
    v_codes: np.ndarray = None
    k_params: np.ndarray = None
    v_params: np.ndarray = None

    def __post_init__(self):
        B, nh, cap, hd, g = self.B, self.n_heads, self.capacity, self.head_dim, self.group
        if hd % g:
            raise ValueError("group must divide head_dim")
        if self.k_codes is None:
            self.k_codes = np.zeros((B, nh, cap, hd // 2), np.uint8)
            self.v_codes = np.zeros((B, nh, cap, hd // 2), np.uint8)
            self.k_params = np.zeros((B, nh, cap, hd // g, 2), np.float16)
            self.v_params = np.zeros((B, nh, cap, hd // g, 2), np.float16)


def kv_append(cache: KVCache, k16: np.ndarray, v16: np.ndarray, pos: int) -> None:
    """Quantize tokens' K and V rows ([B, T, h] or [B, h]) into positions pos.. of the cache."""
    k16 = np.asarray(k16, np.float16)
    v16 = np.asarray(v16, np.float16)
    if k16.ndim == 2:
        k16, v16 = k16[:, None, :], v16[:, None, :]
    B, T, h = k16.shape
    nh, hd, g = cache.n_heads, cache.head_dim, cache.group
    if pos + T > cache.capacity:
        raise ValueError("KV cache capacity exceeded")
    for src, codes_dst, params_dst in ((k16, cache.k_codes, cache.k_params),
                                       (v16, cache.v_codes, cache.v_params)):
        codes, params = quantize_pack(src.reshape(B * T, h), g, axis=1)
        codes_dst[:, :, pos:pos + T, :] = codes.reshape(B, T, nh, hd // 2).transpose(0, 2, 1, 3)
        params_dst[:, :, pos:pos + T] = params.reshape(B, T, nh, hd // g, 2).transpose(0, 2, 1, 3, 4)


def cache_dequant(cache: KVCache, which: str, b: int, head: int, S: int) -> np.ndarray:
    """Dequantized K or V of one (sequence, head) for positions 0..S-1, fp16 [S, hd]
    (the storage form, as fg_dequantize would write it)."""
    codes = (cache.k_codes if which == "k" else cache.v_codes)[b, head, :S]
    params = (cache.k_params if which == "k" else cache.v_params)[b, head, :S]
    return dequantize(codes, params.reshape(-1, 2), S, cache.head_dim, cache.group, 1)


def cache_values(cache: KVCache, which: str, b: int, head: int, S: int) -> np.ndarray:
    """Exact values mn + code*s of one (sequence, head), positions 0..S-1, float64 [S, hd].

    This is what attention consumes: the value the 4-bit code stands for, without a
    second rounding to fp16 (the product and sum are exact in float64)."""
    codes = (cache.k_codes if which == "k" else cache.v_codes)[b, head, :S]
    params = (cache.k_params if which == "k" else cache.v_params)[b, head, :S].astype(np.float64)
    g = cache.group
    q = np.empty((S, cache.head_dim), np.float64)
    q[:, 0::2] = codes & 0x0F
    q[:, 1::2] = codes >> 4
    mn = np.repeat(params[..., 0], g, axis=1)
    sc = np.repeat(params[..., 1], g, axis=1)
    return mn + q * sc


def _softmax_rows(s: np.ndarray) -> np.ndarray:
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=-1, keepdims=True)


def prefill_attention(qkv16: np.ndarray, n_heads: int, head_dim: int) -> np.ndarray:
    """Causal multi-head attention over [B, L, 3h] fp16 projections -> fp16 [B, L, h]."""
    qkv = _f64(qkv16)
    B, L, h3 = qkv.shape
    h = h3 // 3
    out = np.empty((B, L, h), np.float64)
    scale = 1.0 / np.sqrt(head_dim)
    mask = np.triu(np.ones((L, L), bool), k=1)          # key j > query i is masked
    for j in range(n_heads):
        c = slice(j * head_dim, (j + 1) * head_dim)
        q = qkv[:, :, 0 * h:1 * h][:, :, c]
        k = qkv[:, :, 1 * h:2 * h][:, :, c]
        v = qkv[:, :, 2 * h:3 * h][:, :, c]
        s = np.einsum("bid,bjd->bij", q, k) * scale
        s[:, mask] = -np.inf
        out[:, :, c] = np.einsum("bij,bjd->bid", _softmax_rows(s), v)
    return out.astype(np.float16)


def decode_attention(q16: np.ndarray, cache: KVCache, S: int) -> np.ndarray:
    """One query per sequence over cached positions 0..S-1 (dequantized) -> fp16 [B, h]."""
    q = _f64(q16)
    B = q.shape[0]
    nh, hd = cache.n_heads, cache.head_dim
    out = np.empty((B, nh * hd), np.float64)
    scale = 1.0 / np.sqrt(hd)
    for b in range(B):
        for j in range(nh):
            c = slice(j * hd, (j + 1) * hd)
            K = cache_values(cache, "k", b, j, S)
            V = cache_values(cache, "v", b, j, S)
            p = _softmax_rows((K @ q[b, c]) * scale)
            out[b, c] = p @ V
    return out.astype(np.float16)


def prefill_layer(layer: QLayer, cache: KVCache, x16: np.ndarray) -> np.ndarray:
    """One decoder block over a whole prompt [B, L, h]; writes cache positions 0..L-1."""
    B, L, h = x16.shape
    xf = np.asarray(x16, np.float16).reshape(B * L, h)
    h1 = layernorm(xf, layer.ln1_g, layer.ln1_b)
    qkv = qlinear(h1, layer.qkv)
    kv_append(cache, qkv[:, h:2 * h].reshape(B, L, h), qkv[:, 2 * h:].reshape(B, L, h), 0)
    cache.length = L
    att = prefill_attention(qkv.reshape(B, L, 3 * h), cache.n_heads, cache.head_dim)
    x = qlinear(att.reshape(B * L, h), layer.out, residual16=xf)
    f = qlinear(layernorm(x, layer.ln2_g, layer.ln2_b), layer.fc1, relu=True)
    x = qlinear(f, layer.fc2, residual16=x)
    return x.reshape(B, L, h)


def decode_layer(layer: QLayer, cache: KVCache, x16: np.ndarray) -> np.ndarray:
    """One decoder block for one new token per sequence [B, h]; appends at cache.length."""
    x16 = np.asarray(x16, np.float16)
    h = x16.shape[1]
    h1 = layernorm(x16, layer.ln1_g, layer.ln1_b)
    qkv = qlinear(h1, layer.qkv)
    pos = cache.length
    kv_append(cache, qkv[:, h:2 * h], qkv[:, 2 * h:], pos)
    cache.length = pos + 1
    att = decode_attention(qkv[:, :h], cache, pos + 1)
    x = qlinear(att, layer.out, residual16=x16)
    f = qlinear(layernorm(x, layer.ln2_g, layer.ln2_b), layer.fc1, relu=True)
    return qlinear(f, layer.fc2, residual16=x)


@dataclass
class Model:
    n_layers: int
    hidden: int
    n_heads: int
    head_dim: int
    ffn: int
    vocab: int
    max_pos: int
    group: int
    embed: np.ndarray           # fp16 [vocab, h]
    pos_embed: np.ndarray       # fp16 [max_pos, h]
    lnf_g: np.ndarray
    lnf_b: np.ndarray
    layers: List[QLayer]


def embed(model: Model, ids: np.ndarray, pos0: int) -> np.ndarray:
    """fp16(E[id] + P[pos]) with one rounding; ids [B, T] -> [B, T, h]."""
    ids = np.asarray(ids)
    T = ids.shape[1]
    pos = np.arange(pos0, pos0 + T)
    return (_f64(model.embed[ids]) + _f64(model.pos_embed[pos])[None]).astype(np.float16)


def lm_head_argmax(model: Model, x16: np.ndarray):
    """Final LayerNorm, tied LM head, greedy argmax (lowest id on ties).  x16 [B, h]."""
    logits = linear_fp16(layernorm(x16, model.lnf_g, model.lnf_b), model.embed)
    return np.argmax(logits, axis=-1).astype(np.int32), logits   # argmax returns the first max


def generate(model: Model, ids: np.ndarray, gen_len: int, return_logits: bool = False):
    """Greedy generation: prefill over the prompt, then gen_len-1 decode steps.

    Returns tokens [B, gen_len] (and the float64 logits [gen_len, B, vocab] if asked).
    """
    ids = np.asarray(ids, np.int32)
    B, L = ids.shape
    caches = [KVCache(B, model.n_heads, model.head_dim, model.group, L + gen_len)
              for _ in range(model.n_layers)]
    x = embed(model, ids, 0)
    for layer, cache in zip(model.layers, caches):
        x = prefill_layer(layer, cache, x)
    tok, logits = lm_head_argmax(model, x[:, -1, :])
    toks, all_logits = [tok], [logits]
    for step in range(1, gen_len):
        x = embed(model, tok[:, None], L + step - 1)[:, 0, :]
        for layer, cache in zip(model.layers, caches):
            x = decode_layer(layer, cache, x)
        tok, logits = lm_head_argmax(model, x)
        toks.append(tok)
        all_logits.append(logits)
    out = np.stack(toks, axis=1)
    if return_logits:
        return out, np.stack(all_logits, axis=0)
    return out
