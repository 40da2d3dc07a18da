"""The OPT-shaped decoder over 4-bit weights and a 4-bit KV cache: the oracle's decoder
(test infrastructure only).

Every value here is computed by the C++ oracle (``fg_oracle.cpp``: LayerNorm, the linear
layer, prefill and decode attention, the KV append, the layers, the embedding, the LM head
and the generation loop); this module holds the model state as numpy arrays and shapes
buffers for those calls.

The pages name the model family and workload only: OPT-6.7B/30B/175B generation with
input length 512 and output length 32, throughput = generated tokens / (prompt time +
generation time) ("FlexGen" README mirror, benchmark table and its workload/metric
notes), with weights and attention cache compressed to 4 bits (same page, key features;
arXiv 2303.06865 record, abstract).  The block is the standard OPT decoder block
(pre-LayerNorm, multi-head causal attention, ReLU FFN, learned positions, tied LM head).
Readings taken where the pages are silent (D1-D7 in the C++ file):

* Y = X @ W + b with W stored [in][out] (out contiguous) and quantized in groups along
  `out`; Q, K and V come from one [h, 3h] projection, columns q | k | v, head j owning
  columns j*hd .. (j+1)*hd-1 of each part.
* fp16 at the storage points (residual stream, LayerNorm outputs, projection outputs,
  attention outputs, the dequantized weights and K/V), float64 in between.
* LayerNorm eps = 1e-5 inside the square root, population variance over the hidden dim.
* Attention scale 1/sqrt(hd).  Prefill attention uses this pass's unquantized fp16 K/V;
  every token's K and V is then appended to the 4-bit cache in groups of g along the
  hidden dimension.  A decode step appends the new token first and then attends over
  positions 0..len (the new one included), consuming the exact values mn + code*s.
* Embedding x = fp16(E[id] + P[pos]) (one rounding), positions 0..L-1 for the prompt and
  L+j-1 for the j-th generated token; no position offset.
* LM head logits = LN_f(x) @ E^T with the tied fp16 embedding; greedy token = argmax,
  ties to the lowest id.
* T output tokens = 1 from the prompt pass + T-1 decode steps.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

from . import _lib
from ._lib import f16, lib, p
from .quant import quantize_pack, dequantize

LN_EPS = 1e-5


def layernorm(x16: np.ndarray, g16: np.ndarray, b16: np.ndarray, eps: float = LN_EPS) -> np.ndarray:
    """y = (x - mean) / sqrt(var + eps) * gamma + beta over the last axis -> fp16."""
    x = f16(x16)
    h = x.shape[-1]
    y = np.empty_like(x)
    lib().orc_layernorm(p(x), x.size // h, h, p(f16(g16)), p(f16(b16)), float(eps), p(y))
    return y


@dataclass
class QLinear:
    """A linear layer whose [K][N] weight is stored as 4-bit codes + {min, scale} params."""
    codes: np.ndarray           # uint8 [K, N/2]
    params: np.ndarray          # fp16 [K, N/group, 2]
    bias: np.ndarray            # fp16 [N]
    K: int
    N: int
    group: int = 64
    axis: int = 1               # 1: groups along N (output channel), 0: along K (input dim)
    _w16: Optional[np.ndarray] = field(default=None, repr=False)

    @staticmethod
    def from_fp16(w16: np.ndarray, b16: np.ndarray, group: int = 64, axis: int = 1) -> "QLinear":
        K, N = w16.shape
        codes, params = quantize_pack(w16, group, axis=axis)
        return QLinear(codes, params, f16(b16), K, N, group, axis)

    def weight16(self) -> np.ndarray:
        """W_hat as fp16 [K, N] (the oracle's dequantization of the stored weight)."""
        if self._w16 is None:
            self._w16 = dequantize(self.codes, self.params, self.K, self.N, self.group, self.axis)
        return self._w16

    def weight(self) -> np.ndarray:
        """W_hat as float64 [K, N] (the exact fp16 values)."""
        return self.weight16().astype(np.float64)

    def columns(self, cols) -> np.ndarray:
        """Dequantized columns ``cols`` only, float64 [K, len(cols)]; only the groups holding
        them are dequantized (for sampled checks of large weights)."""
        assert self.axis == 1, "column sampling reads groups along N"
        cols = np.asarray(cols)
        g = self.group
        out = np.empty((self.K, len(cols)), np.float64)
        for gi in np.unique(cols // g):
            gi = int(gi)
            codes = np.ascontiguousarray(self.codes[:, gi * g // 2:(gi + 1) * g // 2])
            params = np.ascontiguousarray(np.asarray(self.params, np.float16).reshape(self.K, -1, 2)[:, gi])
            wg = dequantize(codes, params, self.K, g, g, 1)
            sel = np.nonzero(cols // g == gi)[0]
            out[:, sel] = wg[:, cols[sel] - gi * g].astype(np.float64)
        return out


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

    def weight16(self) -> np.ndarray:
        return f16(self.w16)

    def weight(self) -> np.ndarray:
        return self.weight16().astype(np.float64)


def qlinear(a16: np.ndarray, lin, relu: bool = False, residual16: Optional[np.ndarray] = None) -> np.ndarray:
    """fp16( [relu](a @ W_hat + b) [+ residual] ), float64 in between (QLinear or Linear16)."""
    a = f16(a16)
    K = a.shape[-1]
    M = a.size // K
    W = lin.weight16()
    assert W.shape == (K, lin.N)
    r = None if residual16 is None else f16(residual16).reshape(M, lin.N)
    y = np.empty(a.shape[:-1] + (lin.N,), np.float16)
    lib().orc_linear(p(a), M, K, p(W), K, lin.N, p(None if lin.bias is None else f16(lin.bias)), int(relu), p(r),
                     p(y))
    return y


def linear_fp16(a16: np.ndarray, w_nk16: np.ndarray) -> np.ndarray:
    """a @ W^T for an fp16 weight stored [N][K]; float64 result (logits)."""
    a = f16(a16)
    E = f16(w_nk16)
    M, K = a.shape
    out = np.empty((M, E.shape[0]), np.float64)
    lib().orc_linear_nk(p(a), M, p(E), E.shape[0], K, p(out))
    return out


@dataclass
class QLayer:
    ln1_g: np.ndarray
    ln1_b: np.ndarray
    ln2_g: np.ndarray
    ln2_b: np.ndarray
    qkv: object
    out: object
    fc1: object
    fc2: object


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

    def c(self) -> _lib.Cache:
        """The C view of this cache (pointers into the numpy arrays)."""
        return _lib.Cache(p(self.k_codes), p(self.v_codes), p(self.k_params), p(self.v_params), self.B,
                          self.n_heads, self.head_dim, self.group, self.capacity, self.length)


def kv_append(cache: KVCache, k16: np.ndarray, v16: np.ndarray, pos: int) -> None:
    """Quantize tokens' K and V rows ([B, T, h] or [B, h]) into positions pos.. of the cache."""
    k = f16(k16)
    v = f16(v16)
    if k.ndim == 2:
        k, v = k[:, None, :], v[:, None, :]
    B, T, h = k.shape
    if pos + T > cache.capacity:
        raise ValueError("KV cache capacity exceeded")
    c = cache.c()
    assert lib().orc_kv_append(ctypes.byref(c), p(k), p(v), h, T, pos) == 0


def cache_dequant(cache: KVCache, which: str, b: int, head: int, S: int) -> np.ndarray:
    """Dequantized K or V of one (sequence, head) for positions 0..S-1, fp16 [S, hd]
    (the storage form, as fg_dequantize would write it)."""
    codes = np.ascontiguousarray((cache.k_codes if which == "k" else cache.v_codes)[b, head, :S])
    params = np.ascontiguousarray((cache.k_params if which == "k" else cache.v_params)[b, head, :S])
    return dequantize(codes, params, S, cache.head_dim, cache.group, 1)


def cache_values(cache: KVCache, which: str, b: int, head: int, S: int) -> np.ndarray:
    """Exact values mn + code*s of one (sequence, head), positions 0..S-1, float64 [S, hd]:
    what attention consumes (no second rounding to fp16)."""
    codes = np.ascontiguousarray((cache.k_codes if which == "k" else cache.v_codes)[b, head, :S])
    params = np.ascontiguousarray((cache.k_params if which == "k" else cache.v_params)[b, head, :S])
    out = np.empty((S, cache.head_dim), np.float64)
    lib().orc_code_values(p(codes), p(params), S, cache.head_dim, cache.group, p(out))
    return out


def prefill_attention(qkv16: np.ndarray, n_heads: int, head_dim: int) -> np.ndarray:
    """Causal multi-head attention over [B, L, 3h] fp16 projections -> fp16 [B, L, h]."""
    qkv = f16(qkv16)
    B, L, h3 = qkv.shape
    out = np.empty((B, L, h3 // 3), np.float16)
    lib().orc_prefill_attention(p(qkv), B, L, n_heads, head_dim, p(out))
    return out


def decode_attention(q16: np.ndarray, cache: KVCache, S: int) -> np.ndarray:
    """One query per sequence over cached positions 0..S-1 (exact code values) -> fp16 [B, h]."""
    q = f16(q16)
    B = q.shape[0]
    out = np.empty((B, cache.n_heads * cache.head_dim), np.float16)
    c = cache.c()
    lib().orc_decode_attention(p(q), q.shape[1], ctypes.byref(c), S, p(out))
    return out


def _linear_c(lin) -> _lib.LinearW:
    return _lib.LinearW(p(lin.weight16()), p(None if lin.bias is None else f16(lin.bias)), lin.K, lin.N)


class _LayerC:
    """C view of a QLayer, holding references to every buffer it points at."""

    def __init__(self, layer: QLayer):
        self.keep = [f16(layer.ln1_g), f16(layer.ln1_b), f16(layer.ln2_g), f16(layer.ln2_b)]
        for lin in (layer.qkv, layer.out, layer.fc1, layer.fc2):
            self.keep += [lin.weight16(), None if lin.bias is None else f16(lin.bias)]
        lins = []
        for i in range(4):
            w, b = self.keep[4 + 2 * i], self.keep[5 + 2 * i]
            lin = (layer.qkv, layer.out, layer.fc1, layer.fc2)[i]
            lins.append(_lib.LinearW(p(w), p(b), lin.K, lin.N))
        self.c = _lib.Layer(*[p(a) for a in self.keep[:4]], *lins)


def prefill_layer(layer: QLayer, cache: KVCache, x16: np.ndarray) -> np.ndarray:
    """One decoder block over a whole prompt [B, L, h]; writes cache positions 0..L-1."""
    x = np.array(x16, dtype=np.float16, copy=True, order="C")
    B, L, h = x.shape
    lc = _LayerC(layer)
    cc = cache.c()
    cc.len = 0
    assert lib().orc_prefill_layer(ctypes.byref(lc.c), ctypes.byref(cc), p(x), B, L) == 0
    cache.length = cc.len
    return x


def decode_layer(layer: QLayer, cache: KVCache, x16: np.ndarray) -> np.ndarray:
    """One decoder block for one new token per sequence [B, h]; appends at cache.length."""
    x = f16(x16)
    B, h = x.shape
    y = np.empty_like(x)
    lc = _LayerC(layer)
    cc = cache.c()
    assert lib().orc_decode_layer(ctypes.byref(lc.c), ctypes.byref(cc), p(x), p(y), B) == 0
    cache.length = cc.len
    return y


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


class _ModelC:
    def __init__(self, m: Model):
        self.keep = [f16(m.embed), f16(m.pos_embed), f16(m.lnf_g), f16(m.lnf_b)]
        self.layers = [_LayerC(l) for l in m.layers]
        arr = (_lib.Layer * max(1, len(self.layers)))(*[l.c for l in self.layers])
        self.arr = arr
        self.c = _lib.Model(m.n_layers, m.hidden, m.n_heads, m.head_dim, m.ffn, m.vocab, m.max_pos, m.group,
                            *[p(a) for a in self.keep], ctypes.cast(arr, ctypes.POINTER(_lib.Layer)))


def embed(model: Model, ids: np.ndarray, pos0: int) -> np.ndarray:
    """fp16(E[id] + P[pos]) with one rounding; ids [B, T] -> [B, T, h]."""
    ids = np.ascontiguousarray(ids, np.int32)
    B, T = ids.shape
    mc = _ModelC(model)
    out = np.empty((B, T, model.hidden), np.float16)
    lib().orc_embed(ctypes.byref(mc.c), p(ids), B, T, pos0, p(out))
    return out


def lm_head_argmax(model: Model, x16: np.ndarray):
    """Final LayerNorm, tied LM head, greedy argmax (lowest id on ties).  x16 [B, h]."""
    x = f16(x16)
    B = x.shape[0]
    mc = _ModelC(model)
    logits = np.empty((B, model.vocab), np.float64)
    tok = np.empty(B, np.int32)
    lib().orc_lm_head_argmax(ctypes.byref(mc.c), p(x), B, p(logits), p(tok))
    return tok, logits


def generate(model: Model, ids: np.ndarray, gen_len: int, return_logits: bool = False):
    """Greedy generation: prefill over the prompt, then gen_len-1 decode steps.

    Returns tokens [B, gen_len] (and the float64 logits [gen_len, B, vocab] if asked).
    """
    ids = np.ascontiguousarray(ids, np.int32)
    B, L = ids.shape
    caches = [KVCache(B, model.n_heads, model.head_dim, model.group, L + gen_len) for _ in range(model.n_layers)]
    cc = (_lib.Cache * max(1, len(caches)))(*[c.c() for c in caches])
    mc = _ModelC(model)
    out = np.empty((B, gen_len), np.int32)
    logits = np.empty((gen_len, B, model.vocab), np.float64) if return_logits else None
    assert lib().orc_generate(ctypes.byref(mc.c), p(ids), B, L, gen_len, p(out), cc, p(logits)) == 0
    if return_logits:
        return out, logits
    return out
