"""Python binding of the 4-bit group-wise compressed decode path (B200, sm_100a).

Argument marshalling only: every step runs in the CUDA kernels of ``libfg.so`` behind the
C ABI of ``include/fg.h``; PyTorch supplies device memory and streams.  There is no CPU
path: importing works without a GPU (for builds and symbol checks), but every call needs
the compiled library and a CUDA device and raises otherwise.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_double, c_float, c_int, c_int64, c_size_t, c_void_p

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfg.so")

FG_OK = 0
STATUS = {0: "FG_OK", -1: "FG_ERR_INVALID_ARG", -2: "FG_ERR_SHAPE", -3: "FG_ERR_ALIGN",
          -4: "FG_ERR_CAPACITY", -5: "FG_ERR_CUDA", -6: "FG_ERR_UNSUPPORTED", -7: "FG_ERR_WORKSPACE"}
(PROF_GEMM, PROF_DECODE_ATTN, PROF_PREFILL_ATTN, PROF_QUANT, PROF_OTHER, PROF_GEMM_DECODE,
 PROF_LM_HEAD) = range(7)
PROF_NAMES = ["gemm_prefill", "decode_attention", "prefill_attention", "quantize_append", "other",
              "gemm_decode", "lm_head"]


class FGError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class QLinear(ctypes.Structure):
    _fields_ = [("codes", c_void_p), ("params", c_void_p), ("bias", c_void_p),
                ("K", c_int), ("N", c_int), ("group", c_int), ("w16", c_void_p), ("group_along_k", c_int)]


class Layer(ctypes.Structure):
    _fields_ = [("ln1_g", c_void_p), ("ln1_b", c_void_p), ("ln2_g", c_void_p), ("ln2_b", c_void_p),
                ("qkv", QLinear), ("out", QLinear), ("fc1", QLinear), ("fc2", QLinear)]


class KVCache(ctypes.Structure):
    _fields_ = [("k_codes", c_void_p), ("v_codes", c_void_p), ("k_params", c_void_p),
                ("v_params", c_void_p), ("B", c_int), ("n_heads", c_int), ("head_dim", c_int),
                ("group", c_int), ("capacity", c_int), ("len", c_int)]


class Model(ctypes.Structure):
    _fields_ = [("n_layers", c_int), ("hidden", c_int), ("n_heads", c_int), ("head_dim", c_int),
                ("ffn", c_int), ("vocab", c_int), ("max_pos", c_int), ("group", c_int),
                ("embed", c_void_p), ("pos_embed", c_void_p), ("lnf_g", c_void_p), ("lnf_b", c_void_p),
                ("layers", POINTER(Layer))]


class Timing(ctypes.Structure):
    _fields_ = [("prefill_ms", c_float), ("decode_ms", c_float), ("tokens", c_int64),
                ("tok_per_s", c_double)]


_SIGS = {
    "fg_status_string": (ctypes.c_char_p, [c_int]),
    "fg_last_error": (ctypes.c_char_p, []),
    "fg_version": (c_int, []),
    "fg_quantize_pack": (c_int, [c_void_p, c_int64, c_int64, c_int, c_int, c_void_p, c_void_p, c_void_p]),
    "fg_dequantize": (c_int, [c_void_p, c_void_p, c_int64, c_int64, c_int, c_int, c_void_p, c_void_p]),
    "fg_kv_append": (c_int, [POINTER(KVCache), c_void_p, c_void_p, c_int64, c_int, c_void_p]),
    "fg_qgemm_workspace_bytes": (c_size_t, [c_int64, c_int, c_int]),
    "fg_qgemm": (c_int, [c_void_p, c_int64, POINTER(QLinear), c_void_p, c_int, c_void_p, c_void_p, c_size_t,
                         c_void_p]),
    "fg_gemm_f16_workspace_bytes": (c_size_t, [c_int64, c_int, c_int]),
    "fg_gemm_f16": (c_int, [c_void_p, c_int64, c_void_p, c_int, c_int, c_void_p, c_void_p, c_int, c_void_p,
                            c_void_p, c_size_t, c_void_p]),
    "fg_decode_attention_workspace_bytes": (c_size_t, [c_int, c_int, c_int, c_int]),
    "fg_decode_attention": (c_int, [c_void_p, c_int64, POINTER(KVCache), c_void_p, c_void_p, c_size_t,
                                    c_void_p]),
    "fg_decode_attention_noalloc": (c_int, [c_void_p, c_int64, POINTER(KVCache), c_void_p, c_void_p]),
    "fg_prefill_attention": (c_int, [c_void_p, c_int, c_int, c_int, c_int, c_void_p, c_void_p]),
    "fg_layernorm": (c_int, [c_void_p, c_int64, c_int, c_void_p, c_void_p, c_void_p, c_void_p]),
    "fg_embed": (c_int, [c_void_p, c_int, c_int, c_int, c_void_p, c_void_p, c_int, c_void_p, c_void_p]),
    "fg_lm_head_workspace_bytes": (c_size_t, [c_int, c_int]),
    "fg_lm_head_argmax": (c_int, [c_void_p, c_int, c_int, c_void_p, c_int, c_void_p, c_void_p, c_void_p,
                                  c_size_t, c_void_p]),
    "fg_decode_layer_workspace_bytes": (c_size_t, [c_int, c_int, c_int, c_int, c_int]),
    "fg_decode_layer": (c_int, [POINTER(Layer), POINTER(KVCache), c_void_p, c_void_p, c_int, c_void_p,
                                c_size_t, c_void_p]),
    "fg_prefill_layer_workspace_bytes": (c_size_t, [c_int, c_int, c_int, c_int]),
    "fg_prefill_layer": (c_int, [POINTER(Layer), POINTER(KVCache), c_void_p, c_int, c_int, c_void_p,
                                 c_size_t, c_void_p]),
    "fg_workspace_bytes": (c_size_t, [POINTER(Model), c_int, c_int, c_int]),
    "fg_generate": (c_int, [POINTER(Model), c_void_p, c_int, c_int, c_int, c_void_p, POINTER(KVCache),
                            c_void_p, c_size_t, POINTER(Timing), c_void_p]),
    "fg_offload_workspace_bytes": (c_size_t, [POINTER(Model), c_int, c_int, c_int]),
    "fg_generate_offload": (c_int, [POINTER(Model), c_void_p, c_int, c_int, c_int, c_void_p, POINTER(KVCache),
                                    c_void_p, c_size_t, POINTER(Timing), POINTER(c_double), c_void_p]),
    "fg_profile_enable": (c_int, [c_int]),
    "fg_profile_select": (c_int, [ctypes.c_uint]),
    "fg_profile_read": (c_int, [c_int, POINTER(c_double), POINTER(c_int64), POINTER(c_double),
                                POINTER(c_double)]),
    "fg_profile_reset": (c_int, []),
    "fg_launch_count": (c_int64, []),
}

_lib = None


def lib():
    """Load libfg.so (raises if it has not been built: there is no fallback path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with bit_group_quantized_fg_b200/build.py")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(status: int):
    if status != FG_OK:
        raise FGError(status, lib().fg_last_error().decode())


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def _empty(shape, dtype, device):
    import torch
    return torch.empty(shape, dtype=dtype, device=device)


# ------------------------------------------------------------------------- compression
def fg_quantize_pack(x, group: int = 64, axis: int = 1, codes=None, params=None, stream=None):
    """x fp16 [rows, cols] (CUDA) -> (codes uint8 [rows, cols/2], params fp16 [..., 2])."""
    import torch
    rows, cols = x.shape
    if codes is None:
        codes = _empty((rows, cols // 2), torch.uint8, x.device)
    if params is None:
        pshape = (rows, cols // group, 2) if axis == 1 else (rows // group, cols, 2)
        params = _empty(pshape, torch.float16, x.device)
    _check(lib().fg_quantize_pack(_ptr(x), rows, cols, group, axis, _ptr(codes), _ptr(params), _stream(stream)))
    return codes, params


def fg_dequantize(codes, params, rows: int, cols: int, group: int = 64, axis: int = 1, out=None, stream=None):
    import torch
    if out is None:
        out = _empty((rows, cols), torch.float16, codes.device)
    _check(lib().fg_dequantize(_ptr(codes), _ptr(params), rows, cols, group, axis, _ptr(out), _stream(stream)))
    return out


# ------------------------------------------------------------------------- state holders
class DeviceQLinear:
    """A 4-bit linear layer resident in HBM (keeps the tensors alive for the C struct)."""

    def __init__(self, codes, params, bias, K: int, N: int, group: int = 64, w16=None, along_k: bool = False):
        self.codes, self.params, self.bias, self.w16 = codes, params, bias, w16
        self.K, self.N, self.group, self.along_k = K, N, group, along_k
        self.c = QLinear(_ptr(codes), _ptr(params), _ptr(bias), K, N, group, _ptr(w16), int(along_k))

    @staticmethod
    def from_fp16(w, bias, group: int = 64, stream=None, along_k: bool = False) -> "DeviceQLinear":
        """Quantize an fp16 weight [K][N] on the GPU: groups along N (output channel) by
        default, along K (input dimension) with along_k."""
        K, N = w.shape
        codes, params = fg_quantize_pack(w, group, 0 if along_k else 1, stream=stream)
        return DeviceQLinear(codes, params, bias, K, N, group, along_k=along_k)

    @staticmethod
    def uncompressed(w, bias) -> "DeviceQLinear":
        """The same layer over the fp16 weight itself (no compression)."""
        K, N = w.shape
        return DeviceQLinear(None, None, bias, K, N, 64, w16=w)


class DeviceLayer:
    def __init__(self, ln1_g, ln1_b, ln2_g, ln2_b, qkv: DeviceQLinear, out: DeviceQLinear,
                 fc1: DeviceQLinear, fc2: DeviceQLinear):
        self.t = (ln1_g, ln1_b, ln2_g, ln2_b)
        self.qkv, self.out, self.fc1, self.fc2 = qkv, out, fc1, fc2
        self.c = Layer(_ptr(ln1_g), _ptr(ln1_b), _ptr(ln2_g), _ptr(ln2_b), qkv.c, out.c, fc1.c, fc2.c)


class DeviceKVCache:
    """4-bit KV cache of one layer in HBM: codes [B][nh][cap][hd/2], params [B][nh][cap][hd/g][2]."""

    def __init__(self, B: int, n_heads: int, head_dim: int, capacity: int, group: int = 64, device="cuda"):
        import torch
        self.k_codes = torch.zeros((B, n_heads, capacity, head_dim // 2), dtype=torch.uint8, device=device)
        self.v_codes = torch.zeros_like(self.k_codes)
        self.k_params = torch.zeros((B, n_heads, capacity, head_dim // group, 2), dtype=torch.float16,
                                    device=device)
        self.v_params = torch.zeros_like(self.k_params)
        self.c = KVCache(_ptr(self.k_codes), _ptr(self.v_codes), _ptr(self.k_params), _ptr(self.v_params),
                         B, n_heads, head_dim, group, capacity, 0)

    @property
    def length(self) -> int:
        return self.c.len

    @length.setter
    def length(self, v: int):
        self.c.len = v


class DeviceModel:
    def __init__(self, n_layers, hidden, n_heads, head_dim, ffn, vocab, max_pos, group, embed, pos_embed,
                 lnf_g, lnf_b, layers):
        self.tensors = (embed, pos_embed, lnf_g, lnf_b)
        self.layers = list(layers)
        self._arr = (Layer * max(1, len(self.layers)))(*[l.c for l in self.layers])
        self.c = Model(n_layers, hidden, n_heads, head_dim, ffn, vocab, max_pos, group, _ptr(embed),
                       _ptr(pos_embed), _ptr(lnf_g), _ptr(lnf_b), ctypes.cast(self._arr, POINTER(Layer)))


# ------------------------------------------------------------------------- steps
def fg_kv_append(cache: DeviceKVCache, k, v, row_stride: int, n_tokens: int, stream=None):
    _check(lib().fg_kv_append(ctypes.byref(cache.c), _ptr(k), _ptr(v), row_stride, n_tokens, _stream(stream)))


def fg_qgemm_workspace_bytes(M: int, N: int, K: int) -> int:
    return lib().fg_qgemm_workspace_bytes(M, N, K)


def fg_qgemm(X, W: DeviceQLinear, R=None, relu: bool = False, Y=None, workspace=None, stream=None):
    import torch
    M = X.shape[0]
    if Y is None:
        Y = _empty((M, W.N), torch.float16, X.device)
    wsb = fg_qgemm_workspace_bytes(M, W.N, W.K)
    if workspace is None and wsb:
        workspace = _empty((wsb,), torch.uint8, X.device)
    _check(lib().fg_qgemm(_ptr(X), M, ctypes.byref(W.c), _ptr(R), int(relu), _ptr(Y), _ptr(workspace),
                          0 if workspace is None else workspace.numel(), _stream(stream)))
    return Y


def fg_gemm_f16(X, W, bias=None, R=None, relu: bool = False, Y=None, workspace=None, stream=None):
    """Y = [relu](X @ W + b) [+ R] with an uncompressed fp16 weight W [K, N] on the tensor cores."""
    import torch
    M = X.shape[0]
    K, N = W.shape
    if Y is None:
        Y = _empty((M, N), torch.float16, X.device)
    wsb = lib().fg_gemm_f16_workspace_bytes(M, N, K)
    if workspace is None and wsb:
        workspace = _empty((wsb,), torch.uint8, X.device)
    _check(lib().fg_gemm_f16(_ptr(X), M, _ptr(W), K, N, _ptr(bias), _ptr(R), int(relu), _ptr(Y), _ptr(workspace),
                             0 if workspace is None else workspace.numel(), _stream(stream)))
    return Y


def fg_decode_attention(q, q_stride: int, cache: DeviceKVCache, out=None, workspace=None, stream=None):
    import torch
    B, nh, hd = cache.c.B, cache.c.n_heads, cache.c.head_dim
    if out is None:
        out = _empty((B, nh * hd), torch.float16, q.device)
    wsb = lib().fg_decode_attention_workspace_bytes(B, nh, hd, cache.c.len)
    if workspace is None and wsb:
        workspace = _empty((wsb,), torch.uint8, q.device)
    _check(lib().fg_decode_attention(_ptr(q), q_stride, ctypes.byref(cache.c), _ptr(out), _ptr(workspace),
                                     0 if workspace is None else workspace.numel(), _stream(stream)))
    return out


def fg_decode_attention_noalloc(q, q_stride: int, cache: DeviceKVCache, out=None, stream=None):
    """fg_decode_attention with its scratch in the library's fixed device array (no workspace).
    Only `out` may be allocated here, and only when the caller passes none."""
    import torch
    B, nh, hd = cache.c.B, cache.c.n_heads, cache.c.head_dim
    if out is None:
        out = _empty((B, nh * hd), torch.float16, q.device)
    _check(lib().fg_decode_attention_noalloc(_ptr(q), q_stride, ctypes.byref(cache.c), _ptr(out), _stream(stream)))
    return out


def fg_prefill_attention(qkv, B: int, L: int, n_heads: int, head_dim: int, out=None, stream=None):
    import torch
    if out is None:
        out = _empty((B * L, n_heads * head_dim), torch.float16, qkv.device)
    _check(lib().fg_prefill_attention(_ptr(qkv), B, L, n_heads, head_dim, _ptr(out), _stream(stream)))
    return out


def fg_layernorm(x, g, b, y=None, stream=None):
    rows, cols = x.shape
    if y is None:
        y = _empty((rows, cols), x.dtype, x.device)
    _check(lib().fg_layernorm(_ptr(x), rows, cols, _ptr(g), _ptr(b), _ptr(y), _stream(stream)))
    return y


def fg_embed(ids, pos0: int, E, P, out=None, stream=None):
    import torch
    B, T = ids.shape
    h = E.shape[1]
    if out is None:
        out = _empty((B * T, h), torch.float16, E.device)
    _check(lib().fg_embed(_ptr(ids), B, T, pos0, _ptr(E), _ptr(P), h, _ptr(out), _stream(stream)))
    return out


def fg_lm_head_argmax(x, E, logits=None, tokens=None, workspace=None, stream=None):
    import torch
    B, h = x.shape
    V = E.shape[0]
    if tokens is None:
        tokens = _empty((B,), torch.int32, x.device)
    if logits is None and workspace is None:
        workspace = _empty((lib().fg_lm_head_workspace_bytes(B, V),), torch.uint8, x.device)
    _check(lib().fg_lm_head_argmax(_ptr(x), B, h, _ptr(E), V, _ptr(logits), _ptr(tokens), _ptr(workspace),
                                   0 if workspace is None else workspace.numel(), _stream(stream)))
    return tokens


def fg_decode_layer(layer: DeviceLayer, cache: DeviceKVCache, x_in, x_out=None, workspace=None, stream=None):
    import torch
    B, h = x_in.shape
    F = layer.fc1.N
    if x_out is None:
        x_out = _empty((B, h), torch.float16, x_in.device)
    if workspace is None:
        wsb = lib().fg_decode_layer_workspace_bytes(h, F, cache.c.n_heads, B, cache.c.capacity)
        workspace = _empty((wsb,), torch.uint8, x_in.device)
    _check(lib().fg_decode_layer(ctypes.byref(layer.c), ctypes.byref(cache.c), _ptr(x_in), _ptr(x_out), B,
                                 _ptr(workspace), workspace.numel(), _stream(stream)))
    return x_out


def fg_prefill_layer(layer: DeviceLayer, cache: DeviceKVCache, x, B: int, L: int, workspace=None, stream=None):
    import torch
    h = x.shape[-1]
    F = layer.fc1.N
    if workspace is None:
        wsb = lib().fg_prefill_layer_workspace_bytes(h, F, B, L)
        workspace = _empty((wsb,), torch.uint8, x.device)
    _check(lib().fg_prefill_layer(ctypes.byref(layer.c), ctypes.byref(cache.c), _ptr(x), B, L, _ptr(workspace),
                                  workspace.numel(), _stream(stream)))
    return x


def fg_workspace_bytes(model: DeviceModel, B: int, L: int, gen_len: int) -> int:
    return lib().fg_workspace_bytes(ctypes.byref(model.c), B, L, gen_len)


def fg_generate(model: DeviceModel, prompt_ids, gen_len: int, caches, out_ids=None, workspace=None,
                stream=None):
    """Greedy generation; returns (out_ids int32 [B, gen_len] on the device, Timing)."""
    import torch
    B, L = prompt_ids.shape
    if out_ids is None:
        out_ids = _empty((B, gen_len), torch.int32, prompt_ids.device)
    if workspace is None:
        workspace = _empty((fg_workspace_bytes(model, B, L, gen_len),), torch.uint8, prompt_ids.device)
    arr = (KVCache * len(caches))(*[c.c for c in caches])
    timing = Timing()
    st = lib().fg_generate(ctypes.byref(model.c), _ptr(prompt_ids), B, L, gen_len, _ptr(out_ids), arr,
                           _ptr(workspace), workspace.numel(), ctypes.byref(timing), _stream(stream))
    for i, c in enumerate(caches):
        c.c.len = arr[i].len
    _check(st)
    return out_ids, timing


def pinned_layer(layer: DeviceLayer) -> DeviceLayer:
    """A copy of a layer whose tensors live in pinned host memory (for fg_generate_offload)."""
    def pin(t):
        return None if t is None else t.detach().cpu().pin_memory()

    def lin(q: DeviceQLinear) -> DeviceQLinear:
        return DeviceQLinear(pin(q.codes), pin(q.params), pin(q.bias), q.K, q.N, q.group, pin(q.w16), q.along_k)
    return DeviceLayer(*[pin(t) for t in layer.t], lin(layer.qkv), lin(layer.out), lin(layer.fc1), lin(layer.fc2))


def fg_offload_workspace_bytes(model: DeviceModel, B: int, L: int, gen_len: int) -> int:
    return lib().fg_offload_workspace_bytes(ctypes.byref(model.c), B, L, gen_len)


def fg_generate_offload(model: DeviceModel, prompt_ids, gen_len: int, caches, out_ids=None, workspace=None,
                        stream=None):
    """Greedy generation with the layers' weights in pinned host memory, streamed to the GPU
    layer by layer; returns (out_ids int32 [B, gen_len] on the device, Timing, h2d bytes)."""
    import torch
    B, L = prompt_ids.shape
    if out_ids is None:
        out_ids = _empty((B, gen_len), torch.int32, prompt_ids.device)
    if workspace is None:
        workspace = _empty((fg_offload_workspace_bytes(model, B, L, gen_len),), torch.uint8, prompt_ids.device)
    arr = (KVCache * len(caches))(*[c.c for c in caches])
    timing = Timing()
    h2d = c_double()
    st = lib().fg_generate_offload(ctypes.byref(model.c), _ptr(prompt_ids), B, L, gen_len, _ptr(out_ids), arr,
                                   _ptr(workspace), workspace.numel(), ctypes.byref(timing), ctypes.byref(h2d),
                                   _stream(stream))
    for i, c in enumerate(caches):
        c.c.len = arr[i].len
    _check(st)
    return out_ids, timing, h2d.value


def fg_profile_enable(on: bool = True):
    _check(lib().fg_profile_enable(int(on)))


def fg_profile_select(kinds=None):
    """Time only these kinds (indices into PROF_NAMES) while profiling is on; None = all."""
    mask = (1 << len(PROF_NAMES)) - 1 if kinds is None else sum(1 << int(k) for k in kinds)
    _check(lib().fg_profile_select(mask))


def fg_profile_reset():
    _check(lib().fg_profile_reset())


def fg_launch_count() -> int:
    return lib().fg_launch_count()


def fg_profile_read(kind: int):
    ms, n, fl, by = c_double(), c_int64(), c_double(), c_double()
    _check(lib().fg_profile_read(kind, ctypes.byref(ms), ctypes.byref(n), ctypes.byref(fl), ctypes.byref(by)))
    return {"ms": ms.value, "launches": n.value, "flops": fl.value, "bytes": by.value}
