// K4 split-context decode attention over the 4-bit KV cache, and K4r the split combine.
//
// One query token per sequence ("FlexGen" README mirror: generation over a compressed
// attention cache).  For sequence b and head j:
//   score_t = (q . K_t) / sqrt(hd),  K_t = mn_t + code_t * s_t (per group of G dims)
//   out = sum_t softmax(score)_t V_t
// The cache is read exactly once: one CTA per (chunk of positions, head, sequence)
// streams the chunk's K codes (pass 1: scores into shared memory) and V codes (pass 2).
// Codes are never expanded to fp16: with f = 0.5 + code/256 (built by one byte
// permute into the mantissa of 0.5f), sum_i q_i code_i = 256 (sum_i q_i f_i - 0.5 sum_i q_i),
// and a group contributes s * sum(q code) + mn * sum(q).  The V side uses the same
// identity with weights p_t s_t.  Softmax is fp32 with exp2 (q pre-scaled by
// log2(e)/sqrt(hd)); chunks are merged with the usual (max, sum, acc) rescaling.
#include <algorithm>
#include <mutex>

#include "fg_common.cuh"

namespace fg {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kUnroll = 4;
constexpr float kLog2e = 1.4426950408889634f;

// f_i = 0.5 + c_i/256 for the 8 codes of w (element i in bits 4i..4i+3).
// even = w & 0x0F0F0F0F holds codes 0,2,4,6 in bytes 0..3; odd = (w>>4) & 0x0F0F0F0F
// codes 1,3,5,7.  __byte_perm(src, 0x3F000000, sel) puts byte k of src into byte 2 of
// 0x3F000000 (0.5f), i.e. into mantissa bits 16..19.
__device__ __forceinline__ void code_floats(uint32_t w, float f[8]) {
  const uint32_t even = w & 0x0F0F0F0Fu;
  const uint32_t odd = (w >> 4) & 0x0F0F0F0Fu;
  const uint32_t half = 0x3F000000u;
  // selector nibbles: result byte r takes byte sel_r of {b (4..7), a (0..3)} = {half, src}
  // result = [half.b0, half.b1, src.bk, half.b3] -> sel = 0x7 k 5 4 (byte3..byte0)
  f[0] = __uint_as_float(__byte_perm(even, half, 0x7054));
  f[1] = __uint_as_float(__byte_perm(odd, half, 0x7054));
  f[2] = __uint_as_float(__byte_perm(even, half, 0x7154));
  f[3] = __uint_as_float(__byte_perm(odd, half, 0x7154));
  f[4] = __uint_as_float(__byte_perm(even, half, 0x7254));
  f[5] = __uint_as_float(__byte_perm(odd, half, 0x7254));
  f[6] = __uint_as_float(__byte_perm(even, half, 0x7354));
  f[7] = __uint_as_float(__byte_perm(odd, half, 0x7354));
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// HD = head dim (64 or 128), G = group size (divides HD).
template <int HD, int G>
__global__ void __launch_bounds__(kThreads) decode_attn_kernel(
    const __half* __restrict__ q, int64_t q_stride, const uint32_t* __restrict__ kc,
    const __half2* __restrict__ kp, const uint32_t* __restrict__ vc, const __half2* __restrict__ vp,
    int nh, int cap, int S, int chunk_len, __half* __restrict__ out, float* __restrict__ part_ml,
    float* __restrict__ part_acc) {
  constexpr int LPT = HD / 8;   // lanes per token: each lane owns 8 dims (one code word)
  constexpr int TPW = 32 / LPT; // tokens per warp step
  constexpr int STEP = kWarps * TPW;
  constexpr int WPT = HD / 8;   // code words per token
  constexpr int PPT = HD / G;   // params per token
  extern __shared__ float smem[];  // [chunk_len] scores, then reduction scratch
  float* sc = smem;
  __shared__ float red[kWarps][HD];
  __shared__ float red2[2][kWarps];

  const int b = blockIdx.z, head = blockIdx.y, chunk = blockIdx.x;
  const int t0 = chunk * chunk_len;
  const int t1 = min(S, t0 + chunk_len);
  const int n = t1 - t0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane % LPT, slot = lane / LPT;
  const int d0 = sub * 8;

  // query slice, pre-scaled so that scores are in log2 units
  float qf[8];
  {
    const uint4 raw = *reinterpret_cast<const uint4*>(q + int64_t(b) * q_stride + head * HD + d0);
    const __half2* h = reinterpret_cast<const __half2*>(&raw);
    const float scale = kLog2e * rsqrtf(float(HD));
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float2 f = __half22float2(h[j]);
      qf[2 * j] = f.x * scale;
      qf[2 * j + 1] = f.y * scale;
    }
  }
  float qs = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) qs += qf[i];

  const int64_t slot0 = (int64_t(b) * nh + head) * cap;
  const uint32_t* kw = kc + slot0 * WPT + sub;
  const uint32_t* vw = vc + slot0 * WPT + sub;
  const __half2* kpp = kp + slot0 * PPT + d0 / G;
  const __half2* vpp = vp + slot0 * PPT + d0 / G;

  // ---------------- pass 1: scores
  for (int tb = t0 + warp * TPW; tb < t1; tb += STEP * kUnroll) {
    uint32_t w[kUnroll];
    __half2 p[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int t = tb + u * STEP + slot;
      const bool ok = t < t1;
      w[u] = ok ? __ldg(kw + int64_t(t) * WPT) : 0u;
      p[u] = ok ? __ldg(kpp + int64_t(t) * PPT) : __half2();
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int t = tb + u * STEP + slot;
      float f[8];
      code_floats(w[u], f);
      float dot = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) dot = fmaf(qf[i], f[i], dot);
      const float2 ms = __half22float2(p[u]);  // {mn, s}
      const float cq = (dot - 0.5f * qs) * 256.f;
      float part = fmaf(ms.y, cq, ms.x * qs);
#pragma unroll
      for (int o = 1; o < LPT; o <<= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
      if (sub == 0 && t < t1) sc[t - t0] = part;
    }
  }
  __syncthreads();

  // ---------------- softmax over the chunk
  float m = -INFINITY;
  for (int i = threadIdx.x; i < n; i += kThreads) m = fmaxf(m, sc[i]);
  m = warp_max(m);
  if (lane == 0) red2[0][warp] = m;
  __syncthreads();
  m = red2[0][0];
#pragma unroll
  for (int i = 1; i < kWarps; ++i) m = fmaxf(m, red2[0][i]);
  float l = 0.f;
  for (int i = threadIdx.x; i < n; i += kThreads) {
    const float e = exp2f(sc[i] - m);
    sc[i] = e;
    l += e;
  }
  l = warp_sum(l);
  if (lane == 0) red2[1][warp] = l;
  __syncthreads();
  l = 0.f;
#pragma unroll
  for (int i = 0; i < kWarps; ++i) l += red2[1][i];

  // ---------------- pass 2: weighted sum of V
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  float accb = 0.f, accm = 0.f;
  for (int tb = t0 + warp * TPW; tb < t1; tb += STEP * kUnroll) {
    uint32_t w[kUnroll];
    __half2 p[kUnroll];
    float pt[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int t = tb + u * STEP + slot;
      const bool ok = t < t1;
      w[u] = ok ? __ldg(vw + int64_t(t) * WPT) : 0u;
      p[u] = ok ? __ldg(vpp + int64_t(t) * PPT) : __half2();
      pt[u] = ok ? sc[t - t0] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      float f[8];
      code_floats(w[u], f);
      const float2 ms = __half22float2(p[u]);
      const float bt = pt[u] * ms.y;
      accm = fmaf(pt[u], ms.x, accm);
      accb += bt;
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = fmaf(bt, f[i], acc[i]);
    }
  }
  float vals[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float v = fmaf(256.f, acc[i] - 0.5f * accb, accm);
    // sum over the token slots of this warp (lanes with equal `sub`)
#pragma unroll
    for (int o = LPT; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    vals[i] = v;
  }
  if (slot == 0) {
#pragma unroll
    for (int i = 0; i < 8; ++i) red[warp][d0 + i] = vals[i];
  }
  __syncthreads();
  const int64_t bh = int64_t(b) * nh + head;
  for (int d = threadIdx.x; d < HD; d += kThreads) {
    float v = 0.f;
#pragma unroll
    for (int i = 0; i < kWarps; ++i) v += red[i][d];
    if (part_ml == nullptr) {
      out[int64_t(b) * nh * HD + head * HD + d] = __float2half_rn(v / l);
    } else {
      part_acc[(bh * gridDim.x + chunk) * HD + d] = v;
    }
  }
  if (part_ml != nullptr && threadIdx.x == 0) {
    part_ml[(bh * gridDim.x + chunk) * 2 + 0] = m;
    part_ml[(bh * gridDim.x + chunk) * 2 + 1] = l;
  }
}

// K4r: one warp per (sequence, head) merges the chunk partials.
template <int HD>
__global__ void __launch_bounds__(128) decode_combine_kernel(const float* __restrict__ part_ml,
                                                             const float* __restrict__ part_acc,
                                                             int n_bh, int n_chunks, int nh,
                                                             __half* __restrict__ out) {
  const int bh = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (bh >= n_bh) return;
  float M = -INFINITY;
  for (int c = 0; c < n_chunks; ++c) M = fmaxf(M, part_ml[(int64_t(bh) * n_chunks + c) * 2]);
  float L = 0.f;
  float acc[HD / 32];
#pragma unroll
  for (int i = 0; i < HD / 32; ++i) acc[i] = 0.f;
  for (int c = 0; c < n_chunks; ++c) {
    const float mc = part_ml[(int64_t(bh) * n_chunks + c) * 2];
    const float lc = part_ml[(int64_t(bh) * n_chunks + c) * 2 + 1];
    const float w = exp2f(mc - M);
    L = fmaf(lc, w, L);
#pragma unroll
    for (int i = 0; i < HD / 32; ++i)
      acc[i] = fmaf(part_acc[(int64_t(bh) * n_chunks + c) * HD + i * 32 + lane], w, acc[i]);
  }
  const int b = bh / nh, head = bh - b * nh;
#pragma unroll
  for (int i = 0; i < HD / 32; ++i)
    out[int64_t(b) * nh * HD + head * HD + i * 32 + lane] = __float2half_rn(acc[i] / L);
}

int pick_chunks(int B, int nh, int S) {
  const int target = num_sms() * 8;
  const int bh = B * nh;
  int nc = (target + bh - 1) / bh;
  const int max_by_len = (S + 127) / 128;  // at least 128 positions per chunk
  nc = std::min(nc, std::max(1, max_by_len));
  const int min_by_smem = (S + 4095) / 4096;  // at most 4096 positions per chunk
  return std::max(nc, std::max(1, min_by_smem));
}

}  // namespace

size_t decode_attention_ws_bytes(int B, int nh, int hd, int ctx) {
  if (B <= 0 || nh <= 0 || hd <= 0 || ctx <= 0) return 0;
  const int nc = pick_chunks(B, nh, ctx);
  if (nc <= 1) return 0;
  return size_t(B) * nh * nc * (2 + hd) * sizeof(float) + 256;
}

int decode_attention_impl(const void* q, int64_t q_stride, const fg_kv_cache* c, void* out,
                          void* ws, size_t ws_bytes, cudaStream_t s) {
  if (!q || !c || !out) return fail(FG_ERR_INVALID_ARG, "null pointer");
  const int B = c->B, nh = c->n_heads, hd = c->head_dim, G = c->group, S = c->len;
  if (hd != 64 && hd != 128) return fail(FG_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (G != 32 && G != 64 && G != 128) return fail(FG_ERR_SHAPE, "group must be 32, 64 or 128");
  if (hd % G) return fail(FG_ERR_SHAPE, "group must divide head_dim");
  if (B <= 0 || nh <= 0 || S <= 0 || S > c->capacity) return fail(FG_ERR_SHAPE, "bad cache length/shape");
  if (q_stride < int64_t(nh) * hd || q_stride % 8) return fail(FG_ERR_ALIGN, "q_stride must be >= h and a multiple of 8");
  if (!aligned16(q) || !aligned16(out) || !aligned16(c->k_codes) || !aligned16(c->v_codes) ||
      !aligned16(c->k_params) || !aligned16(c->v_params))
    return fail(FG_ERR_ALIGN, "pointers must be 16-byte aligned");
  const int nc = pick_chunks(B, nh, S);
  const int chunk_len = (S + nc - 1) / nc;
  float* ml = nullptr;
  float* acc = nullptr;
  if (nc > 1) {
    const size_t need = decode_attention_ws_bytes(B, nh, hd, S);
    if (!ws || ws_bytes < need) return fail(FG_ERR_WORKSPACE, "decode attention needs %zu workspace bytes", need);
    if (!aligned16(ws)) return fail(FG_ERR_ALIGN, "workspace must be 16-byte aligned");
    ml = reinterpret_cast<float*>(ws);
    acc = ml + size_t(B) * nh * nc * 2;
    acc = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(acc) + 15) & ~uintptr_t(15));
  }
  const double bytes = double(B) * nh * S * 2.0 * (hd / 2 + 4.0 * hd / G) + 4.0 * B * nh * hd;
  ProfScope ps(PROF_DECODE_ATTN, s, 4.0 * B * nh * double(S) * hd, bytes);
  dim3 grid(nc, nh, B);
  const size_t smem = size_t(chunk_len) * sizeof(float);
  auto* qh = reinterpret_cast<const __half*>(q);
  auto* kc = reinterpret_cast<const uint32_t*>(c->k_codes);
  auto* vc = reinterpret_cast<const uint32_t*>(c->v_codes);
  auto* kp = reinterpret_cast<const __half2*>(c->k_params);
  auto* vp = reinterpret_cast<const __half2*>(c->v_params);
  auto* o = reinterpret_cast<__half*>(out);
#define FG_ATTN_LAUNCH(HD_, G_)                                                                   \
  decode_attn_kernel<HD_, G_><<<grid, kThreads, smem, s>>>(qh, q_stride, kc, kp, vc, vp, nh,    \
                                                            c->capacity, S, chunk_len, o, ml, acc)
  if (hd == 128 && G == 128) FG_ATTN_LAUNCH(128, 128);
  else if (hd == 128 && G == 64) FG_ATTN_LAUNCH(128, 64);
  else if (hd == 128 && G == 32) FG_ATTN_LAUNCH(128, 32);
  else if (hd == 64 && G == 64) FG_ATTN_LAUNCH(64, 64);
  else FG_ATTN_LAUNCH(64, 32);
#undef FG_ATTN_LAUNCH
  FG_CHECK_LAUNCH("decode attention kernel");
  if (nc > 1) {
    const int n_bh = B * nh;
    if (hd == 128)
      decode_combine_kernel<128><<<(n_bh + 3) / 4, 128, 0, s>>>(ml, acc, n_bh, nc, nh, o);
    else
      decode_combine_kernel<64><<<(n_bh + 3) / 4, 128, 0, s>>>(ml, acc, n_bh, nc, nh, o);
    FG_CHECK_LAUNCH("decode combine kernel");
  }
  return FG_OK;
}

}  // namespace fg

// ==================================================================== no-allocation variant
// fg_decode_attention_noalloc: the same kernels, with the split-context partials in a fixed
// array compiled into the library instead of a caller-provided workspace.  It serves callers
// that may not allocate device memory themselves (see include/fg.h).  The array is held by
// every GPU that loads the library until the process exits.
namespace fg {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB of fp32 partials

}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

// Device address of the array for the current device, looked up once per device (with
// that device current) on the first call; host code must not use the symbol itself.
int noalloc_scratch(void** out) {
  static std::mutex mu;
  static void* addr[64] = {nullptr};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(FG_ERR_UNSUPPORTED, "device ordinal %d above 63", dev);
  std::lock_guard<std::mutex> lk(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-allocation scratch)");
    addr[dev] = p;
  }
  *out = addr[dev];
  return FG_OK;
}

}  // namespace
}  // namespace fg

extern "C" int fg_decode_attention_noalloc(const void* q, int64_t q_stride, const fg_kv_cache* cache, void* out,
                                           void* stream) {
  using namespace fg;
  if (!cache) return fail(FG_ERR_INVALID_ARG, "null cache");
  const size_t need = decode_attention_ws_bytes(cache->B, cache->n_heads, cache->head_dim, cache->len);
  if (need > kNoAllocScratchBytes)
    return fail(FG_ERR_WORKSPACE,
                "this shape needs %zu bytes of split-context scratch; the fixed no-allocation array holds %zu "
                "(use fg_decode_attention with a workspace)",
                need, kNoAllocScratchBytes);
  void* scratch = nullptr;
  FG_TRY(noalloc_scratch(&scratch));
  // Every partial the combine step reads is written by this call first: nothing to clear.
  return decode_attention_impl(q, q_stride, cache, out, scratch, kNoAllocScratchBytes, as_stream(stream));
}
