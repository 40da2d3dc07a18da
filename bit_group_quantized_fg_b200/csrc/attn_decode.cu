// K4 split-context decode attention over the 4-bit KV cache, and K4r the split combine.
//
// One query token per sequence ("FlexGen" README mirror: generation over a compressed
// attention cache).  For sequence b and head j:
//   score_t = (q . K_t) / sqrt(hd),  K_t = mn_t + code_t * s_t (per group of G dims)
//   out = sum_t softmax(score)_t V_t
// The cache is read exactly once: one CTA per (chunk of positions, head, sequence)
// streams the chunk's K and V codes together in a single pass with an online softmax.
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
  // result bytes (3..0) = [half.b3, src.bk, half.b1, half.b0] -> selector 0x7k54
  f[0] = __uint_as_float(__byte_perm(even, half, 0x7054));
  f[1] = __uint_as_float(__byte_perm(odd, half, 0x7054));
  f[2] = __uint_as_float(__byte_perm(even, half, 0x7154));
  f[3] = __uint_as_float(__byte_perm(odd, half, 0x7154));
  f[4] = __uint_as_float(__byte_perm(even, half, 0x7254));
  f[5] = __uint_as_float(__byte_perm(odd, half, 0x7254));
  f[6] = __uint_as_float(__byte_perm(even, half, 0x7354));
  f[7] = __uint_as_float(__byte_perm(odd, half, 0x7354));
}

__device__ __forceinline__ uint4 ldg_v4(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// HD = head dim (64 or 128), G = group size (divides HD, >= 32).
// Lane layout: LPT = HD/32 lanes per token, each owning 32 dims (one 16-byte load of K
// codes and one of V codes per token, inside one group); TPW = 32/LPT tokens per warp
// step.  Every lane keeps an online-softmax state (max m, sum l, weighted sums) for the
// tokens of its slot; slots, warps and chunks are merged at the end with the usual rescaling.
template <int HD, int G>
__global__ void __launch_bounds__(kThreads) decode_attn_kernel(
    const __half* __restrict__ q, int64_t q_stride, const uint4* __restrict__ kc,
    const __half2* __restrict__ kp, const uint4* __restrict__ vc, const __half2* __restrict__ vp,
    int nh, int cap, int S, int chunk_len, __half* __restrict__ out, float* __restrict__ part_ml,
    float* __restrict__ part_acc) {
  constexpr int LPT = HD / 32;
  constexpr int TPW = 32 / LPT;
  constexpr int STEP = kWarps * TPW;
  constexpr int VPT = HD / 32;  // 16-byte code vectors per token
  constexpr int PPT = HD / G;   // params per token
  constexpr int U = 2;          // token steps in flight per lane
  __shared__ float red_v[kWarps][HD];
  __shared__ float red_ml[kWarps][2];

  const int b = blockIdx.z, head = blockIdx.y, chunk = blockIdx.x;
  const int t0 = chunk * chunk_len;
  const int t1 = min(S, t0 + chunk_len);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane % LPT, slot = lane / LPT;
  const int d0 = sub * 32;

  // query slice (32 dims), pre-scaled so scores are in log2 units
  float qf[32];
  {
    const uint4* qp = reinterpret_cast<const uint4*>(q + int64_t(b) * q_stride + head * HD + d0);
    const float scale = kLog2e * rsqrtf(float(HD));
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const uint4 raw = qp[v];
      const __half2* h = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __half22float2(h[j]);
        qf[8 * v + 2 * j] = f.x * scale;
        qf[8 * v + 2 * j + 1] = f.y * scale;
      }
    }
  }
  float qs = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) qs += qf[i];

  const int64_t slot0 = (int64_t(b) * nh + head) * cap;
  const uint4* kw = kc + slot0 * VPT + sub;
  const uint4* vw = vc + slot0 * VPT + sub;
  const __half2* kpp = kp + slot0 * PPT + d0 / G;
  const __half2* vpp = vp + slot0 * PPT + d0 / G;

  float m = -INFINITY, l = 0.f, accb = 0.f, accm = 0.f;
  float acc[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) acc[i] = 0.f;

  for (int tb = t0 + warp * TPW; tb < t1; tb += STEP * U) {
    uint4 kq[U], vq[U];
    __half2 kpar[U], vpar[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int t = tb + u * STEP + slot;
      const bool ok = t < t1;
      kq[u] = ok ? ldg_v4(kw + int64_t(t) * VPT) : make_uint4(0, 0, 0, 0);
      vq[u] = ok ? ldg_v4(vw + int64_t(t) * VPT) : make_uint4(0, 0, 0, 0);
      kpar[u] = ok ? __ldg(kpp + int64_t(t) * PPT) : __half2();
      vpar[u] = ok ? __ldg(vpp + int64_t(t) * PPT) : __half2();
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const bool ok = tb + u * STEP + slot < t1;
      // score partial over this lane's 32 dims: s*sum(q code) + mn*sum(q)
      float dot = 0.f;
      {
        const uint32_t wv[4] = {kq[u].x, kq[u].y, kq[u].z, kq[u].w};
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          float f[8];
          code_floats(wv[v], f);
#pragma unroll
          for (int i = 0; i < 8; ++i) dot = fmaf(qf[8 * v + i], f[i], dot);
        }
      }
      const float2 km = __half22float2(kpar[u]);  // {mn, s}
      float part = fmaf(km.y, (dot - 0.5f * qs) * 256.f, km.x * qs);
#pragma unroll
      for (int o = 1; o < LPT; o <<= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
      if (!ok) continue;
      if (part > m) {  // new running max for this slot: rescale its sums
        const float sc = exp2f(m - part);  // m = -inf -> 0
        l *= sc;
        accb *= sc;
        accm *= sc;
#pragma unroll
        for (int i = 0; i < 32; ++i) acc[i] *= sc;
        m = part;
      }
      const float p = exp2f(part - m);
      l += p;
      const float2 vm = __half22float2(vpar[u]);
      const float bt = p * vm.y;
      accm = fmaf(p, vm.x, accm);
      accb += bt;
      const uint32_t wv[4] = {vq[u].x, vq[u].y, vq[u].z, vq[u].w};
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        float f[8];
        code_floats(wv[v], f);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[8 * v + i] = fmaf(bt, f[i], acc[8 * v + i]);
      }
    }
  }

  // sum_t p_t (mn_t + s_t c_td) = accm + 256 (acc_d - 0.5 accb), then merge the slots of the warp
  float M = m;
#pragma unroll
  for (int o = LPT; o < 32; o <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float sc = (m == -INFINITY) ? 0.f : exp2f(m - M);
  float lw = l * sc;
#pragma unroll
  for (int o = LPT; o < 32; o <<= 1) lw += __shfl_xor_sync(0xffffffffu, lw, o);
  const float base = accm * sc;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    float v = fmaf(256.f * sc, acc[i] - 0.5f * accb, base);
#pragma unroll
    for (int o = LPT; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (slot == 0) red_v[warp][d0 + i] = v;
  }
  if (lane == 0) {
    red_ml[warp][0] = M;
    red_ml[warp][1] = lw;
  }
  __syncthreads();
  // merge the warps
  float Mc = red_ml[0][0];
#pragma unroll
  for (int w = 1; w < kWarps; ++w) Mc = fmaxf(Mc, red_ml[w][0]);
  float wsc[kWarps];
  float L = 0.f;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    wsc[w] = (red_ml[w][0] == -INFINITY) ? 0.f : exp2f(red_ml[w][0] - Mc);
    L = fmaf(red_ml[w][1], wsc[w], L);
  }
  const int64_t bh = int64_t(b) * nh + head;
  for (int d = threadIdx.x; d < HD; d += kThreads) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) v = fmaf(red_v[w][d], wsc[w], v);
    if (part_ml == nullptr) {
      out[int64_t(b) * nh * HD + head * HD + d] = __float2half_rn(v / L);
    } else {
      part_acc[(bh * gridDim.x + chunk) * HD + d] = v;
    }
  }
  if (part_ml != nullptr && threadIdx.x == 0) {
    part_ml[(bh * gridDim.x + chunk) * 2 + 0] = Mc;
    part_ml[(bh * gridDim.x + chunk) * 2 + 1] = L;
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
  const int min_by_len = (S + 4095) / 4096;  // at most 4096 positions per chunk
  return std::max(nc, std::max(1, min_by_len));
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
  const size_t smem = 0;
  auto* qh = reinterpret_cast<const __half*>(q);
  auto* kc = reinterpret_cast<const uint4*>(c->k_codes);
  auto* vc = reinterpret_cast<const uint4*>(c->v_codes);
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
