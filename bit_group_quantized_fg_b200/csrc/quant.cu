// K1 quantize/pack (weights and KV append) and K2 dequantize.
//
// Definition ("FlexGen" README mirror, key features "Extreme Compression": weights and
// attention cache to 4 bits; group-wise asymmetric min-max with fp16 {min, scale} per
// group of G consecutive elements), per group:
//   mn = min, mx = max (zero extremes as +0); s = fp16(fp32(mx - mn) / 15);
//   code = clamp(rint(fp32(x - mn) / s), 0, 15), every code 0 when s == 0.
// All fp32 steps use explicitly rounded intrinsics (__fsub_rn/__fdiv_rn), so no FMA
// contraction or reciprocal approximation can change a code.
//
// Layout of a row-grouped (axis=1) tensor: 16-byte chunks of 8 fp16 values; one thread
// owns one chunk, G/8 adjacent lanes own one group and combine min/max with xor
// shuffles.  A chunk's 8 codes form one 32-bit word (element i in bits 4i..4i+3, i.e.
// byte j = code(2j) | code(2j+1) << 4).  Loads are 128-bit and read-only cached; the
// loop is grid-stride over tiles of blockDim*U chunks with all U loads issued first.
#include <algorithm>

#include "fg_common.cuh"
#include "quant_common.cuh"

namespace fg {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// ------------------------------------------------------------------ K1, axis = 1
// One thread per 16 consecutive elements (a "chunk"); G/16 lanes per group.
template <int G>
__global__ void __launch_bounds__(kThreads) quantize_rows_kernel(const uint4* __restrict__ x,
                                                                 int64_t n_chunks,
                                                                 uint2* __restrict__ codes,
                                                                 __half2* __restrict__ params) {
  pdl_wait();  // the previous kernel in the stream has finished (see fg_launch)
  constexpr int TPG = G / 16;
  const int64_t tile = int64_t(kThreads) * kUnroll;
  for (int64_t base = int64_t(blockIdx.x) * tile; base < n_chunks; base += int64_t(gridDim.x) * tile) {
    uint4 va[kUnroll], vb[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t c = base + u * kThreads + threadIdx.x;
      const bool ok = c < n_chunks;
      va[u] = ok ? ld_nc_v4(x + 2 * c) : make_uint4(0, 0, 0, 0);
      vb[u] = ok ? ld_nc_v4(x + 2 * c + 1) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t c = base + u * kThreads + threadIdx.x;
      GroupQ q = quantize_chunk16<TPG>(va[u], vb[u]);
      if (c < n_chunks) {
        codes[c] = q.words;
        if ((threadIdx.x % TPG) == 0) params[c / TPG] = q.params;
      }
    }
  }
}

// ------------------------------------------------------------------ KV append
// n / d for 0 <= n < 2^31 by a multiply-high and a shift (Granlund and Montgomery, "Division
// by invariant integers using multiplication", 1994): with l = ceil(log2 d) and
// m = ceil(2^(31 + l) / d) < 2^32, n / d = (n m) >> (31 + l), because m d - 2^(31 + l) < d
// keeps the error term n (m d - 2^(31 + l)) / (d 2^(31 + l)) below 1/d.  d = 1 is passed
// through.  The append splits every 16-value chunk index into (row, chunk, sequence, token,
// head): 64-bit divisions there cost more than the quantization itself.
struct FastDiv {
  uint32_t m;
  int s;      // shift after the multiply-high: l - 1
  int one;    // d == 1
};
FastDiv make_fastdiv(uint32_t d) {
  FastDiv f{0, 0, d == 1};
  if (d > 1) {
    int l = 0;
    while ((uint64_t(1) << l) < d) ++l;
    f.m = uint32_t(((uint64_t(1) << (31 + l)) + d - 1) / d);
    f.s = l - 1;
  }
  return f;
}
__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv& f) {
  return f.one ? n : (__umulhi(n, f.m) >> f.s);
}

// Rows r = b*T + t of k (blockIdx.y == 0) or v (== 1); h valid values per row, quantized in
// chunks of 16 along the hidden dimension.  The group of head `head` lands at cache
// position pos0 + t.  FAST: fewer than 2^31 chunks, indices split with FastDiv.
template <int G, int U, bool FAST>
__global__ void __launch_bounds__(kThreads) kv_append_kernel(
    const __half* __restrict__ k, const __half* __restrict__ v, int64_t row_stride, int T, int h,
    int hd, int cap, int pos0, int64_t n_chunks, uint2* __restrict__ kc, uint2* __restrict__ vc,
    __half2* __restrict__ kp, __half2* __restrict__ vp, FastDiv f_cpr, FastDiv f_T, FastDiv f_hd) {
  pdl_wait();  // the previous kernel in the stream has finished (see fg_launch)
  constexpr int TPG = G / 16;
  const __half* src = blockIdx.y == 0 ? k : v;
  uint2* dc = blockIdx.y == 0 ? kc : vc;
  __half2* dp = blockIdx.y == 0 ? kp : vp;
  const int chunks_per_row = h / 16;
  const int nh = h / hd;
  const int64_t tile = int64_t(kThreads) * U;
  for (int64_t base = int64_t(blockIdx.x) * tile; base < n_chunks; base += int64_t(gridDim.x) * tile) {
    uint4 va[U], vb[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t c = base + u * kThreads + threadIdx.x;
      if (c < n_chunks) {
        const int64_t row = FAST ? int64_t(fdiv(uint32_t(c), f_cpr)) : c / chunks_per_row;
        const int cc = int(c - row * chunks_per_row);
        const uint4* p = reinterpret_cast<const uint4*>(src + row * row_stride + cc * 16);
        va[u] = ld_nc_v4(p);
        vb[u] = ld_nc_v4(p + 1);
      } else {
        va[u] = make_uint4(0, 0, 0, 0);
        vb[u] = va[u];
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t c = base + u * kThreads + threadIdx.x;
      GroupQ q = quantize_chunk16<TPG>(va[u], vb[u]);
      if (c < n_chunks) {
        const int64_t row = FAST ? int64_t(fdiv(uint32_t(c), f_cpr)) : c / chunks_per_row;
        const int cc = int(c - row * chunks_per_row);
        const int64_t b = FAST ? int64_t(fdiv(uint32_t(row), f_T)) : row / T;
        const int t = int(row - b * T);
        const int d = cc * 16;
        const int head = FAST ? int(fdiv(uint32_t(d), f_hd)) : d / hd;
        const int dh = d - head * hd;
        const int64_t slot = (b * nh + head) * int64_t(cap) + (pos0 + t);
        dc[slot * (hd / 16) + dh / 16] = q.words;
        if ((threadIdx.x % TPG) == 0) dp[slot * (hd / G) + dh / G] = q.params;
      }
    }
  }
}

// ------------------------------------------------------------------ K1, axis = 0
// One thread per (column pair, row group); min/max down the G rows of its two columns.
__global__ void __launch_bounds__(kThreads) quantize_cols_kernel(const __half2* __restrict__ x,
                                                                 int64_t rows, int64_t cols, int G,
                                                                 uint8_t* __restrict__ codes,
                                                                 __half2* __restrict__ params) {
  pdl_wait();  // the previous kernel in the stream has finished (see fg_launch)
  const int64_t pairs = cols / 2;
  const int64_t p = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (p >= pairs) return;
  for (int64_t rg = blockIdx.y; rg < rows / G; rg += gridDim.y) {
    const __half2* col = x + rg * G * pairs + p;
    float mn0 = INFINITY, mx0 = -INFINITY, mn1 = INFINITY, mx1 = -INFINITY;
    for (int r = 0; r < G; ++r) {
      float2 f = __half22float2(col[int64_t(r) * pairs]);
      mn0 = fminf(mn0, f.x);
      mx0 = fmaxf(mx0, f.x);
      mn1 = fminf(mn1, f.y);
      mx1 = fmaxf(mx1, f.y);
    }
    mn0 = __fadd_rn(mn0, 0.0f);
    mx0 = __fadd_rn(mx0, 0.0f);
    mn1 = __fadd_rn(mn1, 0.0f);
    mx1 = __fadd_rn(mx1, 0.0f);
    const __half s0 = __float2half_rn(__fdiv_rn(__fsub_rn(mx0, mn0), 15.0f));
    const __half s1 = __float2half_rn(__fdiv_rn(__fsub_rn(mx1, mn1), 15.0f));
    const float sf0 = __half2float(s0), sf1 = __half2float(s1);
    const float d0 = sf0 == 0.0f ? 1.0f : sf0, d1 = sf1 == 0.0f ? 1.0f : sf1;
    params[rg * cols + 2 * p] = __halves2half2(__float2half_rn(mn0), s0);
    params[rg * cols + 2 * p + 1] = __halves2half2(__float2half_rn(mn1), s1);
    for (int r = 0; r < G; ++r) {
      float2 f = __half22float2(col[int64_t(r) * pairs]);
      int q0 = __float2int_rn(__fdiv_rn(__fsub_rn(f.x, mn0), d0));
      int q1 = __float2int_rn(__fdiv_rn(__fsub_rn(f.y, mn1), d1));
      q0 = q0 < 0 ? 0 : (q0 > 15 ? 15 : q0);
      q1 = q1 < 0 ? 0 : (q1 > 15 ? 15 : q1);
      if (sf0 == 0.0f) q0 = 0;
      if (sf1 == 0.0f) q1 = 0;
      codes[(rg * G + r) * pairs + p] = uint8_t(q0 | (q1 << 4));
    }
  }
}

// ------------------------------------------------------------------ K2 dequantize
// axis = 1: one thread per code word (8 elements, one group's params).
template <int G>
__global__ void __launch_bounds__(kThreads) dequant_rows_kernel(const uint32_t* __restrict__ codes,
                                                                const __half2* __restrict__ params,
                                                                int64_t n_words,
                                                                uint4* __restrict__ out) {
  pdl_wait();  // the previous kernel in the stream has finished (see fg_launch)
  constexpr int WPG = G / 8;
  const int64_t tile = int64_t(kThreads) * kUnroll;
  for (int64_t base = int64_t(blockIdx.x) * tile; base < n_words; base += int64_t(gridDim.x) * tile) {
    uint32_t w[kUnroll];
    __half2 p[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t c = base + u * kThreads + threadIdx.x;
      w[u] = c < n_words ? __ldg(codes + c) : 0u;
      p[u] = c < n_words ? __ldg(params + c / WPG) : __half2();
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t c = base + u * kThreads + threadIdx.x;
      if (c < n_words) {
        uint32_t o[4];
        dequant8(w[u], __high2half2(p[u]), __low2half2(p[u]), o);
        out[c] = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
  }
}

// axis = 0: one thread per code word; the 8 columns have their own params.
__global__ void __launch_bounds__(kThreads) dequant_cols_kernel(const uint32_t* __restrict__ codes,
                                                                const __half2* __restrict__ params,
                                                                int64_t rows, int64_t cols, int G,
                                                                uint4* __restrict__ out) {
  pdl_wait();  // the previous kernel in the stream has finished (see fg_launch)
  const int64_t words_per_row = cols / 8;
  const int64_t n_words = rows * words_per_row;
  for (int64_t c = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; c < n_words;
       c += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = c / words_per_row;
    const int64_t col0 = (c - r * words_per_row) * 8;
    const uint32_t w = __ldg(codes + c);
    const __half2* pr = params + (r / G) * cols + col0;
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      __half2 pa = __ldg(pr + 2 * j), pb = __ldg(pr + 2 * j + 1);
      const __half2 s2 = __halves2half2(__high2half(pa), __high2half(pb));
      const __half2 m2 = __halves2half2(__low2half(pa), __low2half(pb));
      uint32_t pair[4];
      dequant8((w >> (8 * j)) & 0xFFu, s2, m2, pair);  // only pair[0] is used
      o[j] = pair[0];
    }
    out[c] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

int grid_for(int64_t units, int64_t per_block) {
  int64_t blocks = (units + per_block - 1) / per_block;
  const int64_t cap = int64_t(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return int(blocks);
}

int check_qargs(const void* a, const void* b, const void* c, int64_t rows, int64_t cols, int group,
                int axis) {
  if (rows < 0 || cols < 0) return fail(FG_ERR_SHAPE, "negative size");
  if (group != 32 && group != 64 && group != 128)
    return fail(FG_ERR_SHAPE, "group must be 32, 64 or 128 (got %d)", group);
  if (axis != 0 && axis != 1) return fail(FG_ERR_INVALID_ARG, "axis must be 0 or 1");
  if (cols % 8) return fail(FG_ERR_SHAPE, "cols must be a multiple of 8");
  if (axis == 1 && cols % group) return fail(FG_ERR_SHAPE, "cols %% group != 0");
  if (axis == 0 && rows % group) return fail(FG_ERR_SHAPE, "rows %% group != 0");
  if (rows > 0 && cols > 0 && rows > (int64_t(1) << 34) / cols)
    return fail(FG_ERR_SHAPE, "tensor larger than 2^34 elements");
  if (rows == 0 || cols == 0) return FG_OK;  // nothing to touch: pointers may be null
  if (!a || !b || !c) return fail(FG_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(a) || !aligned16(b) || !aligned16(c)) return fail(FG_ERR_ALIGN, "pointers must be 16-byte aligned");
  return FG_OK;
}

}  // namespace

// ------------------------------------------------------------------ host entry points
int quantize_pack_impl(const void* x, int64_t rows, int64_t cols, int group, int axis,
                       uint8_t* codes, void* params, cudaStream_t s) {
  FG_TRY(check_qargs(x, codes, params, rows, cols, group, axis));
  const int64_t n = rows * cols;
  if (n == 0) return FG_OK;
  ProfScope ps(PROF_QUANT, s, 0.0, double(n) * (2.0 + 0.5 + 4.0 / group));
  if (axis == 1) {
    const int64_t chunks = n / 16;
    const int grid = grid_for(chunks, int64_t(kThreads) * kUnroll);
    auto* xin = reinterpret_cast<const uint4*>(x);
    auto* cw = reinterpret_cast<uint2*>(codes);
    auto* pw = reinterpret_cast<__half2*>(params);
    if (group == 32) FG_LAUNCH("quantize kernel", quantize_rows_kernel<32>, dim3(grid), dim3(kThreads), size_t(0), s, xin, chunks, cw, pw);
    else if (group == 64) FG_LAUNCH("quantize kernel", quantize_rows_kernel<64>, dim3(grid), dim3(kThreads), size_t(0), s, xin, chunks, cw, pw);
    else FG_LAUNCH("quantize kernel", quantize_rows_kernel<128>, dim3(grid), dim3(kThreads), size_t(0), s, xin, chunks, cw, pw);
  } else {
    const int64_t pairs = cols / 2;
    dim3 grid(unsigned((pairs + kThreads - 1) / kThreads),
              unsigned(std::min<int64_t>(rows / group, 65535)));
    FG_LAUNCH("quantize kernel", quantize_cols_kernel, dim3(grid), dim3(kThreads), size_t(0), s, reinterpret_cast<const __half2*>(x), rows, cols,
                                                   group, codes, reinterpret_cast<__half2*>(params));
  }
  return FG_OK;
}

int dequantize_impl(const uint8_t* codes, const void* params, int64_t rows, int64_t cols, int group,
                    int axis, void* out, cudaStream_t s) {
  FG_TRY(check_qargs(codes, params, out, rows, cols, group, axis));
  const int64_t n = rows * cols;
  if (n == 0) return FG_OK;
  ProfScope ps(PROF_QUANT, s, 0.0, double(n) * (2.0 + 0.5 + 4.0 / group));
  const int64_t words = n / 8;
  auto* cw = reinterpret_cast<const uint32_t*>(codes);
  auto* pw = reinterpret_cast<const __half2*>(params);
  auto* o = reinterpret_cast<uint4*>(out);
  if (axis == 1) {
    const int grid = grid_for(words, int64_t(kThreads) * kUnroll);
    if (group == 32) FG_LAUNCH("dequantize kernel", dequant_rows_kernel<32>, dim3(grid), dim3(kThreads), size_t(0), s, cw, pw, words, o);
    else if (group == 64) FG_LAUNCH("dequantize kernel", dequant_rows_kernel<64>, dim3(grid), dim3(kThreads), size_t(0), s, cw, pw, words, o);
    else FG_LAUNCH("dequantize kernel", dequant_rows_kernel<128>, dim3(grid), dim3(kThreads), size_t(0), s, cw, pw, words, o);
  } else {
    const int grid = grid_for(words, kThreads);
    FG_LAUNCH("dequantize kernel", dequant_cols_kernel, dim3(grid), dim3(kThreads), size_t(0), s, cw, pw, rows, cols, group, o);
  }
  return FG_OK;
}

int kv_append_impl(fg_kv_cache* c, const void* k, const void* v, int64_t row_stride, int n_tokens,
                   cudaStream_t s) {
  if (!c || !k || !v) return fail(FG_ERR_INVALID_ARG, "null pointer");
  if (!c->k_codes || !c->v_codes || !c->k_params || !c->v_params)
    return fail(FG_ERR_INVALID_ARG, "cache buffers not set");
  const int hd = c->head_dim, G = c->group;
  if (G != 32 && G != 64 && G != 128) return fail(FG_ERR_SHAPE, "cache group must be 32, 64 or 128");
  if (hd <= 0 || hd % G || hd % 8) return fail(FG_ERR_SHAPE, "group must divide head_dim");
  if (c->B <= 0 || c->n_heads <= 0 || n_tokens < 0) return fail(FG_ERR_SHAPE, "bad cache shape");
  const int h = c->n_heads * hd;
  if (row_stride < h || row_stride % 8) return fail(FG_ERR_ALIGN, "row_stride must be >= h and a multiple of 8");
  if (c->len < 0 || int64_t(c->len) + n_tokens > c->capacity)
    return fail(FG_ERR_CAPACITY, "KV cache capacity %d exceeded (len %d + %d)", c->capacity, c->len, n_tokens);
  if (!aligned16(k) || !aligned16(v) || !aligned16(c->k_codes) || !aligned16(c->v_codes) ||
      !aligned16(c->k_params) || !aligned16(c->v_params))
    return fail(FG_ERR_ALIGN, "pointers must be 16-byte aligned");
  if (n_tokens == 0) return FG_OK;
  const int64_t chunks = int64_t(c->B) * n_tokens * (h / 16);
  ProfScope ps(PROF_QUANT, s, 0.0, double(chunks) * 16 * 2 * (2.0 + 0.5 + 4.0 / G));
  // few chunks (a decode step's tokens): one chunk per thread and more CTAs, so the
  // latency of the loads is spread over the SMs instead of queueing in a few CTAs
  const bool small = chunks < int64_t(num_sms()) * kThreads * 2;
  dim3 grid(unsigned(grid_for(chunks, int64_t(kThreads) * (small ? 1 : kUnroll))), 2);
  auto* K = reinterpret_cast<const __half*>(k);
  auto* V = reinterpret_cast<const __half*>(v);
  auto* kc = reinterpret_cast<uint2*>(c->k_codes);
  auto* vc = reinterpret_cast<uint2*>(c->v_codes);
  auto* kp = reinterpret_cast<__half2*>(c->k_params);
  auto* vp = reinterpret_cast<__half2*>(c->v_params);
  const bool fast = chunks < (int64_t(1) << 31);
  const FastDiv f_cpr = make_fastdiv(uint32_t(h / 16)), f_T = make_fastdiv(uint32_t(n_tokens)),
                f_hd = make_fastdiv(uint32_t(hd));
  using KernelT = void (*)(const __half*, const __half*, int64_t, int, int, int, int, int, int64_t, uint2*, uint2*,
                           __half2*, __half2*, FastDiv, FastDiv, FastDiv);
  // [group 32 / 64 / 128][one chunk per thread, kUnroll][64-bit, fast indices]
  static const KernelT table[3][2][2] = {
      {{kv_append_kernel<32, 1, false>, kv_append_kernel<32, 1, true>},
       {kv_append_kernel<32, kUnroll, false>, kv_append_kernel<32, kUnroll, true>}},
      {{kv_append_kernel<64, 1, false>, kv_append_kernel<64, 1, true>},
       {kv_append_kernel<64, kUnroll, false>, kv_append_kernel<64, kUnroll, true>}},
      {{kv_append_kernel<128, 1, false>, kv_append_kernel<128, 1, true>},
       {kv_append_kernel<128, kUnroll, false>, kv_append_kernel<128, kUnroll, true>}}};
  const KernelT kern = table[G == 32 ? 0 : (G == 64 ? 1 : 2)][small ? 0 : 1][fast ? 1 : 0];
  FG_LAUNCH("kv append kernel", kern, dim3(grid), dim3(kThreads), size_t(0), s, K, V, row_stride, n_tokens, h, hd,
            c->capacity, c->len, chunks, kc, vc, kp, vp, f_cpr, f_T, f_hd);
  c->len += n_tokens;
  return FG_OK;
}

}  // namespace fg
