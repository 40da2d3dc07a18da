// K6 LayerNorm, K7 embedding gather, K8 greedy argmax.
//
// OPT decoder plumbing (model family of the "FlexGen" README mirror's benchmark table):
// pre-LayerNorm with fp32 statistics (eps 1e-5), learned positions added to token
// embeddings, and greedy decoding (argmax, ties to the lowest token id).
#include <algorithm>

#include "fg_common.cuh"

namespace fg {
namespace {

constexpr int kLnThreads = 128;
constexpr int kLnMaxChunks = 12;  // 12 * 8 * 128 = 12288 = largest hidden size served

__device__ __forceinline__ float block_sum_128(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  return red[0] + red[1] + red[2] + red[3];
}

// One CTA per row; the row lives in registers (<= 12 chunks of 8 per thread).
__global__ void __launch_bounds__(kLnThreads) layernorm_kernel(const uint4* __restrict__ x, int cols,
                                                               const uint4* __restrict__ g,
                                                               const uint4* __restrict__ bta,
                                                               uint4* __restrict__ y) {
  pdl_wait();  // the previous kernel in the stream has finished (see fg_launch)
  __shared__ float red[4];
  const int chunks = cols / 8;
  const int64_t row = blockIdx.x;
  const uint4* xr = x + row * chunks;
  float v[kLnMaxChunks][8];
  float sum = 0.f;
#pragma unroll
  for (int i = 0; i < kLnMaxChunks; ++i) {
    const int c = threadIdx.x + i * kLnThreads;
    if (c < chunks) {
      const uint4 raw = __ldg(xr + c);
      const __half2* h = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __half22float2(h[j]);
        v[i][2 * j] = f.x;
        v[i][2 * j + 1] = f.y;
        sum += f.x + f.y;
      }
    }
  }
  const float mean = block_sum_128(sum, red) / float(cols);
  float sq = 0.f;
#pragma unroll
  for (int i = 0; i < kLnMaxChunks; ++i) {
    const int c = threadIdx.x + i * kLnThreads;
    if (c < chunks) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float d = v[i][j] - mean;
        sq = fmaf(d, d, sq);
      }
    }
  }
  const float var = block_sum_128(sq, red) / float(cols);
  const float rstd = 1.0f / sqrtf(var + 1e-5f);
#pragma unroll
  for (int i = 0; i < kLnMaxChunks; ++i) {
    const int c = threadIdx.x + i * kLnThreads;
    if (c < chunks) {
      const uint4 gr = __ldg(g + c), br = __ldg(bta + c);
      const __half2* gh = reinterpret_cast<const __half2*>(&gr);
      const __half2* bh = reinterpret_cast<const __half2*>(&br);
      uint4 o;
      uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 gg = __half22float2(gh[j]), bb = __half22float2(bh[j]);
        const float a = fmaf((v[i][2 * j] - mean) * rstd, gg.x, bb.x);
        const float b = fmaf((v[i][2 * j + 1] - mean) * rstd, gg.y, bb.y);
        ow[j] = h2_as_u32(__floats2half2_rn(a, b));
      }
      y[row * chunks + c] = o;
    }
  }
}

// One warp per row for hidden sizes up to 4096 (multiples of 256): the row stays in
// registers as fp16 (CPL 16-byte chunks per lane, a compile-time count so that every load
// of the row is issued before the first is used) and both statistics are warp shuffles, so
// no block barrier sits on the path.  Same fp32 two-pass statistics as above.
constexpr int kLnWarpMaxChunks = 16;
constexpr int kLnWarpRows = 8;  // rows (warps) per CTA

template <int CPL>
__global__ void __launch_bounds__(kLnWarpRows * 32) layernorm_warp_kernel(const uint4* __restrict__ x, int64_t rows,
                                                                           const uint4* __restrict__ g,
                                                                           const uint4* __restrict__ bta,
                                                                           uint4* __restrict__ y) {
  pdl_wait();  // the previous kernel in the stream has finished (see fg_launch)
  const int lane = threadIdx.x & 31;
  const int64_t row = int64_t(blockIdx.x) * kLnWarpRows + (threadIdx.x >> 5);
  if (row >= rows) return;
  constexpr int cols = CPL * 256;  // CPL chunks of 8 values per lane
  const uint4* xr = x + row * (cols / 8);
  uint4 v[CPL];
#pragma unroll
  for (int i = 0; i < CPL; ++i) v[i] = __ldg(xr + i * 32 + lane);  // all loads in flight at once
  float sum = 0.f;
#pragma unroll
  for (int i = 0; i < CPL; ++i) {
    const __half2* h = reinterpret_cast<const __half2*>(&v[i]);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __half22float2(h[j]);
      sum += f.x + f.y;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float mean = sum / float(cols);
  float sq = 0.f;
#pragma unroll
  for (int i = 0; i < CPL; ++i) {
    const __half2* h = reinterpret_cast<const __half2*>(&v[i]);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __half22float2(h[j]);
      const float d0 = f.x - mean, d1 = f.y - mean;
      sq = fmaf(d0, d0, sq);
      sq = fmaf(d1, d1, sq);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
  const float rstd = 1.0f / sqrtf(sq / float(cols) + 1e-5f);
#pragma unroll
  for (int i = 0; i < CPL; ++i) {
    const int c = i * 32 + lane;
    const uint4 gr = __ldg(g + c), br = __ldg(bta + c);
    const __half2* xh = reinterpret_cast<const __half2*>(&v[i]);
    const __half2* gh = reinterpret_cast<const __half2*>(&gr);
    const __half2* bh = reinterpret_cast<const __half2*>(&br);
    uint4 o;
    uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __half22float2(xh[j]), gg = __half22float2(gh[j]), bb = __half22float2(bh[j]);
      const float a = fmaf((f.x - mean) * rstd, gg.x, bb.x);
      const float b = fmaf((f.y - mean) * rstd, gg.y, bb.y);
      ow[j] = h2_as_u32(__floats2half2_rn(a, b));
    }
    y[row * (cols / 8) + c] = o;
  }
}

// x[r] = fp16(E[ids[r]] + P[pos0 + r % T]); __hadd2 rounds the exact sum once.
__global__ void embed_kernel(const int32_t* __restrict__ ids, int T, int ids_stride, int pos0,
                             const uint4* __restrict__ E, const uint4* __restrict__ P, int chunks,
                             int64_t n, uint4* __restrict__ out) {
  pdl_wait();  // the previous kernel in the stream has finished (see fg_launch)
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = i / chunks;
    const int c = int(i - r * chunks);
    const int64_t bb = r / T;
    const int t = int(r - bb * T);
    const int id = __ldg(ids + bb * ids_stride + t);
    const uint4 e = __ldg(E + int64_t(id) * chunks + c);
    const uint4 p = __ldg(P + int64_t(pos0 + t) * chunks + c);
    uint4 o;
    o.x = h2_as_u32(__hadd2(u32_as_h2(e.x), u32_as_h2(p.x)));
    o.y = h2_as_u32(__hadd2(u32_as_h2(e.y), u32_as_h2(p.y)));
    o.z = h2_as_u32(__hadd2(u32_as_h2(e.z), u32_as_h2(p.z)));
    o.w = h2_as_u32(__hadd2(u32_as_h2(e.w), u32_as_h2(p.w)));
    out[i] = o;
  }
}

// One CTA per row of fp32 logits; ties resolve to the lowest index.
__global__ void __launch_bounds__(512) argmax_kernel(const float* __restrict__ logits, int V,
                                                     int32_t* __restrict__ tokens, int64_t tok_stride) {
  pdl_wait();  // the previous kernel in the stream has finished (see fg_launch)
  __shared__ float sv[16];
  __shared__ int si[16];
  const float* row = logits + int64_t(blockIdx.x) * V;
  float best = -INFINITY;
  int bi = 0x7fffffff;
  for (int i = threadIdx.x; i < V; i += blockDim.x) {
    const float x = row[i];
    if (x > best) {  // strictly greater: the first (lowest) index of a tie is kept
      best = x;
      bi = i;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (ov > best || (ov == best && oi < bi)) {
      best = ov;
      bi = oi;
    }
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    sv[warp] = best;
    si[warp] = bi;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const int nw = blockDim.x >> 5;
    float b = sv[0];
    int ix = si[0];
    for (int w = 1; w < nw; ++w) {
      if (sv[w] > b || (sv[w] == b && si[w] < ix)) {
        b = sv[w];
        ix = si[w];
      }
    }
    tokens[int64_t(blockIdx.x) * tok_stride] = ix == 0x7fffffff ? 0 : ix;
  }
}

}  // namespace

int layernorm_impl(const void* x, int64_t rows, int cols, const void* g, const void* b, void* y,
                   cudaStream_t s) {
  if (!x || !g || !b || !y) return fail(FG_ERR_INVALID_ARG, "null pointer");
  if (rows < 0 || cols <= 0 || cols % 8) return fail(FG_ERR_SHAPE, "cols must be a positive multiple of 8");
  if (cols > kLnMaxChunks * 8 * kLnThreads) return fail(FG_ERR_UNSUPPORTED, "hidden size above 12288");
  if (!aligned16(x) || !aligned16(g) || !aligned16(b) || !aligned16(y)) return fail(FG_ERR_ALIGN, "pointers must be 16-byte aligned");
  if (rows == 0) return FG_OK;
  if (rows > 0x7fffffff) return fail(FG_ERR_SHAPE, "too many rows");
  ProfScope ps(PROF_OTHER, s, 0.0, double(rows) * cols * 4.0);
  if (cols % 256 == 0 && cols / 256 <= kLnWarpMaxChunks) {
    using K = void (*)(const uint4*, int64_t, const uint4*, const uint4*, uint4*);
    static const K table[kLnWarpMaxChunks] = {
        layernorm_warp_kernel<1>,  layernorm_warp_kernel<2>,  layernorm_warp_kernel<3>,  layernorm_warp_kernel<4>,
        layernorm_warp_kernel<5>,  layernorm_warp_kernel<6>,  layernorm_warp_kernel<7>,  layernorm_warp_kernel<8>,
        layernorm_warp_kernel<9>,  layernorm_warp_kernel<10>, layernorm_warp_kernel<11>, layernorm_warp_kernel<12>,
        layernorm_warp_kernel<13>, layernorm_warp_kernel<14>, layernorm_warp_kernel<15>, layernorm_warp_kernel<16>};
    FG_LAUNCH("layernorm kernel", table[cols / 256 - 1], dim3(unsigned((rows + kLnWarpRows - 1) / kLnWarpRows)),
              dim3(kLnWarpRows * 32), size_t(0), s, reinterpret_cast<const uint4*>(x), rows,
              reinterpret_cast<const uint4*>(g), reinterpret_cast<const uint4*>(b), reinterpret_cast<uint4*>(y));
    return FG_OK;
  }
  FG_LAUNCH("layernorm kernel", layernorm_kernel, dim3(unsigned(rows)), dim3(kLnThreads), size_t(0), s, 
      reinterpret_cast<const uint4*>(x), cols, reinterpret_cast<const uint4*>(g),
      reinterpret_cast<const uint4*>(b), reinterpret_cast<uint4*>(y));
  return FG_OK;
}

int embed_impl(const int32_t* ids, int64_t B, int T, int ids_stride, int pos0, const void* E, const void* P,
               int hidden, void* out, cudaStream_t s) {
  if (!ids || !E || !P || !out) return fail(FG_ERR_INVALID_ARG, "null pointer");
  if (B < 0 || T < 0 || pos0 < 0 || hidden <= 0 || hidden % 8 || ids_stride < T)
    return fail(FG_ERR_SHAPE, "bad embed shape");
  if (!aligned16(E) || !aligned16(P) || !aligned16(out)) return fail(FG_ERR_ALIGN, "pointers must be 16-byte aligned");
  const int chunks = hidden / 8;
  const int64_t n = int64_t(B) * T * chunks;
  if (n == 0) return FG_OK;
  ProfScope ps(PROF_OTHER, s, 0.0, double(n) * 48.0);
  const int grid = int(std::min<int64_t>((n + 255) / 256, int64_t(num_sms()) * 16));
  FG_LAUNCH("embed kernel", embed_kernel, dim3(grid), dim3(256), size_t(0), s, ids, T, ids_stride, pos0, reinterpret_cast<const uint4*>(E),
                                    reinterpret_cast<const uint4*>(P), chunks, n,
                                    reinterpret_cast<uint4*>(out));
  return FG_OK;
}

int argmax_impl(const float* logits, int B, int V, int32_t* tokens, int64_t tok_stride, cudaStream_t s) {
  if (B <= 0) return FG_OK;
  FG_LAUNCH("argmax kernel", argmax_kernel, dim3(B), dim3(512), size_t(0), s, logits, V, tokens, tok_stride);
  return FG_OK;
}

}  // namespace fg
