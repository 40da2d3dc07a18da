// K5 causal prefill attention over this pass's unquantized fp16 projections.
//
// "FlexGen" README mirror, benchmark notes: the prompt pass (input length 512) is part of
// the measured time.  For each sequence b, head j and query i:
//   out_i = sum_{t <= i} softmax_t(q_i . k_t / sqrt(hd)) v_t
// computed flash-style so the L x L scores never reach memory: one CTA per (64-query tile,
// head, sequence), 4 warps x 16 query rows, key/value tiles of 64 staged in shared
// memory, S = Q K^T and O += P V on mma.sync m16n8k16 (fp16 in, fp32 accumulate), fp32
// online softmax in registers.  P is rounded to fp16 for the second product.  The next
// key tile is copied (cp.async) while the softmax and P V of this one run, the next value
// tile while the next Q K^T runs.
#include "fg_common.cuh"

namespace fg {
namespace {

constexpr int kQT = 64;   // queries per CTA
constexpr int kKT = 64;   // keys per tile
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* g, bool valid) {
  const int n = valid ? 16 : 0;  // 0 source bytes -> zero fill
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(saddr), "l"(g), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_group() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ uint32_t pack_h2(float a, float b) { return h2_as_u32(__floats2half2_rn(a, b)); }

template <int HD>
__global__ void __launch_bounds__(128, HD == 128 ? 3 : 4) prefill_attn_kernel(const __half* __restrict__ qkv, int L, int nh,
                                                           __half* __restrict__ out) {
  pdl_wait();  // the previous kernel in the stream has finished (see fg_launch)
  constexpr int LD = HD + 8;  // padded smem row (halves)
  constexpr int NKS = HD / 16;  // k-steps over head dim
  constexpr int NDB = HD / 8;   // n-blocks over head dim
  extern __shared__ __align__(16) __half sm[];
  __half* sQ = sm;
  __half* sK = sQ + kQT * LD;
  __half* sV = sK + kKT * LD;

  const int qt = gridDim.x - 1 - blockIdx.x;  // heavy (late) tiles first
  const int head = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const int h = nh * HD;
  const int64_t row_stride = 3 * int64_t(h);
  const __half* base = qkv + int64_t(b) * L * row_stride + head * HD;
  const int q0 = qt * kQT;

  // load Q tile
  for (int i = threadIdx.x; i < kQT * (HD / 8); i += 128) {
    const int r = i / (HD / 8), c = (i % (HD / 8)) * 8;
    const int qi = q0 + r;
    cp_async16(static_cast<uint32_t>(__cvta_generic_to_shared(sQ + r * LD + c)),
               base + int64_t(qi < L ? qi : 0) * row_stride + c, qi < L);
  }
  cp_async_wait_all();
  __syncthreads();

  // Q fragments are re-read from shared memory at each k-step (registers go to O and S)
  const uint32_t q_frag_addr =
      static_cast<uint32_t>(__cvta_generic_to_shared(sQ + (warp * 16 + (lane & 15)) * LD + (lane >> 4) * 8));

  float o[NDB][4];
#pragma unroll
  for (int i = 0; i < NDB; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
  const float sl2 = kLog2e * rsqrtf(float(HD));
  const int qrow0 = q0 + warp * 16 + g;  // rows qrow0 and qrow0 + 8

  const int n_kt = qt + 1;  // causal: key tiles 0..qt
  auto load_tile = [&](__half* dst, int k0, int which) {  // which: 1 = K, 2 = V
    for (int i = threadIdx.x; i < kKT * (HD / 8); i += 128) {
      const int r = i / (HD / 8), c = (i % (HD / 8)) * 8;
      const int kj = k0 + r;
      const bool ok = kj < L;
      const __half* src = base + int64_t(ok ? kj : 0) * row_stride + c + which * h;
      cp_async16(static_cast<uint32_t>(__cvta_generic_to_shared(dst + r * LD + c)), src, ok);
    }
    cp_async_commit();
  };
  load_tile(sK, 0, 1);
  load_tile(sV, 0, 2);
  for (int kt = 0; kt < n_kt; ++kt) {
    const int k0 = kt * kKT;
    const bool more = kt + 1 < n_kt;
    cp_async_wait_group<1>();  // this key tile has landed (its value tile may still be in flight)
    __syncthreads();

    // S = Q K^T  (16 x 64 per warp)
    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < NKS; ++ks) {
      uint32_t qa[4];
      ldsm_x4(q_frag_addr + ks * 32, qa[0], qa[1], qa[2], qa[3]);
#pragma unroll
      for (int nb2 = 0; nb2 < 4; ++nb2) {  // pairs of 8-key blocks
        const int j = lane >> 3, r = lane & 7;
        const int key = nb2 * 16 + (j >> 1) * 8 + r;
        const int d = ks * 16 + (j & 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(static_cast<uint32_t>(__cvta_generic_to_shared(sK + key * LD + d)), b0, b1, b2, b3);
        mma16816(s[2 * nb2], qa, b0, b1);
        mma16816(s[2 * nb2 + 1], qa, b2, b3);
      }
    }
    __syncthreads();  // every warp is done with this key tile
    if (more) load_tile(sK, k0 + kKT, 1);
    // scale, mask, online softmax
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int qi = qrow0 + (e >> 1) * 8;
        const int kj = k0 + nb * 8 + 2 * t4 + (e & 1);
        float v = s[nb][e] * sl2;
        if (kj > qi) v = -INFINITY;
        s[nb][e] = v;
        mx[e >> 1] = fmaxf(mx[e >> 1], v);
      }
    }
    float alpha[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
      const float mnew = fmaxf(m_r[r], mx[r]);
      alpha[r] = (m_r[r] == -INFINITY) ? 0.f : exp2f(m_r[r] - mnew);
      m_r[r] = mnew;
    }
    float ls[2] = {0.f, 0.f};
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = e >> 1;
        const float p = (s[nb][e] == -INFINITY) ? 0.f : exp2f(s[nb][e] - m_r[r]);
        s[nb][e] = p;
        ls[r] += p;
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      ls[r] += __shfl_xor_sync(0xffffffffu, ls[r], 1);
      ls[r] += __shfl_xor_sync(0xffffffffu, ls[r], 2);
      l_r[r] = l_r[r] * alpha[r] + ls[r];
    }
#pragma unroll
    for (int i = 0; i < NDB; ++i) {
      o[i][0] *= alpha[0];
      o[i][1] *= alpha[0];
      o[i][2] *= alpha[1];
      o[i][3] *= alpha[1];
    }
    // O += P V (the value tile of this step must have landed)
    if (more) cp_async_wait_group<1>();
    else cp_async_wait_group<0>();
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {  // 16 keys per k-step
      uint32_t a[4];
      a[0] = pack_h2(s[2 * kk][0], s[2 * kk][1]);
      a[1] = pack_h2(s[2 * kk][2], s[2 * kk][3]);
      a[2] = pack_h2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      a[3] = pack_h2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int db2 = 0; db2 < NDB / 2; ++db2) {  // pairs of 8-wide d blocks
        const int j = lane >> 3, r = lane & 7;
        const int key = kk * 16 + (j & 1) * 8 + r;
        const int d = db2 * 16 + (j >> 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(static_cast<uint32_t>(__cvta_generic_to_shared(sV + key * LD + d)), b0, b1, b2, b3);
        mma16816(o[2 * db2], a, b0, b1);
        mma16816(o[2 * db2 + 1], a, b2, b3);
      }
    }
    __syncthreads();  // every warp is done with this value tile
    if (more) load_tile(sV, k0 + kKT, 2);
  }

  // normalize and store
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int qi = qrow0 + r * 8;
    if (qi >= L) continue;
    const float inv = 1.0f / l_r[r];
    __half* dst = out + (int64_t(b) * L + qi) * h + head * HD;
#pragma unroll
    for (int i = 0; i < NDB; ++i) {
      const int d = i * 8 + 2 * t4;
      *reinterpret_cast<__half2*>(dst + d) = __floats2half2_rn(o[i][2 * r] * inv, o[i][2 * r + 1] * inv);
    }
  }
}

}  // namespace

int prefill_attention_impl(const void* qkv, int B, int L, int nh, int hd, void* out, cudaStream_t s) {
  if (!qkv || !out) return fail(FG_ERR_INVALID_ARG, "null pointer");
  if (B <= 0 || L <= 0 || nh <= 0) return fail(FG_ERR_SHAPE, "bad prefill attention shape");
  if (hd != 64 && hd != 128) return fail(FG_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (!aligned16(qkv) || !aligned16(out)) return fail(FG_ERR_ALIGN, "pointers must be 16-byte aligned");
  const double flops = 4.0 * B * nh * double(L) * (L + 1) / 2.0 * hd;
  ProfScope ps(PROF_PREFILL_ATTN, s, flops, double(B) * L * nh * hd * 2.0 * 4.0);
  dim3 grid((L + kQT - 1) / kQT, nh, B);
  const size_t smem = size_t(kQT + 2 * kKT) * (hd + 8) * sizeof(__half);
  if (hd == 128) {
    static bool set = false;
    if (!set) {
      FG_CHECK_CUDA(cudaFuncSetAttribute(prefill_attn_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)));
      set = true;
    }
    FG_LAUNCH("prefill attention kernel", prefill_attn_kernel<128>, dim3(grid), dim3(128), size_t(smem), s, reinterpret_cast<const __half*>(qkv), L, nh,
                                                      reinterpret_cast<__half*>(out));
  } else {
    FG_LAUNCH("prefill attention kernel", prefill_attn_kernel<64>, dim3(grid), dim3(128), size_t(smem), s, reinterpret_cast<const __half*>(qkv), L, nh,
                                                     reinterpret_cast<__half*>(out));
  }
  return FG_OK;
}

}  // namespace fg
