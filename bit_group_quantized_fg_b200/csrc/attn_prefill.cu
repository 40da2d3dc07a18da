// K5 causal prefill attention over this pass's unquantized fp16 projections.
//
// "FlexGen" README mirror, benchmark notes: the prompt pass (input length 512) is part of
// the measured time.  For each sequence b, head j and query i:
//   out_i = sum_{t <= i} softmax_t(q_i . k_t / sqrt(hd)) v_t
// computed flash-style so the L x L scores never reach memory, fp32 online softmax, P
// rounded to fp16 for the second product.
#include <cudaTypedefs.h>

#include "fg_common.cuh"
#include "sm100.cuh"

namespace fg {
namespace {

// ---------------------------------------------------------------------------------------
// On the 5th-generation tensor cores.  One CTA of 4 warps per
// (128-query tile, head, sequence); thread r of the CTA owns query row q0 + r.
//   TMA       Q tile [128 x HD] once, key and value tiles [128 x HD] per step, straight
//             from the interleaved projection rows (128-byte swizzle, 64-column boxes).
//   S         = Q K^T: HD/16 x tcgen05.mma M128 N128 K16 into TMEM columns [0, 128).
//   softmax   each thread loads its row of S (fp32), applies the scale and the causal
//             mask, and writes P = 2^(s - m) as fp16 pairs over the first 64 columns of S
//             (TMEM lane r, column c = keys 2c, 2c+1: the A layout the MMA reads).
//   O         += P V: 8 x tcgen05.mma M128 N=HD K16 with A from TMEM, V (MN-major) from
//             shared memory, accumulating in TMEM columns [128, 128 + HD).
// The running maximum m of a row is only raised when a new score exceeds it by more than
// 2^8 (then O and the running sum are rescaled by 2^(m_old - m_new)); otherwise P is taken
// against the stale maximum, at most 256, which fp16 and the fp32 sums hold exactly as
// well.  The result is the same softmax: numerator and denominator share the maximum.
// One thread issues all copies and MMAs; the next key tile is copied while the softmax
// runs, the next value tile while the next Q K^T and softmax run.  Two CTAs fit on an SM
// (96 KB of shared memory and 256 TMEM columns each), so one CTA's softmax overlaps the
// other's MMAs.  Every wait is bounded; a wait that gives up raises the device error flag,
// and the CTA drains its copies and MMAs before it frees TMEM and exits.
constexpr int kTQ = 128;       // queries per CTA (MMA M)
constexpr int kTK = 128;       // keys per step (MMA N of Q K^T, K of P V)
constexpr int kBox = 128 * 128;  // one [128 rows x 64 fp16] swizzled box

template <int HD>
struct TcAttnCfg {
  static constexpr int NB = HD / 64;                 // 64-column boxes per tile
  static constexpr int kTileBytes = NB * kBox;
  static constexpr int kOffQ = 0, kOffK = kTileBytes, kOffV = 2 * kTileBytes;
  static constexpr int kOffBar = 3 * kTileBytes;
  static constexpr int kSmem = kOffBar + 64 + 1024;  // barriers + alignment slack
  static constexpr uint32_t kTmemCols = 256;         // S/P [0, 128), O [128, 128 + HD)
};

template <int HD>
__global__ void __launch_bounds__(128, 2)
    prefill_attn_tc_kernel(const __grid_constant__ CUtensorMap tm, int L, int nh, __half* __restrict__ out,
                           int* __restrict__ err_flag) {
  using namespace sm100;
  using C = TcAttnCfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* bar_k = bars + 0;   // Q (first step) and key tile landed
  uint64_t* bar_v = bars + 1;   // value tile landed
  uint64_t* bar_s = bars + 2;   // S = Q K^T complete
  uint64_t* bar_o = bars + 3;   // O += P V complete
  uint64_t* bar_d = bars + 4;   // drain on abort
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 6);

  const int warp = threadIdx.x >> 5;
  const int nqt = gridDim.x;
  const int qt = nqt - 1 - blockIdx.x;  // heavy (late) tiles first
  const int head = blockIdx.y, b = blockIdx.z;
  const int q0 = qt * kTQ;
  const int h = nh * HD;
  const int row0 = b * L;  // first projection row of this sequence
  const int n_kt = qt + 1;  // causal: key tiles 0..qt

  pdl_wait();  // the projections come from the previous kernel in the stream
  if (threadIdx.x == 0) {
    prefetch_tmap(&tm);
    for (int i = 0; i < 5; ++i) mbar_init(&bars[i], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tO = tmem + 128;
  const uint32_t lane_off = uint32_t(warp * 32) << 16;

  // copies issued / completions waited, per barrier (thread 0 only), for the abort drain
  int k_issued = 0, v_issued = 0, k_done = 0, v_done = 0, mma_open = 0;
  if (threadIdx.x == 0) {
    mbar_expect_tx(bar_k, 2 * C::kTileBytes);
    for (int bb = 0; bb < C::NB; ++bb) {
      tma_load_2d(sQ + bb * kBox, &tm, head * HD + 64 * bb, row0 + q0, bar_k);
      tma_load_2d(sK + bb * kBox, &tm, h + head * HD + 64 * bb, row0, bar_k);
    }
    mbar_expect_tx(bar_v, C::kTileBytes);
    for (int bb = 0; bb < C::NB; ++bb) tma_load_2d(sV + bb * kBox, &tm, 2 * h + head * HD + 64 * bb, row0, bar_v);
    k_issued = v_issued = 1;
  }

  constexpr uint32_t idesc_qk = idesc_f16_f32(kTQ, kTK, false);
  constexpr uint32_t idesc_pv = idesc_f16_f32(kTQ, HD, true);
  const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK), v_addr = smem_u32(sV);
  const float sl2 = 1.4426950408889634f * rsqrtf(float(HD));  // log2(e) / sqrt(hd)
  const int qi = q0 + threadIdx.x;
  float m_run = -INFINITY, l_run = 0.f;
  bool ok = true;

  for (int kt = 0; kt < n_kt; ++kt) {
    const uint32_t ph = kt & 1;
    // ---- S = Q K^T
    if (threadIdx.x == 0 && ok) {
      ok = mbar_wait(bar_k, ph, abort_flag, err_flag, 0x100);
      if (ok) {
        k_done++;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kBox + (kk & 3) * 32;
          mma_f16_ss(tS, smem_desc_sw128(q_addr + off, 16, 1024), smem_desc_sw128(k_addr + off, 16, 1024),
                     idesc_qk, kk > 0);
        }
        mma_commit(bar_s);
        mma_open++;
      }
    }
    if (ok) ok = mbar_wait(bar_s, ph, abort_flag, err_flag, 0x200);
    ok = __all_sync(0xffffffffu, ok);
    if (threadIdx.x == 0 && ok) {
      mma_open--;
      if (kt + 1 < n_kt) {  // the key tile is free: fetch the next one under the softmax
        mbar_expect_tx(bar_k, C::kTileBytes);
        for (int bb = 0; bb < C::NB; ++bb)
          tma_load_2d(sK + bb * kBox, &tm, h + head * HD + 64 * bb, row0 + (kt + 1) * kTK, bar_k);
        k_issued++;
      }
    }
    // ---- softmax on this thread's row
    if (ok) {
      tc_fence_after();
      uint32_t sr[128];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        tmem_ld_32x32b_x32(tS + lane_off + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * c]));
      tmem_ld_wait();
      const int k0 = kt * kTK;
      const bool diag = kt == qt;
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        float v = __uint_as_float(sr[c]) * sl2;
        if (diag && k0 + c > qi) v = -INFINITY;
        sr[c] = __float_as_uint(v);
        mx = fmaxf(mx, v);
      }
      // raise the running maximum only when it grew by more than 8 (p <= 2^8 otherwise)
      const bool raise = mx > m_run + 8.f;
      if (__any_sync(0xffffffffu, raise && kt > 0)) {
        const float alpha = raise ? exp2f(m_run - mx) : 1.f;
#pragma unroll
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t o[32];
          tmem_ld_32x32b_x32(tO + lane_off + 32 * c, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st_32x32b_x32(tO + lane_off + 32 * c, o);
        }
      }
      if (raise) {
        l_run *= (kt > 0) ? exp2f(m_run - mx) : 0.f;
        m_run = mx;
      }
      float ls = 0.f;
      uint32_t pr[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float p0 = exp2f(__uint_as_float(sr[2 * c]) - m_run);
        const float p1 = exp2f(__uint_as_float(sr[2 * c + 1]) - m_run);
        ls += p0 + p1;
        pr[c] = h2_as_u32(__floats2half2_rn(p0, p1));
      }
      l_run += ls;
      tmem_st_32x32b_x32(tS + lane_off, *reinterpret_cast<uint32_t(*)[32]>(&pr[0]));
      tmem_st_32x32b_x32(tS + lane_off + 32, *reinterpret_cast<uint32_t(*)[32]>(&pr[32]));
      tmem_st_wait();
    }
    tc_fence_before();
    __syncthreads();
    ok = ok && !*abort_flag;
    // ---- O += P V
    if (threadIdx.x == 0 && ok) {
      tc_fence_after();
      ok = mbar_wait(bar_v, ph, abort_flag, err_flag, 0x400);
      if (ok) {
        v_done++;
#pragma unroll
        for (int kk = 0; kk < kTK / 16; ++kk)
          mma_f16_ts(tO, tS + 8 * kk, smem_desc_sw128(v_addr + kk * 2048, kBox, 1024), idesc_pv,
                     (kt > 0 || kk > 0) ? 1u : 0u);
        mma_commit(bar_o);
        mma_open++;
        // P and the value tile are read once P V completes: then S may be overwritten
        ok = mbar_wait(bar_o, ph, abort_flag, err_flag, 0x800);
        if (ok) {
          mma_open--;
          if (kt + 1 < n_kt) {
            mbar_expect_tx(bar_v, C::kTileBytes);
            for (int bb = 0; bb < C::NB; ++bb)
              tma_load_2d(sV + bb * kBox, &tm, 2 * h + head * HD + 64 * bb, row0 + (kt + 1) * kTK, bar_v);
            v_issued++;
          }
        }
      }
    }
  }

  // ---- epilogue: O / l to fp16
  if (ok) ok = mbar_wait(bar_o, (n_kt - 1) & 1, abort_flag, err_flag, 0x1000);
  ok = __all_sync(0xffffffffu, ok);
  if (ok) {
    tc_fence_after();
    const float inv = 1.f / l_run;
    __half* dst = out + (int64_t(row0) + qi) * h + head * HD;
#pragma unroll
    for (int c = 0; c < HD / 32; ++c) {
      uint32_t o[32];
      tmem_ld_32x32b_x32(tO + lane_off + 32 * c, o);
      tmem_ld_wait();
      if (qi < L) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          uint4 w;
          w.x = h2_as_u32(__floats2half2_rn(__uint_as_float(o[8 * e + 0]) * inv, __uint_as_float(o[8 * e + 1]) * inv));
          w.y = h2_as_u32(__floats2half2_rn(__uint_as_float(o[8 * e + 2]) * inv, __uint_as_float(o[8 * e + 3]) * inv));
          w.z = h2_as_u32(__floats2half2_rn(__uint_as_float(o[8 * e + 4]) * inv, __uint_as_float(o[8 * e + 5]) * inv));
          w.w = h2_as_u32(__floats2half2_rn(__uint_as_float(o[8 * e + 6]) * inv, __uint_as_float(o[8 * e + 7]) * inv));
          reinterpret_cast<uint4*>(dst + 32 * c)[e] = w;
        }
      }
    }
  }
  // ---- abort drain: wait (bounded) for this CTA's copies and MMAs still in flight
  if (threadIdx.x == 0 && !ok) {
    for (; k_done < k_issued; ++k_done) mbar_wait_drain(bar_k, k_done & 1);
    for (; v_done < v_issued; ++v_done) mbar_wait_drain(bar_v, v_done & 1);
    if (mma_open > 0) {
      mma_commit(bar_d);
      mbar_wait_drain(bar_d, 0);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, C::kTmemCols);
}
}  // namespace

int make_map_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes, uint64_t inner,
                uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz);

int prefill_attention_impl(const void* qkv, int B, int L, int nh, int hd, void* out, cudaStream_t s) {
  if (!qkv || !out) return fail(FG_ERR_INVALID_ARG, "null pointer");
  if (B <= 0 || L <= 0 || nh <= 0) return fail(FG_ERR_SHAPE, "bad prefill attention shape");
  if (hd != 64 && hd != 128) return fail(FG_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (int64_t(B) * L > 0x7fffffff - kTQ) return fail(FG_ERR_SHAPE, "too many rows");
  if (!aligned16(qkv) || !aligned16(out)) return fail(FG_ERR_ALIGN, "pointers must be 16-byte aligned");
  const double flops = 4.0 * B * nh * double(L) * (L + 1) / 2.0 * hd;
  ProfScope ps(PROF_PREFILL_ATTN, s, flops, double(B) * L * nh * hd * 2.0 * 4.0);
  const uint64_t h = uint64_t(nh) * hd;
  CUtensorMap tm;
  FG_TRY(make_map_2d(&tm, qkv, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, 3 * h, uint64_t(B) * L, 3 * h * 2, 64, kTQ,
                     CU_TENSOR_MAP_SWIZZLE_128B));
  int* err = device_error_ptr();
  if (!err) return fail(FG_ERR_CUDA, "device error flag unavailable");
  const dim3 grid((L + kTQ - 1) / kTQ, nh, B);
  if (hd == 128) {
    static bool set = false;
    if (!set) {
      FG_CHECK_CUDA(cudaFuncSetAttribute(prefill_attn_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         TcAttnCfg<128>::kSmem));
      set = true;
    }
    FG_LAUNCH("prefill attention kernel", prefill_attn_tc_kernel<128>, grid, dim3(128), size_t(TcAttnCfg<128>::kSmem),
              s, tm, L, nh, reinterpret_cast<__half*>(out), err);
  } else {
    static bool set = false;
    if (!set) {
      FG_CHECK_CUDA(cudaFuncSetAttribute(prefill_attn_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         TcAttnCfg<64>::kSmem));
      set = true;
    }
    FG_LAUNCH("prefill attention kernel", prefill_attn_tc_kernel<64>, grid, dim3(128), size_t(TcAttnCfg<64>::kSmem),
              s, tm, L, nh, reinterpret_cast<__half*>(out), err);
  }
  return FG_OK;
}

}  // namespace fg
