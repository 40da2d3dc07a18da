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
// On the 5th-generation tensor cores.  One CTA of 5 warps per (128-query tile, head,
// sequence); thread r of warps 0-3 owns query row q0 + r, warp 4 issues every copy and MMA.
//   TMA       Q tile [128 x HD] once; key and value tiles [64 x HD], two of each in flight,
//             straight from the interleaved projection rows (128-byte swizzle, 64-column boxes).
//   S_j       = Q K_j^T: HD/16 x tcgen05.mma M128 N64 K16 into one of two 64-column TMEM
//             buffers, so Q K_{j+1}^T can run while the softmax of tile j does.
//   softmax   each thread loads its row of S_j (fp32), applies the causal mask, and writes
//             P = 2^(s/sqrt(hd) log2 e - m) as fp16 pairs over the first 32 columns of the
//             same buffer (TMEM lane r, column c = keys 2c, 2c+1: the A layout the MMA reads).
//   O         += P_j V_j: 4 x tcgen05.mma M128 N=HD K16 with A from TMEM and V (MN-major)
//             from shared memory, accumulating in TMEM columns [128, 128 + HD).
// The running maximum m of a row is only raised when a new score exceeds it by more than
// 2^8 (then O and the running sum are rescaled by 2^(m_old - m_new), after the previous
// P V has completed); otherwise P is taken against the stale maximum, at most 256, which
// fp16 and the fp32 sums hold exactly as well.  The result is the same softmax: numerator
// and denominator share the maximum.  Two CTAs fit on an SM (96 KB of shared memory and
// 256 TMEM columns each).  Every wait is bounded; a wait that gives up raises the device
// error flag, and the CTA drains its copies and MMAs before it frees TMEM and exits.
constexpr int kTQ = 128;         // queries per CTA (MMA M)
constexpr int kTK = 64;          // keys per tile (MMA N of Q K^T, K of P V)
constexpr int kBox = 64 * 128;   // one [64 rows x 64 fp16] swizzled box (8 KB)

template <int HD>
struct TcAttnCfg {
  static constexpr int NB = HD / 64;                  // 64-column boxes across the head dim
  static constexpr int kQBytes = NB * 2 * kBox;      // [NB][128 rows][64]
  static constexpr int kKVBytes = NB * kBox;         // [NB][64 rows][64]
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kQBytes;               // two key buffers
  static constexpr int kOffV = kQBytes + 2 * kKVBytes;  // two value buffers
  static constexpr int kOffBar = kQBytes + 4 * kKVBytes;
  static constexpr int kSmem = kOffBar + 128 + 1024;  // barriers + alignment slack
  static constexpr uint32_t kTmemCols = 256;          // S/P 2 x 64, O [128, 128 + HD)
  static constexpr int kThreads = 160;
};

template <int HD>
__global__ void __launch_bounds__(160, 2)
    prefill_attn_tc_kernel(const __grid_constant__ CUtensorMap tm, int L, int nh, __half* __restrict__ out,
                           int* __restrict__ err_flag) {
  using namespace sm100;
  using C = TcAttnCfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* kfull = bars + 0;   // [2] key tile (and, first, Q) landed
  uint64_t* vfull = bars + 2;   // [2] value tile landed
  uint64_t* sfull = bars + 4;   // [2] S_j = Q K_j^T complete
  uint64_t* pfull = bars + 6;   // [2] P_j written (one arrival per softmax warp)
  uint64_t* ofull = bars + 8;   // O += P_j V_j complete (one phase per tile)
  uint64_t* bar_d = bars + 9;   // drain on abort
  uint64_t* ofin = bars + 10;   // every P V complete (one phase, for the epilogue)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 11);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 12);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = gridDim.x - 1 - blockIdx.x;  // heavy (late) tiles first
  const int head = blockIdx.y, b = blockIdx.z;
  const int q0 = qt * kTQ;
  const int h = nh * HD;
  const int row0 = b * L;            // first projection row of this sequence
  const int n_kt = 2 * (qt + 1);     // causal: key tiles 0 .. q0 + 127
  const int kt_diag = 2 * qt;        // tiles from here on need the causal mask

  const bool issuer = warp == 4 && lane == 0;
  // tiles whose copies were issued / waited for, in tile order (issuer only; abort drain)
  int k_iss = 0, k_wt = 0, v_iss = 0, v_wt = 0;
  auto load_k = [&](int j, int extra_bytes) {  // key tile j into buffer j & 1
    const int bb = j & 1;
    mbar_expect_tx(&kfull[bb], C::kKVBytes + extra_bytes);  // the one arrival of this phase
    for (int x = 0; x < C::NB; ++x)
      tma_load_2d(smem + C::kOffK + bb * C::kKVBytes + x * kBox, &tm, h + head * HD + 64 * x, row0 + j * kTK,
                  &kfull[bb]);
    k_iss++;
  };
  auto load_v = [&](int j) {
    const int bb = j & 1;
    mbar_expect_tx(&vfull[bb], C::kKVBytes);
    for (int x = 0; x < C::NB; ++x)
      tma_load_2d(smem + C::kOffV + bb * C::kKVBytes + x * kBox, &tm, 2 * h + head * HD + 64 * x, row0 + j * kTK,
                  &vfull[bb]);
    v_iss++;
  };

  pdl_wait();  // the projections come from the previous kernel in the stream
  if (issuer) {
    // barriers, then the first copies at once: their latency overlaps the TMEM allocation
    prefetch_tmap(&tm);
    for (int i = 0; i < 11; ++i) mbar_init(&bars[i], (i == 6 || i == 7) ? 4 : 1);
    *abort_flag = 0;
    fence_barrier_init();
    // Q rides on the first key tile's barrier (its bytes counted in that phase's expect_tx)
    load_k(0, C::kQBytes);
    for (int x = 0; x < C::NB; ++x)
      for (int r = 0; r < 2; ++r)
        tma_load_2d(smem + C::kOffQ + x * 2 * kBox + r * kBox, &tm, head * HD + 64 * x, row0 + q0 + 64 * r,
                    &kfull[0]);
    load_v(0);
    load_k(1, 0);  // n_kt >= 2
    load_v(1);
  }
  if (warp == 4) {
    __syncwarp();  // the warp-wide allocation after lane 0's copies
    tmem_alloc(tmem_slot, C::kTmemCols);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tO = tmem + 128;

  if (warp == 4) {
    // ------------------------------------------------------------ copies and MMAs
    if (lane == 0) {
      const uint32_t q_addr = smem_u32(smem + C::kOffQ);
      const uint32_t k_addr = smem_u32(smem + C::kOffK), v_addr = smem_u32(smem + C::kOffV);
      constexpr uint32_t idesc_qk = idesc_f16_f32(kTQ, kTK, false);
      constexpr uint32_t idesc_pv = idesc_f16_f32(kTQ, HD, true);
      bool ok = true;
      auto issue_qk = [&](int j) {  // waits for key tile j, S_j into buffer j & 1
        const int bb = j & 1;
        if (!mbar_wait(&kfull[bb], (j >> 1) & 1, abort_flag, err_flag, 0x100)) return false;
        k_wt++;
        tc_fence_after();
        const uint32_t kb = k_addr + bb * C::kKVBytes;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          mma_f16_ss(tmem + 64 * bb, smem_desc_sw128(q_addr + (kk >> 2) * (2 * kBox) + (kk & 3) * 32, 16, 1024),
                     smem_desc_sw128(kb + (kk >> 2) * kBox + (kk & 3) * 32, 16, 1024), idesc_qk, kk > 0);
        }
        mma_commit(&sfull[bb]);
        return true;
      };
      ok = issue_qk(0) && issue_qk(1);
      for (int j = 0; j < n_kt && ok; ++j) {
        const int bb = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        // S_j complete: its key buffer is free for tile j + 2
        if (!(ok = mbar_wait(&sfull[bb], ph, abort_flag, err_flag, 0x200))) break;
        if (j + 2 < n_kt) load_k(j + 2, 0);
        if (!(ok = mbar_wait(&pfull[bb], ph, abort_flag, err_flag, 0x400))) break;
        if (!(ok = mbar_wait(&vfull[bb], ph, abort_flag, err_flag, 0x800))) break;
        v_wt++;
        tc_fence_after();
        const uint32_t vb = v_addr + bb * C::kKVBytes;
#pragma unroll
        for (int kk = 0; kk < kTK / 16; ++kk)
          mma_f16_ts(tO, tmem + 64 * bb + 8 * kk, smem_desc_sw128(vb + kk * 2048, kBox, 1024), idesc_pv,
                     (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(ofull);
        if (j + 2 < n_kt) {
          // P_j and the value tile are read once P V completes: then S_j's buffer and the
          // value buffer take tile j + 2
          if (!(ok = mbar_wait(ofull, j & 1, abort_flag, err_flag, 0x1000))) break;
          load_v(j + 2);
          if (!(ok = issue_qk(j + 2))) break;
        }
      }
      // The epilogue cannot wait for the last tile on ofull: the issuer never waits for
      // P_{n-2} V_{n-2}, so two phases of ofull may be pending then, which a parity wait cannot
      // tell from none.  This commit arrives once every MMA issued so far has completed.
      if (ok) mma_commit(ofin);
      if (!ok) {
        // drain: copies still in flight, then every MMA issued so far
        for (; k_wt < k_iss; ++k_wt) mbar_wait_drain(&kfull[k_wt & 1], (k_wt >> 1) & 1);
        for (; v_wt < v_iss; ++v_wt) mbar_wait_drain(&vfull[v_wt & 1], (v_wt >> 1) & 1);
        mma_commit(bar_d);
        mbar_wait_drain(bar_d, 0);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax and epilogue
    const uint32_t lane_off = uint32_t(warp * 32) << 16;
    const float sl2 = 1.4426950408889634f * rsqrtf(float(HD));  // log2(e) / sqrt(hd)
    const int qi = q0 + threadIdx.x;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kt; ++j) {
      const int bb = j & 1;
      ok = mbar_wait(&sfull[bb], (j >> 1) & 1, abort_flag, err_flag, 0x2000);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      const uint32_t ts = tmem + 64 * bb + lane_off;
      uint32_t sr[64];
      tmem_ld_32x32b_x32(ts, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld_32x32b_x32(ts + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_ld_wait();
      float mx = -INFINITY;
      if (j >= kt_diag) {
        const int last = qi - j * kTK;  // keys of this tile with index <= last are visible
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float v = c <= last ? __uint_as_float(sr[c]) * sl2 : -INFINITY;
          sr[c] = __float_as_uint(v);
          mx = fmaxf(mx, v);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float v = __uint_as_float(sr[c]) * sl2;
          sr[c] = __float_as_uint(v);
          mx = fmaxf(mx, v);
        }
      }
      // raise the running maximum only when it grew by more than 8 (p <= 2^8 otherwise)
      const bool raise = mx > m_run + 8.f;
      if (__any_sync(0xffffffffu, raise && j > 0)) {
        // O is rescaled after P_{j-1} V_{j-1} has landed in it
        ok = mbar_wait(ofull, (j - 1) & 1, abort_flag, err_flag, 0x4000);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
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
        l_run *= (j > 0) ? exp2f(m_run - mx) : 0.f;
        m_run = mx;
      }
      float ls = 0.f;
      uint32_t pr[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float p0 = exp2f(__uint_as_float(sr[2 * c]) - m_run);
        const float p1 = exp2f(__uint_as_float(sr[2 * c + 1]) - m_run);
        ls += p0 + p1;
        pr[c] = h2_as_u32(__floats2half2_rn(p0, p1));
      }
      l_run += ls;
      tmem_st_32x32b_x32(ts, pr);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&pfull[bb]);
    }
    // epilogue: O / l to fp16, once the last P V has landed
    if (ok) ok = mbar_wait(ofin, 0, abort_flag, err_flag, 0x8000);
    if (__all_sync(0xffffffffu, ok)) {
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
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
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
  FG_TRY(make_map_2d(&tm, qkv, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, 3 * h, uint64_t(B) * L, 3 * h * 2, 64, kTK,
                     CU_TENSOR_MAP_SWIZZLE_128B));
  int* err = device_error_ptr();
  if (!err) return fail(FG_ERR_CUDA, "device error flag unavailable");
  const dim3 grid((L + kTQ - 1) / kTQ, nh, B);
  if (hd == 128) {
    static std::atomic<uint64_t> attr_done{0};
    FG_TRY(ensure_smem_attr(prefill_attn_tc_kernel<128>, TcAttnCfg<128>::kSmem, attr_done));
    FG_LAUNCH("prefill attention kernel", prefill_attn_tc_kernel<128>, grid, dim3(TcAttnCfg<128>::kThreads), size_t(TcAttnCfg<128>::kSmem),
              s, tm, L, nh, reinterpret_cast<__half*>(out), err);
  } else {
    static std::atomic<uint64_t> attr_done{0};
    FG_TRY(ensure_smem_attr(prefill_attn_tc_kernel<64>, TcAttnCfg<64>::kSmem, attr_done));
    FG_LAUNCH("prefill attention kernel", prefill_attn_tc_kernel<64>, grid, dim3(TcAttnCfg<64>::kThreads), size_t(TcAttnCfg<64>::kSmem),
              s, tm, L, nh, reinterpret_cast<__half*>(out), err);
  }
  return FG_OK;
}

}  // namespace fg
