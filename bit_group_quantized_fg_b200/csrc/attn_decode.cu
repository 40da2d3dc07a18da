// K4 split-context decode attention over the 4-bit KV cache, and K4r the split combine.
//
// One query token per sequence ("FlexGen" README mirror: generation over a compressed
// attention cache).  For sequence b and head j:
//   score_t = (q . K_t) / sqrt(hd),  K_t = mn_t + code_t * s_t (per group of G dims)
//   out = sum_t softmax(score)_t V_t
// The cache is read exactly once: one CTA per (chunk of positions, head, sequence)
// streams the chunk's K and V codes together in a single pass with an online softmax.
// Both contractions run on the tensor cores (mma.sync) over codes that are only unpacked
// into exact fp16 (offset + code) values, with the per-group {min, scale} applied to the
// fp32 results.  Softmax is fp32 with exp2 (scores scaled by log2(e)/sqrt(hd)); warps and
// chunks are merged with the usual (max, sum, acc) rescaling.  The small mma.sync tile, not
// tcgen05, because each (sequence, head) has a single query row: the contractions are
// matrix-vector products over streamed codes (about 3.6 FLOP per byte), so a 128-row tcgen05
// tile would hold one useful row; the MMA only takes the multiply-adds off the FMA pipe, and
// HBM stays the bound.
#include <algorithm>
#include <mutex>

#include "fg_common.cuh"
#include "quant_common.cuh"

namespace fg {
namespace {

constexpr int kWarps = 2;
// Blocks of positions a warp keeps in flight (cp.async into its shared-memory ring) ahead of
// the one it computes on: the bytes in flight no longer cost registers.
constexpr int kDepth = 4;
constexpr int kThreads = kWarps * 32;
constexpr float kLog2e = 1.4426950408889634f;

// 16-byte global -> shared copy of which the first `bytes` (0..16) are read and the rest is
// zero-filled (L2 only: the cache is streamed once); both addresses 16-byte aligned.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, int bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src), "r"(bytes)
               : "memory");
}
// 4-byte copy (`bytes` 0 or 4; 0 writes a zero word without reading).
__device__ __forceinline__ void cp_async4(void* dst, const void* src, int bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ------------------------------------------------------------------ K4, tensor-core form
// The same attention with both contractions on mma.sync (m16n8k16, fp16 in, fp32 out), so
// that the codes are only unpacked, never multiplied on the FMA pipe.  A warp takes blocks
// of 16 positions.
//   scores:  D[t][n] = sum over the dims d of group n of q_d (o_d + c_td)   (A = codes,
//            B = q masked per group): a code becomes an exact fp16 o + c by putting the
//            nibble into the mantissa of 1024.0 (low nibbles, bits 0-3: o = 1024) or of 64.0
//            (high nibbles, bits 4-7: o = 64); K dims are taken in any order that A and B
//            agree on.  score_t = sum_n s_tn (D[t][n] - O_n) + mn_tn Q_n, with
//            O_n = sum q_d o_d and Q_n = sum q_d over the group.
//   values:  E[d][n] = sum_t w_tn (64 + c_td) with w_tn = fp16(p_t s_tn) (A = codes with
//            pairs of positions per register, B = w), and
//            out_d = (sum_t p_t mn_tn + E[d][n] - 64 sum_t w_tn) / sum_t p_t, n = group(d).
//            Here both nibbles use o = 64 (low nibbles shifted up): the offset sum grows with
//            the number of positions, and the small offset keeps its cancellation small.
// Thread (g = lane/4, q4 = lane%4) holds positions g and g + 8 of a block for the scores and
// dims DPT*g .. DPT*g + DPT-1 for the values (DPT = HD/8).
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The four fp16 pairs (o + c) of one code word (dims 8w .. 8w+7): P0 = dims (0, 2),
// P1 = (4, 6) from the low nibbles (o = 1024), P2 = (1, 3), P3 = (5, 7) from the high nibbles
// (o = 64).
__device__ __forceinline__ void code_pairs(uint32_t w, uint32_t (&P)[4]) {
  const uint32_t x = w & 0x0F0F0F0Fu, y = w & 0xF0F0F0F0u;
  P[0] = __byte_perm(x, 0x64646464u, 0x4140);
  P[1] = __byte_perm(x, 0x64646464u, 0x4342);
  P[2] = __byte_perm(y, 0x54545454u, 0x4140);
  P[3] = __byte_perm(y, 0x54545454u, 0x4342);
}

template <int HD, int G>
struct AttnMma {
  static constexpr int NG = HD / G;    // groups per head: 1, 2 or 4
  static constexpr int KW = HD / 32;   // code words a thread reads of a K row
  static constexpr int KS = HD / 16;   // k-steps of the score MMA
  static constexpr int MT = HD / 16;   // 16-dim tiles of the value MMA
  static constexpr int DPT = HD / 8;   // dims per value row-thread
  static constexpr int VW = HD / 64;   // code words a thread reads of a V row
  static constexpr int TB = 16;        // positions per block
  // a block in a warp's ring: K codes, V codes (TB rows of HD/2 bytes), K params, V params
  // (TB rows of NG {min, scale} pairs), each a contiguous run of the cache
  static constexpr int RC = HD / 2, RP = NG * 4;                // row bytes
  static constexpr int SLOT = 2 * TB * RC + 2 * TB * RP;      // bytes of one block
  static_assert(SLOT % 16 == 0 && RC % 16 == 0, "16-byte copies");
};

// Fused append (the decode step's KV append): when `knew` is not NULL, position S - 1 is the
// step's new token, whose K and V rows (knew/vnew + b * new_stride, fp16) are not yet in the
// cache.  The CTA of each (sequence, head) that owns the last chunk quantizes them with the
// same group quantizer as the append kernel (warp 0: K, warp 1: V), stores codes and params
// at position S - 1, and attends over that position from shared memory (no other CTA reads it).
template <int HD, int G>
__global__ void __launch_bounds__(kThreads) decode_attn_mma_kernel(
    const __half* __restrict__ q, int64_t q_stride, const uint8_t* __restrict__ kc,
    const __half2* __restrict__ kp, const uint8_t* __restrict__ vc, const __half2* __restrict__ vp,
    int nh, int cap, int S, int chunk_len, __half* __restrict__ out, float* __restrict__ part_ml,
    float* __restrict__ part_acc, const __half* knew, const __half* vnew, int64_t new_stride, uint8_t* kc_w,
    __half2* kp_w, uint8_t* vc_w, __half2* vp_w) {
  pdl_wait();  // the previous kernel in the stream has finished (see fg_launch)
  using C = AttnMma<HD, G>;
  constexpr int NG = C::NG, KW = C::KW, KS = C::KS, MT = C::MT, DPT = C::DPT, VW = C::VW, TB = C::TB;
  __shared__ float red_v[kWarps][HD];
  __shared__ float red_ml[kWarps][2];
  __shared__ uint32_t new_codes[2][HD / 8];  // the new token's K / V code words
  __shared__ uint32_t new_par[2][NG];        // and {min, scale} pairs

  const int b = blockIdx.z, head = blockIdx.y, chunk = blockIdx.x;
  const int t0 = chunk * chunk_len;
  const int t1 = min(S, t0 + chunk_len);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, q4 = lane & 3;
  const __half* qh = q + int64_t(b) * q_stride + head * HD;
  const bool app = knew != nullptr && chunk == int(gridDim.x) - 1;
  const int tnew = S - 1;
  if (app) {
    static_assert(kWarps == 2, "one warp quantizes K, the other V");
    constexpr int TPG = G / 16;  // lanes per group (16 values per lane)
    const __half* src = (warp == 0 ? knew : vnew) + int64_t(b) * new_stride + head * HD;
    uint4 xa = make_uint4(0, 0, 0, 0), xb = xa;
    if (lane < HD / 16) {
      xa = *reinterpret_cast<const uint4*>(src + lane * 16);
      xb = *reinterpret_cast<const uint4*>(src + lane * 16 + 8);
    }
    const GroupQ r = quantize_chunk16<TPG>(xa, xb);  // every lane takes part in the shuffles
    if (lane < HD / 16) {
      const int64_t slot = (int64_t(b) * nh + head) * cap + tnew;
      uint8_t* cw = warp == 0 ? kc_w : vc_w;
      __half2* pw = warp == 0 ? kp_w : vp_w;
      *reinterpret_cast<uint2*>(cw + slot * (HD / 2) + lane * 8) = r.words;
      new_codes[warp][2 * lane] = r.words.x;
      new_codes[warp][2 * lane + 1] = r.words.y;
      if (lane % TPG == 0) {
        pw[slot * NG + lane / TPG] = r.params;
        new_par[warp][lane / TPG] = h2_as_u32(r.params);
      }
    }
    __syncthreads();
  }

  // ---- query: B fragments of the score MMA, and per-group O_n, Q_n
  uint32_t qb[KS][2];
#pragma unroll
  for (int st = 0; st < KS; ++st) {
    const int w = KW * q4 + st / 2, e = st & 1;
    const bool mine = (8 * w) / G == g;  // column g of B is group g
    const int d0 = 8 * w + e;
    const __half z = __float2half(0.f);
    const __half h0 = mine ? qh[d0] : z, h1 = mine ? qh[d0 + 2] : z;
    const __half h2 = mine ? qh[d0 + 4] : z, h3 = mine ? qh[d0 + 6] : z;
    qb[st][0] = h2_as_u32(__halves2half2(h0, h1));
    qb[st][1] = h2_as_u32(__halves2half2(h2, h3));
  }
  float On[NG], Qn[NG];
#pragma unroll
  for (int n = 0; n < NG; ++n) On[n] = Qn[n] = 0.f;
#pragma unroll
  for (int i = 0; i < HD / 32; ++i) {
    const int d = lane + 32 * i;
    const float qd = __half2float(qh[d]);
#pragma unroll
    for (int n = 0; n < NG; ++n) {
      if (d / G == n) {
        Qn[n] += qd;
        On[n] += qd * ((d & 1) ? 64.f : 1024.f);
      }
    }
  }
#pragma unroll
  for (int n = 0; n < NG; ++n) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      Qn[n] += __shfl_xor_sync(0xffffffffu, Qn[n], o);
      On[n] += __shfl_xor_sync(0xffffffffu, On[n], o);
    }
  }
  const float sc = kLog2e * rsqrtf(float(HD));

  const int64_t slot0 = (int64_t(b) * nh + head) * cap;
  const uint8_t* kbase = kc + slot0 * (HD / 2);
  const uint8_t* vbase = vc + slot0 * (HD / 2);
  const __half2* kpb = kp + slot0 * NG;
  const __half2* vpb = vp + slot0 * NG;

  float m = -INFINITY, lsum = 0.f, amn = 0.f, ssum = 0.f;
  float acc[MT][4];
#pragma unroll
  for (int i = 0; i < MT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;

  // One block's registers: K rows g, g+8 (KW words from word KW*q4), V rows 2q4, 2q4+1,
  // 2q4+8, 2q4+9 (VW words at dim DPT*g), K params of (row, groups 2q4, 2q4+1), V params of
  // (row, group q4); positions past t1 hold zeros (the ring copies zero-fill them).
  struct Blk {
    uint32_t kA[KW], kB[KW], vw[4][VW], kpA[2], kpB[2], vpA, vpB;
  };
  __shared__ __align__(16) uint8_t ring[kWarps][kDepth][C::SLOT];
  // the copies of block `blk` into ring slot `sl` of this warp; rows at or past t1 are
  // written as zeros without being read.  Codes go in 16-byte chunks (a row is HD/2 bytes,
  // a multiple of 16); the {min, scale} rows of one (sequence, head) start only 4 * NG-byte
  // aligned (at (b * nh + head) * cap * NG pairs), so they go word by word.
  auto issue = [&](int sl, int blk) {
    uint8_t* dst = ring[warp][sl];
    const int nv = max(0, min(TB, t1 - blk));   // valid rows of the block
    constexpr int kCodeChunks = 2 * TB * C::RC / 16;
#pragma unroll
    for (int j = 0; j < (kCodeChunks + 31) / 32; ++j) {
      const int i = lane + 32 * j;
      if (i < kCodeChunks) {
        const int o = i * 16;
        const bool v = o >= TB * C::RC;
        const int off = v ? o - TB * C::RC : o;
        const bool ok = off / C::RC < nv;
        cp_async16(dst + o, ok ? (v ? vbase : kbase) + int64_t(blk) * C::RC + off : kbase, ok ? 16 : 0);
      }
    }
    constexpr int kParWords = 2 * TB * NG;
    const uint32_t* kpu = reinterpret_cast<const uint32_t*>(kpb);
    const uint32_t* vpu = reinterpret_cast<const uint32_t*>(vpb);
#pragma unroll
    for (int j = 0; j < (kParWords + 31) / 32; ++j) {
      const int i = lane + 32 * j;
      if (i < kParWords) {
        const bool v = i >= TB * NG;
        const int wi = v ? i - TB * NG : i;   // word of the block's param run
        const bool ok = wi / NG < nv;
        cp_async4(dst + 2 * TB * C::RC + 4 * i, ok ? (v ? vpu : kpu) + int64_t(blk) * NG + wi : kpu, ok ? 4 : 0);
      }
    }
  };
  // the block in ring slot `sl` into registers; the new token's position comes from the
  // quantizer's shared-memory copy
  auto fetch = [&](Blk& o, int sl, int blk) {
    const uint8_t* r = ring[warp][sl];
    const uint8_t* kr = r;
    const uint8_t* vr = r + TB * C::RC;
    const uint32_t* kpr = reinterpret_cast<const uint32_t*>(r + 2 * TB * C::RC);
    const uint32_t* vpr = reinterpret_cast<const uint32_t*>(r + 2 * TB * C::RC + TB * C::RP);
#pragma unroll
    for (int i = 0; i < KW; ++i) {
      o.kA[i] = reinterpret_cast<const uint32_t*>(kr + g * C::RC)[KW * q4 + i];
      o.kB[i] = reinterpret_cast<const uint32_t*>(kr + (g + 8) * C::RC)[KW * q4 + i];
    }
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      const int t = 2 * q4 + (rr & 1) + (rr >> 1) * 8;
#pragma unroll
      for (int w = 0; w < VW; ++w) o.vw[rr][w] = reinterpret_cast<const uint32_t*>(vr + t * C::RC)[VW * g + w];
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int n = 2 * q4 + j;
      o.kpA[j] = n < NG ? kpr[g * NG + (n < NG ? n : 0)] : 0u;
      o.kpB[j] = n < NG ? kpr[(g + 8) * NG + (n < NG ? n : 0)] : 0u;
    }
    o.vpA = q4 < NG ? vpr[g * NG + (q4 < NG ? q4 : 0)] : 0u;
    o.vpB = q4 < NG ? vpr[(g + 8) * NG + (q4 < NG ? q4 : 0)] : 0u;
    if (app && tnew >= blk && tnew < blk + TB) {
      const int tA = blk + g, tB = blk + g + 8;
      const bool pA = tA == tnew, pB = tB == tnew;
      if (pA || pB) {
#pragma unroll
        for (int i = 0; i < KW; ++i) {
          const uint32_t w = new_codes[0][KW * q4 + i];
          if (pA) o.kA[i] = w;
          if (pB) o.kB[i] = w;
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int n = 2 * q4 + j;
          const uint32_t pk = n < NG ? new_par[0][n < NG ? n : 0] : 0u;
          if (pA) o.kpA[j] = pk;
          if (pB) o.kpB[j] = pk;
        }
        const uint32_t pv = q4 < NG ? new_par[1][q4 < NG ? q4 : 0] : 0u;
        if (pA) o.vpA = pv;
        if (pB) o.vpB = pv;
      }
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) {
        if (blk + 2 * q4 + (rr & 1) + (rr >> 1) * 8 == tnew) {
#pragma unroll
          for (int w = 0; w < VW; ++w) o.vw[rr][w] = new_codes[1][VW * g + w];
        }
      }
    }
  };

  // one commit group per block, empty ones past t1, so that the wait count stays uniform
#pragma unroll
  for (int i = 0; i < kDepth; ++i) {
    issue(i, t0 + warp * TB + i * kWarps * TB);
    cp_async_commit();
  }
  int sl = 0;
  for (int blk = t0 + warp * TB; blk < t1; blk += kWarps * TB) {
    Blk cur;
    cp_async_wait<kDepth - 1>();
    __syncwarp();   // every lane's copies of this block have landed
    fetch(cur, sl, blk);
    __syncwarp();   // every lane has read the slot before it is refilled
    issue(sl, blk + kDepth * kWarps * TB);
    cp_async_commit();
    if (++sl == kDepth) sl = 0;
    const int tA = blk + g, tB = blk + g + 8;
    const bool okA = tA < t1, okB = tB < t1;
    const uint32_t(&kA)[KW] = cur.kA;
    const uint32_t(&kB)[KW] = cur.kB;
    const uint32_t(&vw)[4][VW] = cur.vw;
    float ksA[2], kmA[2], ksB[2], kmB[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const float2 fa = __half22float2(u32_as_h2(cur.kpA[j])), fb = __half22float2(u32_as_h2(cur.kpB[j]));
      kmA[j] = fa.x;
      ksA[j] = fa.y;
      kmB[j] = fb.x;
      ksB[j] = fb.y;
    }
    const float2 fva = __half22float2(u32_as_h2(cur.vpA)), fvb = __half22float2(u32_as_h2(cur.vpB));
    const float vmA = fva.x, vsA = fva.y, vmB = fvb.x, vsB = fvb.y;

    // ---- scores
    float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int wi = 0; wi < KW; ++wi) {
      uint32_t PA[4], PB[4];
      code_pairs(kA[wi], PA);
      code_pairs(kB[wi], PB);
      mma16816(d, PA[0], PB[0], PA[1], PB[1], qb[2 * wi][0], qb[2 * wi][1]);
      mma16816(d, PA[2], PB[2], PA[3], PB[3], qb[2 * wi + 1][0], qb[2 * wi + 1][1]);
    }
    float pa = 0.f, pb = 0.f;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int n = 2 * q4 + j;
      float o = 0.f, qs = 0.f;
#pragma unroll
      for (int k = 0; k < NG; ++k) {
        if (n == k) {
          o = On[k];
          qs = Qn[k];
        }
      }
      if (n < NG) {
        pa += fmaf(ksA[j], d[j] - o, kmA[j] * qs);
        pb += fmaf(ksB[j], d[2 + j] - o, kmB[j] * qs);
      }
    }
    if (NG > 2) {
      pa += __shfl_xor_sync(0xffffffffu, pa, 1);
      pb += __shfl_xor_sync(0xffffffffu, pb, 1);
    }
    // every lane of a row now holds the scores (lanes with q4 >= 2 hold 0 when NG <= 2)
    pa = __shfl_sync(0xffffffffu, pa, lane & ~3);
    pb = __shfl_sync(0xffffffffu, pb, lane & ~3);
    const float sA = okA ? pa * sc : -INFINITY, sB = okB ? pb * sc : -INFINITY;
    float bm = fmaxf(sA, sB);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
    if (bm > m) {
      const float r = exp2f(m - bm);  // m = -inf -> 0
      lsum *= r;
      amn *= r;
      ssum *= r;
#pragma unroll
      for (int i = 0; i < MT; ++i) {
        acc[i][0] *= r; acc[i][1] *= r; acc[i][2] *= r; acc[i][3] *= r;
      }
      m = bm;
    }
    const float pA = exp2f(sA - m), pB = exp2f(sB - m);  // 0 for positions past the end
    if (q4 == 0) lsum += pA + pB;
    // value weights of (row, group q4): w = fp16(p * s)
    const __half wA = __float2half_rn(pA * vsA), wB = __float2half_rn(pB * vsB);
    amn = fmaf(pA, vmA, fmaf(pB, vmB, amn));
    ssum += __half2float(wA) + __half2float(wB);
    // B fragment of the value MMA for group g: positions 2q4, 2q4+1 (rows of lanes 8q4 + g,
    // 8q4 + 4 + g as "A"), and 2q4 + 8, 2q4 + 9 (the same lanes' "B" rows)
    const uint32_t wAu = __half_as_ushort(wA), wBu = __half_as_ushort(wB);
    const int src0 = 8 * q4 + (g & 3), src1 = src0 + 4;
    const uint32_t w0 = __shfl_sync(0xffffffffu, wAu, src0), w1 = __shfl_sync(0xffffffffu, wAu, src1);
    const uint32_t w2 = __shfl_sync(0xffffffffu, wBu, src0), w3 = __shfl_sync(0xffffffffu, wBu, src1);
    const bool gv = g < NG;
    const uint32_t b0 = gv ? (w0 | (w1 << 16)) : 0u, b1 = gv ? (w2 | (w3 << 16)) : 0u;

    // ---- values: tile mt covers byte mt of the thread's V words (dims DPT*g + 2mt, +1)
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const int wd = mt / 4, by = mt % 4;
      const uint32_t sel = uint32_t(by | (by << 4) | ((4 + by) << 8) | ((4 + by) << 12));
      const uint32_t r01 = __byte_perm(vw[0][wd], vw[1][wd], sel);
      const uint32_t r23 = __byte_perm(vw[2][wd], vw[3][wd], sel);
      const uint32_t a0 = ((r01 << 4) & 0x00F000F0u) | 0x54005400u, a1 = (r01 & 0x00F000F0u) | 0x54005400u;
      const uint32_t a2 = ((r23 << 4) & 0x00F000F0u) | 0x54005400u, a3 = (r23 & 0x00F000F0u) | 0x54005400u;
      mma16816(acc[mt], a0, a1, a2, a3, b0, b1);
    }
  }
  cp_async_wait<0>();   // nothing in flight when the warp leaves its ring

  // ---- finish the warp: sums over rows, then out_d for the dims this lane holds
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    amn += __shfl_xor_sync(0xffffffffu, amn, o);
    ssum += __shfl_xor_sync(0xffffffffu, ssum, o);
  }
  float amn_n[NG], ss_n[NG];
#pragma unroll
  for (int n = 0; n < NG; ++n) {
    amn_n[n] = __shfl_sync(0xffffffffu, amn, n);
    ss_n[n] = __shfl_sync(0xffffffffu, ssum, n);
  }
  // acc[mt][0/1]: dim DPT*g + 2mt (low nibble), groups 2q4 / 2q4+1;
  // acc[mt][2/3]: dim DPT*g + 2mt + 1 (high nibble)
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
    for (int hv = 0; hv < 2; ++hv) {
      const int dd = DPT * g + 2 * mt + hv;
      const int n = dd / G;
      if ((n >> 1) == q4) {
        const float e = (n & 1) ? acc[mt][2 * hv + 1] : acc[mt][2 * hv];
        float an = amn_n[0], sn = ss_n[0];
#pragma unroll
        for (int k = 1; k < NG; ++k) {
          if (n == k) {
            an = amn_n[k];
            sn = ss_n[k];
          }
        }
        red_v[warp][dd] = an + e - 64.f * sn;
      }
    }
  }
  if (lane == 0) {
    red_ml[warp][0] = m;
    red_ml[warp][1] = lsum;
  }
  __syncthreads();
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
  for (int dd = threadIdx.x; dd < HD; dd += kThreads) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w)
      if (wsc[w] != 0.f) v = fmaf(red_v[w][dd], wsc[w], v);
    if (part_ml == nullptr) {
      out[int64_t(b) * nh * HD + head * HD + dd] = __float2half_rn(v / L);
    } else {
      part_acc[(bh * gridDim.x + chunk) * HD + dd] = v;
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
  pdl_wait();  // the previous kernel in the stream has finished (see fg_launch)
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
  // At most 2048 positions per chunk: the offset codes' cancellation error (the value MMA
  // sums w (64 + c) over the chunk in fp32, then 64 * sum(w) is subtracted) grows with the
  // chunk while the output of a near-uniform softmax shrinks; chunks of 4096 measured
  // 1.24e-2 * RMS at context 8192, chunks of 2048 stay near 4e-3.
  const int min_by_len = (S + 2047) / 2048;
  return std::max(nc, std::max(1, min_by_len));
}

}  // namespace

size_t decode_attention_ws_bytes(int B, int nh, int hd, int ctx) {
  if (B <= 0 || nh <= 0 || hd <= 0 || ctx <= 0) return 0;
  const int nc = pick_chunks(B, nh, ctx);
  if (nc <= 1) return 0;
  return size_t(B) * nh * nc * (2 + hd) * sizeof(float) + 256;
}

// With knew/vnew (rows of the step's new K and V, new_stride elements apart) the step's token
// is appended at position len inside the attention kernel, attention covers 0..len, and len
// advances (the cache must be non-const then).
int decode_attention_impl(const void* q, int64_t q_stride, const fg_kv_cache* c, void* out,
                          void* ws, size_t ws_bytes, cudaStream_t s, const void* knew = nullptr,
                          const void* vnew = nullptr, int64_t new_stride = 0, fg_kv_cache* cw = nullptr) {
  if (!q || !c || !out) return fail(FG_ERR_INVALID_ARG, "null pointer");
  const bool append = knew != nullptr;
  if (append && (!vnew || cw != c)) return fail(FG_ERR_INVALID_ARG, "fused append needs K, V and the cache");
  if (append && c->len + 1 > c->capacity) return fail(FG_ERR_CAPACITY, "KV cache full (capacity %d)", c->capacity);
  if (append && (new_stride < int64_t(c->n_heads) * c->head_dim || new_stride % 8 || !aligned16(knew) ||
                 !aligned16(vnew)))
    return fail(FG_ERR_ALIGN, "new K/V rows must be 16-byte aligned with a stride >= h, multiple of 8");
  const int B = c->B, nh = c->n_heads, hd = c->head_dim, G = c->group, S = c->len + (append ? 1 : 0);
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
  auto* kp = reinterpret_cast<const __half2*>(c->k_params);
  auto* vp = reinterpret_cast<const __half2*>(c->v_params);
  auto* o = reinterpret_cast<__half*>(out);
  auto* kc8 = reinterpret_cast<const uint8_t*>(c->k_codes);
  auto* vc8 = reinterpret_cast<const uint8_t*>(c->v_codes);
  auto* kn = reinterpret_cast<const __half*>(knew);
  auto* vn = reinterpret_cast<const __half*>(vnew);
  auto* kcw = append ? cw->k_codes : nullptr;
  auto* vcw = append ? cw->v_codes : nullptr;
  auto* kpw = append ? reinterpret_cast<__half2*>(cw->k_params) : nullptr;
  auto* vpw = append ? reinterpret_cast<__half2*>(cw->v_params) : nullptr;
#define FG_ATTN_LAUNCH(HD_, G_)                                                                      \
  FG_LAUNCH("decode attention kernel", decode_attn_mma_kernel<HD_, G_>, dim3(grid), dim3(kThreads), size_t(smem), s, qh, q_stride, kc8, kp, vc8, vp, nh, \
                                                                c->capacity, S, chunk_len, o, ml, acc, kn, vn, new_stride, kcw, kpw, vcw, vpw)
  if (hd == 128 && G == 128) FG_ATTN_LAUNCH(128, 128);
  else if (hd == 128 && G == 64) FG_ATTN_LAUNCH(128, 64);
  else if (hd == 128 && G == 32) FG_ATTN_LAUNCH(128, 32);
  else if (hd == 64 && G == 64) FG_ATTN_LAUNCH(64, 64);
  else FG_ATTN_LAUNCH(64, 32);
#undef FG_ATTN_LAUNCH
  if (nc > 1) {
    const int n_bh = B * nh;
    if (hd == 128)
      FG_LAUNCH("decode combine kernel", decode_combine_kernel<128>, dim3((n_bh + 3) / 4), dim3(128), size_t(0), s, ml, acc, n_bh, nc, nh, o);
    else
      FG_LAUNCH("decode combine kernel", decode_combine_kernel<64>, dim3((n_bh + 3) / 4), dim3(128), size_t(0), s, ml, acc, n_bh, nc, nh, o);
  }
  if (append) cw->len += 1;
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
