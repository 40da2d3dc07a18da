// The group quantizer of a 16-value chunk, shared by the quantize/append kernels and by the
// decode attention kernel that appends a step's new token (include/fg.h, fg_quantize_pack:
// mn = min, mx = max with zero extremes as +0, s = fp16(fp32(mx - mn) / 15),
// code = clamp(rint(fp32(x - mn) / s), 0, 15), every code 0 when s == 0).  Both callers get
// the same codes bit for bit.
#pragma once

#include "fg_common.cuh"

namespace fg {
namespace {

struct GroupQ {
  uint2 words;     // 16 packed codes (element i in bits 4i..4i+3 of words.x, then words.y)
  __half2 params;  // {mn, s}
};

// Packed fp32 pairs (sm_100 f32x2 arithmetic: two IEEE fp32 operations, each rounded to
// nearest even, in one instruction).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// Codes of 16 values by the definition itself: rint(RN(fp32(x - mn) / s)) with the IEEE
// quotient, clamped to 15 (kept out of line: only reached when the fast path is unsure).
__device__ __noinline__ uint2 exact_codes16(uint4 a, uint4 b, float mn, float sf) {
  const __half2* ha = reinterpret_cast<const __half2*>(&a);
  const __half2* hb = reinterpret_cast<const __half2*>(&b);
  uint32_t w[2] = {0u, 0u};
  for (int i = 0; i < 16; ++i) {
    const __half2 pr = (i < 8) ? ha[i / 2] : hb[(i - 8) / 2];
    const float x = (i & 1) ? __high2float(pr) : __low2float(pr);
    int q = sf == 0.0f ? 0 : __float2int_rn(__fdiv_rn(__fsub_rn(x, mn), sf));
    q = q > 15 ? 15 : q;
    w[i / 8] |= uint32_t(q) << (4 * (i % 8));
  }
  return make_uint2(w[0], w[1]);
}

// Quantize 16 consecutive values (two 16-byte vectors) that are part of a group spread over
// TPG = G/16 adjacent lanes.  Every lane of the warp must call this (full-mask shuffles).
// min/max run on packed fp16 (comparisons are exact); the scale and the reciprocal are
// computed once per 16 values, the per-value steps on packed fp32 pairs.
template <int TPG>
__device__ __forceinline__ GroupQ quantize_chunk16(uint4 a, uint4 b) {
  const __half2* ha = reinterpret_cast<const __half2*>(&a);
  const __half2* hb = reinterpret_cast<const __half2*>(&b);
  __half2 lo = __hmin2(__hmin2(ha[0], ha[1]), __hmin2(ha[2], ha[3]));
  __half2 hi = __hmax2(__hmax2(ha[0], ha[1]), __hmax2(ha[2], ha[3]));
  lo = __hmin2(lo, __hmin2(__hmin2(hb[0], hb[1]), __hmin2(hb[2], hb[3])));
  hi = __hmax2(hi, __hmax2(__hmax2(hb[0], hb[1]), __hmax2(hb[2], hb[3])));
  float mn = fminf(__low2float(lo), __high2float(lo));
  float mx = fmaxf(__low2float(hi), __high2float(hi));
#pragma unroll
  for (int o = 1; o < TPG; o <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  mn = __fadd_rn(mn, 0.0f);  // -0 -> +0
  mx = __fadd_rn(mx, 0.0f);
  const __half s16 = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), 15.0f));
  const float sf = __half2float(s16);
  // The code is rint of r = RN(d / s).  r1 = RN(d * RN(1/s)) differs from r by less than
  // 1.5 * 2^-23 * |r| < 2^-18 (r < 16), so rint(r1) == rint(r) unless r1 lies within 2^-18 of
  // a half-integer; inside the wider 2^-17 window the exact IEEE quotient is used instead.
  // rint is taken by adding 1.5 * 2^23 (for 0 <= r1 < 2^22 the sum's ulp is 1, so the add
  // rounds half to even and the low mantissa bits hold the integer).  A zero scale gets a
  // zero reciprocal, which makes every code 0.
  const float rcp = sf == 0.0f ? 0.0f : __frcp_rn(sf);
  const float kMagic = 12582912.0f;  // 1.5 * 2^23
  const uint64_t MN2 = f2_pack(mn, mn), RCP2 = f2_pack(rcp, rcp), MAG2 = f2_pack(kMagic, kMagic);
  uint32_t w[2] = {0u, 0u};
  bool unsure = false;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float2 xf = __half22float2(j < 4 ? ha[j] : hb[j - 4]);
    const uint64_t R = f2_mul(f2_sub(f2_pack(xf.x, xf.y), MN2), RCP2);
    const uint64_t T = f2_add(R, MAG2);
    float f0, f1, t0, t1;
    f2_unpack(f2_sub(R, f2_sub(T, MAG2)), f0, f1);
    f2_unpack(T, t0, t1);
    unsure |= fabsf(f0) > 0.5f - 7.62939453125e-06f;  // 2^-17
    unsure |= fabsf(f1) > 0.5f - 7.62939453125e-06f;
    const uint32_t q0 = min(__float_as_uint(t0) - 0x4B400000u, 15u);
    const uint32_t q1 = min(__float_as_uint(t1) - 0x4B400000u, 15u);
    w[j / 4] |= (q0 | (q1 << 4)) << (8 * (j % 4));
  }
  GroupQ r;
  r.words = unsure ? exact_codes16(a, b, mn, sf) : make_uint2(w[0], w[1]);
  r.params = __halves2half2(__float2half_rn(mn), s16);
  return r;
}

}  // namespace
}  // namespace fg
