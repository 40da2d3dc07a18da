// K3: dequant-fused GEMM on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
//   Y[M][N] = [relu](X[M][K] * W_hat[K][N] + b) [+ R]
//
// The weights W ("FlexGen" README mirror, key features: parameters compressed to 4 bits)
// are 4-bit codes [K][N/2] with {min, scale} fp16 pairs per group of G along N.  W_hat is
// exactly fg_dequantize's fp16 value, so fp16 x fp16 products accumulated in fp32 are the
// contraction the layer defines.
//
// Structure (one CTA per SM, persistent over output tiles of 128 x 256):
//   warp 0      TMA producer: X tile [128 x 64] (128-byte swizzle, K-major) and the code
//               tile [64 x 128 B] + param tile [64 x PB] of the k-block into a stage.
//   warp 1      MMA issuer: 4 x tcgen05.mma (M128 N256 K16) per k-block into one of two
//               TMEM accumulators (2 x 256 fp32 columns); tcgen05.commit frees the stage.
//   warps 4-7   epilogue: tcgen05.ld rows of the finished accumulator, bias / ReLU /
//               residual, fp16 (or fp32) stores; frees the accumulator for tile i+2.
//   warps 8-15  dequant (4-bit mode): expand the stage's codes to fp16 directly into
//               the MN-major 128-byte-swizzled operand layout the MMA reads.
// Other operand modes reuse the skeleton: B as a ready fp16 [K][N] tensor (MN-major, by
// TMA) or as an fp16 [N][K] tensor (K-major by TMA, the tied LM head).  Tiles are
// rasterized in bands of row tiles (at most 64 MiB of X) so a band of X stays in L2 while
// the weight streams past it.
// With few tiles (decode batches) the K loop is split and fp32 partials are reduced by a
// second kernel that applies the epilogue.  Prompt-pass fp16 [K][N] GEMMs (from kPairRows
// rows) run on CTA pairs instead (gemm_pair.cu), and so do 4-bit GEMMs grouped along N of
// 129-256 rows (gemm_q4pair.cu: each CTA of a pair expands half of a 256-column weight
// tile); this kernel keeps decode batches of up to 128 rows, weights grouped along K, the
// LM head and the smaller fp16 GEMMs.
#include <algorithm>
#include <cstring>
#include <cudaTypedefs.h>

#include "fg_common.cuh"
#include "sm100.cuh"

namespace fg {

__device__ int g_device_error = 0;  // set by bounded waits that gave up (host-readable)

namespace {

using namespace sm100;

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int kABytes = BM * BK * 2;   // 16 KB
constexpr int kBBytes = BN * BK * 2;   // 32 KB
constexpr int kCodeBytes = BK * BN / 2; // 8 KB
constexpr int kParamBytesMax = BK * 8 * 4;  // up to 8 half2 per k row (G = 32)

// B_Q4: 4-bit weight, groups along N (params [K][N/G]); B_Q4K: 4-bit weight, groups along K
// (params [K/G][N]); B_F16_MN: fp16 [K][N]; B_F16_K: fp16 [N][K].
enum BMode { B_Q4 = 0, B_F16_MN = 1, B_F16_K = 2, B_Q4K = 3 };

// Shared memory: a ring of TMA stages, then (4-bit mode) a ring of expanded fp16 B tiles.
// 4-bit mode: TMA stage = X tile + code tile + param tile (26 KB), 6 deep, so that the loads
// run far enough ahead of the tensor cores to cover their latency; the dequant warps fill a
// separate 2-deep ring of 32 KB fp16 B tiles.  fp16 modes: TMA stage = X tile + B tile, 4 deep.
template <int MODE>
struct Cfg {
  static constexpr bool kQ4 = MODE == B_Q4 || MODE == B_Q4K;
  static constexpr int kStages = kQ4 ? 6 : 4;
  static constexpr int kCodeOff = kABytes;
  static constexpr int kParamOff = kABytes + kCodeBytes;
  static constexpr int kStageBytes = kQ4 ? kABytes + kCodeBytes + kParamBytesMax : kABytes + kBBytes;
  static constexpr int kBStages = kQ4 ? 2 : 0;
  static constexpr int kBRingOff = kStages * kStageBytes;
  static constexpr int kDequantWarps = kQ4 ? 8 : 0;
  static constexpr int kThreads = 256 + kDequantWarps * 32;
  static constexpr int kSmem = kBRingOff + kBStages * kBBytes + 1024 /*align*/ + 256 /*barriers*/;
  static_assert(kBRingOff % 1024 == 0 && kStageBytes % 1024 == 0, "1024-byte aligned operand tiles");
  static_assert(kSmem <= 232448, "shared memory budget");
};

struct GemmArgs {
  int M, N, K;
  int m_tiles, n_tiles, k_blocks, splits;
  int band;         // row tiles per rasterization band
  int prefetch_w;   // weight tiles may be requested before the previous kernel completes
  int total;        // m_tiles * n_tiles * splits
  int G, PB;        // group size, params per k row in a stage (B_Q4)
  int param_bytes;  // bytes of a stage's param tile
  const __half* bias;
  const __half* R;
  int relu;
  void* Y;          // fp16 or fp32 [M][N]
  float* partial;   // [splits][M][N] when splits > 1
  // Wave tail (splits == 1): tiles [0, full_units) run whole, gridDim.x at a time; the
  // k-blocks of the remaining tail_tiles are divided evenly over all CTAs (CTA b takes the
  // flat range [I b / grid, I (b + 1) / grid) of I = tail_tiles * k_blocks), which cuts
  // at most two tiles per CTA; those segments go to tail_part[b][segment][BM][BN] in fp32
  // and tail_fixup_kernel sums them per tile.
  int full_units, tail_tiles;
  float* tail_part;
};

struct TileCoord {
  int m0, n0, kb0, kb1, ks;
  int seg;          // tail segment of this CTA (0 or 1), -1 for a whole tile or split-K slice
};

__device__ __forceinline__ TileCoord tile_coord(const GemmArgs& a, int t) {
  TileCoord c;
  c.ks = t % a.splits;
  const int r = t / a.splits;
  const int band_tiles = a.band * a.n_tiles;
  const int bi = r / band_tiles;
  const int rr = r - bi * band_tiles;
  const int mt_in_band = min(a.band, a.m_tiles - bi * a.band);
  const int n = rr / mt_in_band;
  const int m = bi * a.band + (rr - n * mt_in_band);
  c.m0 = m * BM;
  c.n0 = n * BN;
  c.kb0 = int((int64_t(c.ks) * a.k_blocks) / a.splits);
  c.kb1 = int((int64_t(c.ks + 1) * a.k_blocks) / a.splits);
  c.seg = -1;
  return c;
}

// First flat k-block of the wave tail that CTA b computes.
__host__ __device__ __forceinline__ int64_t tail_start(int64_t I, int b, int grid) { return I * b / grid; }

// Work units of this CTA, in the order every role walks them.
__device__ __forceinline__ int unit_count(const GemmArgs& a) {
  const int b = blockIdx.x, G = gridDim.x;
  if (a.tail_tiles == 0) return b < a.total ? (a.total - 1 - b) / G + 1 : 0;
  const int64_t I = int64_t(a.tail_tiles) * a.k_blocks;
  const int64_t s0 = tail_start(I, b, G), s1 = tail_start(I, b + 1, G);
  int n = a.full_units / G;
  if (s1 > s0) n += (s0 / a.k_blocks == (s1 - 1) / a.k_blocks) ? 1 : 2;
  return n;
}

__device__ __forceinline__ TileCoord unit_coord(const GemmArgs& a, int u) {
  const int b = blockIdx.x, G = gridDim.x;
  const int nf = a.tail_tiles == 0 ? 0x7fffffff : a.full_units / G;
  if (u < nf) return tile_coord(a, b + u * G);
  const int64_t I = int64_t(a.tail_tiles) * a.k_blocks;
  const int64_t s0 = tail_start(I, b, G), s1 = tail_start(I, b + 1, G);
  const int seg = u - nf;
  const int tile0 = int(s0 / a.k_blocks);
  const int tile = tile0 + seg;
  TileCoord c = tile_coord(a, a.full_units + tile);
  c.kb0 = seg == 0 ? int(s0 - int64_t(tile0) * a.k_blocks) : 0;
  c.kb1 = int(min(int64_t(a.k_blocks), s1 - int64_t(tile) * a.k_blocks));
  c.seg = seg;
  return c;
}

template <int MODE, bool OUT_F32>
__global__ void __launch_bounds__(Cfg<MODE>::kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                   const __grid_constant__ CUtensorMap tm_p, const GemmArgs args) {
  using C = Cfg<MODE>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base_u32 = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024 - (base_u32 & 1023)) & 1023);
  constexpr int SB = C::kBStages > 0 ? C::kBStages : 1;  // B-ring depth (4-bit mode)
  uint8_t* bring = smem + C::kBRingOff;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBRingOff + C::kBStages * kBBytes);
  uint64_t* full = bars;                   // [S]  TMA stage landed
  uint64_t* empty = bars + S;              // [S]  MMA finished reading the TMA stage
  uint64_t* bfull = bars + 2 * S;          // [SB] dequant wrote a B tile
  uint64_t* bempty = bars + 2 * S + SB;    // [SB] MMA finished reading a B tile
  uint64_t* acc_full = bars + 2 * S + 2 * SB;       // [2]
  uint64_t* acc_empty = bars + 2 * S + 2 * SB + 2;  // [2]
  uint64_t* drain = bars + 2 * S + 2 * SB + 4;      // [1] MMA drain on abort
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 2 * SB + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * S + 2 * SB + 6);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < SB; ++i) {
      mbar_init(&bfull[i], C::kDequantWarps > 0 ? C::kDequantWarps : 1);
      mbar_init(&bempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    if (C::kQ4) prefetch_tmap(&tm_p);
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t tx = kABytes + (C::kQ4 ? (kCodeBytes + args.param_bytes) : kBBytes);
      bool ok = true;
      // the weight operand of k-block kb of tile c into stage buffer st
      auto load_w = [&](uint8_t* st, const TileCoord& c, int kb, uint64_t* bar) {
        if (MODE == B_Q4) {
          tma_load_2d(st + C::kCodeOff, &tm_b, c.n0 / 2, kb * BK, bar);
          const int px = (c.n0 / args.G) & ~3;
          tma_load_2d(st + C::kParamOff, &tm_p, px, kb * BK, bar);
        } else if (MODE == B_Q4K) {
          tma_load_2d(st + C::kCodeOff, &tm_b, c.n0 / 2, kb * BK, bar);
          tma_load_2d(st + C::kParamOff, &tm_p, c.n0, (kb * BK) / args.G, bar);
        } else if (MODE == B_F16_MN) {
#pragma unroll
          for (int j = 0; j < BN / 64; ++j) tma_load_2d(st + kABytes + j * 8192, &tm_b, c.n0 + 64 * j, kb * BK, bar);
        } else {
          tma_load_2d(st + kABytes, &tm_b, kb * BK, c.n0, bar);
        }
      };
      // Weights are never written by an earlier kernel: the first stages' weight tiles are
      // requested before waiting for the previous kernel, whose output X may still be in
      // the making (programmatic dependent launch).
      int pre = 0;
      const int n_units = unit_count(args);
      if (args.prefetch_w && n_units > 0) {
        const TileCoord c0 = unit_coord(args, 0);
        pre = min(S, c0.kb1 - c0.kb0);
        for (int i = 0; i < pre; ++i) {
          mbar_expect_tx(&full[i], tx);
          load_w(smem + i * C::kStageBytes, c0, c0.kb0 + i, &full[i]);
        }
      }
      pdl_wait();
      int issued = 0;
      for (int u = 0; u < n_units && ok; ++u) {
        const TileCoord c = unit_coord(args, u);
        for (int kb = c.kb0; kb < c.kb1; ++kb, ++issued) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, &g_device_error, 1)) { ok = false; break; }
          uint8_t* st = smem + stage * C::kStageBytes;
          if (issued >= pre) {
            mbar_expect_tx(&full[stage], tx);
            load_w(st, c, kb, &full[stage]);
          }
          tma_load_2d(st, &tm_a, kb * BK, c.m0, &full[stage]);
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
      }
      if (*abort_flag) {
        // stages whose weight tiles were requested up front but whose X copy was never
        // issued get it now, so that their barriers complete; then let every copy this
        // thread issued land before the CTA exits
        if (issued < pre) {
          const TileCoord c0 = unit_coord(args, 0);
          for (int i = issued; i < pre; ++i)
            tma_load_2d(smem + i * C::kStageBytes, &tm_a, (c0.kb0 + i) * BK, c0.m0, &full[i]);
        }
        // stage q (in issue order) went to slot q % S in phase (q / S) & 1; only the last S
        // can still be in flight
        const int armed = max(issued, pre);
        for (int q = max(0, armed - S); q < armed; ++q) mbar_wait_drain(&full[q % S], uint32_t(q / S) & 1u);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(BM, BN, MODE != B_F16_K);
      int stage = 0, bs = 0;
      uint32_t phase = 0, bphase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      const int n_units = unit_count(args);
      for (int u = 0; u < n_units && ok; ++u) {
        const TileCoord c = unit_coord(args, u);
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1, abort_flag, &g_device_error, 2)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + uint32_t(acc * BN);
        for (int kb = c.kb0; kb < c.kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, &g_device_error, 4)) { ok = false; break; }
          if (C::kQ4 && !mbar_wait(&bfull[bs], bphase, abort_flag, &g_device_error, 8)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * C::kStageBytes);
          const uint32_t b_addr = C::kQ4 ? smem_u32(bring + bs * kBBytes) : a_addr + kABytes;
          // the k-th 16-deep slice: +32 bytes along K (K-major) or +2048 (MN-major: two 8-row
          // groups of 1024 bytes); the descriptor's address field counts 16-byte units
          const uint64_t ad0 = smem_desc_sw128(a_addr, 16, 1024);
          const uint64_t bd0 = MODE == B_F16_K ? smem_desc_sw128(b_addr, 16, 1024) : smem_desc_sw128(b_addr, 8192, 1024);
          constexpr uint64_t kBStep = MODE == B_F16_K ? 2 : 128;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            mma_f16_ss(d_tmem, ad0 + uint64_t(2 * k), bd0 + kBStep * k, idesc, (kb > c.kb0 || k > 0) ? 1u : 0u);
          mma_commit(&empty[stage]);
          if (++stage == S) { stage = 0; phase ^= 1; }
          if (C::kQ4) {
            mma_commit(&bempty[bs]);
            if (++bs == SB) { bs = 0; bphase ^= 1; }
          }
        }
        if (!ok) break;
        mma_commit(&acc_full[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
      if (*abort_flag) {
        // wait for the MMAs already issued before TMEM is released
        mma_commit(drain);
        mbar_wait_drain(drain, 0);
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ epilogue
    const int q = warp - 4;  // TMEM lane quarter
    int acc = 0;
    uint32_t acc_phase = 0;
    const int n_units = unit_count(args);
    for (int u = 0; u < n_units; ++u) {
      const TileCoord c = unit_coord(args, u);
      if (!mbar_wait(&acc_full[acc], acc_phase, abort_flag, &g_device_error, 16)) break;
      tc_fence_after();
      const int m = c.m0 + q * 32 + lane;
      const bool row_ok = m < args.M;
      for (int cc = 0; cc < BN; cc += 32) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem_base + (uint32_t(q * 32) << 16) + uint32_t(acc * BN + cc), r);
        tmem_ld_wait();
        if (C::kQ4) {
          // the dequant warps stored each 8 columns in the order [0,4,1,5,2,6,3,7]:
          // natural column j of a group sits at position (j < 4 ? 2j : 2(j-4)+1)
          uint32_t t[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int jj = j & 7;
            t[j] = r[(j & ~7) + (jj < 4 ? 2 * jj : 2 * (jj - 4) + 1)];
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = t[j];
        }
        const int n = c.n0 + cc;
        if (!row_ok || n >= args.N) continue;
        if (c.seg >= 0) {
          float4* dst = reinterpret_cast<float4*>(
              args.tail_part + ((int64_t(blockIdx.x) * 2 + c.seg) * BM + (m - c.m0)) * BN + cc);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            dst[j] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                 __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
          continue;
        }
        if (args.partial != nullptr) {
          float4* dst = reinterpret_cast<float4*>(args.partial + (int64_t(c.ks) * args.M + m) * args.N + n);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            dst[j] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                 __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
          continue;
        }
        if (OUT_F32) {
          float* dst = reinterpret_cast<float*>(args.Y) + int64_t(m) * args.N + n;
          if (n + 32 <= args.N) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
              reinterpret_cast<float4*>(dst)[j] =
                  make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                              __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
          } else {
            for (int j = 0; j < 32 && n + j < args.N; ++j) dst[j] = __uint_as_float(r[j]);
          }
          continue;
        }
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
        if (args.bias != nullptr) {
          const uint4* bp = reinterpret_cast<const uint4*>(args.bias + n);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint4 bw = __ldg(bp + j);
            const __half2* bh = reinterpret_cast<const __half2*>(&bw);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __half22float2(bh[e]);
              v[8 * j + 2 * e] += f.x;
              v[8 * j + 2 * e + 1] += f.y;
            }
          }
        }
        if (args.relu) {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = fmaxf(v[j], 0.f);
        }
        if (args.R != nullptr) {
          const uint4* rp = reinterpret_cast<const uint4*>(args.R + int64_t(m) * args.N + n);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint4 rw = __ldg(rp + j);
            const __half2* rh = reinterpret_cast<const __half2*>(&rw);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __half22float2(rh[e]);
              v[8 * j + 2 * e] += f.x;
              v[8 * j + 2 * e + 1] += f.y;
            }
          }
        }
        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__half*>(args.Y) + int64_t(m) * args.N + n);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint4 o;
          o.x = h2_as_u32(__floats2half2_rn(v[8 * j + 0], v[8 * j + 1]));
          o.y = h2_as_u32(__floats2half2_rn(v[8 * j + 2], v[8 * j + 3]));
          o.z = h2_as_u32(__floats2half2_rn(v[8 * j + 4], v[8 * j + 5]));
          o.w = h2_as_u32(__floats2half2_rn(v[8 * j + 6], v[8 * j + 7]));
          dst[j] = o;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
  } else if (C::kQ4 && warp >= 8) {
    // ------------------------------------------------------------ dequant warps
    constexpr int DW = C::kDequantWarps > 0 ? C::kDequantWarps : 1;
    constexpr int RPW = BK / DW;   // k rows per warp: dw, dw + DW, ...
    const int dw = warp - 8;
    const int nb = lane >> 3;      // 64-wide MN block of the word
    const int ch = lane & 7;       // 16-byte chunk inside the block
    int stage = 0, bs = 0;
    uint32_t phase = 0, bphase = 0;
    bool ok = true;
    const int n_units = unit_count(args);
    for (int u = 0; u < n_units && ok; ++u) {
      const TileCoord c = unit_coord(args, u);
      const int poff = (c.n0 / args.G) & 3;
      const int pcol = poff + (lane * 8) / args.G;
      for (int kb = c.kb0; kb < c.kb1; ++kb) {
        if (!mbar_wait(&full[stage], phase, abort_flag, &g_device_error, 32)) { ok = false; break; }
        const uint8_t* st = smem + stage * C::kStageBytes;
        const uint32_t* codes = reinterpret_cast<const uint32_t*>(st + C::kCodeOff);
        const uint32_t* prm = reinterpret_cast<const uint32_t*>(st + C::kParamOff);
        uint32_t w[RPW];
        uint32_t o[RPW][4];
#pragma unroll
        for (int i = 0; i < RPW; ++i) w[i] = codes[(dw + DW * i) * (BN / 8) + lane];
        if (MODE == B_Q4) {
          uint32_t p[RPW];
#pragma unroll
          for (int i = 0; i < RPW; ++i) p[i] = prm[(dw + DW * i) * args.PB + pcol];
#pragma unroll
          for (int i = 0; i < RPW; ++i) {
            const __half2 pr = u32_as_h2(p[i]);
            dequant8_interleaved(w[i], __high2half2(pr), __low2half2(pr), o[i]);
          }
        } else {
          // groups along K: one {min, scale} per column for each group of G rows; the rows of
          // this k-block lie in one group (G >= 64) or two (G = 32: rows 0-31, 32-63)
          // rows dw + 8i: i < 4 lie in rows 0-31, i >= 4 in rows 32-63 of the k-block
          const bool two = args.G == 32;
          const uint4* pp0 = reinterpret_cast<const uint4*>(prm + lane * 8);
          const uint4* pp1 = reinterpret_cast<const uint4*>(prm + (two ? BN : 0) + lane * 8);
          const uint4 a0 = pp0[0], b0 = pp0[1], a1 = pp1[0], b1 = pp1[1];  // columns +0..3, +4..7
          __half2 s_lo[4], m_lo[4], s_hi[4], m_hi[4];
          {
            const uint32_t la[4] = {a0.x, a0.y, a0.z, a0.w}, ha[4] = {b0.x, b0.y, b0.z, b0.w};
            const uint32_t lb[4] = {a1.x, a1.y, a1.z, a1.w}, hb[4] = {b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {   // pair j holds columns j and j + 4 (interleaved order)
              m_lo[j] = u32_as_h2(__byte_perm(la[j], ha[j], 0x5410));
              s_lo[j] = u32_as_h2(__byte_perm(la[j], ha[j], 0x7632));
              m_hi[j] = u32_as_h2(__byte_perm(lb[j], hb[j], 0x5410));
              s_hi[j] = u32_as_h2(__byte_perm(lb[j], hb[j], 0x7632));
            }
          }
#pragma unroll
          for (int i = 0; i < RPW; ++i) {
            if (i < RPW / 2) dequant8_interleaved_pairs(w[i], s_lo, m_lo, o[i]);
            else dequant8_interleaved_pairs(w[i], s_hi, m_hi, o[i]);
          }
        }
        // the B tile this k-block fills must have been consumed by the MMA two blocks ago
        if (!mbar_wait(&bempty[bs], bphase ^ 1, abort_flag, &g_device_error, 64)) { ok = false; break; }
        uint8_t* bt = bring + bs * kBBytes;
#pragma unroll
        for (int i = 0; i < RPW; ++i) {
          const int row = dw + DW * i;  // k index inside the block
          const int kg = row >> 3, rr = row & 7;
          uint4* dst = reinterpret_cast<uint4*>(bt + nb * 8192 + kg * 1024 + rr * 128 + ((ch ^ rr) << 4));
          *dst = make_uint4(o[i][0], o[i][1], o[i][2], o[i][3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bfull[bs]);
        if (++stage == S) { stage = 0; phase ^= 1; }
        if (++bs == SB) { bs = 0; bphase ^= 1; }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// Split-K reduction + epilogue: Y = [relu](sum_s P[s] + b) [+ R], 8 columns per thread.
__global__ void splitk_reduce_kernel(const float* __restrict__ P, int splits, int64_t MN, int N,
                                     const __half* __restrict__ bias, const __half* __restrict__ R,
                                     int relu, __half* __restrict__ Y) {
  pdl_wait();  // the previous kernel in the stream has finished (see fg_launch)
  const int64_t n8 = MN / 8;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n8; i += int64_t(gridDim.x) * blockDim.x) {
    float v[8];
    const float4* p0 = reinterpret_cast<const float4*>(P) + i * 2;
    float4 a = p0[0], b = p0[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    for (int s = 1; s < splits; ++s) {
      const float4* ps = reinterpret_cast<const float4*>(P + s * MN) + i * 2;
      a = ps[0];
      b = ps[1];
      v[0] += a.x; v[1] += a.y; v[2] += a.z; v[3] += a.w; v[4] += b.x; v[5] += b.y; v[6] += b.z; v[7] += b.w;
    }
    const int n = int((i * 8) % N);
    if (bias) {
      const uint4 bw = __ldg(reinterpret_cast<const uint4*>(bias + n));
      const __half2* bh = reinterpret_cast<const __half2*>(&bw);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(bh[e]);
        v[2 * e] += f.x;
        v[2 * e + 1] += f.y;
      }
    }
    if (relu) {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = fmaxf(v[j], 0.f);
    }
    if (R) {
      const uint4 rw = __ldg(reinterpret_cast<const uint4*>(R) + i);
      const __half2* rh = reinterpret_cast<const __half2*>(&rw);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(rh[e]);
        v[2 * e] += f.x;
        v[2 * e + 1] += f.y;
      }
    }
    uint4 o;
    o.x = h2_as_u32(__floats2half2_rn(v[0], v[1]));
    o.y = h2_as_u32(__floats2half2_rn(v[2], v[3]));
    o.z = h2_as_u32(__floats2half2_rn(v[4], v[5]));
    o.w = h2_as_u32(__floats2half2_rn(v[6], v[7]));
    reinterpret_cast<uint4*>(Y)[i] = o;
  }
}

// Wave tail of a GEMM (see GemmArgs): each tail tile's segments summed in CTA order, then
// Y = [relu](sum + b) [+ R].  A block covers 8 rows of one tile (32 threads x 8 columns
// per row); grid = tail_tiles * BM / 8.
__global__ void __launch_bounds__(256) tail_fixup_kernel(const GemmArgs a, int grid) {
  pdl_wait();  // the GEMM's partial tiles are complete (see fg_launch)
  const int tau = blockIdx.x / (BM / 8);
  const int row = (blockIdx.x % (BM / 8)) * 8 + (threadIdx.x >> 5);
  const int col = (threadIdx.x & 31) * 8;
  const TileCoord c = tile_coord(a, a.full_units + tau);
  const int m = c.m0 + row, n = c.n0 + col;
  if (m >= a.M || n >= a.N) return;
  const int64_t kb = a.k_blocks, I = int64_t(a.tail_tiles) * kb;
  const int64_t x0 = int64_t(tau) * kb, x1 = x0 + kb;
  // first CTA whose range reaches past x0
  int g = int(x0 * grid / I);
  while (g + 1 < grid && tail_start(I, g + 1, grid) <= x0) ++g;
  while (g > 0 && tail_start(I, g, grid) > x0) --g;
  float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (; g < grid; ++g) {
    const int64_t s0 = tail_start(I, g, grid), s1 = tail_start(I, g + 1, grid);
    if (s0 >= x1) break;
    if (s1 <= s0 || s1 <= x0) continue;
    const int seg = s0 >= x0 ? 0 : 1;  // tau is this CTA's first tile, or its second
    const float4* p = reinterpret_cast<const float4*>(a.tail_part + ((int64_t(g) * 2 + seg) * BM + row) * BN + col);
    const float4 p0 = p[0], p1 = p[1];
    v[0] += p0.x; v[1] += p0.y; v[2] += p0.z; v[3] += p0.w;
    v[4] += p1.x; v[5] += p1.y; v[6] += p1.z; v[7] += p1.w;
  }
  if (a.bias) {
    const uint4 bw = __ldg(reinterpret_cast<const uint4*>(a.bias + n));
    const __half2* bh = reinterpret_cast<const __half2*>(&bw);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __half22float2(bh[e]);
      v[2 * e] += f.x;
      v[2 * e + 1] += f.y;
    }
  }
  if (a.relu) {
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = fmaxf(v[j], 0.f);
  }
  const int64_t e0 = int64_t(m) * a.N + n;
  if (a.R) {
    const uint4 rw = __ldg(reinterpret_cast<const uint4*>(a.R + e0));
    const __half2* rh = reinterpret_cast<const __half2*>(&rw);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __half22float2(rh[e]);
      v[2 * e] += f.x;
      v[2 * e + 1] += f.y;
    }
  }
  uint4 o;
  o.x = h2_as_u32(__floats2half2_rn(v[0], v[1]));
  o.y = h2_as_u32(__floats2half2_rn(v[2], v[3]));
  o.z = h2_as_u32(__floats2half2_rn(v[4], v[5]));
  o.w = h2_as_u32(__floats2half2_rn(v[6], v[7]));
  *reinterpret_cast<uint4*>(reinterpret_cast<__half*>(a.Y) + e0) = o;
}

// Split-K reduction + epilogue + LayerNorm of the row, for a GEMM whose output row feeds a
// LayerNorm (the out-projection's residual sum x1 -> LN2, fc2's -> the next block's LN1):
// one CTA per row reduces the partials, adds bias and residual, stores the fp16 row Y, and
// normalizes the stored fp16 values: H = fp16((y - mean) / sqrt(var + 1e-5) * g + b), fp32
// two-pass statistics, population variance (the same definition as the LayerNorm kernel).
// CPT = 8-column chunks per thread (N <= 256 * 8 * CPT).
template <int CPT>
__global__ void __launch_bounds__(256) splitk_reduce_ln_kernel(const float* __restrict__ P, int splits, int M, int N,
                                                               const __half* __restrict__ bias,
                                                               const __half* __restrict__ R, __half* __restrict__ Y,
                                                               const __half* __restrict__ g,
                                                               const __half* __restrict__ b, __half* __restrict__ H) {
  pdl_wait();  // the previous kernel in the stream has finished (see fg_launch)
  __shared__ float red[8];
  const int row = blockIdx.x;
  const int chunks = N / 8;
  const int64_t MN = int64_t(M) * N;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto block_sum = [&](float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    __syncthreads();  // earlier readers of red[] are done
    if (lane == 0) red[warp] = x;
    __syncthreads();
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) t += red[w];
    return t;
  };
  float v[CPT][8];
  float sum = 0.f;
#pragma unroll
  for (int i = 0; i < CPT; ++i) {
    const int c = threadIdx.x + i * 256;
    if (c >= chunks) continue;
    const int64_t e = int64_t(row) * N + int64_t(c) * 8;
    const float4* p0 = reinterpret_cast<const float4*>(P + e);
    float4 a = p0[0], bb = p0[1];
    float t[8] = {a.x, a.y, a.z, a.w, bb.x, bb.y, bb.z, bb.w};
    for (int sp = 1; sp < splits; ++sp) {
      const float4* ps = reinterpret_cast<const float4*>(P + sp * MN + e);
      a = ps[0];
      bb = ps[1];
      t[0] += a.x; t[1] += a.y; t[2] += a.z; t[3] += a.w; t[4] += bb.x; t[5] += bb.y; t[6] += bb.z; t[7] += bb.w;
    }
    if (bias) {
      const uint4 bw = __ldg(reinterpret_cast<const uint4*>(bias + int64_t(c) * 8));
      const __half2* bh = reinterpret_cast<const __half2*>(&bw);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = __half22float2(bh[k]);
        t[2 * k] += f.x;
        t[2 * k + 1] += f.y;
      }
    }
    if (R) {
      const uint4 rw = __ldg(reinterpret_cast<const uint4*>(R + e));
      const __half2* rh = reinterpret_cast<const __half2*>(&rw);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = __half22float2(rh[k]);
        t[2 * k] += f.x;
        t[2 * k + 1] += f.y;
      }
    }
    uint4 o;
    uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const __half2 hv = __floats2half2_rn(t[2 * k], t[2 * k + 1]);
      ow[k] = h2_as_u32(hv);
      const float2 f = __half22float2(hv);  // the stored fp16 values are what LayerNorm reads
      v[i][2 * k] = f.x;
      v[i][2 * k + 1] = f.y;
      sum += f.x + f.y;
    }
    *reinterpret_cast<uint4*>(Y + e) = o;
  }
  const float mean = block_sum(sum) / float(N);
  float sq = 0.f;
#pragma unroll
  for (int i = 0; i < CPT; ++i) {
    const int c = threadIdx.x + i * 256;
    if (c >= chunks) continue;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float d = v[i][k] - mean;
      sq = fmaf(d, d, sq);
    }
  }
  const float var = block_sum(sq) / float(N);
  const float rstd = 1.0f / sqrtf(var + 1e-5f);
#pragma unroll
  for (int i = 0; i < CPT; ++i) {
    const int c = threadIdx.x + i * 256;
    if (c >= chunks) continue;
    const uint4 gw = __ldg(reinterpret_cast<const uint4*>(g + int64_t(c) * 8));
    const uint4 bw = __ldg(reinterpret_cast<const uint4*>(b + int64_t(c) * 8));
    const __half2* gh = reinterpret_cast<const __half2*>(&gw);
    const __half2* bh = reinterpret_cast<const __half2*>(&bw);
    uint4 o;
    uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 gg = __half22float2(gh[k]), be = __half22float2(bh[k]);
      const float y0 = fmaf((v[i][2 * k] - mean) * rstd, gg.x, be.x);
      const float y1 = fmaf((v[i][2 * k + 1] - mean) * rstd, gg.y, be.y);
      ow[k] = h2_as_u32(__floats2half2_rn(y0, y1));
    }
    *reinterpret_cast<uint4*>(H + int64_t(row) * N + int64_t(c) * 8) = o;
  }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

}  // namespace

int make_map_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes, uint64_t inner,
                uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (!fn) return fail(FG_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  (void)elem_bytes;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FG_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return FG_OK;
}

namespace {

template <int MODE, bool F32>
int launch(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& p, const GemmArgs& args, cudaStream_t s) {
  using C = Cfg<MODE>;
  static std::atomic<uint64_t> attr_done{0};
  FG_TRY(ensure_smem_attr(gemm_tc_kernel<MODE, F32>, C::kSmem, attr_done));
  // a wave tail is spread over every SM (tail_fixup_kernel assumes that grid)
  const int grid = args.tail_tiles > 0 ? num_sms() : std::min(args.total, num_sms());
  FG_LAUNCH("tcgen05 gemm kernel", gemm_tc_kernel<MODE, F32>, dim3(grid), dim3(C::kThreads), size_t(C::kSmem), s, a, b, p, args);
  return FG_OK;
}

int pick_splits(int tiles, int k_blocks) {
  const int sms = num_sms();
  if (tiles >= sms / 2) return 1;
  int sp = sms / tiles;
  sp = std::min(sp, k_blocks / 2);
  return std::max(sp, 1);
}

// Tiles of a GEMM with one K-split that fill the SMs unevenly (a last, partial wave) spread
// that wave's k-blocks over every SM when the estimated time, in k-blocks per SM, drops by
// more than the fix-up's cost (taken as 16 k-blocks: the segments' fp32 write and the second
// kernel; at 8 the OPT-175B QKV shape, 1.95 waves, chose the tail and ran 2 % slower).
// Returns the number of tail tiles (0: tiles run whole, in waves).
int pick_tail(int tiles, int k_blocks, int N) {
  const int sms = num_sms();
  if (N % BN || tiles < sms / 2 || tiles % sms == 0 || tiles >= 4 * sms) return 0;
  const int tail = tiles % sms;
  const int64_t waves = int64_t((tiles + sms - 1) / sms) * k_blocks;
  const int64_t spread = int64_t(tiles / sms) * k_blocks + (int64_t(tail) * k_blocks + sms - 1) / sms;
  return spread + 16 < waves ? tail : 0;
}

}  // namespace

int splitk_reduce_launch(const float* P, int splits, int64_t M, int N, const void* bias, const void* R, int relu,
                         void* Y, cudaStream_t s) {
  const int64_t MN = M * N;
  const int grid = int(std::min<int64_t>((MN / 8 + 255) / 256, int64_t(num_sms()) * 8));
  FG_LAUNCH("split-K reduce kernel", splitk_reduce_kernel, dim3(grid), dim3(256), size_t(0), s, P, splits, MN, N, reinterpret_cast<const __half*>(bias),
                                            reinterpret_cast<const __half*>(R), relu, reinterpret_cast<__half*>(Y));
  return FG_OK;
}

// One CTA per row: reduce + epilogue + LayerNorm (see splitk_reduce_ln_kernel).
int splitk_reduce_ln_launch(const float* P, int splits, int64_t M, int N, const void* bias, const void* R, void* Y,
                            const void* g, const void* b, void* H, cudaStream_t s) {
  const int cpt = (N / 8 + 255) / 256;
  using K = void (*)(const float*, int, int, int, const __half*, const __half*, __half*, const __half*,
                     const __half*, __half*);
  static const K table[6] = {splitk_reduce_ln_kernel<1>, splitk_reduce_ln_kernel<2>, splitk_reduce_ln_kernel<3>,
                             splitk_reduce_ln_kernel<4>, splitk_reduce_ln_kernel<5>, splitk_reduce_ln_kernel<6>};
  if (cpt < 1 || cpt > 6) return fail(FG_ERR_UNSUPPORTED, "fused LayerNorm supports rows of up to 12288");
  FG_LAUNCH("split-K reduce + LayerNorm kernel", table[cpt - 1], dim3(unsigned(M)), dim3(256), size_t(0), s, P, splits,
            int(M), N, reinterpret_cast<const __half*>(bias), reinterpret_cast<const __half*>(R),
            reinterpret_cast<__half*>(Y), reinterpret_cast<const __half*>(g), reinterpret_cast<const __half*>(b),
            reinterpret_cast<__half*>(H));
  return FG_OK;
}

int read_device_error(int* out) {
  return cudaMemcpyFromSymbol(out, g_device_error, sizeof(int)) == cudaSuccess ? FG_OK : FG_ERR_CUDA;
}

// Device address of the flag, for kernels compiled in other translation units.
int* device_error_ptr() {
  static int* ptr[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
    ptr[dev] = static_cast<int*>(p);
  }
  return ptr[dev];
}

// Split-K partials of one GEMM, or the fp32 segments of its wave tail (0 when the tiles
// alone fill the GPU evenly).
size_t q4_pair_ws_bytes(int64_t M, int N, int K);

size_t splitk_ws_bytes(int64_t M, int N, int K) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  if (M > BM && M <= 2 * BM && N % BN == 0 && K % BK == 0) {
    // 4-bit weights at these batch sizes run on CTA pairs (gemm_q4pair.cu); the fp16 path
    // still runs single CTAs, so the workspace covers both plans
    const size_t q = q4_pair_ws_bytes(M, N, K);
    const int m_tiles = int((M + BM - 1) / BM), n_tiles = N / BN;
    const int sp = pick_splits(m_tiles * n_tiles, K / BK);
    size_t one = 0;
    if (sp > 1) one = size_t(sp) * size_t(M) * size_t(N) * sizeof(float);
    else if (pick_tail(m_tiles * n_tiles, K / BK, N) > 0) one = size_t(num_sms()) * 2 * BM * BN * sizeof(float);
    return std::max(q, one);
  }
  const int m_tiles = int((M + BM - 1) / BM);
  const int n_tiles = (N + BN - 1) / BN;
  const int sp = pick_splits(m_tiles * n_tiles, K / BK);
  if (sp <= 1) {
    if (pick_tail(m_tiles * n_tiles, K / BK, N) == 0) return 0;
    return size_t(num_sms()) * 2 * BM * BN * sizeof(float);
  }
  return size_t(sp) * size_t(M) * size_t(N) * sizeof(float);
}

// Workspace of a 4-bit GEMM: with M >= kExpandRows the fp16 copy of the weight, then the
// partials (both 256-byte aligned).
size_t qgemm_ws_bytes(int64_t M, int N, int K) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  size_t w = 0;
  if (M >= kExpandRows) w = (size_t(K) * size_t(N) * 2 + 255) & ~size_t(255);
  return w + splitk_ws_bytes(M, N, K);
}

int gemm_pair_launch(const void* X, int64_t M, int N, int K, const void* W, const void* bias, const void* R,
                     int relu, void* Y, cudaStream_t s);
int gemm_q4_pair_launch(const void* X, int64_t M, int N, int K, const void* w, const void* wparams, int G,
                        const void* bias, const void* R, int relu, void* Y, void* ws, size_t ws_bytes,
                        cudaStream_t s, int* splits_out, float** partial_out);

// mode: 0 = 4-bit weight W grouped along N, 1 = fp16 [K][N] weight, 2 = fp16 [N][K] weight,
// 3 = 4-bit weight grouped along K.  An fp16 [K][N] weight with many rows (the prompt pass)
// runs on CTA pairs (gemm_pair.cu), a 4-bit weight grouped along N at 129-256 rows too
// (gemm_q4pair.cu).
int gemm_impl(int mode, const void* X, int64_t M, int N, int K, const void* w, const void* wparams, int G,
              const void* bias, const void* R, int relu, void* Y, bool out_f32, void* ws, size_t ws_bytes,
              cudaStream_t s, bool w_ready, LnFuse* ln) {
  if (ln) ln->done = false;
  if (!X || !w || !Y) return fail(FG_ERR_INVALID_ARG, "null pointer");
  if (M < 0 || N <= 0 || K <= 0) return fail(FG_ERR_SHAPE, "bad GEMM shape");
  if (K % BK) return fail(FG_ERR_SHAPE, "K must be a multiple of 64");
  if (M > 0x7fffff00LL) return fail(FG_ERR_SHAPE, "M too large");
  if (mode == B_Q4 || mode == B_Q4K) {
    if (!wparams) return fail(FG_ERR_INVALID_ARG, "null params");
    if (G != 32 && G != 64 && G != 128) return fail(FG_ERR_SHAPE, "group must be 32, 64 or 128");
    if (N % BN) return fail(FG_ERR_SHAPE, "N must be a multiple of 256");
    if (mode == B_Q4 && N % (4 * G)) return fail(FG_ERR_SHAPE, "N must be a multiple of 4*group");
    if (mode == B_Q4K && K % G) return fail(FG_ERR_SHAPE, "K must be a multiple of the group (groups along K)");
  } else if (mode == B_F16_MN) {
    if (N % BN) return fail(FG_ERR_SHAPE, "N must be a multiple of 256");
  } else if (N % 8) {
    return fail(FG_ERR_SHAPE, "N must be a multiple of 8");
  }
  if (!out_f32 && N % 8) return fail(FG_ERR_SHAPE, "N must be a multiple of 8");
  if (!aligned16(X) || !aligned16(w) || !aligned16(Y) || (wparams && !aligned16(wparams)) ||
      (bias && !aligned16(bias)) || (R && !aligned16(R)))
    return fail(FG_ERR_ALIGN, "pointers must be 16-byte aligned");
  if (M == 0) return FG_OK;

  if (mode == B_Q4 && !out_f32 && M > BM && M <= 2 * BM) {
    // 129-256 rows: 256 x 256 tiles on CTA pairs, each CTA expanding half the weight tile
    const double flops = 2.0 * double(M) * N * K;
    const double bytes = double(N) * K * (0.5 + 4.0 / G) + double(M) * K * 2.0 + double(M) * N * 2.0 +
                         (R ? double(M) * N * 2.0 : 0.0);
    ProfScope ps(PROF_GEMM_DECODE, s, flops, bytes);
    int sp = 1;
    float* part = nullptr;
    FG_TRY(gemm_q4_pair_launch(X, M, N, K, w, wparams, G, bias, R, relu, Y, ws, ws_bytes, s, &sp, &part));
    if (sp > 1) {
      if (ln && ln->g && ln->b && ln->H && !relu && N % 8 == 0 && N <= 12288 && aligned16(ln->g) &&
          aligned16(ln->b) && aligned16(ln->H)) {
        FG_TRY(splitk_reduce_ln_launch(part, sp, M, N, bias, R, Y, ln->g, ln->b, ln->H, s));
        ln->done = true;
      } else {
        FG_TRY(splitk_reduce_launch(part, sp, M, N, bias, R, relu, Y, s));
      }
    }
    return FG_OK;
  }

  GemmArgs a{};
  a.M = int(M);
  a.N = N;
  a.K = K;
  a.m_tiles = int((M + BM - 1) / BM);
  a.n_tiles = (N + BN - 1) / BN;
  a.k_blocks = K / BK;
  a.splits = out_f32 ? 1 : pick_splits(a.m_tiles * a.n_tiles, a.k_blocks);
  // Rasterization: bands of row tiles whose X rows stay in L2 while every column tile of the
  // band runs; the weight is read once per band, so larger bands read it less often.  A band
  // holds at most 64 MiB of X (half the L2): 16 row tiles up to K 16384, 8 at K 28672.  On the
  // OPT-30B prompt-pass shapes (K 7168 and 28672) that ran 2.5 % faster than bands of ~16 MB,
  // and 23 % faster than 16 row tiles at K 28672 (117 MB of X).
  a.band = 16;
  while (a.band > 2 && int64_t(BM) * a.band * K * 2 > (int64_t(64) << 20)) a.band /= 2;
  a.total = a.m_tiles * a.n_tiles * a.splits;
  a.G = G;
  a.PB = G == 32 ? 8 : 4;
  a.param_bytes = mode == B_Q4 ? BK * a.PB * 4 : (mode == B_Q4K ? std::max(1, BK / G) * BN * 4 : 0);
  a.bias = reinterpret_cast<const __half*>(bias);
  a.R = reinterpret_cast<const __half*>(R);
  a.relu = relu;
  a.Y = Y;
  a.prefetch_w = w_ready ? 1 : 0;
  a.partial = nullptr;
  a.full_units = 0;
  a.tail_tiles = (a.splits == 1 && !out_f32) ? pick_tail(a.m_tiles * a.n_tiles, a.k_blocks, N) : 0;
  a.tail_part = nullptr;
  if (a.tail_tiles > 0) {
    const size_t need = size_t(num_sms()) * 2 * BM * BN * sizeof(float);
    if (!ws || ws_bytes < need) return fail(FG_ERR_WORKSPACE, "GEMM wave tail needs %zu workspace bytes", need);
    if (!aligned16(ws)) return fail(FG_ERR_ALIGN, "workspace must be 16-byte aligned");
    a.full_units = a.total - a.tail_tiles;
    a.tail_part = reinterpret_cast<float*>(ws);
  }
  if (a.splits > 1) {
    const size_t need = size_t(a.splits) * size_t(M) * size_t(N) * sizeof(float);
    if (!ws || ws_bytes < need) return fail(FG_ERR_WORKSPACE, "GEMM split-K needs %zu workspace bytes", need);
    if (!aligned16(ws)) return fail(FG_ERR_ALIGN, "workspace must be 16-byte aligned");
    a.partial = reinterpret_cast<float*>(ws);
  }

  CUtensorMap ta, tb, tp;
  memset(&tp, 0, sizeof(tp));
  FG_TRY(make_map_2d(&ta, X, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, uint64_t(K), uint64_t(M), uint64_t(K) * 2, BK, BM,
                     CU_TENSOR_MAP_SWIZZLE_128B));
  if (mode == B_Q4) {
    FG_TRY(make_map_2d(&tb, w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, uint64_t(N / 2), uint64_t(K), uint64_t(N / 2),
                       BN / 2, BK, CU_TENSOR_MAP_SWIZZLE_NONE));
    FG_TRY(make_map_2d(&tp, wparams, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, uint64_t(N / G), uint64_t(K),
                       uint64_t(N / G) * 4, uint32_t(a.PB), BK, CU_TENSOR_MAP_SWIZZLE_NONE));
  } else if (mode == B_Q4K) {
    FG_TRY(make_map_2d(&tb, w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, uint64_t(N / 2), uint64_t(K), uint64_t(N / 2),
                       BN / 2, BK, CU_TENSOR_MAP_SWIZZLE_NONE));
    FG_TRY(make_map_2d(&tp, wparams, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, uint64_t(N), uint64_t(K / G), uint64_t(N) * 4,
                       BN, uint32_t(std::max(1, BK / G)), CU_TENSOR_MAP_SWIZZLE_NONE));
  } else if (mode == B_F16_MN) {
    FG_TRY(make_map_2d(&tb, w, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, uint64_t(N), uint64_t(K), uint64_t(N) * 2, 64, BK,
                       CU_TENSOR_MAP_SWIZZLE_128B));
  } else {
    FG_TRY(make_map_2d(&tb, w, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, uint64_t(K), uint64_t(N), uint64_t(K) * 2, BK, BN,
                       CU_TENSOR_MAP_SWIZZLE_128B));
  }
  if (mode != B_Q4 && mode != B_Q4K) tp = tb;

  const double flops = 2.0 * double(M) * N * K;
  const double bytes = (mode == B_Q4 || mode == B_Q4K ? double(N) * K * (0.5 + 4.0 / G) : double(N) * K * 2.0) +
                       double(M) * K * 2.0 + double(M) * N * (out_f32 ? 4.0 : 2.0) + (R ? double(M) * N * 2.0 : 0.0);
  {
    ProfScope ps(out_f32 ? PROF_LM_HEAD : (M > 256 ? PROF_GEMM : PROF_GEMM_DECODE), s, flops, bytes);
    int st;
    if (mode == B_F16_MN && !out_f32 && a.splits == 1 && a.tail_tiles == 0 && M >= kPairRows)
      st = gemm_pair_launch(X, M, N, K, w, bias, R, relu, Y, s);   // 256 x 256 tiles on CTA pairs
    else if (mode == B_Q4) st = launch<B_Q4, false>(ta, tb, tp, a, s);
    else if (mode == B_Q4K) st = launch<B_Q4K, false>(ta, tb, tp, a, s);
    else if (mode == B_F16_MN) st = launch<B_F16_MN, false>(ta, tb, tp, a, s);
    else st = out_f32 ? launch<B_F16_K, true>(ta, tb, tp, a, s) : launch<B_F16_K, false>(ta, tb, tp, a, s);
    if (st != FG_OK) return st;
    // the split-K reduction (and a fused LayerNorm), or the wave tail's fix-up, is timed
    // with its GEMM
    if (a.tail_tiles > 0) {
      FG_LAUNCH("wave-tail fix-up kernel", tail_fixup_kernel, dim3(a.tail_tiles * (BM / 8)), dim3(256), size_t(0), s,
                a, num_sms());
    }
    if (a.splits > 1) {
      if (ln && ln->g && ln->b && ln->H && !relu && N % 8 == 0 && N <= 12288 && aligned16(ln->g) &&
          aligned16(ln->b) && aligned16(ln->H)) {
        FG_TRY(splitk_reduce_ln_launch(a.partial, a.splits, M, N, a.bias, a.R, Y, ln->g, ln->b, ln->H, s));
        ln->done = true;
      } else {
        FG_TRY(splitk_reduce_launch(a.partial, a.splits, M, N, a.bias, a.R, relu, Y, s));
      }
    }
  }
  return FG_OK;
}

}  // namespace fg
