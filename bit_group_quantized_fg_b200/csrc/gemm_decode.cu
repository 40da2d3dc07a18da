// K3 for decode batches (M <= 256 rows): the dequant GEMM with the expanded weight tile
// held in tensor memory.
//
//   Y[M][N] = [relu](X[M][K] * W_hat[K][N] + b) [+ R]
//
// The weight is the 128-row operand of tcgen05.mma and the rows of X are its N (swap-AB):
// D[channel][row] = sum_k W_hat[k][channel] X[row][k].  The 4-bit codes never pass through
// shared memory as fp16: the dequant warps read a 16 x 16 byte code tile transposed
// (ldmatrix .trans .b8, so each thread holds two channels x four consecutive k), expand it
// to the exact fp16 values mn + code * s, and store them with tcgen05.st straight into the
// tensor-memory A operand.  Shared memory carries only the TMA stream of codes, params and
// the X tile, which leaves its bandwidth to the tensor core's B reads.
//
// One CTA computes a 256-channel x (up to) 128-row tile over a range of k; the CTAs of a
// thread-block cluster split K, and the split is reduced inside the kernel through
// distributed shared memory (fixed order, so the result is deterministic), followed by the
// bias / ReLU / residual epilogue.  No workspace, no second kernel.
//
// Warp roles (896 threads):
//   0-7    producers: k-block j goes to warp j % 8.  Lane 0 issues the TMA copies of the X
//          tile and the code tile (128-byte rows); the 32 lanes load the tile's {mn, s} words
//          of two consecutive k each with plain loads (a 64 x 16-byte TMA box would be
//          fetched row by row) and store them regrouped as (s_k, s_k+1), (mn_k, mn_k+1)
//   8      TMEM allocation and MMA issue (8 x M128 N<=128 K16 per k-block)
//   9-11   no role in the main loop
//   12-27  dequant into TMEM, in two teams of 8 warps that take alternate k-blocks (a warp
//          expands all 64 k of its 32 channels per block); then the epilogue (TMEM -> shared
//          memory, cluster reduction)
#include <algorithm>
#include <cstring>
#include <map>
#include <mutex>
#include <cudaTypedefs.h>

#include "fg_common.cuh"
#include "sm100.cuh"

namespace fg {

int make_map_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes, uint64_t inner,
                uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz);

namespace {

using namespace sm100;

constexpr int kTileN = 256;     // weight channels per CTA: two 128-lane A tiles
constexpr int kBK = 64;         // k per block
constexpr int kMaxRows = 128;   // X rows per CTA (the MMA's N)
constexpr int kAStages = 4;     // TMEM A ring
constexpr int kMaxStages = 12;  // TMA ring
constexpr int kProdWarps = 8;
constexpr int kMmaWarp = 8;
constexpr int kDqWarp0 = 12;    // first dequant warp (a multiple of 4: warp % 4 = lane quarter)
constexpr int kDqWarps = 16;
constexpr int kThreads = (kDqWarp0 + kDqWarps) * 32;
constexpr int kCodeBytes = kBK * kTileN / 2;   // 8 KB: [64 k][128 B], 128-byte swizzle
constexpr int kPairBytes = 8 * 32 * 8;         // 2 KB: [group][32 k pairs] {s pair, mn pair}
constexpr int kAColBase = 2 * kMaxRows;        // TMEM: D0 at 0, D1 at 128, A ring from 256
constexpr int kSmemBudget = 232448 - 1024;

struct DecArgs {
  int M, N, K;
  int k_blocks, splits, rows;  // rows: the MMA N (X rows per CTA, multiple of 16)
  int G, pcols, stages, stage_bytes, x_bytes;
  const uint32_t* params;  // [K][pcols] {mn, s} words
  const __half* bias;
  const __half* R;
  int relu;
  __half* Y;
  int* err;
};

// Channel (0..31 inside a lane quarter) that TMEM lane L holds: the transposed code load
// gives thread t byte columns t/4 and 8 + t/4, whose low / high nibbles are channels 2j and
// 2j + 1, and the 16x256b store puts them in lanes t/4 and t/4 + 8 (+16 for the second).
__device__ __forceinline__ int lane_channel(int L) { return (L & 16) + 2 * (L & 7) + ((L >> 3) & 1); }

// One code register (4 consecutive k of a low-nibble and a high-nibble channel) to four
// fp16 pairs: o[0] = lo(k0, k1), o[1] = lo(k2, k3), o[2] = hi(k0, k1), o[3] = hi(k2, k3).
// Each value is mn + code * s with one rounding: the code sits in the mantissa of 1024.0
// (low nibble) or, already shifted by 4, in that of 64.0 (high nibble), the constant is
// subtracted exactly, and fma.rn.f16x2 rounds the exact product-sum once.
__device__ __forceinline__ void dequant_pairs(uint32_t w, uint32_t s01, uint32_t mn01, uint32_t s23, uint32_t mn23,
                                              uint32_t* o) {
  const uint32_t x = w & 0x0F0F0F0Fu;
  const uint32_t y = w & 0xF0F0F0F0u;
  const __half2 k1024 = u32_as_h2(0x64006400u), k64 = u32_as_h2(0x54005400u);
  const __half2 q0 = __hsub2(u32_as_h2(__byte_perm(x, 0x64646464u, 0x4140)), k1024);
  const __half2 q1 = __hsub2(u32_as_h2(__byte_perm(x, 0x64646464u, 0x4342)), k1024);
  const __half2 q2 = __hsub2(u32_as_h2(__byte_perm(y, 0x54545454u, 0x4140)), k64);
  const __half2 q3 = __hsub2(u32_as_h2(__byte_perm(y, 0x54545454u, 0x4342)), k64);
  o[0] = h2_as_u32(__hfma2(q0, u32_as_h2(s01), u32_as_h2(mn01)));
  o[1] = h2_as_u32(__hfma2(q1, u32_as_h2(s23), u32_as_h2(mn23)));
  o[2] = h2_as_u32(__hfma2(q2, u32_as_h2(s01), u32_as_h2(mn01)));
  o[3] = h2_as_u32(__hfma2(q3, u32_as_h2(s23), u32_as_h2(mn23)));
}

__global__ void __launch_bounds__(kThreads, 1)
    qgemm_dec_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_c,
                     const DecArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base_u32 = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024 - (base_u32 & 1023)) & 1023);
  const int S = a.stages;
  uint8_t* ring = smem;                                   // [S][X tile | codes]
  uint8_t* pairs = smem + S * a.stage_bytes;              // [S][kPairBytes]
  uint64_t* bars = reinterpret_cast<uint64_t*>(pairs + S * kPairBytes);
  uint64_t* full = bars;                                  // [S] TMA stage landed
  uint64_t* empty = bars + kMaxStages;                    // [S] MMA done with the stage
  uint64_t* pfull = bars + 2 * kMaxStages;                // [S] param pairs ready
  uint64_t* afull = bars + 3 * kMaxStages;                // [kAStages] A tile in TMEM
  uint64_t* aempty = afull + kAStages;                    // [kAStages] MMA done with the A tile
  uint64_t* accf = aempty + kAStages;                     // accumulators final
  uint64_t* drain = accf + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(drain + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int S_split = a.splits;
  const int rank = int(cluster_ctarank());
  const int tile = blockIdx.x / S_split;
  const int n0 = tile * kTileN;
  const int m0 = blockIdx.y * kMaxRows;
  const int kb0 = int((int64_t(rank) * a.k_blocks) / S_split);
  const int kb1 = int((int64_t(rank + 1) * a.k_blocks) / S_split);
  const int nkb = kb1 - kb0;
  const int groups = kTileN / a.G;              // param groups in the tile (2, 4 or 8)

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
      mbar_init(&pfull[i], 32);
    }
    for (int i = 0; i < kAStages; ++i) {
      mbar_init(&afull[i], kDqWarps / 2);  // one team of dequant warps per k-block
      mbar_init(&aempty[i], 1);
    }
    mbar_init(accf, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_x);
    prefetch_tmap(&tm_c);
  }
  if (warp == kMmaWarp) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < kProdWarps) {
    // ------------------------------------------------------------ producers
    const uint32_t tx = uint32_t(a.x_bytes + kCodeBytes);
    const uint32_t* prm = a.params + (n0 / a.G);
    int last_j = -1;
    for (int j = warp; j < nkb; j += kProdWarps) {
      const int s = j % S;
      const uint32_t ph = uint32_t(j / S) & 1u;
      if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, a.err, 1)) break;
      const int ky = (kb0 + j) * kBK;
      if (lane == 0) {
        uint8_t* st = ring + s * a.stage_bytes;
        mbar_expect_tx(&full[s], tx);
        tma_load_2d(st, &tm_x, ky, m0, &full[s]);
        tma_load_2d(st + a.x_bytes, &tm_c, n0 / 2, ky, &full[s]);
      }
      last_j = j;
      // rows ky + 2 lane and ky + 2 lane + 1: the k pair this lane regroups
      const uint32_t* r0 = prm + int64_t(ky + 2 * lane) * a.pcols;
      const uint32_t* r1 = r0 + a.pcols;
      uint32_t w0[8], w1[8];
      if (groups == 2) {
        const uint2 x0 = __ldg(reinterpret_cast<const uint2*>(r0)), x1 = __ldg(reinterpret_cast<const uint2*>(r1));
        w0[0] = x0.x; w0[1] = x0.y; w1[0] = x1.x; w1[1] = x1.y;
      } else {
#pragma unroll
        for (int v = 0; v < 2; ++v) {
          if (v == 0 || groups == 8) {
            const uint4 x0 = __ldg(reinterpret_cast<const uint4*>(r0) + v);
            const uint4 x1 = __ldg(reinterpret_cast<const uint4*>(r1) + v);
            w0[4 * v] = x0.x; w0[4 * v + 1] = x0.y; w0[4 * v + 2] = x0.z; w0[4 * v + 3] = x0.w;
            w1[4 * v] = x1.x; w1[4 * v + 1] = x1.y; w1[4 * v + 2] = x1.z; w1[4 * v + 3] = x1.w;
          }
        }
      }
      uint2* pp = reinterpret_cast<uint2*>(pairs + s * kPairBytes);
#pragma unroll
      for (int g = 0; g < 8; ++g)
        if (g < groups) pp[g * 32 + lane] = make_uint2(__byte_perm(w0[g], w1[g], 0x7632), __byte_perm(w0[g], w1[g], 0x5410));
      __syncwarp();
      mbar_arrive(&pfull[s]);
    }
    if (lane == 0 && *abort_flag) {
      // let the copies this warp issued land before the CTA winds down
      for (int j = warp; j <= last_j; j += kProdWarps) mbar_wait_drain(&full[j % S], uint32_t(j / S) & 1u);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_f16_f32(128, a.rows, false);
      bool ok = true;
      for (int j = 0; j < nkb && ok; ++j) {
        const int s = j % S, sa = j % kAStages;
        const uint32_t ph = uint32_t(j / S) & 1u, pha = uint32_t(j / kAStages) & 1u;
        if (!mbar_wait(&afull[sa], pha, abort_flag, a.err, 2)) { ok = false; break; }
        if (!mbar_wait(&full[s], ph, abort_flag, a.err, 4)) { ok = false; break; }
        tc_fence_after();
        const uint32_t x_addr = smem_u32(ring + s * a.stage_bytes);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint32_t a_tmem = tmem_base + uint32_t(kAColBase + sa * 64 + h * 32 + kk * 8);
            const uint64_t bd = smem_desc_sw128(x_addr + kk * 32, 16, 1024);
            mma_f16_ts(tmem_base + uint32_t(h * kMaxRows), a_tmem, bd, idesc, (j > 0 || kk > 0) ? 1u : 0u);
          }
        }
        mma_commit(&empty[s]);
        mma_commit(&aempty[sa]);
      }
      if (ok) mma_commit(accf);
      if (*abort_flag) {
        mma_commit(drain);
        mbar_wait_drain(drain, 0);
      }
    }
  } else if (warp >= kDqWarp0) {
    // ------------------------------------------------------------ dequant into TMEM
    const int d = warp - kDqWarp0;
    const int q = warp & 3;        // TMEM lane quarter (fixed by the warp id)
    const int h = (d >> 2) & 1;    // which 128-channel half of the tile
    const int team = d >> 3;       // k-blocks j with j % 2 == team
    const int cb = h * 128 + q * 32;   // first channel of this warp inside the tile
    const int g = cb / a.G;            // its param group (G >= 32)
    const int chunk = cb >> 5;         // its 16-byte column of the code rows (32 channels)
    const uint32_t lane_addr = uint32_t(q * 32) << 16;
    bool ok = true;
    for (int j = team; j < nkb && ok; j += 2) {
      const int s = j % S, sa = j % kAStages;
      const uint32_t ph = uint32_t(j / S) & 1u, pha = uint32_t(j / kAStages) & 1u;
      if (!mbar_wait(&pfull[s], ph, abort_flag, a.err, 16)) { ok = false; break; }
      if (!mbar_wait(&full[s], ph, abort_flag, a.err, 16)) { ok = false; break; }
      const uint8_t* codes = ring + s * a.stage_bytes + a.x_bytes;
      const uint4* pp = reinterpret_cast<const uint4*>(pairs + s * kPairBytes + g * 256);
      // the whole 64-k block of this warp's 32 channels: four transposed 16 x 16 loads
      uint32_t c[4][2];
      uint4 pr[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int row = 16 * i + (lane & 15);
        ldsm_16x16_trans_b8(smem_u32(codes + row * 128 + ((chunk ^ (row & 7)) << 4)), c[i][0], c[i][1]);
        // this thread's k: 16i + 4(t%4) + {0..3} -> pairs (kp, kp+1), kp = 8i + 2(t%4)
        pr[i] = pp[4 * i + (lane & 3)];
      }
      if (!mbar_wait(&aempty[sa], pha ^ 1u, abort_flag, a.err, 32)) { ok = false; break; }
      tc_fence_after();
      const uint32_t col = tmem_base + uint32_t(kAColBase + sa * 64 + h * 32);
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {  // k 0-31, then 32-63 (16 TMEM columns each)
        uint32_t lo[8], hi[8];  // [i*4 + r]: TMEM words for lanes t/4 (+8) and 16 + t/4 (+8)
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const uint4 p4 = pr[2 * hb + i];
          dequant_pairs(c[2 * hb + i][0], p4.x, p4.y, p4.z, p4.w, &lo[i * 4]);
          dequant_pairs(c[2 * hb + i][1], p4.x, p4.y, p4.z, p4.w, &hi[i * 4]);
        }
        tmem_st_16x256b_x2(col + uint32_t(16 * hb) + lane_addr, lo);
        tmem_st_16x256b_x2(col + uint32_t(16 * hb) + lane_addr + (16u << 16), hi);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[sa]);
    }
    // ------------------------------------------------------------ epilogue part 1:
    // accumulators -> shared memory, fp32 [row][256 channels] (the TMA ring is idle now)
    if (ok && nkb > 0 && mbar_wait(accf, 0, abort_flag, a.err, 64)) {
      tc_fence_after();
      float* red = reinterpret_cast<float*>(ring);
      const int ch = cb + lane_channel(lane);
      const int half_cols = a.rows / 2;
      for (int c0 = team * half_cols; c0 < (team + 1) * half_cols; c0 += 8) {
        uint32_t r[8];
        tmem_ld_32x32b_x8(tmem_base + lane_addr + uint32_t(h * kMaxRows + c0), r);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 8; ++e) red[(c0 + e) * kTileN + ch] = __uint_as_float(r[e]);
      }
    } else if (nkb == 0) {
      float* red = reinterpret_cast<float*>(ring);
      const int ch = cb + lane_channel(lane);
      for (int c = team * (a.rows / 2); c < (team + 1) * (a.rows / 2); ++c) red[c * kTileN + ch] = 0.f;
    }
  }

  // ------------------------------------------------------------ epilogue part 2:
  // the cluster's partial tiles are summed in rank order; this CTA finishes rows
  // [lo, hi) of the tile: bias, ReLU, residual, fp16 stores.
  tc_fence_before();
  cluster_sync();
  {
    const int rows_here = min(kMaxRows, a.M - m0);
    const int lo = (rank * rows_here) / S_split, hi = ((rank + 1) * rows_here) / S_split;
    const uint32_t red_local = smem_u32(ring);
    for (int item = threadIdx.x; item < (hi - lo) * (kTileN / 8); item += kThreads) {
      const int r = lo + item / (kTileN / 8);
      const int c8 = (item % (kTileN / 8)) * 8;
      float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      const uint32_t off = uint32_t((r * kTileN + c8) * 4);
      for (int p = 0; p < S_split; ++p) {
        const uint32_t ra = mapa_shared(red_local + off, uint32_t(p));
        const float4 x0 = ld_dsmem_f4(ra), x1 = ld_dsmem_f4(ra + 16);
        v[0] += x0.x; v[1] += x0.y; v[2] += x0.z; v[3] += x0.w;
        v[4] += x1.x; v[5] += x1.y; v[6] += x1.z; v[7] += x1.w;
      }
      const int n = n0 + c8;
      const int64_t m = int64_t(m0) + r;
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
        for (int e = 0; e < 8; ++e) v[e] = fmaxf(v[e], 0.f);
      }
      if (a.R) {
        const uint4 rw = __ldg(reinterpret_cast<const uint4*>(a.R + m * a.N + n));
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
      *reinterpret_cast<uint4*>(a.Y + m * a.N + n) = o;
    }
  }
  cluster_sync();  // peers may still be reading this CTA's partial tile until here
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

struct DecPlan {
  int rows, chunks, tiles, splits, stages, stage_bytes, x_bytes, smem;
};

int plan_smem(int stages, int stage_bytes) {
  return 1024 + stages * (stage_bytes + kPairBytes) + (3 * kMaxStages + 2 * kAStages + 4) * 8;
}

// Clusters of `splits` CTAs with `smem` bytes each that can be resident at once (cached per
// device: the occupancy query is a slow driver call).
int active_clusters(int splits, int smem, int grid_x, int grid_y) {
  static std::mutex mu;
  static std::map<std::pair<int, int>, int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lk(mu);
  const auto key = std::make_pair(splits, smem);
  auto it = cache[dev].find(key);
  if (it != cache[dev].end()) return it->second;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(grid_x), unsigned(grid_y));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = size_t(smem);
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = unsigned(splits);
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, qgemm_dec_kernel, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  cache[dev][key] = n;
  return n;
}

DecPlan make_plan(int64_t M, int N, int K) {
  DecPlan p{};
  p.rows = int(std::min<int64_t>(kMaxRows, (M + 15) / 16 * 16));
  p.chunks = int((M + kMaxRows - 1) / kMaxRows);
  p.tiles = (N / kTileN) * p.chunks;
  p.x_bytes = p.rows * kBK * 2;
  p.stage_bytes = p.x_bytes + kCodeBytes;
  p.stages = kMaxStages;
  while (p.stages > 2 && plan_smem(p.stages, p.stage_bytes) > kSmemBudget) --p.stages;
  p.smem = plan_smem(p.stages, p.stage_bytes);
  // Split K over a cluster of `sp` CTAs: pick the split with the least estimated time,
  // waves of resident clusters x k-blocks per CTA (at most 8 CTAs a cluster, >= 2 k-blocks each).
  const int k_blocks = K / kBK;
  int best = 1;
  double best_t = 1e30;
  for (int sp = 1; sp <= 8 && sp <= std::max(1, k_blocks / 2); ++sp) {
    const int act = active_clusters(sp, p.smem, (N / kTileN) * sp, p.chunks);
    if (act <= 0) continue;
    const int waves = (p.tiles + act - 1) / act;
    const double t = double(waves) * ((k_blocks + sp - 1) / sp) + 2.0 * sp;  // + reduction cost
    if (t < best_t) {
      best_t = t;
      best = sp;
    }
  }
  p.splits = best;
  return p;
}

}  // namespace

bool qgemm_dec_supported(int64_t M, int N, int K, int G) {
  return M > 0 && M <= 2 * kMaxRows && N % kTileN == 0 && K % kBK == 0 && (G == 32 || G == 64 || G == 128) &&
         N % (4 * G) == 0;
}

int qgemm_dec_impl(const void* X, int64_t M, int N, int K, const void* codes, const void* params, int G,
                   const void* bias, const void* R, int relu, void* Y, cudaStream_t s) {
  if (!X || !codes || !params || !Y) return fail(FG_ERR_INVALID_ARG, "null pointer");
  if (!qgemm_dec_supported(M, N, K, G)) return fail(FG_ERR_SHAPE, "unsupported decode GEMM shape");
  if (!aligned16(X) || !aligned16(codes) || !aligned16(params) || !aligned16(Y) || (bias && !aligned16(bias)) ||
      (R && !aligned16(R)))
    return fail(FG_ERR_ALIGN, "pointers must be 16-byte aligned");
  static bool attr_set[64] = {false};
  int dev = 0;
  FG_CHECK_CUDA(cudaGetDevice(&dev));
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    FG_CHECK_CUDA(cudaFuncSetAttribute(qgemm_dec_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBudget));
    attr_set[dev] = true;
  }
  const DecPlan p = make_plan(M, N, K);

  DecArgs a{};
  a.M = int(M);
  a.N = N;
  a.K = K;
  a.k_blocks = K / kBK;
  a.splits = p.splits;
  a.rows = p.rows;
  a.G = G;
  a.pcols = N / G;
  a.params = reinterpret_cast<const uint32_t*>(params);
  a.stages = p.stages;
  a.stage_bytes = p.stage_bytes;
  a.x_bytes = p.x_bytes;
  a.bias = reinterpret_cast<const __half*>(bias);
  a.R = reinterpret_cast<const __half*>(R);
  a.relu = relu;
  a.Y = reinterpret_cast<__half*>(Y);
  a.err = device_error_ptr();
  if (!a.err) return fail(FG_ERR_CUDA, "device error flag unavailable");

  CUtensorMap tx, tc;
  FG_TRY(make_map_2d(&tx, X, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, uint64_t(K), uint64_t(M), uint64_t(K) * 2, kBK,
                     uint32_t(p.rows), CU_TENSOR_MAP_SWIZZLE_128B));
  FG_TRY(make_map_2d(&tc, codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, uint64_t(N / 2), uint64_t(K), uint64_t(N / 2),
                     kTileN / 2, kBK, CU_TENSOR_MAP_SWIZZLE_128B));

  const double flops = 2.0 * double(M) * N * K;
  const double bytes = double(N) * K * (0.5 + 4.0 / G) + double(M) * K * 2.0 + double(M) * N * 2.0 +
                       (R ? double(M) * N * 2.0 : 0.0);
  ProfScope ps(PROF_GEMM_DECODE, s, flops, bytes);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned((N / kTileN) * p.splits), unsigned(p.chunks));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = size_t(p.smem);
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = unsigned(p.splits);
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  FG_CHECK_CUDA(cudaLaunchKernelEx(&cfg, qgemm_dec_kernel, tx, tc, a));
  count_launch();
  return FG_OK;
}

}  // namespace fg
