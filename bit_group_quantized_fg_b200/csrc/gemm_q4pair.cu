// K3q: the decode-step 4-bit GEMM on CTA pairs (tcgen05 cta_group::2), for batches of
// 129-256 rows.
//
//   Y[M][N] = [relu](X[M][K] * W_hat[K][N] + b) [+ R]      W_hat = mn + code * s per group
//
// The same contraction as the one-CTA 4-bit kernel (gemm.cu, B_Q4: groups of G along N),
// over 256 x 256 output tiles shared by the two CTAs of a cluster, on the two SMs of a TPC:
//   - each CTA loads its own 128 rows of X and the codes and {min, scale} pairs of its own
//     128 columns of the weight tile per 64-deep k-block,
//   - each CTA's eight expansion warps write the fp16 values of those 128 columns (the same
//     single-rounding fma(code, s, mn) as the one-CTA kernel) into its half of the B tile,
//   - the leader issues tcgen05.mma.cta_group::2 M256 N256 K16, which reads each CTA's X rows
//     and B half once and accumulates each CTA's 128 rows in its own tensor memory.
// With one CTA expanding a whole 128 x 256 tile per k-block, an SM moves ~121 KB through
// shared memory per k-block (TMA writes, code reads, the fp16 tile's writes, the MMA's operand
// reads); here each SM expands 128 columns and the MMA reads 16 + 16 KB, ~77 KB for the same
// 128 x 256 x 64 of work.  At batch <= 256 a weight column tile is one pair tile (M <= 256),
// so every weight byte is read and expanded once per launch.
//
// Scheduling is the one-CTA kernel's, with clusters in place of CTAs: whole tiles in waves
// over the clusters, and either split-K (few tiles; fp32 partials summed by the split-K
// reduction, which can fuse the next LayerNorm) or a wave tail whose k-blocks are spread
// over every cluster (fp32 partial tiles summed by tail_fixup_pair_kernel).
//
// Barriers (same offsets in both CTAs):
//   full[s]      leader: both CTAs' X tiles of stage s landed (cta_group::2 loads, armed
//                by the leader's producer with both CTAs' bytes).
//   cfull[s]     each CTA: its codes and params of stage s landed.
//   empty[s]     each CTA: the leader's commit (signalled to both) frees stage s.
//   ready[b]     leader: 16 arrivals (8 expansion warps of each CTA) say B slot b is full
//                (CTA-scope release: a cluster-scope one made the kernel 1.6x slower).
//   bempty[b]    each CTA: the leader's commit (signalled to both) frees B slot b.
//   acc_full[a]  each CTA: the leader's commit (signalled to both): accumulator a complete.
//   acc_empty[a] leader: 8 arrivals (4 epilogue warps of each CTA) free accumulator a.
//   drain        each CTA: the leader's last commit, before tensor memory is freed.
// Every wait is bounded (about 2 s); a wait that gives up records an error code for the host
// and the kernel winds down.
#include <algorithm>
#include <cstring>
#include <cudaTypedefs.h>

#include "fg_common.cuh"
#include "sm100.cuh"

namespace fg {

int make_map_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes, uint64_t inner,
                uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz);

namespace {

using namespace sm100;

constexpr int QM = 256;                                   // rows of a pair tile (128 per CTA)
constexpr int QN = 256;                                   // columns (128 expanded by each CTA)
constexpr int QK = 64;                                    // k-block
constexpr int kStages = 7;                                // TMA stages
constexpr int kBSlots = 3;                                // fp16 B half-tiles
constexpr int kXBytes = 128 * QK * 2;                     // 16 KB: this CTA's rows of X
constexpr int kCodeBytes = QK * (QN / 2) / 2;             // 4 KB: codes of its 128 columns
constexpr int kParamWords = 4;                            // {min, scale} words per k row
constexpr int kParamBytes = QK * kParamWords * 4;         // 1 KB
constexpr int kStageBytes = kXBytes + kCodeBytes + kParamBytes;
constexpr int kBHalfBytes = QK * (QN / 2) * 2;            // 16 KB: two 64-column MN blocks
constexpr int kBRingOff = kStages * kStageBytes;
constexpr int kBarOff = kBRingOff + kBSlots * kBHalfBytes;
constexpr int kThreads = 512;   // warp 0 loads, warp 1 MMA (leader), 4-7 epilogue, 8-15 expand
constexpr int kExpandWarps = 8;
constexpr int kSmem = kBarOff + 1024 /*barriers*/ + 1024 /*alignment of the base*/;
static_assert(kStageBytes % 1024 == 0 && kBRingOff % 1024 == 0, "1024-byte aligned operand tiles");
static_assert(kSmem <= 232448, "shared memory budget");

struct QArgs {
  int M, N, K;
  int n_tiles, k_blocks, splits, total;   // total = n_tiles * splits (one row tile: M <= 256)
  int G;
  const __half* bias;
  const __half* R;
  int relu;
  __half* Y;
  float* partial;   // [splits][M][N] when splits > 1
  // wave tail (splits == 1): tiles [0, full_units) run whole, a cluster at a time; the
  // k-blocks of the remaining tail_tiles are divided evenly over all clusters (cluster b
  // takes [I b / C, I (b + 1) / C) of I = tail_tiles * k_blocks, at most two tiles); those
  // segments go to tail_part[b][segment][QM][QN] in fp32
  int full_units, tail_tiles;
  float* tail_part;
};

struct QCoord {
  int n0, kb0, kb1, ks;
  int seg;   // tail segment of this cluster (0 or 1), -1 for a whole tile or a split-K slice
};

__device__ __forceinline__ QCoord q_tile(const QArgs& a, int t) {
  QCoord c;
  c.ks = t % a.splits;
  c.n0 = (t / a.splits) * QN;
  c.kb0 = int((int64_t(c.ks) * a.k_blocks) / a.splits);
  c.kb1 = int((int64_t(c.ks + 1) * a.k_blocks) / a.splits);
  c.seg = -1;
  return c;
}

__host__ __device__ __forceinline__ int64_t q_tail_start(int64_t I, int b, int clusters) {
  return I * b / clusters;
}

// Work units of cluster b of C, in the order every role of both CTAs walks them.
__device__ __forceinline__ int q_unit_count(const QArgs& a, int b, int C) {
  if (a.tail_tiles == 0) return b < a.total ? (a.total - 1 - b) / C + 1 : 0;
  const int64_t I = int64_t(a.tail_tiles) * a.k_blocks;
  const int64_t s0 = q_tail_start(I, b, C), s1 = q_tail_start(I, b + 1, C);
  int n = a.full_units / C;
  if (s1 > s0) n += (s0 / a.k_blocks == (s1 - 1) / a.k_blocks) ? 1 : 2;
  return n;
}

__device__ __forceinline__ QCoord q_unit(const QArgs& a, int b, int C, int u) {
  const int nf = a.tail_tiles == 0 ? 0x7fffffff : a.full_units / C;
  if (u < nf) return q_tile(a, b + u * C);
  const int64_t I = int64_t(a.tail_tiles) * a.k_blocks;
  const int64_t s0 = q_tail_start(I, b, C), s1 = q_tail_start(I, b + 1, C);
  const int seg = u - nf;
  const int tile0 = int(s0 / a.k_blocks);
  const int tile = tile0 + seg;
  QCoord c = q_tile(a, a.full_units + tile);
  c.kb0 = seg == 0 ? int(s0 - int64_t(tile0) * a.k_blocks) : 0;
  c.kb1 = int(min(int64_t(a.k_blocks), s1 - int64_t(tile) * a.k_blocks));
  c.seg = seg;
  return c;
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_q4_pair_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_c,
                        const __grid_constant__ CUtensorMap tm_p, const QArgs args, int* err) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base_u32 = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024 - (base_u32 & 1023)) & 1023);
  uint8_t* bring = smem + kBRingOff;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOff);
  uint64_t* full = bars;                                   // [kStages] (leader)
  uint64_t* cfull = bars + kStages;                        // [kStages]
  uint64_t* empty = bars + 2 * kStages;                    // [kStages]
  uint64_t* ready = bars + 3 * kStages;                    // [kBSlots] (leader)
  uint64_t* bempty = bars + 3 * kStages + kBSlots;         // [kBSlots]
  uint64_t* acc_full = bars + 3 * kStages + 2 * kBSlots;   // [2]
  uint64_t* acc_empty = acc_full + 2;                      // [2] (leader)
  uint64_t* drain = acc_full + 4;                          // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(acc_full + 6);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster = blockIdx.x >> 1;
  const int n_clusters = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&cfull[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < kBSlots; ++i) {
      mbar_init(&ready[i], 2 * kExpandWarps);
      mbar_init(&bempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 8);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_x);
    prefetch_tmap(&tm_c);
    prefetch_tmap(&tm_p);
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, 2 * QN);
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers are initialized before any cross-CTA arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();      // X comes from the previous kernel, which may also still read the workspace

  const int n_units = q_unit_count(args, cluster, n_clusters);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      const uint32_t full_leader = mapa_shared(smem_u32(full), 0);
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int u = 0; u < n_units && ok; ++u) {
        const QCoord c = q_unit(args, cluster, n_clusters, u);
        const int nh = c.n0 + (QN / 2) * int(rank);           // this CTA's first column
        const int px = (nh / args.G) & ~(kParamWords - 1);    // 16-byte aligned param box
        for (int kb = c.kb0; kb < c.kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, err, 0x10000)) { ok = false; break; }
          uint8_t* st = smem + stage * kStageBytes;
          if (leader) mbar_expect_tx(&full[stage], 2 * kXBytes);
          mbar_expect_tx(&cfull[stage], kCodeBytes + kParamBytes);
          tma_load_2d_pair(st, &tm_x, kb * QK, 128 * int(rank), full_leader + uint32_t(stage) * 8u);
          tma_load_2d(st + kXBytes, &tm_c, nh / 2, kb * QK, &cfull[stage]);
          tma_load_2d(st + kXBytes + kCodeBytes, &tm_p, px, kb * QK, &cfull[stage]);
          ++issued;
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
      }
      if (*abort_flag) {
        // let this CTA's own copies land before it exits (the last kStages can be in flight)
        for (int q = max(0, issued - kStages); q < issued; ++q)
          mbar_wait_drain(&cfull[q % kStages], uint32_t(q / kStages) & 1u);
        if (leader)
          for (int q = max(0, issued - kStages); q < issued; ++q)
            mbar_wait_drain(&full[q % kStages], uint32_t(q / kStages) & 1u);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (lane == 0 && leader) {
      constexpr uint32_t idesc = idesc_f16_f32(QM, QN, true);
      int stage = 0, bs = 0;
      uint32_t phase = 0, bphase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int u = 0; u < n_units && ok; ++u) {
        const QCoord c = q_unit(args, cluster, n_clusters, u);
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1, abort_flag, err, 0x20000)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + uint32_t(acc * QN);
        for (int kb = c.kb0; kb < c.kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, err, 0x40000)) { ok = false; break; }
          if (!mbar_wait(&ready[bs], bphase, abort_flag, err, 0x80000)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * kStageBytes);
          const uint32_t b_addr = smem_u32(bring + bs * kBHalfBytes);
          // the k-th 16-deep slice: +32 bytes along K for X (K-major), +2048 bytes (two
          // 8-row groups) for the MN-major B half; descriptor addresses count 16-byte units
          const uint64_t ad0 = smem_desc_sw128(a_addr, 16, 1024);
          const uint64_t bd0 = smem_desc_sw128(b_addr, 8192, 1024);
#pragma unroll
          for (int k = 0; k < QK / 16; ++k)
            mma_f16_ss_pair(d_tmem, ad0 + uint64_t(2 * k), bd0 + uint64_t(128 * k), idesc,
                            (kb > c.kb0 || k > 0) ? 1u : 0u);
          mma_commit_pair(&empty[stage], 0x3);
          mma_commit_pair(&bempty[bs], 0x3);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
          if (++bs == kBSlots) { bs = 0; bphase ^= 1; }
        }
        if (!ok) break;
        mma_commit_pair(&acc_full[acc], 0x3);
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
      // every MMA issued above has completed once this arrives (in both CTAs)
      mma_commit_pair(drain, 0x3);
    }
    if (lane == 0) mbar_wait_drain(drain, 0);
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp - 4;  // TMEM lane quarter
    const uint32_t acc_empty_leader = mapa_shared(smem_u32(acc_empty), 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int u = 0; u < n_units; ++u) {
      const QCoord c = q_unit(args, cluster, n_clusters, u);
      if (!mbar_wait(&acc_full[acc], acc_phase, abort_flag, err, 0x100000)) break;
      tc_fence_after();
      const int row = 128 * int(rank) + q * 32 + lane;   // row of the pair tile = row of Y
      const bool row_ok = row < args.M;
      for (int cc = 0; cc < QN; cc += 32) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem_base + (uint32_t(q * 32) << 16) + uint32_t(acc * QN + cc), r);
        tmem_ld_wait();
        {
          // the expansion warps stored each 8 columns in the order [0,4,1,5,2,6,3,7]:
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
        if (!row_ok) continue;
        if (c.seg >= 0 || args.partial != nullptr) {
          float4* dst = c.seg >= 0
                            ? reinterpret_cast<float4*>(args.tail_part +
                                                        ((int64_t(cluster) * 2 + c.seg) * QM + row) * QN + cc)
                            : reinterpret_cast<float4*>(args.partial + (int64_t(c.ks) * args.M + row) * args.N + n);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            dst[j] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                 __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
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
          const uint4* rp = reinterpret_cast<const uint4*>(args.R + int64_t(row) * args.N + n);
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
        uint4* dst = reinterpret_cast<uint4*>(args.Y + int64_t(row) * args.N + n);
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
      if (lane == 0) mbar_arrive_cluster(acc_empty_leader + uint32_t(acc) * 8u);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ expansion warps (both CTAs)
    // warp e expands k rows 8e .. 8e+7 of each block, two rows per pass: lanes 0-15 take row
    // 8e + 2j and lanes 16-31 row 8e + 2j + 1, one code word (8 columns) per lane
    const int e = warp - 8;
    const int hi = lane >> 4;
    const int word = lane & 15;
    const int nb = word >> 3;      // 64-column MN block of the word
    const int ch = word & 7;       // 16-byte chunk inside the block
    const uint32_t ready_leader = mapa_shared(smem_u32(ready), 0);
    int stage = 0, bs = 0;
    uint32_t phase = 0, bphase = 0;
    bool ok = true;
    for (int u = 0; u < n_units && ok; ++u) {
      const QCoord c = q_unit(args, cluster, n_clusters, u);
      const int nh = c.n0 + (QN / 2) * int(rank);
      const int pcol = ((nh / args.G) & (kParamWords - 1)) + (word * 8) / args.G;
      for (int kb = c.kb0; kb < c.kb1; ++kb) {
        if (!mbar_wait(&cfull[stage], phase, abort_flag, err, 0x200000)) { ok = false; break; }
        const uint8_t* st = smem + stage * kStageBytes;
        const uint32_t* codes = reinterpret_cast<const uint32_t*>(st + kXBytes);
        const uint32_t* prm = reinterpret_cast<const uint32_t*>(st + kXBytes + kCodeBytes);
        uint32_t w[4], p[4], o[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int row = 8 * e + 2 * j + hi;
          w[j] = codes[row * (QN / 16) + word];
          p[j] = prm[row * kParamWords + pcol];
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const __half2 pr = u32_as_h2(p[j]);
          dequant8_interleaved(w[j], __high2half2(pr), __low2half2(pr), o[j]);
        }
        // the B slot this block fills was read by the MMAs of the block kBSlots back
        if (!mbar_wait(&bempty[bs], bphase ^ 1, abort_flag, err, 0x400000)) { ok = false; break; }
        uint8_t* bt = bring + bs * kBHalfBytes;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int rr = 2 * j + hi;   // row inside the 8-row group e
          uint4* dst = reinterpret_cast<uint4*>(bt + nb * 8192 + e * 1024 + rr * 128 + ((ch ^ rr) << 4));
          *dst = make_uint4(o[j][0], o[j][1], o[j][2], o[j][3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(ready_leader + uint32_t(bs) * 8u);
        if (++stage == kStages) { stage = 0; phase ^= 1; }
        if (++bs == kBSlots) { bs = 0; bphase ^= 1; }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // neither CTA frees tensor memory or exits while the pair still works
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 2 * QN);
  }
}

// Wave tail of the pair GEMM: each tail tile's segments summed in cluster order, then
// Y = [relu](sum + b) [+ R].  A block covers 8 rows of one tile (32 threads x 8 columns per
// row); grid = tail_tiles * QM / 8.
__global__ void __launch_bounds__(256) tail_fixup_pair_kernel(const QArgs a, int clusters) {
  pdl_wait();  // the GEMM's partial tiles are complete (see fg_launch)
  const int tau = blockIdx.x / (QM / 8);
  const int row = (blockIdx.x % (QM / 8)) * 8 + (threadIdx.x >> 5);
  const int col = (threadIdx.x & 31) * 8;
  const QCoord c = q_tile(a, a.full_units + tau);
  const int m = row, n = c.n0 + col;
  if (m >= a.M || n >= a.N) return;
  const int64_t kb = a.k_blocks, I = int64_t(a.tail_tiles) * kb;
  const int64_t x0 = int64_t(tau) * kb, x1 = x0 + kb;
  // first cluster whose range reaches past x0
  int g = int(x0 * clusters / I);
  while (g + 1 < clusters && q_tail_start(I, g + 1, clusters) <= x0) ++g;
  while (g > 0 && q_tail_start(I, g, clusters) > x0) --g;
  float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (; g < clusters; ++g) {
    const int64_t s0 = q_tail_start(I, g, clusters), s1 = q_tail_start(I, g + 1, clusters);
    if (s0 >= x1) break;
    if (s1 <= s0 || s1 <= x0) continue;
    const int seg = s0 >= x0 ? 0 : 1;  // tau is this cluster's first tail tile, or its second
    const float4* p = reinterpret_cast<const float4*>(a.tail_part + ((int64_t(g) * 2 + seg) * QM + row) * QN + col);
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
  *reinterpret_cast<uint4*>(a.Y + e0) = o;
}

// Plan of a pair GEMM: K-splits and wave tail over `clusters` pairs (the one-CTA kernel's
// rules, with clusters in place of SMs).
void q_plan(int tiles, int k_blocks, int clusters, int& splits, int& tail) {
  splits = 1;
  tail = 0;
  if (tiles < clusters / 2) {
    splits = std::max(1, std::min(clusters / tiles, k_blocks / 2));
    return;
  }
  if (tiles % clusters == 0 || tiles >= 4 * clusters) return;
  const int t = tiles % clusters;
  const int64_t waves = int64_t((tiles + clusters - 1) / clusters) * k_blocks;
  const int64_t spread = int64_t(tiles / clusters) * k_blocks + (int64_t(t) * k_blocks + clusters - 1) / clusters;
  if (spread + 16 < waves) tail = t;
}

}  // namespace

// Workspace of a pair GEMM of M rows (128 < M <= 256): fp32 split-K partials or the wave
// tail's partial tiles, 0 when the tiles fill the pairs evenly.
size_t q4_pair_ws_bytes(int64_t M, int N, int K) {
  const int clusters = num_sms() / 2;
  int splits = 1, tail = 0;
  q_plan(N / QN, K / QK, clusters, splits, tail);
  if (splits > 1) return size_t(splits) * size_t(M) * size_t(N) * sizeof(float);
  if (tail > 0) return size_t(clusters) * 2 * QM * QN * sizeof(float);
  return 0;
}

// Y = [relu](X W_hat + b) [+ R] on CTA pairs for a 4-bit weight grouped along N; 128 < M <=
// 256, N % 256 == 0, N % (4 G) == 0, K % 64 == 0, pointers 16-byte aligned (checked by the
// caller).  With a K-split the fp32 partials are left in the workspace for the caller's
// reduction: *splits_out > 1 and *partial_out points at them.
int gemm_q4_pair_launch(const void* X, int64_t M, int N, int K, const void* w, const void* wparams, int G,
                        const void* bias, const void* R, int relu, void* Y, void* ws, size_t ws_bytes,
                        cudaStream_t s, int* splits_out, float** partial_out) {
  int* err = device_error_ptr();
  if (!err) return fail(FG_ERR_CUDA, "device error flag unavailable");
  const int clusters = num_sms() / 2;
  QArgs a{};
  a.M = int(M);
  a.N = N;
  a.K = K;
  a.n_tiles = N / QN;
  a.k_blocks = K / QK;
  q_plan(a.n_tiles, a.k_blocks, clusters, a.splits, a.tail_tiles);
  a.total = a.n_tiles * a.splits;
  a.G = G;
  a.bias = reinterpret_cast<const __half*>(bias);
  a.R = reinterpret_cast<const __half*>(R);
  a.relu = relu;
  a.Y = reinterpret_cast<__half*>(Y);
  a.partial = nullptr;
  a.tail_part = nullptr;
  a.full_units = 0;
  const size_t need = q4_pair_ws_bytes(M, N, K);
  if (need > 0) {
    if (!ws || ws_bytes < need) return fail(FG_ERR_WORKSPACE, "pair GEMM needs %zu workspace bytes", need);
    if (!aligned16(ws)) return fail(FG_ERR_ALIGN, "workspace must be 16-byte aligned");
  }
  if (a.splits > 1) {
    a.partial = reinterpret_cast<float*>(ws);
  } else if (a.tail_tiles > 0) {
    a.full_units = a.total - a.tail_tiles;
    a.tail_part = reinterpret_cast<float*>(ws);
  }
  *splits_out = a.splits;
  *partial_out = a.partial;

  CUtensorMap tx, tc, tp;
  FG_TRY(make_map_2d(&tx, X, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, uint64_t(K), uint64_t(M), uint64_t(K) * 2, QK, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B));
  FG_TRY(make_map_2d(&tc, w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, uint64_t(N / 2), uint64_t(K), uint64_t(N / 2),
                     QN / 4, QK, CU_TENSOR_MAP_SWIZZLE_NONE));
  FG_TRY(make_map_2d(&tp, wparams, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, uint64_t(N / G), uint64_t(K),
                     uint64_t(N / G) * 4, kParamWords, QK, CU_TENSOR_MAP_SWIZZLE_NONE));
  static std::atomic<uint64_t> attr_done{0};
  FG_TRY(ensure_smem_attr(gemm_q4_pair_kernel, kSmem, attr_done));
  // a wave tail is spread over every cluster (tail_fixup_pair_kernel assumes that grid)
  const int grid_clusters = a.tail_tiles > 0 ? clusters : std::min(a.total, clusters);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * grid_clusters);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = s;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  count_launch();
  const cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_q4_pair_kernel, tx, tc, tp, a, err);
  if (e != cudaSuccess) return cuda_fail(e, "tcgen05 4-bit pair gemm kernel");
  if (a.tail_tiles > 0) {
    FG_LAUNCH("pair wave-tail fix-up kernel", tail_fixup_pair_kernel, dim3(a.tail_tiles * (QM / 8)), dim3(256),
              size_t(0), s, a, clusters);
  }
  return FG_OK;
}

}  // namespace fg
