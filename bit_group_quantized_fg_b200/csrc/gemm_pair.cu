// K3p: the prompt-pass GEMM on CTA pairs (tcgen05 cta_group::2).
//
//   Y[M][N] = [relu](X[M][K] * W[K][N] + b) [+ R]      X, W fp16, fp32 accumulation, Y fp16
//
// In the prompt pass every 4-bit weight has just been expanded to its fp16 values W_hat
// (the same values fg_dequantize writes), so this is a plain fp16 contraction of
// M = B * L rows ("FlexGen" README mirror, benchmark notes: prompt processing time is part
// of the throughput metric).  One output tile is 256 x 256; the two CTAs of a cluster, on
// the two SMs of one TPC, share it:
//   - each CTA stages its own 128 rows of X and its own 128 columns of W per 64-deep k-block
//     (32 KB per stage instead of the 48 KB one SM would need for a 128 x 256 tile alone),
//   - the leader (rank 0) issues tcgen05.mma.cta_group::2 M256 N256 K16, which reads both
//     CTAs' shared memory and accumulates each CTA's 128 rows in its own tensor memory,
//   - each CTA's epilogue warps read their 128 rows, apply bias / ReLU / residual, and write
//     each 32 x 32 fp16 box through shared memory with one TMA store (about 1 % faster at the
//     OPT-30B prompt shapes than 16-byte stores from registers, under the same power cap).
// Per SM, every MMA of 128 x 256 x 16 now reads 8 KB of shared memory instead of 12 KB.
//
// Scheduling: one cluster per tile, two CTAs per SM (3 stages of 32 KB, one 256-column
// accumulator each), so one pair's epilogue runs while another pair's k-loop keeps the tensor
// pipe busy, and the hardware hands out tiles in raster order as pairs finish.  A persistent
// grid (74 pairs walking fixed tile sequences) measured 94-96 % tensor-pipe activity but read
// ~5x the DRAM bytes its band order needs (the pairs' positions in the raster drift apart) and
// ran ~30 % below this launch's SM clock under the power cap; it was slower than the one-CTA
// kernel.  With one cluster per tile the OPT-30B prompt-pass projections take 133 ms instead
// of 149-151 for the one-CTA kernel on the same box, at 84 % tensor-pipe activity.
//
// Barriers (same offsets in both CTAs):
//   full[s]      leader only: the leader's producer arms it with both CTAs' bytes; each
//                CTA's tile loads count their bytes on it (cta_group::2 loads).
//   empty[s]     each CTA: the leader's commit (signalled to both CTAs) frees stage s.
//   acc_full[a]  each CTA: the leader's commit (signalled to both) says accumulator a is complete.
//   acc_empty[a] leader only: 8 arrivals (4 epilogue warps of each CTA) free accumulator a.
//   drain        each CTA: the leader's last commit (signalled to both), before TMEM is freed.
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

constexpr int PM = 256;        // rows of a pair tile (128 per CTA)
constexpr int PN = 256;        // columns of a pair tile (128 staged by each CTA)
constexpr int PK = 64;         // k-block
constexpr int kStages = 3;
constexpr int kAccs = 1;       // accumulators per CTA (one tile per cluster)
constexpr int kABytes = 128 * PK * 2;         // 16 KB: this CTA's rows of X
constexpr int kBBytes = PK * (PN / 2) * 2;    // 16 KB: this CTA's columns of W (two 64-column blocks)
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kThreads = 256;  // warp 0 loads, warp 1 MMA (leader) / drain, warps 4-7 epilogue
constexpr int kStageOut = 4 * 32 * 32 * 2;  // one 32 x 32 fp16 output box per epilogue warp
// stages, barriers (padded to 1 KB so the output boxes stay 1 KB aligned), output boxes, and
// the alignment slack of the dynamic shared-memory base
constexpr int kSmem = kStages * kStageBytes + 1024 + kStageOut + 1024;
static_assert(kSmem <= 232448, "shared memory budget");

struct PairArgs {
  int M, N, K;
  int m_tiles, n_tiles, k_blocks, total;
  int band;   // pair tiles (of 256 rows) per rasterization band
  const __half* bias;
  const __half* R;
  int relu;
  __half* Y;
};

__device__ __forceinline__ void pair_tile(const PairArgs& a, int t, int& m0, int& n0) {
  const int band_tiles = a.band * a.n_tiles;
  const int bi = t / band_tiles;
  const int rr = t - bi * band_tiles;
  const int mt_in_band = min(a.band, a.m_tiles - bi * a.band);
  const int n = rr / mt_in_band;
  const int m = bi * a.band + (rr - n * mt_in_band);
  m0 = m * PM;
  n0 = n * PN;
}

__global__ void __launch_bounds__(kThreads, 2)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_y, const PairArgs args, int* err) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base_u32 = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024 - (base_u32 & 1023)) & 1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint8_t* out_box = smem + kStages * kStageBytes + 1024;
  uint64_t* full = bars;                         // [kStages] (leader)
  uint64_t* empty = bars + kStages;              // [kStages]
  uint64_t* acc_full = bars + 2 * kStages;       // [2]
  uint64_t* acc_empty = bars + 2 * kStages + 2;  // [2] (leader)
  uint64_t* drain = bars + 2 * kStages + 4;      // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * kStages + 6);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster = blockIdx.x >> 1;
  const int n_clusters = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
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
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, kAccs * PN);
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers are initialized before any cross-CTA arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();      // X (and W, just expanded) come from earlier kernels in the stream

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      const uint32_t full_leader = mapa_shared(smem_u32(full), 0);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = cluster; t < args.total && ok; t += n_clusters) {
        int m0, n0;
        pair_tile(args, t, m0, n0);
        for (int kb = 0; kb < args.k_blocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, err, 0x100)) { ok = false; break; }
          if (leader) mbar_expect_tx(&full[stage], 2 * kStageBytes);
          uint8_t* st = smem + stage * kStageBytes;
          const uint32_t fb = full_leader + uint32_t(stage) * 8u;
          tma_load_2d_pair(st, &tm_a, kb * PK, m0 + 128 * int(rank), fb);
          const int nb = n0 + (PN / 2) * int(rank);
          tma_load_2d_pair(st + kABytes, &tm_b, nb, kb * PK, fb);
          tma_load_2d_pair(st + kABytes + 8192, &tm_b, nb + 64, kb * PK, fb);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (lane == 0 && leader) {
      constexpr uint32_t idesc = idesc_f16_f32(PM, PN, true);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = cluster; t < args.total && ok; t += n_clusters) {
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1, abort_flag, err, 0x200)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + uint32_t(acc * PN);
        for (int kb = 0; kb < args.k_blocks; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, err, 0x400)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * kStageBytes);
          const uint32_t b_addr = a_addr + kABytes;
#pragma unroll
          for (int k = 0; k < PK / 16; ++k) {
            const uint64_t ad = smem_desc_sw128(a_addr + k * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(b_addr + k * 2048, 8192, 1024);
            mma_f16_ss_pair(d_tmem, ad, bd, idesc, (kb > 0 || k > 0) ? 1u : 0u);
          }
          mma_commit_pair(&empty[stage], 0x3);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        mma_commit_pair(&acc_full[acc], 0x3);
        if (++acc == kAccs) { acc = 0; acc_phase ^= 1; }
      }
      // every MMA issued above has completed once this arrives (in both CTAs)
      mma_commit_pair(drain, 0x3);
    }
    if (lane == 0) mbar_wait_drain(drain, 0);
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp - 4;  // TMEM lane quarter
    const uint32_t acc_empty_leader = mapa_shared(smem_u32(acc_empty), 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = cluster; t < args.total; t += n_clusters) {
      int m0, n0;
      pair_tile(args, t, m0, n0);
      if (!mbar_wait(&acc_full[acc], acc_phase, abort_flag, err, 0x800)) break;
      tc_fence_after();
      const int m = m0 + 128 * int(rank) + q * 32 + lane;
      const bool row_ok = m < args.M;
      for (int cc = 0; cc < PN; cc += 32) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem_base + (uint32_t(q * 32) << 16) + uint32_t(acc * PN + cc), r);
        tmem_ld_wait();
        const int n = n0 + cc;
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
        if (args.R != nullptr && row_ok) {
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
        // the warp's 32 x 32 box goes out through shared memory as one TMA store (the tensor
        // map clips rows past M).  Lane l holds row l; with the 64-byte swizzle its four 16-byte
        // pieces land in distinct banks for every 8 consecutive lanes.
        uint8_t* box = out_box + q * 2048;
        if (lane == 0) bulk_wait_read0();  // this warp's previous box has left shared memory
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint4 o;
          o.x = h2_as_u32(__floats2half2_rn(v[8 * j + 0], v[8 * j + 1]));
          o.y = h2_as_u32(__floats2half2_rn(v[8 * j + 2], v[8 * j + 3]));
          o.z = h2_as_u32(__floats2half2_rn(v[8 * j + 4], v[8 * j + 5]));
          o.w = h2_as_u32(__floats2half2_rn(v[8 * j + 6], v[8 * j + 7]));
          *reinterpret_cast<uint4*>(box + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4)) = o;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && m < args.M) {
          tma_store_2d(&tm_y, n, m, box);
          bulk_commit();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty_leader + uint32_t(acc) * 8u);
      if (++acc == kAccs) { acc = 0; acc_phase ^= 1; }
    }
    if (lane == 0) bulk_wait0();  // every box written before the CTA exits
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // neither CTA frees tensor memory or exits while the pair still works
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kAccs * PN);
  }
}

}  // namespace

// Y = [relu](X W + b) [+ R] on CTA pairs for fp16 W [K][N]; M rows (any), N % 256 == 0,
// K % 64 == 0, pointers 16-byte aligned (checked by the caller).
int gemm_pair_launch(const void* X, int64_t M, int N, int K, const void* W, const void* bias, const void* R,
                     int relu, void* Y, cudaStream_t s) {
  int* err = device_error_ptr();
  if (!err) return fail(FG_ERR_CUDA, "device error flag unavailable");
  PairArgs a{};
  a.M = int(M);
  a.N = N;
  a.K = K;
  a.m_tiles = int((M + PM - 1) / PM);
  a.n_tiles = N / PN;
  a.k_blocks = K / PK;
  a.total = a.m_tiles * a.n_tiles;
  // tiles in raster order: bands of 8 pair tiles (2048 rows of X) walk every column tile
  // (bands of 16 measured 6-7 % slower at K 7168)
  a.band = 8;
  a.bias = reinterpret_cast<const __half*>(bias);
  a.R = reinterpret_cast<const __half*>(R);
  a.relu = relu;
  a.Y = reinterpret_cast<__half*>(Y);
  CUtensorMap ta, tb, ty;
  FG_TRY(make_map_2d(&ta, X, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, uint64_t(K), uint64_t(M), uint64_t(K) * 2, PK, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B));
  FG_TRY(make_map_2d(&tb, W, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, uint64_t(N), uint64_t(K), uint64_t(N) * 2, 64, PK,
                     CU_TENSOR_MAP_SWIZZLE_128B));
  FG_TRY(make_map_2d(&ty, Y, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, uint64_t(N), uint64_t(M), uint64_t(N) * 2, 32, 32,
                     CU_TENSOR_MAP_SWIZZLE_64B));
  static std::atomic<uint64_t> attr_done{0};
  FG_TRY(ensure_smem_attr(gemm_pair_kernel, kSmem, attr_done));
  const int clusters = a.total;   // one cluster per tile (see the header)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters);
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
  const cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_pair_kernel, ta, tb, ty, a, err);
  if (e != cudaSuccess) return cuda_fail(e, "tcgen05 pair gemm kernel");
  return FG_OK;
}

}  // namespace fg
