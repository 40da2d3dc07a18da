// GPU twin of fg_synth's seeded input generator (see fg_synth/__init__.py for the
// definition).  Same counter-based SplitMix64 bits, same exact integer sums and the same
// IEEE-rounded float64 steps (explicit __dmul_rn/__dadd_rn/__ddiv_rn/__dsqrt_rn so that no
// FMA contraction changes a bit), one cvt.rn.f16.f64 rounding at the end.  It holds no
// arithmetic of the compression method or the decoder.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr uint64_t GAMMA = 0x9E3779B97F4A7C15ull;
constexpr uint64_t DELTA = 0xD1B54A32D192ED03ull;
constexpr uint64_t OUTLIER_TAG = 0x5A5Aull;

__host__ __device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}
__host__ __device__ __forceinline__ uint64_t key_of(uint64_t seed, uint64_t stream) {
  return mix64(seed * GAMMA + stream * DELTA);
}
__device__ __forceinline__ uint64_t bits_at(uint64_t key, uint64_t i) { return mix64(key + (i + 1) * GAMMA); }

__device__ __forceinline__ double normal_z(uint64_t key, uint64_t i) {
  int64_t s = 0;
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    const uint64_t b = bits_at(key, i * 3 + c);
#pragma unroll
    for (int f = 0; f < 4; ++f) s += int64_t((b >> (16 * f)) & 0xFFFF);
  }
  return __dmul_rn(double(s - 393210), 1.0 / 65536.0);  // exact
}

__device__ __forceinline__ __half to_half(double v) {
  unsigned short h;
  asm("cvt.rn.f16.f64 %0, %1;" : "=h"(h) : "d"(v));
  return __ushort_as_half(h);
}

__global__ void gen_kernel(uint64_t key, uint64_t okey, int dist, double scale, int64_t cols, int64_t offset,
                           int64_t n, __half* __restrict__ out) {
  for (int64_t j = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; j < n; j += int64_t(gridDim.x) * blockDim.x) {
    const uint64_t i = uint64_t(offset + j);
    double v;
    if (dist == 0) {
      v = __dmul_rn(normal_z(key, i), scale);
    } else if (dist == 1) {
      const double u = __dmul_rn(double(bits_at(key, i) >> 11), 1.0 / 9007199254740992.0);
      v = __dadd_rn(-scale, __dmul_rn(2.0 * scale, u));
    } else if (dist == 2) {
      const double z0 = normal_z(key, 4 * i), z1 = normal_z(key, 4 * i + 1);
      const double z2 = normal_z(key, 4 * i + 2), z3 = normal_z(key, 4 * i + 3);
      double chi = __dadd_rn(__dmul_rn(z1, z1), __dmul_rn(z2, z2));
      chi = __dadd_rn(chi, __dmul_rn(z3, z3));
      const double den = __dsqrt_rn(__ddiv_rn(chi, 3.0));
      v = chi == 0.0 ? 0.0 : __ddiv_rn(z0, den);
      v = fmin(fmax(__dmul_rn(v, scale), -65504.0), 65504.0);
    } else {
      const uint64_t col = i % uint64_t(cols);
      const uint64_t tag = bits_at(okey, col) >> 40;
      const double mult = (tag % 100 == 0) ? 50.0 : 1.0;
      v = __dmul_rn(__dmul_rn(normal_z(key, i), mult), scale);
    }
    out[j] = to_half(v);
  }
}

__global__ void ids_kernel(uint64_t key, int64_t n, uint32_t vocab, int32_t* __restrict__ out) {
  for (int64_t j = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; j < n; j += int64_t(gridDim.x) * blockDim.x)
    out[j] = int32_t((bits_at(key, uint64_t(j)) >> 32) % vocab);
}

}  // namespace

extern "C" {

// Fill out[0..n) (fp16, device) with elements offset..offset+n-1 of tensor (seed, stream).
// dist: 0 normal(scale), 1 uniform(-scale, scale), 2 t3 * scale, 3 outlier columns (cols).
int fgsynth_fill(uint64_t seed, uint64_t stream, int dist, double scale, int64_t cols, int64_t offset, int64_t n,
                 void* out, void* cuda_stream) {
  if (n <= 0) return 0;
  if (dist == 3 && cols <= 0) return -1;
  const uint64_t key = key_of(seed, stream);
  const uint64_t okey = key_of(seed, stream ^ OUTLIER_TAG);
  const int64_t blocks = (n + 255) / 256;
  const int grid = int(blocks < 148 * 32 ? blocks : 148 * 32);
  gen_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(cuda_stream)>>>(key, okey, dist, scale,
                                                                            cols > 0 ? cols : 1, offset, n,
                                                                            reinterpret_cast<__half*>(out));
  return cudaGetLastError() == cudaSuccess ? 0 : -2;
}

int fgsynth_ids(uint64_t seed, uint64_t stream, int64_t n, int vocab, void* out, void* cuda_stream) {
  if (n <= 0) return 0;
  if (vocab <= 0) return -1;
  const int64_t blocks = (n + 255) / 256;
  const int grid = int(blocks < 148 * 32 ? blocks : 148 * 32);
  ids_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(cuda_stream)>>>(key_of(seed, stream), n, uint32_t(vocab),
                                                                            reinterpret_cast<int32_t*>(out));
  return cudaGetLastError() == cudaSuccess ? 0 : -2;
}

}  // extern "C"
