// Shared host/device helpers of the fg library (status handling, fp16 bit helpers,
// 4-bit code expansion).  Nothing here allocates device memory.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

#include <atomic>

#include "../../include/fg.h"

namespace fg {

// ------------------------------------------------------------------ host-side errors
void set_error(const char* fmt, ...);
int fail(int status, const char* fmt, ...);
int cuda_fail(cudaError_t e, const char* what);

#define FG_CHECK_CUDA(expr)                               \
  do {                                                    \
    cudaError_t _e = (expr);                              \
    if (_e != cudaSuccess) return ::fg::cuda_fail(_e, #expr); \
  } while (0)

void count_launch();

#define FG_CHECK_LAUNCH(what)                               \
  do {                                                      \
    ::fg::count_launch();                                   \
    cudaError_t _e = cudaGetLastError();                    \
    if (_e != cudaSuccess) return ::fg::cuda_fail(_e, what); \
  } while (0)

#define FG_TRY(expr)                 \
  do {                               \
    int _s = (expr);                 \
    if (_s != FG_OK) return _s;      \
  } while (0)

// Every kernel of the library is launched with programmatic stream serialization: a kernel
// may start (prologue, loads of data no earlier kernel writes) while the previous kernel
// in the stream finishes, and waits in pdl_wait() before it touches that kernel's results
// or writes memory the previous kernel may still read.  Every kernel calls pdl_wait(), so
// completion stays ordered along the stream.
template <typename... KArgs, typename... Args>
inline cudaError_t fg_launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                             Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

#define FG_LAUNCH(what, ...)                                  \
  do {                                                        \
    ::fg::count_launch();                                     \
    cudaError_t _e = ::fg::fg_launch(__VA_ARGS__);            \
    if (_e != cudaSuccess) return ::fg::cuda_fail(_e, what);  \
  } while (0)

// Waits until the previous kernel in the stream has completed and its writes are visible
// (no-op for a kernel launched without programmatic serialization).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

int num_sms();

// Raises a kernel's dynamic shared-memory limit once per device: the attribute belongs to
// the device's context, so a process that drives several GPUs sets it on each of them.
// `done` holds one bit per device ordinal (0..63).
template <typename Kernel>
int ensure_smem_attr(Kernel kernel, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  FG_CHECK_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(FG_ERR_UNSUPPORTED, "device ordinal %d above 63", dev);
  const uint64_t bit = uint64_t(1) << dev;
  if (done.load(std::memory_order_acquire) & bit) return FG_OK;
  FG_CHECK_CUDA(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  done.fetch_or(bit, std::memory_order_acq_rel);
  return FG_OK;
}

// Row count from which a 4-bit GEMM expands its weight to fp16 once and runs the plain
// fp16 tensor-core GEMM (measured break-even ~700 rows on B200).
constexpr int64_t kExpandRows = 1024;

// Row count from which an fp16 [K][N] GEMM runs 256 x 256 tiles on CTA pairs
// (tcgen05 cta_group::2) instead of 128 x 256 tiles on single CTAs.
constexpr int64_t kPairRows = 1024;

// Device address of the flag that bounded device-side waits set when they give up.
int* device_error_ptr();

// A LayerNorm of a GEMM's output rows to fuse into its split-K reduction when there is one
// (H = LN(Y) with gamma g, beta b); `done` reports whether it was fused.
struct LnFuse {
  const void* g;
  const void* b;
  void* H;
  bool done;
};

int splitk_reduce_launch(const float* P, int splits, int64_t M, int N, const void* bias, const void* R, int relu,
                         void* Y, cudaStream_t s);

// Kernel classes for fg_profile_* (same numbering as the header).
enum ProfKind { PROF_GEMM = 0, PROF_DECODE_ATTN = 1, PROF_PREFILL_ATTN = 2, PROF_QUANT = 3,
                PROF_OTHER = 4, PROF_GEMM_DECODE = 5, PROF_LM_HEAD = 6, PROF_NKINDS = 7 };
// RAII pair of events around a launch when profiling is on.
struct ProfScope {
  int slot;
  cudaStream_t s;
  ProfScope(int kind, cudaStream_t s, double flops, double bytes);
  ~ProfScope();
};

// ------------------------------------------------------------------ device helpers
__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// Eight 4-bit codes of one 32-bit word (element i in bits 4i..4i+3) expanded to the
// exact fp16 values mn + code*s, one rounding each (fma.rn.f16x2 rounds the exact
// a*b+c once).  (1024 + code) is built by OR-ing the code into the mantissa of 1024.0
// (0x6400) and 1024 is then subtracted exactly.  Output pairs in element order:
// out[j] = {x[2j], x[2j+1]}.
__device__ __forceinline__ void dequant8(uint32_t w, __half2 s2, __half2 mn2, uint32_t out[4]) {
  const uint32_t MAGIC = 0x64006400u;  // {1024.0, 1024.0}
  const __half2 K1024 = u32_as_h2(MAGIC);
  // even elements of bytes 0..3 at nibble positions 0,2,4,6 ; odd at 1,3,5,7
  // pair j = {elem 2j, elem 2j+1} = {nibble 2j, nibble 2j+1} of w.
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t byte = (w >> (8 * j)) & 0xFFu;
    uint32_t lohi = (byte & 0x0Fu) | ((byte & 0xF0u) << 12);  // lo -> bits 0..3, hi -> 16..19
    __half2 h = u32_as_h2(lohi | MAGIC);
    __half2 q = __hsub2(h, K1024);
    out[j] = h2_as_u32(__hfma2(q, s2, mn2));
  }
}

// Same values as dequant8 but in the column order [0,4,1,5,2,6,3,7]: out[j] = {x[j], x[j+4]}.
// Each pair is one AND-OR of the word (or of the word shifted by 4j) with the 1024.0 magic,
// about half the instructions of the natural order; consumers that can permute columns
// for free (a GEMM epilogue indexing registers at compile time) use this form.
__device__ __forceinline__ void dequant8_interleaved(uint32_t w, __half2 s2, __half2 mn2, uint32_t out[4]) {
  const uint32_t MAGIC = 0x64006400u;
  const __half2 K1024 = u32_as_h2(MAGIC);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t pair = ((w >> (4 * j)) & 0x000F000Fu) | MAGIC;  // {1024 + c_j, 1024 + c_{j+4}}
    const __half2 q = __hsub2(u32_as_h2(pair), K1024);
    out[j] = h2_as_u32(__hfma2(q, s2, mn2));
  }
}

// dequant8_interleaved with a {min, scale} of its own for each output pair: pair j holds
// columns j and j + 4 of the word (weights grouped along K have one pair per column).
__device__ __forceinline__ void dequant8_interleaved_pairs(uint32_t w, const __half2 (&s2)[4], const __half2 (&mn2)[4],
                                                           uint32_t out[4]) {
  const uint32_t MAGIC = 0x64006400u;
  const __half2 K1024 = u32_as_h2(MAGIC);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t pair = ((w >> (4 * j)) & 0x000F000Fu) | MAGIC;
    const __half2 q = __hsub2(u32_as_h2(pair), K1024);
    out[j] = h2_as_u32(__hfma2(q, s2[j], mn2[j]));
  }
}

}  // namespace fg
