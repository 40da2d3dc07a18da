/*
 * fg.h - C ABI of the 4-bit group-wise compressed decode path (B200, sm_100a).
 *
 * What the path computes comes from the FlexGen pages: weights and the attention (KV)
 * cache are compressed to 4 bits ("FlexGen" README mirror, key features, "Extreme
 * Compression"; arXiv 2303.06865 record, abstract), OPT-shaped models are generated with
 * input length 512 and output length 32, and throughput is generated tokens divided by
 * (prompt time + generation time) ("FlexGen" README mirror, benchmark table notes).
 * The quantizer details the pages leave open (group size/axis, rounding, layout) are
 * stated at each call below.
 *
 * Conventions for every call:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library never
 *    allocates or frees device memory (scratch comes from a caller-provided workspace).
 *  - fp16 means IEEE binary16 ("half"); half2 params are {min, scale} pairs, min first.
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL = legacy
 *    default stream), except fg_generate, which synchronizes to fill its timing record.
 *  - Arguments are validated on the host before any launch; on failure nothing is
 *    launched and a negative fg_status is returned.  fg_last_error() gives a
 *    thread-local message for the last failure.  Launch failures return FG_ERR_CUDA.
 *  - Pointers must be 16-byte aligned unless stated otherwise (FG_ERR_ALIGN).
 */
#ifndef FG_H
#define FG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FG_OK = 0,
  FG_ERR_INVALID_ARG = -1, /* null pointer, bad enum value                        */
  FG_ERR_SHAPE = -2,       /* sizes inconsistent, group does not divide the axis  */
  FG_ERR_ALIGN = -3,       /* pointer or stride not aligned as required          */
  FG_ERR_CAPACITY = -4,    /* KV cache would overflow its capacity                */
  FG_ERR_CUDA = -5,        /* a CUDA runtime/driver call or a launch failed        */
  FG_ERR_UNSUPPORTED = -6, /* valid but not implemented (e.g. head_dim > 256)     */
  FG_ERR_WORKSPACE = -7    /* workspace missing or smaller than required          */
} fg_status;

const char* fg_status_string(int status); /* static string for a status code */
const char* fg_last_error(void);           /* thread-local detail of the last error */
int fg_version(void);                      /* library version (major*10000+minor*100+patch) */

/* ------------------------------------------------------------------------------------
 * Quantize / pack (compression of a weight or KV tensor to 4 bits).
 *
 * Source: "FlexGen" README mirror, key features ("Extreme Compression": parameters and
 * attention cache down to 4 bits) and the out-of-memory tips (weight compression saves
 * about 70 % of weight memory: 4 bits + 2 fp16 per 64 elements = 71.9 %).
 * Definition (readings where the pages are silent), per group of `group` consecutive
 * elements along `axis`:
 *   mn = min, mx = max (a zero extreme is stored as +0)
 *   s  = fp16( fp32(mx - mn) / 15 )          fp32 subtract, fp32 IEEE divide, RNE to fp16
 *   code = clamp( rint( fp32(x - mn) / s ), 0, 15 )   fp32 ops, half-to-even; s==0 -> 0
 * Layout:
 *   x      fp16 [rows][cols], row-major, 16-byte aligned.
 *   codes  uint8 [rows][cols/2]: byte j of a row = code(col 2j) | code(col 2j+1) << 4.
 *   params half2 {mn, s}: axis=1 -> [rows][cols/group]; axis=0 -> [rows/group][cols].
 * group in {32, 64, 128}; axis=1 needs cols % group == 0, axis=0 needs rows % group == 0;
 * cols must be a multiple of 8.  Sizes up to 2^34 elements (64-bit indexing).
 * Non-finite inputs give unspecified codes.
 * ---------------------------------------------------------------------------------- */
int fg_quantize_pack(const void* x, int64_t rows, int64_t cols, int group, int axis,
                     uint8_t* codes, void* params, void* stream);

/* Dequantize: out = fp16(mn + code * s) with ONE rounding of the exact value.
 * Same layouts and preconditions as fg_quantize_pack; out is fp16 [rows][cols]. */
int fg_dequantize(const uint8_t* codes, const void* params, int64_t rows, int64_t cols,
                  int group, int axis, void* out, void* stream);

/* ------------------------------------------------------------------------------------
 * Model state.
 * ---------------------------------------------------------------------------------- */

/* A linear layer Y = X W + b whose weight W [K][N] (math convention, N contiguous) is
 * stored 4-bit in groups of `group` consecutive elements:
 *   group_along_k == 0: groups along N (the output channel), the default:
 *     codes uint8 [K][N/2], params half2 [K][N/group]  = fg_quantize_pack(W, K, N, group, 1)
 *   group_along_k != 0: groups along K (the input dimension, one group per column):
 *     codes uint8 [K][N/2], params half2 [K/group][N]  = fg_quantize_pack(W, K, N, group, 0)
 *     (K % group == 0).  The pages fix neither axis; the README mirror's out-of-memory tips
 *     fix only the storage, about 70 % below fp16, which both axes give.
 * bias fp16 [N] (may be NULL).
 * w16: when not NULL the layer uses this uncompressed fp16 weight [K][N] instead (codes
 * and params are then ignored and may be NULL; N % 256 == 0).  The "FlexGen" README
 * mirror's benchmark table contrasts FlexGen with and without compression; this is the
 * uncompressed side, running through the same layer and generation calls. */
typedef struct {
  const uint8_t* codes;
  const void* params;
  const void* bias;
  int K, N, group;
  const void* w16;
  int group_along_k;
} fg_qlinear;

/* One OPT decoder block (pre-LayerNorm, MHA, ReLU FFN).  qkv: [h][3h] with output
 * columns q | k | v; out: [h][h]; fc1: [h][F]; fc2: [F][h].  LayerNorm params fp16 [h]. */
typedef struct {
  const void *ln1_g, *ln1_b, *ln2_g, *ln2_b;
  fg_qlinear qkv, out, fc1, fc2;
} fg_layer;

/* 4-bit KV cache of one layer ("FlexGen" README mirror: attention cache compressed to 4
 * bits).  Each token's K (and V) row of h = n_heads*head_dim values is quantized in
 * groups of `group` along the hidden dimension (group divides head_dim):
 *   k_codes/v_codes   uint8 [B][n_heads][capacity][head_dim/2]
 *   k_params/v_params half2 [B][n_heads][capacity][head_dim/group]
 * `len` positions are filled, the same for every sequence; the calls below that append
 * advance it on success. */
typedef struct {
  uint8_t *k_codes, *v_codes;
  void *k_params, *v_params;
  int B, n_heads, head_dim, group, capacity;
  int len;
} fg_kv_cache;

typedef struct {
  int n_layers, hidden, n_heads, head_dim, ffn, vocab, max_pos, group;
  const void* embed;     /* fp16 [vocab][hidden], also the (tied) LM head      */
  const void* pos_embed; /* fp16 [max_pos][hidden] learned positions           */
  const void *lnf_g, *lnf_b;
  const fg_layer* layers; /* HOST array of n_layers layers                      */
} fg_model;

typedef struct {
  float prefill_ms, decode_ms; /* device time of the prompt pass and of the decode steps */
  int64_t tokens;              /* generated tokens (B * gen_len)                          */
  double tok_per_s;            /* tokens / (prefill + decode) seconds                     */
} fg_timing;

/* ------------------------------------------------------------------------------------
 * Steps of the path (each one launch or a few), exposed for tests and benchmarks.
 * ---------------------------------------------------------------------------------- */

/* Append n_tokens tokens per sequence to the cache at positions len..len+n_tokens-1 and
 * advance len.  k, v: fp16 rows, row (b*n_tokens + t) at k + row*row_stride (elements),
 * h valid values per row; row_stride % 8 == 0.  FG_ERR_CAPACITY if it would overflow. */
int fg_kv_append(fg_kv_cache* cache, const void* k, const void* v, int64_t row_stride,
                 int n_tokens, void* stream);

/* Dequant-fused GEMM on the tensor cores: Y[M][N] = [relu](X[M][K] W_hat + b) [+ R].
 * X fp16 [M][K] (row stride K), R fp16 [M][N] or NULL, Y fp16 [M][N].  W_hat is the
 * fg_dequantize of the weight (exact fp16; W->w16 itself when set), products accumulate
 * in fp32.  K % 64 == 0, N % 256 == 0, N % (4 * group) == 0, group in {32, 64, 128}.
 * `workspace` may be NULL when fg_qgemm_workspace_bytes(M, N, K) is 0; with M >= 1024 and
 * enough workspace the 4-bit weight is first expanded to fp16 inside it.  The workspace also
 * holds fp32 partial results when the output tiles do not fill the GPU evenly: K-split
 * partials for few tiles, or the partial tiles of the last wave when that wave is spread over
 * every SM (fg_qgemm_workspace_bytes counts them; FG_ERR_WORKSPACE if it is smaller).  From
 * 129 to 256 rows a weight grouped along N runs 256 x 256 tiles on pairs of SMs, with the
 * same kinds of partials per pair of SMs. */
size_t fg_qgemm_workspace_bytes(int64_t M, int N, int K);
int fg_qgemm(const void* X, int64_t M, const fg_qlinear* W, const void* R, int relu, void* Y,
             void* workspace, size_t ws_bytes, void* stream);

/* The same tensor-core GEMM over an uncompressed fp16 weight W [K][N] (N contiguous): the
 * "FlexGen" README mirror's benchmark table contrasts FlexGen with and without compression;
 * this is the uncompressed side.  Y[M][N] = [relu](X W + b) [+ R], fp32 accumulation.
 * K % 64 == 0, N % 256 == 0; workspace >= fg_gemm_f16_workspace_bytes(M, N, K) (fp32 partial
 * results as for fg_qgemm when the output tiles do not fill the GPU; from 1024 rows with
 * enough tiles the GEMM runs on CTA pairs and needs none). */
size_t fg_gemm_f16_workspace_bytes(int64_t M, int N, int K);
int fg_gemm_f16(const void* X, int64_t M, const void* W, int K, int N, const void* bias,
                const void* R, int relu, void* Y, void* workspace, size_t ws_bytes, void* stream);

/* Decode attention over a 4-bit cache: for each sequence b and head j,
 * out = softmax(q K^T / sqrt(hd)) V over positions 0..cache->len-1, with K and V the
 * dequantized cache values (mn + code*s) and an fp32 softmax.  q: fp16, row b at
 * q + b*q_stride (elements); out fp16 [B][h].  Split over the context with partial
 * (max, sum, acc) triples in the workspace (fg_decode_attention_workspace_bytes). */
size_t fg_decode_attention_workspace_bytes(int B, int n_heads, int head_dim, int ctx);
int fg_decode_attention(const void* q, int64_t q_stride, const fg_kv_cache* cache, void* out,
                        void* workspace, size_t ws_bytes, void* stream);

/* Decode attention that needs no device memory from the caller and allocates none itself.
 * The pages have no counterpart to this call; it exists for callers that cannot call
 * cudaMalloc: code embedded in a host program that owns every byte of device memory through
 * its own pool (a stray allocation would break its accounting), or a latency-critical decode
 * loop where an allocation and the synchronization it implies are not allowed.
 * Same arguments and results as fg_decode_attention without the workspace: the partial
 * (max, sum, acc) results of a split context go to a fixed 4 MiB array built into the library,
 * which every GPU that loads the library holds until the process exits.
 *  - A shape whose partials need more than 4 MiB (fg_decode_attention_workspace_bytes tells)
 *    is rejected with FG_ERR_WORKSPACE before any launch.
 *  - The first call on a device looks up the array's address with that device current; make
 *    that first call before any stream capture.  The address is kept for the life of the
 *    process: after cudaDeviceReset on a device, do not call this function on that device again.
 *  - All calls share the array.  Each call writes every partial it reads, so nothing carries
 *    over between calls, but calls that overlap on the GPU (other streams or threads) race. */
int fg_decode_attention_noalloc(const void* q, int64_t q_stride, const fg_kv_cache* cache,
                                void* out, void* stream);

/* Causal prefill attention on unquantized fp16 projections: qkv fp16 [B*L][3h]
 * (q | k | v), out fp16 [B*L][h].  "FlexGen" README mirror: prompt processing time is
 * part of the throughput metric.  head_dim 64 or 128 (FG_ERR_UNSUPPORTED otherwise); qkv
 * and out 16-byte aligned (FG_ERR_ALIGN); B*L below 2^31 (FG_ERR_SHAPE).  Nothing outside
 * the [B*L][3h] qkv rows is read (tiles that reach past row B*L are filled with zeros by
 * the copy engine).  Every wait inside the kernel is bounded (about 2 s);
 * one that gives up leaves the output unwritten and records a device-side error that the
 * next fg_generate reports as FG_ERR_CUDA. */
int fg_prefill_attention(const void* qkv, int B, int L, int n_heads, int head_dim, void* out,
                         void* stream);

/* LayerNorm over rows: y = (x - mean)/sqrt(var + 1e-5) * g + b, fp32 statistics (population
 * variance), fp16 in/out.  The pages benchmark OPT-6.7B/30B/175B ("FlexGen" README mirror,
 * benchmark table); the OPT block is pre-LayerNorm, which this call implements (eps 1e-5 is a
 * reading: the pages give none).  x, y fp16 [rows][cols], g, b fp16 [cols]; cols % 8 == 0 and
 * 16-byte aligned pointers (FG_ERR_SHAPE / FG_ERR_ALIGN). */
int fg_layernorm(const void* x, int64_t rows, int cols, const void* g, const void* b, void* y,
                 void* stream);

/* Token + learned position embedding of the OPT decoders the pages benchmark ("FlexGen" README
 * mirror, benchmark table): x[b*T + t] = fp16(E[ids[b*T+t]] + P[pos0 + t]) with one rounding of
 * the exact sum.  Positions start at 0 for the prompt with no offset (a reading).  ids device
 * int32 [B][T] (each in [0, vocab): not checked, the caller's contract); E fp16 [vocab][hidden],
 * P fp16 [max_pos][hidden] with pos0 + T <= max_pos; out fp16 [B*T][hidden]; hidden % 8 == 0. */
int fg_embed(const int32_t* ids, int B, int T, int pos0, const void* E, const void* P,
             int hidden, void* out, void* stream);

/* Tied LM head + greedy argmax: tokens[b] = argmax_v (x[b] . E[v]) over v < vocab, ties to
 * the lowest id.  Greedy decoding of the generated tokens the "FlexGen" README mirror's
 * benchmark counts (output length 32); the head is the fp16 embedding itself, not
 * compressed, and ties go to the lowest id (readings).  x fp16 [B][hidden] (already
 * final-LayerNormed); E fp16 [vocab][hidden]; logits fp32 [B][vocab] are written when
 * `logits` is not NULL, otherwise the workspace (fg_lm_head_workspace_bytes) holds them;
 * tokens device int32 [B].  hidden % 64 == 0 (FG_ERR_SHAPE). */
size_t fg_lm_head_workspace_bytes(int B, int vocab);
int fg_lm_head_argmax(const void* x, int B, int hidden, const void* E, int vocab, float* logits,
                      int32_t* tokens, void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------------------
 * Layers and generation.
 * ---------------------------------------------------------------------------------- */

/* One decoder block for one new token per sequence, the step the decode phase repeats
 * ("FlexGen" README mirror: generation time is part of the throughput metric; key features:
 * weights and attention cache in 4 bits): x_out = block(x_in), both fp16 [B][h]:
 *   h1 = LN1(x_in); qkv = h1 W_qkv + b; append k, v (4-bit) at cache->len; attention of q over
 *   positions 0..len (the new one included); x1 = x_in + att W_o + b_o;
 *   x_out = x1 + relu(LN2(x1) W_1 + b_1) W_2 + b_2.
 * Advances cache->len.  x_out may alias x_in.  FG_ERR_CAPACITY when the cache is full,
 * FG_ERR_SHAPE when B != cache->B or a weight's shape does not match h and ffn.
 * workspace >= fg_decode_layer_workspace_bytes(h, ffn, n_heads, B, cache->capacity). */
size_t fg_decode_layer_workspace_bytes(int hidden, int ffn, int n_heads, int B, int capacity);
int fg_decode_layer(const fg_layer* layer, fg_kv_cache* cache, const void* x_in, void* x_out,
                    int B, void* workspace, size_t ws_bytes, void* stream);

/* One decoder block over a whole prompt: x fp16 [B*L][h] in place; writes cache positions
 * 0..L-1 (cache->len must be 0) and sets len = L.
 * workspace >= fg_prefill_layer_workspace_bytes(h, ffn, B, L). */
size_t fg_prefill_layer_workspace_bytes(int hidden, int ffn, int B, int L);
int fg_prefill_layer(const fg_layer* layer, fg_kv_cache* cache, void* x, int B, int L,
                     void* workspace, size_t ws_bytes, void* stream);

/* Greedy generation ("FlexGen" README mirror, benchmark notes): prefill over the prompt
 * (B x L ids, device int32) yields token 1, then gen_len-1 decode steps; out_ids device
 * int32 [B][gen_len].  caches: HOST array of n_layers caches (len reset to 0 here),
 * capacity >= L + gen_len.  Timing uses CUDA events on `stream`; this call synchronizes.
 * The first call with a given set of pointers, sizes, stream and profiling state runs
 * eagerly, the second records the prompt pass and the decode steps as two CUDA graphs and
 * every later one replays them.
 * workspace >= fg_workspace_bytes(model, B, L, gen_len). */
size_t fg_workspace_bytes(const fg_model* model, int B, int L, int gen_len);
int fg_generate(const fg_model* model, const int32_t* prompt_ids, int B, int L, int gen_len,
                int32_t* out_ids, fg_kv_cache* caches, void* workspace, size_t ws_bytes,
                fg_timing* timing, void* stream);

/* Greedy generation with the layers' weights in pinned HOST memory ("FlexGen" README mirror:
 * weights offloaded to CPU memory under the --percent placement policy with --pin-weight,
 * and the block schedule that overlaps loading the next layer's weights with computing the
 * current one).  Same arguments and results as fg_generate, except:
 *  - model->layers[l]: every weight, bias and LayerNorm pointer is pinned host memory
 *    (cudaHostAlloc / cudaHostRegister; FG_ERR_INVALID_ARG otherwise), all layers with the same
 *    tensor sizes; embedding, positions and the final LayerNorm stay in device memory.
 *  - Schedule: layer-major over the whole batch; two weight slots in the workspace alternate.
 *    A copy stream owned by the library (one per device) fills the slot of layer visit c + 2
 *    (one cudaMemcpyAsync per tensor) as soon as the kernels of visit c are done, so each
 *    layer's weights cross the host link once per pass (prompt pass, then each decode step)
 *    while the previous layer computes.
 *  - Runs eagerly (no CUDA graphs); returns after the copy stream has drained.
 *  - h2d_bytes (may be NULL) receives the weight bytes copied host -> device.
 * workspace >= fg_offload_workspace_bytes(model, B, L, gen_len) (fg_workspace_bytes plus two
 * weight slots). */
size_t fg_offload_workspace_bytes(const fg_model* model, int B, int L, int gen_len);
int fg_generate_offload(const fg_model* model, const int32_t* prompt_ids, int B, int L, int gen_len,
                        int32_t* out_ids, fg_kv_cache* caches, void* workspace, size_t ws_bytes,
                        fg_timing* timing, double* h2d_bytes, void* stream);

/* Per-kernel device timing of the library's own launches (CUDA events on the launching
 * stream).  kind: 0 = dequant GEMM of a prompt pass (M > 256), 1 = decode attention,
 * 2 = prefill attention, 3 = quantize/append, 4 = other (LayerNorm, embedding, argmax),
 * 5 = dequant GEMM of a decode step (M <= 256), 6 = LM head GEMM.  flops and bytes are the
 * algorithmic work of the timed launches.  Enabling adds one event pair per launch (as
 * event-record nodes inside fg_generate's graphs); fg_profile_read synchronizes the
 * recorded events. */
int fg_profile_enable(int on);
/* Which kinds are timed while profiling is on: bit k selects kind k (default: all).  Timing
 * a few kinds keeps the recorded graphs close to the unprofiled ones. */
int fg_profile_select(unsigned kinds);
int fg_profile_read(int kind, double* total_ms, int64_t* launches, double* flops,
                    double* bytes);
int fg_profile_reset(void);

/* Number of kernels this library has launched in the process so far. */
int64_t fg_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* FG_H */
