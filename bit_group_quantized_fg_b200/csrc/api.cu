// C ABI of the library (include/fg.h): argument checks, workspace carving, per-kernel
// profiling, and the decoder-layer / generation orchestration over the kernels.
//
// Generation follows the "FlexGen" README mirror's benchmark notes: a prompt pass over
// input length L yields the first token, then gen_len-1 decode steps; throughput =
// generated tokens / (prompt time + generation time), both measured with CUDA events.
#include <atomic>
#include <cstdarg>
#include <cstring>
#include <mutex>
#include <vector>

#include "fg_common.cuh"

namespace fg {

// implemented in the kernel files
int quantize_pack_impl(const void*, int64_t, int64_t, int, int, uint8_t*, void*, cudaStream_t);
int dequantize_impl(const uint8_t*, const void*, int64_t, int64_t, int, int, void*, cudaStream_t);
int kv_append_impl(fg_kv_cache*, const void*, const void*, int64_t, int, cudaStream_t);
size_t decode_attention_ws_bytes(int, int, int, int);
int decode_attention_impl(const void*, int64_t, const fg_kv_cache*, void*, void*, size_t, cudaStream_t,
                          const void* = nullptr, const void* = nullptr, int64_t = 0, fg_kv_cache* = nullptr);
int prefill_attention_impl(const void*, int, int, int, int, void*, cudaStream_t);
int layernorm_impl(const void*, int64_t, int, const void*, const void*, void*, cudaStream_t);
int embed_impl(const int32_t*, int64_t, int, int, int, const void*, const void*, int, void*, cudaStream_t);
int argmax_impl(const float*, int, int, int32_t*, int64_t, cudaStream_t);
size_t qgemm_ws_bytes(int64_t, int, int);
size_t splitk_ws_bytes(int64_t, int, int);
int gemm_impl(int, const void*, int64_t, int, int, const void*, const void*, int, const void*, const void*, int,
              void*, bool, void*, size_t, cudaStream_t, bool, LnFuse* = nullptr);
int read_device_error(int*);

// ---------------------------------------------------------------- errors
static thread_local char g_err[512] = "";

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
}

int fail(int status, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return status;
}

int cuda_fail(cudaError_t e, const char* what) {
  snprintf(g_err, sizeof(g_err), "%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
  return FG_ERR_CUDA;
}

int num_sms() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    cached[dev] = v;
  }
  return cached[dev];
}

// ---------------------------------------------------------------- launch counter
static std::atomic<int64_t> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

// ---------------------------------------------------------------- profiling
namespace {
struct ProfRec {
  int kind;
  cudaEvent_t a, b;
  double flops, bytes;
};
// Events are recorded as graph nodes while the stream is being captured, so that a profiled
// generation still replays its CUDA graphs.
void record_event(cudaEvent_t e, cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(e, s, cudaEventRecordExternal);
  else
    cudaEventRecord(e, s);
}
std::mutex g_prof_mu;
constexpr uint32_t kAllKinds = (1u << PROF_NKINDS) - 1;
bool g_prof_on = false;
uint32_t g_prof_sel = kAllKinds;  // kinds timed while profiling is on
uint32_t g_prof_mask = 0;         // g_prof_on ? g_prof_sel : 0
std::vector<ProfRec> g_prof_pending;
double g_prof_ms[PROF_NKINDS] = {0};
int64_t g_prof_n[PROF_NKINDS] = {0};
double g_prof_flops[PROF_NKINDS] = {0};
double g_prof_bytes[PROF_NKINDS] = {0};
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t take_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

void add_record(const ProfRec& r) {
  float ms = 0.f;
  if (cudaEventSynchronize(r.b) == cudaSuccess && cudaEventElapsedTime(&ms, r.a, r.b) == cudaSuccess) {
    g_prof_ms[r.kind] += ms;
    g_prof_n[r.kind] += 1;
    g_prof_flops[r.kind] += r.flops;
    g_prof_bytes[r.kind] += r.bytes;
  }
}
void collect_locked() {
  for (auto& r : g_prof_pending) {
    add_record(r);
    g_event_pool.push_back(r.a);
    g_event_pool.push_back(r.b);
  }
  g_prof_pending.clear();
}
}  // namespace

ProfScope::ProfScope(int kind, cudaStream_t st, double flops, double bytes) : slot(-1), s(st) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (!((g_prof_mask >> kind) & 1u)) return;
  ProfRec r{kind, take_event(), take_event(), flops, bytes};
  record_event(r.a, s);
  g_prof_pending.push_back(r);
  slot = int(g_prof_pending.size()) - 1;
}

ProfScope::~ProfScope() {
  if (slot < 0) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (slot < int(g_prof_pending.size())) record_event(g_prof_pending[slot].b, s);
}

// ---------------------------------------------------------------- workspace carving
namespace {
struct Carver {
  uint8_t* p;
  size_t used = 0, cap;
  Carver(void* base, size_t c) : p(reinterpret_cast<uint8_t*>(base)), cap(c) {}
  void* take(size_t bytes) {
    used = (used + 255) & ~size_t(255);
    void* r = p ? p + used : nullptr;
    used += bytes;
    return r;
  }
  bool ok() const { return used <= cap; }
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int check_qlinear(const fg_qlinear& w, int K, int N, const char* name) {
  if (!w.w16 && (!w.codes || !w.params)) return fail(FG_ERR_INVALID_ARG, "%s: null weight", name);
  if (w.K != K || w.N != N) return fail(FG_ERR_SHAPE, "%s: weight is %dx%d, expected %dx%d", name, w.K, w.N, K, N);
  return FG_OK;
}

int check_layer(const fg_layer* L, int h, int* ffn) {
  if (!L) return fail(FG_ERR_INVALID_ARG, "null layer");
  if (!L->ln1_g || !L->ln1_b || !L->ln2_g || !L->ln2_b) return fail(FG_ERR_INVALID_ARG, "null LayerNorm params");
  const int F = L->fc1.N;
  FG_TRY(check_qlinear(L->qkv, h, 3 * h, "qkv"));
  FG_TRY(check_qlinear(L->out, h, h, "out"));
  FG_TRY(check_qlinear(L->fc1, h, F, "fc1"));
  FG_TRY(check_qlinear(L->fc2, F, h, "fc2"));
  *ffn = F;
  return FG_OK;
}

// Y = [relu](X W_hat + b) [+ R] for a 4-bit weight.  With many rows (a prompt pass) each
// weight tile is reused by M/128 row tiles, so the weight is first expanded once into an
// fp16 copy in the workspace (an HBM-bound pass, ~1 % of the GEMM) and the tensor-core GEMM
// then runs without dequant warps; with fewer rows (decode batches included) the fused kernel
// expands each weight tile into shared memory as it streams the 4-bit weight once.  Both
// compute with the same fp16 values W_hat.
// w_ready: the weight was not written by the kernel just before this one in the stream
// (true inside the layer calls, whose first kernel is a LayerNorm), so its tiles may be
// requested before the previous kernel finishes.
// ln: a LayerNorm of Y's rows to fuse into the GEMM's split-K reduction (decode batches);
// ln->done tells the caller whether it still has to run it.
int qlinear_run(const void* X, int64_t M, const fg_qlinear& w, const void* R, int relu, void* Y, void* ws,
                size_t wsb, cudaStream_t s, bool w_ready = false, LnFuse* ln = nullptr) {
  if (ln) ln->done = false;
  if (w.w16)  // uncompressed weight: the fp16 GEMM over it directly
    return gemm_impl(1, X, M, w.N, w.K, w.w16, nullptr, 0, w.bias, R, relu, Y, false, ws, wsb, s, w_ready, ln);
  const size_t wbytes = (size_t(w.K) * size_t(w.N) * 2 + 255) & ~size_t(255);
  const int axis = w.group_along_k ? 0 : 1;
  if (M >= kExpandRows && ws != nullptr && wsb >= wbytes && aligned16(ws)) {
    FG_TRY(dequantize_impl(w.codes, w.params, w.K, w.N, w.group, axis, ws, s));
    return gemm_impl(1, X, M, w.N, w.K, ws, nullptr, 0, w.bias, R, relu, Y, false,
                     reinterpret_cast<uint8_t*>(ws) + wbytes, wsb - wbytes, s, false);  // weight just written
  }
  return gemm_impl(w.group_along_k ? 3 : 0, X, M, w.N, w.K, w.codes, w.params, w.group, w.bias, R, relu, Y, false, ws,
                   wsb, s, w_ready, ln);
}

size_t gemm_ws_for_layer(int64_t M, int h, int F) {
  size_t m = qgemm_ws_bytes(M, 3 * h, h);
  m = std::max(m, qgemm_ws_bytes(M, h, h));
  m = std::max(m, qgemm_ws_bytes(M, F, h));
  m = std::max(m, qgemm_ws_bytes(M, h, F));
  return m;
}

size_t decode_ws(int h, int F, int nh, int B, int cap) {
  size_t t = 0;
  t += align256(size_t(B) * h * 2) * 4;        // h1, att, x1, h2
  t += align256(size_t(B) * 3 * h * 2);        // qkv
  t += align256(size_t(B) * F * 2);            // f
  t += align256(gemm_ws_for_layer(B, h, F));   // split-K partials
  t += align256(decode_attention_ws_bytes(B, nh, h / nh, cap));
  return t + 256;
}

size_t prefill_ws(int h, int F, int B, int L) {
  const size_t BL = size_t(B) * L;
  size_t t = 0;
  t += align256(BL * h * 2) * 3;     // h1/h2, att, x1
  t += align256(BL * 3 * h * 2);     // qkv
  t += align256(BL * F * 2);         // f
  t += align256(gemm_ws_for_layer(int64_t(BL), h, F));
  return t + 256;
}
}  // namespace

// h1_in: LN1(x_in) already computed (fused into the previous block's fc2 reduction), or NULL.
// next: the LayerNorm that follows this block (the next block's LN1, or the final LN) to fuse
// into fc2's split-K reduction; next->done reports whether it was.
int decode_layer_impl(const fg_layer* layer, fg_kv_cache* cache, const void* x_in, void* x_out, int B, void* ws,
                      size_t ws_bytes, cudaStream_t s, const void* h1_in = nullptr, LnFuse* next = nullptr) {
  if (!cache || !x_in || !x_out) return fail(FG_ERR_INVALID_ARG, "null pointer");
  if (B <= 0 || B != cache->B) return fail(FG_ERR_SHAPE, "B must equal the cache batch");
  const int h = cache->n_heads * cache->head_dim;
  int F = 0;
  FG_TRY(check_layer(layer, h, &F));
  if (cache->len + 1 > cache->capacity) return fail(FG_ERR_CAPACITY, "KV cache full (capacity %d)", cache->capacity);
  const size_t need = decode_ws(h, F, cache->n_heads, B, cache->capacity);
  if (!ws || ws_bytes < need) return fail(FG_ERR_WORKSPACE, "decode layer needs %zu workspace bytes", need);
  Carver c(ws, ws_bytes);
  void* h1 = c.take(size_t(B) * h * 2);
  void* att = c.take(size_t(B) * h * 2);
  void* x1 = c.take(size_t(B) * h * 2);
  void* h2 = c.take(size_t(B) * h * 2);
  void* qkv = c.take(size_t(B) * 3 * h * 2);
  void* f = c.take(size_t(B) * F * 2);
  const size_t gws_b = gemm_ws_for_layer(B, h, F);
  void* gws = c.take(gws_b);
  const size_t aws_b = decode_attention_ws_bytes(B, cache->n_heads, cache->head_dim, cache->capacity);
  void* aws = c.take(aws_b);
  auto* qkvh = reinterpret_cast<__half*>(qkv);

  if (h1_in) h1 = const_cast<void*>(h1_in);
  else FG_TRY(layernorm_impl(x_in, B, h, layer->ln1_g, layer->ln1_b, h1, s));
  FG_TRY(qlinear_run(h1, B, layer->qkv, nullptr, 0, qkv, gws, gws_b, s, true));
  // the step's K/V append runs inside the attention kernel (the last-chunk CTA of each head)
  FG_TRY(decode_attention_impl(qkv, 3 * int64_t(h), cache, att, aws, aws_b, s, qkvh + h, qkvh + 2 * h,
                               3 * int64_t(h), cache));
  LnFuse ln2{layer->ln2_g, layer->ln2_b, h2, false};   // LN2 in the out-projection's reduction
  FG_TRY(qlinear_run(att, B, layer->out, x_in, 0, x1, gws, gws_b, s, true, &ln2));
  if (!ln2.done) FG_TRY(layernorm_impl(x1, B, h, layer->ln2_g, layer->ln2_b, h2, s));
  FG_TRY(qlinear_run(h2, B, layer->fc1, nullptr, 1, f, gws, gws_b, s, true));
  FG_TRY(qlinear_run(f, B, layer->fc2, x1, 0, x_out, gws, gws_b, s, true, next));
  return FG_OK;
}

int prefill_layer_impl(const fg_layer* layer, fg_kv_cache* cache, void* x, int B, int L, void* ws, size_t ws_bytes,
                       cudaStream_t s) {
  if (!cache || !x) return fail(FG_ERR_INVALID_ARG, "null pointer");
  if (B <= 0 || L <= 0 || B != cache->B) return fail(FG_ERR_SHAPE, "B must equal the cache batch and L > 0");
  if (cache->len != 0) return fail(FG_ERR_INVALID_ARG, "prefill needs an empty cache (len 0)");
  if (L > cache->capacity) return fail(FG_ERR_CAPACITY, "prompt longer than the cache capacity");
  const int h = cache->n_heads * cache->head_dim;
  int F = 0;
  FG_TRY(check_layer(layer, h, &F));
  const size_t need = prefill_ws(h, F, B, L);
  if (!ws || ws_bytes < need) return fail(FG_ERR_WORKSPACE, "prefill layer needs %zu workspace bytes", need);
  const int64_t BL = int64_t(B) * L;
  Carver c(ws, ws_bytes);
  void* hn = c.take(size_t(BL) * h * 2);
  void* att = c.take(size_t(BL) * h * 2);
  void* x1 = c.take(size_t(BL) * h * 2);
  void* qkv = c.take(size_t(BL) * 3 * h * 2);
  void* f = c.take(size_t(BL) * F * 2);
  const size_t gws_b = gemm_ws_for_layer(BL, h, F);
  void* gws = c.take(gws_b);
  auto* qkvh = reinterpret_cast<__half*>(qkv);

  FG_TRY(layernorm_impl(x, BL, h, layer->ln1_g, layer->ln1_b, hn, s));
  FG_TRY(qlinear_run(hn, BL, layer->qkv, nullptr, 0, qkv, gws, gws_b, s, true));
  FG_TRY(kv_append_impl(cache, qkvh + h, qkvh + 2 * h, 3 * int64_t(h), L, s));
  FG_TRY(prefill_attention_impl(qkv, B, L, cache->n_heads, cache->head_dim, att, s));
  FG_TRY(qlinear_run(att, BL, layer->out, x, 0, x1, gws, gws_b, s, true));
  FG_TRY(layernorm_impl(x1, BL, h, layer->ln2_g, layer->ln2_b, hn, s));
  FG_TRY(qlinear_run(hn, BL, layer->fc1, nullptr, 1, f, gws, gws_b, s, true));
  FG_TRY(qlinear_run(f, BL, layer->fc2, x1, 0, x, gws, gws_b, s, true));
  return FG_OK;
}

namespace {
size_t lm_ws(int B, int V) { return align256(size_t(B) * V * 4) + 256; }

int lm_head_impl(const void* x, int B, int hidden, const void* E, int V, float* logits, int32_t* tokens,
                 int64_t tok_stride, void* ws, size_t wsb, cudaStream_t s, bool w_ready = false) {
  if (!x || !E || !tokens) return fail(FG_ERR_INVALID_ARG, "null pointer");
  if (B <= 0 || V <= 0 || hidden <= 0 || hidden % 64) return fail(FG_ERR_SHAPE, "bad LM head shape");
  float* lg = logits;
  if (!lg) {
    if (!ws || wsb < lm_ws(B, V)) return fail(FG_ERR_WORKSPACE, "LM head needs %zu workspace bytes", lm_ws(B, V));
    lg = reinterpret_cast<float*>(ws);
  }
  if (!aligned16(lg)) return fail(FG_ERR_ALIGN, "logits must be 16-byte aligned");
  FG_TRY(gemm_impl(2, x, B, V, hidden, E, nullptr, 0, nullptr, nullptr, 0, lg, true, nullptr, 0, s, w_ready));
  return argmax_impl(lg, B, V, tokens, tok_stride, s);
}

size_t generate_ws(const fg_model* m, int B, int L, int T) {
  const int h = m->hidden, F = m->ffn;
  size_t t = 0;
  t += align256(size_t(B) * L * h * 2);                 // x (prompt hidden states)
  t += align256(size_t(B) * h * 2) * 3;                 // decode x, final LN out, next block's LN1
  size_t layer = std::max(prefill_ws(h, F, B, L), decode_ws(h, F, m->n_heads, B, L + T));
  t += align256(layer);
  t += lm_ws(B, m->vocab);
  return t + 256;
}
}  // namespace

// ---------------------------------------------------------------- CUDA graphs for generate
// A generation is ~12k short launches (31 decode steps x 32 layers x ~10 kernels); issuing
// them one by one makes the decode steps host-bound.  The first call with a configuration
// runs eagerly (and loads every kernel); the second records the prompt pass and the decode
// steps as two graphs on a private capture stream; later calls with the same configuration
// replay them.  The key covers every pointer and size the launches bake in.
namespace {
struct GraphKey {
  std::vector<uint8_t> bytes;
  bool operator==(const GraphKey& o) const { return bytes == o.bytes; }
};
template <class T>
void put(std::vector<uint8_t>& v, const T& x) {
  const uint8_t* p = reinterpret_cast<const uint8_t*>(&x);
  v.insert(v.end(), p, p + sizeof(T));
}
GraphKey make_key(const fg_model* m, const int32_t* ids, int B, int L, int T, int32_t* out,
                  const fg_kv_cache* caches, void* ws, size_t wsb, cudaStream_t s, uint32_t prof) {
  GraphKey k;
  int dev = -1;
  cudaGetDevice(&dev);
  put(k.bytes, dev);
  put(k.bytes, *m);
  for (int l = 0; l < m->n_layers; ++l) put(k.bytes, m->layers[l]);
  for (int l = 0; l < m->n_layers; ++l) {
    fg_kv_cache c = caches[l];
    c.len = 0;
    put(k.bytes, c);
  }
  put(k.bytes, ids);
  put(k.bytes, B);
  put(k.bytes, L);
  put(k.bytes, T);
  put(k.bytes, out);
  put(k.bytes, ws);
  put(k.bytes, wsb);
  put(k.bytes, s);
  put(k.bytes, prof);
  return k;
}
struct GraphCache {
  GraphKey key;
  bool seen = false, valid = false;
  cudaGraphExec_t prefill = nullptr, decode = nullptr;
  int64_t n_prefill = 0, n_decode = 0;
  cudaStream_t cap[64] = {nullptr};  // capture stream of each device (created on first use there)
  // timing events the graphs record (captured while profiling was on)
  std::vector<ProfRec> prof_prefill, prof_decode;
};
std::mutex g_graph_mu;
GraphCache g_graph;

uint32_t profiling_mask() {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  return g_prof_mask;
}

void reset_graphs() {
  if (g_graph.prefill) cudaGraphExecDestroy(g_graph.prefill);
  if (g_graph.decode) cudaGraphExecDestroy(g_graph.decode);
  g_graph.prefill = g_graph.decode = nullptr;
  g_graph.valid = g_graph.seen = false;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto* v : {&g_graph.prof_prefill, &g_graph.prof_decode}) {
    for (auto& r : *v) {
      g_event_pool.push_back(r.a);
      g_event_pool.push_back(r.b);
    }
    v->clear();
  }
}

// Adds the durations of the launches that a replayed graph timed.
void collect_graph(const std::vector<ProfRec>& recs) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto& r : recs) add_record(r);
}

template <class F>
int capture_one(F&& seq, cudaStream_t cs, cudaGraphExec_t* exec, int64_t* n_launches, std::vector<ProfRec>* recs) {
  const int64_t before = g_launches.load();
  size_t rec0 = 0;
  {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    rec0 = g_prof_pending.size();
  }
  FG_CHECK_CUDA(cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal));
  const int st = seq(cs);
  cudaGraph_t graph = nullptr;
  const cudaError_t ce = cudaStreamEndCapture(cs, &graph);
  *n_launches = g_launches.load() - before;
  g_launches.fetch_sub(*n_launches);  // recorded, not executed
  {
    // the timing events of the captured launches now belong to the graph
    std::lock_guard<std::mutex> lk(g_prof_mu);
    if (rec0 < g_prof_pending.size()) {
      recs->assign(g_prof_pending.begin() + rec0, g_prof_pending.end());
      g_prof_pending.resize(rec0);
    }
  }
  if (st != FG_OK) {
    if (graph) cudaGraphDestroy(graph);
    return st;
  }
  if (ce != cudaSuccess) return cuda_fail(ce, "stream capture");
  const cudaError_t ie = cudaGraphInstantiate(exec, graph, 0);
  cudaGraphDestroy(graph);
  if (ie != cudaSuccess) return cuda_fail(ie, "graph instantiate");
  return FG_OK;
}

template <class P, class D>
int capture_graphs(P&& prefill_seq, D&& decode_seq) {
  int dev = 0;
  FG_CHECK_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(FG_ERR_UNSUPPORTED, "device ordinal %d above 63", dev);
  if (!g_graph.cap[dev]) FG_CHECK_CUDA(cudaStreamCreateWithFlags(&g_graph.cap[dev], cudaStreamNonBlocking));
  const cudaStream_t cs = g_graph.cap[dev];
  FG_TRY(capture_one(prefill_seq, cs, &g_graph.prefill, &g_graph.n_prefill, &g_graph.prof_prefill));
  FG_TRY(capture_one(decode_seq, cs, &g_graph.decode, &g_graph.n_decode, &g_graph.prof_decode));
  g_graph.valid = true;
  return FG_OK;
}
}  // namespace

int generate_impl(const fg_model* m, const int32_t* ids, int B, int L, int T, int32_t* out, fg_kv_cache* caches,
                  void* ws, size_t wsb, fg_timing* timing, cudaStream_t s) {
  if (!m || !ids || !out || !caches) return fail(FG_ERR_INVALID_ARG, "null pointer");
  if (B <= 0 || L <= 0 || T <= 0) return fail(FG_ERR_SHAPE, "B, L and gen_len must be positive");
  if (!m->embed || !m->pos_embed || !m->lnf_g || !m->lnf_b || !m->layers)
    return fail(FG_ERR_INVALID_ARG, "model tensors not set");
  if (m->hidden != m->n_heads * m->head_dim) return fail(FG_ERR_SHAPE, "hidden != n_heads * head_dim");
  if (L + T - 1 > m->max_pos) return fail(FG_ERR_SHAPE, "L + gen_len - 1 exceeds max_pos");
  const int h = m->hidden;
  for (int l = 0; l < m->n_layers; ++l) {
    fg_kv_cache& c = caches[l];
    if (c.B != B || c.n_heads != m->n_heads || c.head_dim != m->head_dim)
      return fail(FG_ERR_SHAPE, "cache %d shape does not match the model", l);
    if (c.capacity < L + T) return fail(FG_ERR_CAPACITY, "cache %d capacity %d < L + gen_len", l, c.capacity);
  }
  const size_t need = generate_ws(m, B, L, T);
  if (!ws || wsb < need) return fail(FG_ERR_WORKSPACE, "generate needs %zu workspace bytes", need);
  Carver c(ws, wsb);
  void* x = c.take(size_t(B) * L * h * 2);
  void* xd = c.take(size_t(B) * h * 2);
  void* xn = c.take(size_t(B) * h * 2);
  void* hn = c.take(size_t(B) * h * 2);   // LN1 of the next block, from the previous block's fc2
  const size_t layer_b = std::max(prefill_ws(h, m->ffn, B, L), decode_ws(h, m->ffn, m->n_heads, B, L + T));
  void* lws = c.take(layer_b);
  void* lgw = c.take(lm_ws(B, m->vocab));

  // The two launch sequences of a generation (prompt pass; decode steps).  They run directly
  // on `s`, or on the capture stream while a CUDA graph is recorded.  In a decode step each
  // block's fc2 reduction also applies the LayerNorm that follows it (the next block's LN1,
  // or the final LayerNorm before the LM head) whenever that GEMM splits K.
  auto prefill_seq = [&](cudaStream_t st_) -> int {
    for (int l = 0; l < m->n_layers; ++l) caches[l].len = 0;
    FG_TRY(embed_impl(ids, B, L, L, 0, m->embed, m->pos_embed, h, x, st_));
    for (int l = 0; l < m->n_layers; ++l) FG_TRY(prefill_layer_impl(&m->layers[l], &caches[l], x, B, L, lws, layer_b, st_));
    // hidden state of each sequence's last prompt position
    FG_CHECK_CUDA(cudaMemcpy2DAsync(xd, size_t(h) * 2, reinterpret_cast<uint8_t*>(x) + size_t(L - 1) * h * 2,
                                    size_t(L) * h * 2, size_t(h) * 2, B, cudaMemcpyDeviceToDevice, st_));
    FG_TRY(layernorm_impl(xd, B, h, m->lnf_g, m->lnf_b, xn, st_));
    return lm_head_impl(xn, B, h, m->embed, m->vocab, nullptr, out, T, lgw, lm_ws(B, m->vocab), st_, true);
  };
  auto decode_seq = [&](cudaStream_t st_) -> int {
    for (int j = 1; j < T; ++j) {
      // token j-1 sits at position L + j - 1
      FG_TRY(embed_impl(out + (j - 1), B, 1, T, L + j - 1, m->embed, m->pos_embed, h, xd, st_));
      const void* h1 = nullptr;
      for (int l = 0; l < m->n_layers; ++l) {
        const bool last = l + 1 == m->n_layers;
        LnFuse nx{last ? m->lnf_g : m->layers[l + 1].ln1_g, last ? m->lnf_b : m->layers[l + 1].ln1_b,
                  last ? xn : hn, false};
        FG_TRY(decode_layer_impl(&m->layers[l], &caches[l], xd, xd, B, lws, layer_b, st_, h1, &nx));
        if (!nx.done) FG_TRY(layernorm_impl(xd, B, h, nx.g, nx.b, nx.H, st_));
        h1 = last ? nullptr : hn;
      }
      FG_TRY(lm_head_impl(xn, B, h, m->embed, m->vocab, nullptr, out + j, T, lgw, lm_ws(B, m->vocab), st_, true));
    }
    return FG_OK;
  };

  std::lock_guard<std::mutex> glk(g_graph_mu);
  GraphKey key = make_key(m, ids, B, L, T, out, caches, ws, wsb, s, profiling_mask());
  bool replay = false;
  if (g_graph.valid && g_graph.key == key) {
    replay = true;
  } else if (g_graph.seen && g_graph.key == key) {
    // second call with this configuration: record both sequences as graphs, then replay
    FG_TRY(capture_graphs(prefill_seq, decode_seq));
    replay = true;
  } else {
    reset_graphs();
    g_graph.key = key;
    g_graph.seen = true;
  }

  cudaEvent_t e0, e1, e2;
  FG_CHECK_CUDA(cudaEventCreate(&e0));
  FG_CHECK_CUDA(cudaEventCreate(&e1));
  FG_CHECK_CUDA(cudaEventCreate(&e2));
  int st = FG_OK;
  do {
    cudaError_t ce = cudaEventRecord(e0, s);
    if (ce != cudaSuccess) { st = cuda_fail(ce, "event"); break; }
    if (replay) {
      ce = cudaGraphLaunch(g_graph.prefill, s);
      if (ce != cudaSuccess) { st = cuda_fail(ce, "graph launch (prompt pass)"); break; }
      g_launches.fetch_add(g_graph.n_prefill);
    } else if ((st = prefill_seq(s)) != FG_OK) {
      break;
    }
    cudaEventRecord(e1, s);
    if (replay) {
      ce = cudaGraphLaunch(g_graph.decode, s);
      if (ce != cudaSuccess) { st = cuda_fail(ce, "graph launch (decode)"); break; }
      g_launches.fetch_add(g_graph.n_decode);
      for (int l = 0; l < m->n_layers; ++l) caches[l].len = L + T - 1;
    } else if ((st = decode_seq(s)) != FG_OK) {
      break;
    }
    cudaEventRecord(e2, s);
    ce = cudaEventSynchronize(e2);
    if (ce != cudaSuccess) { st = cuda_fail(ce, "generate"); break; }
    if (replay) {
      collect_graph(g_graph.prof_prefill);
      collect_graph(g_graph.prof_decode);
    }
    int derr = 0;
    if (read_device_error(&derr) == FG_OK && derr != 0) {
      st = fail(FG_ERR_CUDA, "a device-side wait timed out (code %d)", derr);
      break;
    }
    float pm = 0.f, dm = 0.f;
    cudaEventElapsedTime(&pm, e0, e1);
    cudaEventElapsedTime(&dm, e1, e2);
    if (timing) {
      timing->prefill_ms = pm;
      timing->decode_ms = dm;
      timing->tokens = int64_t(B) * T;
      timing->tok_per_s = double(B) * T / ((double(pm) + double(dm)) * 1e-3);
    }
  } while (false);
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  cudaEventDestroy(e2);
  return st;
}

// ---------------------------------------------------------------- host-offloaded weights
// Generation with every layer's 4-bit weights resident in pinned HOST memory ("FlexGen"
// README mirror: offloading weights to CPU memory with the --percent policy and pinned weights,
// and the block schedule that overlaps the loading of the next layer's weights with the
// computation of the current one).  The block here is the whole batch: each layer's weights
// cross the host link once per pass (the prompt pass, then each decode step) and serve every
// sequence before the next layer runs.  Two weight slots in the workspace alternate: while the
// compute stream runs layer c out of one slot, a copy stream fills the other slot with layer
// c + 1, and the slot of layer c is refilled with layer c + 2 once layer c's kernels are done.
namespace {

struct LayerSpan {
  size_t off[4][3];   // per linear: codes (or fp16 weight), params, bias
  size_t bytes[4][3];
  size_t ln_off[4];
  size_t total;    // slot bytes (each tensor 256-byte aligned)
  size_t payload;  // bytes copied per layer
};

size_t lin_bytes_codes(const fg_qlinear& w) {
  return w.w16 ? size_t(w.K) * size_t(w.N) * 2 : size_t(w.K) * size_t(w.N) / 2;
}
size_t lin_bytes_params(const fg_qlinear& w) {
  return w.w16 ? 0 : size_t(w.K) * size_t(w.N / w.group) * 4;
}

LayerSpan layer_span(const fg_layer& L, int h) {
  LayerSpan sp{};
  size_t t = 0;
  const fg_qlinear* lins[4] = {&L.qkv, &L.out, &L.fc1, &L.fc2};
  for (int i = 0; i < 4; ++i) {
    const size_t b[3] = {lin_bytes_codes(*lins[i]), lin_bytes_params(*lins[i]),
                         lins[i]->bias ? size_t(lins[i]->N) * 2 : 0};
    for (int j = 0; j < 3; ++j) {
      sp.off[i][j] = t;
      sp.bytes[i][j] = b[j];
      t += align256(b[j]);
      sp.payload += b[j];
    }
  }
  for (int j = 0; j < 4; ++j) {
    sp.ln_off[j] = t;
    t += align256(size_t(h) * 2);
    sp.payload += size_t(h) * 2;
  }
  sp.total = t;
  return sp;
}

bool is_host_memory(const void* p) {
  if (!p) return true;
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeHost;
}

// The device-side layer whose pointers lie in a weight slot.
fg_layer slot_layer(const fg_layer& H, const LayerSpan& sp, uint8_t* slot) {
  fg_layer D = H;
  fg_qlinear* lins[4] = {&D.qkv, &D.out, &D.fc1, &D.fc2};
  for (int i = 0; i < 4; ++i) {
    if (lins[i]->w16) {
      lins[i]->w16 = slot + sp.off[i][0];
    } else {
      lins[i]->codes = slot + sp.off[i][0];
      lins[i]->params = slot + sp.off[i][1];
    }
    if (lins[i]->bias) lins[i]->bias = slot + sp.off[i][2];
  }
  D.ln1_g = slot + sp.ln_off[0];
  D.ln1_b = slot + sp.ln_off[1];
  D.ln2_g = slot + sp.ln_off[2];
  D.ln2_b = slot + sp.ln_off[3];
  return D;
}

// One cudaMemcpyAsync per tensor of layer H into `slot` on stream cs.
int copy_layer(const fg_layer& H, const LayerSpan& sp, uint8_t* slot, int h, cudaStream_t cs) {
  const fg_qlinear* lins[4] = {&H.qkv, &H.out, &H.fc1, &H.fc2};
  for (int i = 0; i < 4; ++i) {
    const void* src[3] = {lins[i]->w16 ? lins[i]->w16 : static_cast<const void*>(lins[i]->codes), lins[i]->params,
                          lins[i]->bias};
    for (int j = 0; j < 3; ++j)
      if (sp.bytes[i][j] && src[j])
        FG_CHECK_CUDA(cudaMemcpyAsync(slot + sp.off[i][j], src[j], sp.bytes[i][j], cudaMemcpyHostToDevice, cs));
  }
  const void* ln[4] = {H.ln1_g, H.ln1_b, H.ln2_g, H.ln2_b};
  for (int j = 0; j < 4; ++j)
    FG_CHECK_CUDA(cudaMemcpyAsync(slot + sp.ln_off[j], ln[j], size_t(h) * 2, cudaMemcpyHostToDevice, cs));
  return FG_OK;
}

cudaStream_t g_copy_stream[64] = {nullptr};
std::mutex g_copy_mu;

size_t offload_ws(const fg_model* m, int B, int L, int T) {
  const LayerSpan sp = layer_span(m->layers[0], m->hidden);
  return generate_ws(m, B, L, T) + 2 * align256(sp.total) + 256;
}

// The weight slots and the events of the double buffer for one generation.
struct Offload {
  const fg_model* m;
  LayerSpan sp;
  uint8_t* slot[2];
  fg_layer dev[2];
  cudaEvent_t loaded[2] = {nullptr, nullptr}, freed[2] = {nullptr, nullptr};
  cudaStream_t cs = nullptr;
  int64_t visits = 0, issued = 0;  // layer visits of the whole generation, copies issued so far
  double bytes = 0;

  ~Offload() {
    for (int i = 0; i < 2; ++i) {
      if (loaded[i]) cudaEventDestroy(loaded[i]);
      if (freed[i]) cudaEventDestroy(freed[i]);
    }
  }
  // enqueue the copy of visit number `c` (layer c % n_layers) into slot c % 2
  int issue(int64_t c) {
    const int l = int(c % m->n_layers), k = int(c % 2);
    if (c >= 2) FG_CHECK_CUDA(cudaStreamWaitEvent(cs, freed[k], 0));
    FG_TRY(copy_layer(m->layers[l], sp, slot[k], m->hidden, cs));
    FG_CHECK_CUDA(cudaEventRecord(loaded[k], cs));
    bytes += double(sp.payload);
    ++issued;
    return FG_OK;
  }
  // the device layer of visit c, ready for the compute stream s
  int acquire(int64_t c, cudaStream_t s, const fg_layer** out) {
    const int k = int(c % 2);
    FG_CHECK_CUDA(cudaStreamWaitEvent(s, loaded[k], 0));
    *out = &dev[k];
    return FG_OK;
  }
  // layer visit c is enqueued on s: its slot is refilled with visit c + 2 after it
  int release(int64_t c, cudaStream_t s) {
    FG_CHECK_CUDA(cudaEventRecord(freed[c % 2], s));
    if (c + 2 < visits) FG_TRY(issue(c + 2));
    return FG_OK;
  }
};

}  // namespace

int generate_offload_impl(const fg_model* m, const int32_t* ids, int B, int L, int T, int32_t* out,
                          fg_kv_cache* caches, void* ws, size_t wsb, fg_timing* timing, double* h2d_bytes,
                          cudaStream_t s) {
  if (!m || !ids || !out || !caches) return fail(FG_ERR_INVALID_ARG, "null pointer");
  if (B <= 0 || L <= 0 || T <= 0) return fail(FG_ERR_SHAPE, "B, L and gen_len must be positive");
  if (!m->embed || !m->pos_embed || !m->lnf_g || !m->lnf_b || !m->layers || m->n_layers <= 0)
    return fail(FG_ERR_INVALID_ARG, "model tensors not set");
  if (m->hidden != m->n_heads * m->head_dim) return fail(FG_ERR_SHAPE, "hidden != n_heads * head_dim");
  if (L + T - 1 > m->max_pos) return fail(FG_ERR_SHAPE, "L + gen_len - 1 exceeds max_pos");
  const int h = m->hidden;
  const LayerSpan sp0 = layer_span(m->layers[0], h);
  for (int l = 0; l < m->n_layers; ++l) {
    int F = 0;
    FG_TRY(check_layer(&m->layers[l], h, &F));
    if (F != m->ffn) return fail(FG_ERR_SHAPE, "layer %d ffn %d != model ffn %d", l, F, m->ffn);
    const fg_layer& H = m->layers[l];
    const void* ptrs[] = {H.ln1_g, H.ln1_b, H.ln2_g, H.ln2_b, H.qkv.codes, H.qkv.params, H.qkv.bias, H.qkv.w16,
                          H.out.codes, H.out.params, H.out.bias, H.out.w16, H.fc1.codes, H.fc1.params,
                          H.fc1.bias, H.fc1.w16, H.fc2.codes, H.fc2.params, H.fc2.bias, H.fc2.w16};
    for (const void* p : ptrs)
      if (!is_host_memory(p))
        return fail(FG_ERR_INVALID_ARG, "layer %d: offloaded weights must be pinned host memory", l);
    const LayerSpan sp = layer_span(H, h);
    if (sp.total != sp0.total || memcmp(sp.bytes, sp0.bytes, sizeof(sp.bytes)) != 0)
      return fail(FG_ERR_SHAPE, "layer %d: every layer must have the same tensor sizes", l);
    fg_kv_cache& c = caches[l];
    if (c.B != B || c.n_heads != m->n_heads || c.head_dim != m->head_dim)
      return fail(FG_ERR_SHAPE, "cache %d shape does not match the model", l);
    if (c.capacity < L + T) return fail(FG_ERR_CAPACITY, "cache %d capacity %d < L + gen_len", l, c.capacity);
  }
  const size_t need = offload_ws(m, B, L, T);
  if (!ws || wsb < need) return fail(FG_ERR_WORKSPACE, "offloaded generate needs %zu workspace bytes", need);

  int dev = 0;
  FG_CHECK_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(FG_ERR_UNSUPPORTED, "device ordinal %d above 63", dev);
  {
    std::lock_guard<std::mutex> lk(g_copy_mu);
    if (!g_copy_stream[dev]) FG_CHECK_CUDA(cudaStreamCreateWithFlags(&g_copy_stream[dev], cudaStreamNonBlocking));
  }
  Carver c(ws, wsb);
  void* x = c.take(size_t(B) * L * h * 2);
  void* xd = c.take(size_t(B) * h * 2);
  void* xn = c.take(size_t(B) * h * 2);
  c.take(size_t(B) * h * 2);  // (the resident path's next-LN1 buffer; unused here: the next
                              // layer's LayerNorm parameters may still be on their way)
  const size_t layer_b = std::max(prefill_ws(h, m->ffn, B, L), decode_ws(h, m->ffn, m->n_heads, B, L + T));
  void* lws = c.take(layer_b);
  void* lgw = c.take(lm_ws(B, m->vocab));
  Offload off;
  off.m = m;
  off.sp = sp0;
  off.cs = g_copy_stream[dev];
  off.visits = int64_t(m->n_layers) * T;  // the prompt pass and T-1 decode steps
  for (int k = 0; k < 2; ++k) {
    off.slot[k] = reinterpret_cast<uint8_t*>(c.take(sp0.total));
    off.dev[k] = slot_layer(m->layers[0], sp0, off.slot[k]);
    FG_CHECK_CUDA(cudaEventCreateWithFlags(&off.loaded[k], cudaEventDisableTiming));
    FG_CHECK_CUDA(cudaEventCreateWithFlags(&off.freed[k], cudaEventDisableTiming));
  }
  for (int l = 0; l < m->n_layers; ++l) caches[l].len = 0;

  cudaEvent_t e0, e1, e2;
  FG_CHECK_CUDA(cudaEventCreate(&e0));
  FG_CHECK_CUDA(cudaEventCreate(&e1));
  FG_CHECK_CUDA(cudaEventCreate(&e2));
  int st = FG_OK;
  int64_t visit = 0;
  do {
    cudaError_t ce = cudaEventRecord(e0, s);
    if (ce != cudaSuccess) { st = cuda_fail(ce, "event"); break; }
    // the copy stream starts after everything already queued on s (the caller's inputs)
    if ((ce = cudaEventRecord(e1, s)) != cudaSuccess || (ce = cudaStreamWaitEvent(off.cs, e1, 0)) != cudaSuccess) {
      st = cuda_fail(ce, "copy stream ordering");
      break;
    }
    if ((st = off.issue(0)) != FG_OK) break;
    if (off.visits > 1 && (st = off.issue(1)) != FG_OK) break;
    // prompt pass, layer-major over the whole batch
    if ((st = embed_impl(ids, B, L, L, 0, m->embed, m->pos_embed, h, x, s)) != FG_OK) break;
    for (int l = 0; l < m->n_layers && st == FG_OK; ++l, ++visit) {
      const fg_layer* ly = nullptr;
      if ((st = off.acquire(visit, s, &ly)) != FG_OK) break;
      if ((st = prefill_layer_impl(ly, &caches[l], x, B, L, lws, layer_b, s)) != FG_OK) break;
      st = off.release(visit, s);
    }
    if (st != FG_OK) break;
    ce = cudaMemcpy2DAsync(xd, size_t(h) * 2, reinterpret_cast<uint8_t*>(x) + size_t(L - 1) * h * 2,
                           size_t(L) * h * 2, size_t(h) * 2, B, cudaMemcpyDeviceToDevice, s);
    if (ce != cudaSuccess) { st = cuda_fail(ce, "last prompt rows"); break; }
    if ((st = layernorm_impl(xd, B, h, m->lnf_g, m->lnf_b, xn, s)) != FG_OK) break;
    if ((st = lm_head_impl(xn, B, h, m->embed, m->vocab, nullptr, out, T, lgw, lm_ws(B, m->vocab), s)) != FG_OK)
      break;
    cudaEventRecord(e1, s);
    for (int j = 1; j < T && st == FG_OK; ++j) {
      if ((st = embed_impl(out + (j - 1), B, 1, T, L + j - 1, m->embed, m->pos_embed, h, xd, s)) != FG_OK) break;
      for (int l = 0; l < m->n_layers && st == FG_OK; ++l, ++visit) {
        const fg_layer* ly = nullptr;
        if ((st = off.acquire(visit, s, &ly)) != FG_OK) break;
        if ((st = decode_layer_impl(ly, &caches[l], xd, xd, B, lws, layer_b, s)) != FG_OK) break;
        st = off.release(visit, s);
      }
      if (st != FG_OK) break;
      if ((st = layernorm_impl(xd, B, h, m->lnf_g, m->lnf_b, xn, s)) != FG_OK) break;
      st = lm_head_impl(xn, B, h, m->embed, m->vocab, nullptr, out + j, T, lgw, lm_ws(B, m->vocab), s);
    }
    if (st != FG_OK) break;
    cudaEventRecord(e2, s);
    ce = cudaEventSynchronize(e2);
    if (ce != cudaSuccess) { st = cuda_fail(ce, "offloaded generate"); break; }
    int derr = 0;
    if (read_device_error(&derr) == FG_OK && derr != 0) {
      st = fail(FG_ERR_CUDA, "a device-side wait timed out (code %d)", derr);
      break;
    }
    float pm = 0.f, dm = 0.f;
    cudaEventElapsedTime(&pm, e0, e1);
    cudaEventElapsedTime(&dm, e1, e2);
    if (timing) {
      timing->prefill_ms = pm;
      timing->decode_ms = dm;
      timing->tokens = int64_t(B) * T;
      timing->tok_per_s = double(B) * T / ((double(pm) + double(dm)) * 1e-3);
    }
    if (h2d_bytes) *h2d_bytes = off.bytes;
  } while (false);
  // nothing of this call may still be copying when it returns (the slots are the caller's)
  cudaStreamSynchronize(off.cs);
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  cudaEventDestroy(e2);
  return st;
}

}  // namespace fg

// ==================================================================== extern "C"
using namespace fg;

extern "C" {

const char* fg_status_string(int status) {
  switch (status) {
    case FG_OK: return "ok";
    case FG_ERR_INVALID_ARG: return "invalid argument";
    case FG_ERR_SHAPE: return "shape error";
    case FG_ERR_ALIGN: return "alignment error";
    case FG_ERR_CAPACITY: return "KV cache capacity exceeded";
    case FG_ERR_CUDA: return "CUDA error";
    case FG_ERR_UNSUPPORTED: return "unsupported configuration";
    case FG_ERR_WORKSPACE: return "workspace too small";
    default: return "unknown status";
  }
}

const char* fg_last_error(void) { return g_err; }
int fg_version(void) { return 100; }

int fg_quantize_pack(const void* x, int64_t rows, int64_t cols, int group, int axis, uint8_t* codes, void* params,
                     void* stream) {
  return quantize_pack_impl(x, rows, cols, group, axis, codes, params, as_stream(stream));
}

int fg_dequantize(const uint8_t* codes, const void* params, int64_t rows, int64_t cols, int group, int axis,
                  void* out, void* stream) {
  return dequantize_impl(codes, params, rows, cols, group, axis, out, as_stream(stream));
}

int fg_kv_append(fg_kv_cache* cache, const void* k, const void* v, int64_t row_stride, int n_tokens, void* stream) {
  return kv_append_impl(cache, k, v, row_stride, n_tokens, as_stream(stream));
}

size_t fg_qgemm_workspace_bytes(int64_t M, int N, int K) { return qgemm_ws_bytes(M, N, K); }

int fg_qgemm(const void* X, int64_t M, const fg_qlinear* W, const void* R, int relu, void* Y, void* workspace,
             size_t ws_bytes, void* stream) {
  if (!W) return fail(FG_ERR_INVALID_ARG, "null weight");
  return qlinear_run(X, M, *W, R, relu, Y, workspace, ws_bytes, as_stream(stream));
}

size_t fg_gemm_f16_workspace_bytes(int64_t M, int N, int K) { return splitk_ws_bytes(M, N, K); }

int fg_gemm_f16(const void* X, int64_t M, const void* W, int K, int N, const void* bias, const void* R, int relu,
                void* Y, void* workspace, size_t ws_bytes, void* stream) {
  return gemm_impl(1, X, M, N, K, W, nullptr, 0, bias, R, relu, Y, false, workspace, ws_bytes, as_stream(stream),
                   false);
}

size_t fg_decode_attention_workspace_bytes(int B, int n_heads, int head_dim, int ctx) {
  return decode_attention_ws_bytes(B, n_heads, head_dim, ctx);
}

int fg_decode_attention(const void* q, int64_t q_stride, const fg_kv_cache* cache, void* out, void* workspace,
                        size_t ws_bytes, void* stream) {
  return decode_attention_impl(q, q_stride, cache, out, workspace, ws_bytes, as_stream(stream));
}

int fg_prefill_attention(const void* qkv, int B, int L, int n_heads, int head_dim, void* out, void* stream) {
  return prefill_attention_impl(qkv, B, L, n_heads, head_dim, out, as_stream(stream));
}

int fg_layernorm(const void* x, int64_t rows, int cols, const void* g, const void* b, void* y, void* stream) {
  return layernorm_impl(x, rows, cols, g, b, y, as_stream(stream));
}

int fg_embed(const int32_t* ids, int B, int T, int pos0, const void* E, const void* P, int hidden, void* out,
             void* stream) {
  return embed_impl(ids, B, T, T, pos0, E, P, hidden, out, as_stream(stream));
}

size_t fg_lm_head_workspace_bytes(int B, int vocab) { return lm_ws(B, vocab); }

int fg_lm_head_argmax(const void* x, int B, int hidden, const void* E, int vocab, float* logits, int32_t* tokens,
                      void* workspace, size_t ws_bytes, void* stream) {
  return lm_head_impl(x, B, hidden, E, vocab, logits, tokens, 1, workspace, ws_bytes, as_stream(stream));
}

size_t fg_decode_layer_workspace_bytes(int hidden, int ffn, int n_heads, int B, int capacity) {
  if (hidden <= 0 || ffn <= 0 || n_heads <= 0 || B <= 0 || capacity <= 0) return 0;
  return decode_ws(hidden, ffn, n_heads, B, capacity);
}

int fg_decode_layer(const fg_layer* layer, fg_kv_cache* cache, const void* x_in, void* x_out, int B, void* workspace,
                    size_t ws_bytes, void* stream) {
  return decode_layer_impl(layer, cache, x_in, x_out, B, workspace, ws_bytes, as_stream(stream));
}

size_t fg_prefill_layer_workspace_bytes(int hidden, int ffn, int B, int L) {
  if (hidden <= 0 || ffn <= 0 || B <= 0 || L <= 0) return 0;
  return prefill_ws(hidden, ffn, B, L);
}

int fg_prefill_layer(const fg_layer* layer, fg_kv_cache* cache, void* x, int B, int L, void* workspace,
                     size_t ws_bytes, void* stream) {
  return prefill_layer_impl(layer, cache, x, B, L, workspace, ws_bytes, as_stream(stream));
}

size_t fg_workspace_bytes(const fg_model* model, int B, int L, int gen_len) {
  if (!model || B <= 0 || L <= 0 || gen_len <= 0) return 0;
  return generate_ws(model, B, L, gen_len);
}

int fg_generate(const fg_model* model, const int32_t* prompt_ids, int B, int L, int gen_len, int32_t* out_ids,
                fg_kv_cache* caches, void* workspace, size_t ws_bytes, fg_timing* timing, void* stream) {
  return generate_impl(model, prompt_ids, B, L, gen_len, out_ids, caches, workspace, ws_bytes, timing,
                       as_stream(stream));
}

size_t fg_offload_workspace_bytes(const fg_model* model, int B, int L, int gen_len) {
  if (!model || !model->layers || model->n_layers <= 0 || B <= 0 || L <= 0 || gen_len <= 0) return 0;
  return offload_ws(model, B, L, gen_len);
}

int fg_generate_offload(const fg_model* model, const int32_t* prompt_ids, int B, int L, int gen_len,
                        int32_t* out_ids, fg_kv_cache* caches, void* workspace, size_t ws_bytes, fg_timing* timing,
                        double* h2d_bytes, void* stream) {
  return generate_offload_impl(model, prompt_ids, B, L, gen_len, out_ids, caches, workspace, ws_bytes, timing,
                               h2d_bytes, as_stream(stream));
}

int fg_profile_enable(int on) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on = on != 0;
  g_prof_mask = g_prof_on ? g_prof_sel : 0u;
  return FG_OK;
}

int fg_profile_select(unsigned kinds) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_sel = kinds & kAllKinds;
  g_prof_mask = g_prof_on ? g_prof_sel : 0u;
  return FG_OK;
}

int fg_profile_read(int kind, double* total_ms, int64_t* launches, double* flops, double* bytes) {
  if (kind < 0 || kind >= PROF_NKINDS) return fail(FG_ERR_INVALID_ARG, "bad profile kind");
  std::lock_guard<std::mutex> lk(g_prof_mu);
  collect_locked();
  if (total_ms) *total_ms = g_prof_ms[kind];
  if (launches) *launches = g_prof_n[kind];
  if (flops) *flops = g_prof_flops[kind];
  if (bytes) *bytes = g_prof_bytes[kind];
  return FG_OK;
}

int64_t fg_launch_count(void) { return g_launches.load(); }

int fg_profile_reset(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  collect_locked();
  for (int i = 0; i < PROF_NKINDS; ++i) {
    g_prof_ms[i] = 0;
    g_prof_n[i] = 0;
    g_prof_flops[i] = 0;
    g_prof_bytes[i] = 0;
  }
  return FG_OK;
}

}  // extern "C"
