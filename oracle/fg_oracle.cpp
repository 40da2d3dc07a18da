// fg_oracle.cpp - plain, slow CPU oracle of the 4-bit group-wise compression path and of the
// OPT-shaped decoder that reads it.  TEST INFRASTRUCTURE ONLY: the tests, the smoke entry
// point and the benchmark's CPU-baseline leg load it (through oracle/_lib.py); the product
// library never does.  It shares no code with the CUDA library: its own fp16 conversion,
// its own quantizer, its own loops.
//
// Build: g++ -std=c++17 -O2 -ffp-contract=off -fno-fast-math -fopenmp -shared -fPIC
// (no contraction of a*b+c into an FMA, no reassociation; OpenMP only splits independent
// outputs - rows, (sequence, head) pairs - across threads and never reorders a sum).
//
// What the pages fix (cited by page title and section):
//  * "FlexGen" README mirror, key features ("Extreme Compression"): weights and the
//    attention cache are compressed to 4 bits; the out-of-memory tips: weight compression
//    cuts weight memory by about 70 %.
//  * arXiv 2303.06865 record (pith.science), abstract: 4-bit weights and attention cache.
//  * "FlexGen" README mirror, benchmark table and its notes: OPT-6.7B/30B/175B generation,
//    input length 512, output length 32, throughput = generated tokens / (prompt time +
//    generation time).
// Everything below that level is a reading, stated where it is used:
//  Q1 a group is g consecutive elements along one axis of a 2-D fp16 tensor;
//  Q2 mn = min, mx = max of the group (a zero extreme taken as +0);
//  Q3 s = fp16(fp32(mx - mn) / 15): fp32 subtract, fp32 division, one RNE rounding;
//  Q4 code = clamp(rint(fp32(x - mn) / s), 0, 15), fp32 subtract and divide by the stored
//     fp16 s, rint half to even; s == 0 -> every code 0;
//  Q5 byte j of a row = code(2j) | code(2j+1) << 4;
//  Q6 params {mn, s} fp16 pairs, [rows][cols/g] (axis 1) or [rows/g][cols] (axis 0);
//  Q7 dequantized value = fp16(mn + code*s), one rounding of the exact value;
//  D1 OPT block: pre-LayerNorm (eps 1e-5), MHA with scale 1/sqrt(hd), ReLU FFN, residuals;
//  D2 Y = X W + b with W [K][N] (N contiguous), columns of the QKV projection q | k | v;
//  D3 fp16 storage at every kernel boundary (LayerNorm output, projections, attention
//     output, residual stream), float64 in between;
//  D4 prefill attention on this pass's unquantized fp16 K/V; the cache then stores them
//     4-bit; a decode step appends its token first and attends over positions 0..len;
//     decode attention consumes the exact values mn + code*s;
//  D5 embedding fp16(E[id] + P[pos]), positions 0..L-1, then L, L+1, ... (no offset);
//  D6 tied fp16 LM head logits = LN_f(x) E^T, greedy argmax with ties to the lowest id;
//  D7 T output tokens = 1 from the prompt pass + T-1 decode steps.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

// ------------------------------------------------------------------ IEEE binary16
// Exact value of an fp16 bit pattern.
double h2d(uint16_t h) {
  const int sign = h >> 15;
  const int e = (h >> 10) & 31;
  const int m = h & 1023;
  double v;
  if (e == 0) {
    v = std::ldexp(double(m), -24);  // subnormal: m * 2^-24
  } else if (e == 31) {
    v = m == 0 ? INFINITY : NAN;
  } else {
    v = std::ldexp(double(1024 + m), e - 25);  // (1 + m/1024) * 2^(e-15)
  }
  return sign ? -v : v;
}

// Round a double to the nearest fp16, ties to even (one rounding); beyond the largest
// finite value the result is infinity.
uint16_t d2h(double x) {
  if (std::isnan(x)) return 0x7E00;
  const uint16_t sign = std::signbit(x) ? 0x8000 : 0;
  const double a = std::fabs(x);
  if (a >= 65520.0) return sign | 0x7C00;  // 65520 is halfway between 65504 and 2^16
  if (a < std::ldexp(1.0, -14)) {
    // subnormal range: multiples of 2^-24 (n = 1024 is the smallest normal, same bits)
    const double n = std::nearbyint(std::ldexp(a, 24));
    return sign | uint16_t(n);
  }
  int ex = 0;
  std::frexp(a, &ex);  // a = f * 2^ex, f in [0.5, 1)
  int e = ex - 1;      // a in [2^e, 2^(e+1))
  double n = std::nearbyint(std::ldexp(a, 10 - e));  // significand as an integer in [1024, 2048]
  if (n == 2048.0) {
    n = 1024.0;
    e += 1;
  }
  if (e > 15) return sign | 0x7C00;
  return sign | uint16_t(((e + 15) << 10) | (int(n) - 1024));
}

float h2f(uint16_t h) { return float(h2d(h)); }  // exact: every fp16 value is a float

// ------------------------------------------------------------------ one group (Q2-Q4)
// x: g fp16 values (consecutive along the group axis, `stride` elements apart).
// Writes the g codes and the fp16 {mn, s}.
void quantize_group(const uint16_t* x, int64_t stride, int g, uint8_t* q, uint16_t* mn_out, uint16_t* s_out) {
  float mn = h2f(x[0]), mx = h2f(x[0]);
  for (int t = 1; t < g; ++t) {
    const float v = h2f(x[t * stride]);
    if (v < mn) mn = v;
    if (v > mx) mx = v;
  }
  mn = mn + 0.0f;  // -0 + 0 = +0: a zero extreme is stored as +0 (Q2)
  mx = mx + 0.0f;
  const float d = mx - mn;        // fp32 subtraction
  const float s32 = d / 15.0f;    // fp32 IEEE division
  const uint16_t s16 = d2h(double(s32));  // one RNE rounding of the fp32 value to fp16 (Q3)
  const float s = h2f(s16);
  for (int t = 0; t < g; ++t) {
    if (s == 0.0f) {
      q[t] = 0;  // constant group, or d/15 below half the smallest subnormal (Q4)
      continue;
    }
    const float r = (h2f(x[t * stride]) - mn) / s;  // fp32 subtract, then fp32 divide
    float c = std::nearbyintf(r);                   // round half to even
    if (c < 0.0f) c = 0.0f;
    if (c > 15.0f) c = 15.0f;
    q[t] = uint8_t(c);
  }
  *mn_out = d2h(double(mn));  // exact: mn is an fp16 value
  *s_out = s16;
}

// Exact value of a code (Q7 before the fp16 rounding): mn + code*s in double (the product
// has at most 15 significant bits, the sum spans 2^-24 .. 2^20: exact).
double code_value(int code, uint16_t mn, uint16_t s) { return h2d(mn) + double(code) * h2d(s); }

int code_at(const uint8_t* codes_row, int64_t col) {
  const uint8_t b = codes_row[col >> 1];
  return (col & 1) ? (b >> 4) : (b & 15);  // Q5: even column in the low nibble
}

}  // namespace

extern "C" {

// ------------------------------------------------------------------ housekeeping
int orc_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
  return omp_get_max_threads();
#else
  (void)n;
  return 1;
#endif
}

uint16_t orc_d2h(double x) { return d2h(x); }
double orc_h2d(uint16_t h) { return h2d(h); }
void orc_d2h_array(const double* x, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = d2h(x[i]);
}

// ------------------------------------------------------------------ quantizer
// Groups given as rows of a [n_groups][g] fp16 array: codes [n_groups][g] (one per byte,
// 0..15), mn/s fp16 [n_groups].
void orc_quantize_groups(const uint16_t* x, int64_t n_groups, int g, uint8_t* q, uint16_t* mn, uint16_t* s) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n_groups; ++i) quantize_group(x + i * g, 1, g, q + i * g, mn + i, s + i);
}

// fp16(mn + code*s), one rounding (Q7); codes [n_groups][g], result [n_groups][g].
void orc_dequantize_groups(const uint8_t* q, const uint16_t* mn, const uint16_t* s, int64_t n_groups, int g,
                           uint16_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n_groups; ++i)
    for (int t = 0; t < g; ++t) out[i * g + t] = d2h(code_value(q[i * g + t], mn[i], s[i]));
}

// codes [rows][cols] one per byte -> packed [rows][cols/2] (Q5).
void orc_pack_nibbles(const uint8_t* q, int64_t rows, int64_t cols, uint8_t* packed) {
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t j = 0; j < cols / 2; ++j)
      packed[r * (cols / 2) + j] = uint8_t((q[r * cols + 2 * j] & 15) | ((q[r * cols + 2 * j + 1] & 15) << 4));
}

void orc_unpack_nibbles(const uint8_t* packed, int64_t rows, int64_t cols, uint8_t* q) {
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c) q[r * cols + c] = uint8_t(code_at(packed + r * (cols / 2), c));
}

// A 2-D fp16 tensor [rows][cols] quantized along `axis` (Q1, Q6): codes [rows][cols/2],
// params {mn, s} pairs: axis 1 -> [rows][cols/g], axis 0 -> [rows/g][cols].
// Returns 0, or -1 when the sizes do not fit the group.
int orc_quantize_pack(const uint16_t* x, int64_t rows, int64_t cols, int g, int axis, uint8_t* codes,
                      uint16_t* params) {
  if (g < 2 || g % 2 || cols % 2 || (axis == 1 && cols % g) || (axis == 0 && rows % g) || (axis != 0 && axis != 1))
    return -1;
  std::vector<uint8_t> q(static_cast<size_t>(rows * cols));
  if (axis == 1) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
      for (int64_t gi = 0; gi < cols / g; ++gi) {
        uint16_t* p = params + 2 * (r * (cols / g) + gi);
        quantize_group(x + r * cols + gi * g, 1, g, q.data() + r * cols + gi * g, p, p + 1);
      }
  } else {
#pragma omp parallel for schedule(static)
    for (int64_t rg = 0; rg < rows / g; ++rg)
      for (int64_t c = 0; c < cols; ++c) {
        std::vector<uint8_t> qq(static_cast<size_t>(g));
        uint16_t* p = params + 2 * (rg * cols + c);
        quantize_group(x + rg * g * cols + c, cols, g, qq.data(), p, p + 1);
        for (int t = 0; t < g; ++t) q[(rg * g + t) * cols + c] = qq[t];
      }
  }
  orc_pack_nibbles(q.data(), rows, cols, codes);
  return 0;
}

// Inverse map: codes + params -> fp16 [rows][cols] (Q7).
int orc_dequantize(const uint8_t* codes, const uint16_t* params, int64_t rows, int64_t cols, int g, int axis,
                   uint16_t* out) {
  if (g < 2 || g % 2 || cols % 2 || (axis == 1 && cols % g) || (axis == 0 && rows % g) || (axis != 0 && axis != 1))
    return -1;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c) {
      const uint16_t* p = axis == 1 ? params + 2 * (r * (cols / g) + c / g) : params + 2 * ((r / g) * cols + c);
      out[r * cols + c] = d2h(code_value(code_at(codes + r * (cols / 2), c), p[0], p[1]));
    }
  return 0;
}

// Exact values mn + code*s (double) of rows of codes grouped along the row: codes
// [rows][cols/2], params [rows][cols/g] pairs, out [rows][cols] (what attention consumes, D4).
void orc_code_values(const uint8_t* codes, const uint16_t* params, int64_t rows, int64_t cols, int g, double* out) {
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c) {
      const uint16_t* p = params + 2 * (r * (cols / g) + c / g);
      out[r * cols + c] = code_value(code_at(codes + r * (cols / 2), c), p[0], p[1]);
    }
}

// ------------------------------------------------------------------ LayerNorm (D1)
// y = (x - mean) / sqrt(var + eps) * gamma + beta over each row of h values, float64
// statistics (population variance), fp16 result.
void orc_layernorm(const uint16_t* x, int64_t rows, int h, const uint16_t* gamma, const uint16_t* beta, double eps,
                   uint16_t* y) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    const uint16_t* xr = x + r * h;
    double sum = 0.0;
    for (int i = 0; i < h; ++i) sum += h2d(xr[i]);
    const double mean = sum / h;
    double ss = 0.0;
    for (int i = 0; i < h; ++i) {
      const double dv = h2d(xr[i]) - mean;
      ss += dv * dv;
    }
    const double var = ss / h;
    const double inv = std::sqrt(var + eps);
    for (int i = 0; i < h; ++i) y[r * h + i] = d2h((h2d(xr[i]) - mean) / inv * h2d(gamma[i]) + h2d(beta[i]));
  }
}

// ------------------------------------------------------------------ linear layer (D2, D3)
// y[i][j] = fp16( [relu]( sum_k a[i][k] W[k][j] + b[j] ) [+ r[i][j]] ), the sum over k in
// ascending order in float64.  a fp16 [M][K] with row stride lda; W the fp16 weight [K][N]
// (the dequantized W_hat, or an uncompressed weight); bias fp16 [N] or NULL; r fp16 [M][N]
// or NULL; y fp16 [M][N].
void orc_linear(const uint16_t* a, int64_t M, int64_t lda, const uint16_t* W, int K, int N, const uint16_t* bias,
                int relu, const uint16_t* r, uint16_t* y) {
  std::vector<float> w(size_t(K) * size_t(N));  // the same values as floats (exact)
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < int64_t(K) * N; ++i) w[size_t(i)] = h2f(W[i]);
#pragma omp parallel
  {
    std::vector<double> acc(static_cast<size_t>(N));
#pragma omp for schedule(static)
    for (int64_t i = 0; i < M; ++i) {
      for (int j = 0; j < N; ++j) acc[j] = 0.0;
      for (int k = 0; k < K; ++k) {
        const double ak = h2d(a[i * lda + k]);
        const float* wk = w.data() + size_t(k) * N;
        for (int j = 0; j < N; ++j) acc[j] += ak * double(wk[j]);
      }
      for (int j = 0; j < N; ++j) {
        double v = acc[j] + (bias ? h2d(bias[j]) : 0.0);
        if (relu && v < 0.0) v = 0.0;
        if (r) v += h2d(r[i * N + j]);
        y[i * N + j] = d2h(v);
      }
    }
  }
}

// logits[i][v] = sum_k a[i][k] E[v][k] (float64) for an fp16 weight stored [V][K] (the tied
// LM head, D6).
void orc_linear_nk(const uint16_t* a, int64_t M, const uint16_t* E, int V, int K, double* logits) {
#pragma omp parallel for schedule(static) collapse(2)
  for (int64_t i = 0; i < M; ++i)
    for (int v = 0; v < V; ++v) {
      double acc = 0.0;
      for (int k = 0; k < K; ++k) acc += h2d(a[i * K + k]) * h2d(E[int64_t(v) * K + k]);
      logits[i * V + v] = acc;
    }
}

// Greedy token per row: the first index of the largest logit (ties to the lowest id, D6).
void orc_argmax(const double* logits, int64_t M, int V, int32_t* tok) {
  for (int64_t i = 0; i < M; ++i) {
    int best = 0;
    for (int v = 1; v < V; ++v)
      if (logits[i * V + v] > logits[i * V + best]) best = v;
    tok[i] = best;
  }
}

// ------------------------------------------------------------------ attention (D1, D4)
// Causal attention over one prompt: qkv fp16 [B][L][3h] (q | k | v, head j owning columns
// j*hd .. (j+1)*hd-1 of each part), out fp16 [B][L][h].  For query i: scores
// s_t = (q_i . k_t) / sqrt(hd) for t <= i, softmax in float64 (max subtracted), output
// sum_t p_t v_t.
void orc_prefill_attention(const uint16_t* qkv, int B, int L, int nh, int hd, uint16_t* out) {
  const int64_t h = int64_t(nh) * hd;
  const double scale = 1.0 / std::sqrt(double(hd));
#pragma omp parallel for schedule(dynamic) collapse(2)
  for (int b = 0; b < B; ++b)
    for (int j = 0; j < nh; ++j) {
      std::vector<double> sc(static_cast<size_t>(L)), o(static_cast<size_t>(hd));
      for (int i = 0; i < L; ++i) {
        const uint16_t* q = qkv + (int64_t(b) * L + i) * 3 * h + int64_t(j) * hd;
        double m = -INFINITY;
        for (int t = 0; t <= i; ++t) {
          const uint16_t* k = qkv + (int64_t(b) * L + t) * 3 * h + h + int64_t(j) * hd;
          double dot = 0.0;
          for (int d = 0; d < hd; ++d) dot += h2d(q[d]) * h2d(k[d]);
          sc[t] = dot * scale;
          if (sc[t] > m) m = sc[t];
        }
        double z = 0.0;
        for (int t = 0; t <= i; ++t) {
          sc[t] = std::exp(sc[t] - m);
          z += sc[t];
        }
        for (int d = 0; d < hd; ++d) o[d] = 0.0;
        for (int t = 0; t <= i; ++t) {
          const double p = sc[t] / z;
          const uint16_t* v = qkv + (int64_t(b) * L + t) * 3 * h + 2 * h + int64_t(j) * hd;
          for (int d = 0; d < hd; ++d) o[d] += p * h2d(v[d]);
        }
        for (int d = 0; d < hd; ++d) out[(int64_t(b) * L + i) * h + int64_t(j) * hd + d] = d2h(o[d]);
      }
    }
}

struct orc_cache {
  uint8_t *k_codes, *v_codes;  // [B][nh][cap][hd/2]
  uint16_t *k_params, *v_params;  // [B][nh][cap][hd/g][2]
  int B, n_heads, head_dim, group, capacity, len;
};

// Quantize n_tokens tokens per sequence into positions pos.. of the cache: k, v fp16 rows,
// row (b*n_tokens + t) at k + row*stride, h = nh*hd values each, grouped along the hidden
// dimension in groups of g (g divides hd, so no group spans two heads).
int orc_kv_append(orc_cache* c, const uint16_t* k, const uint16_t* v, int64_t stride, int n_tokens, int pos) {
  const int nh = c->n_heads, hd = c->head_dim, g = c->group;
  if (hd % g || pos < 0 || pos + n_tokens > c->capacity) return -1;
  for (int which = 0; which < 2; ++which) {
    const uint16_t* src = which == 0 ? k : v;
    uint8_t* codes = which == 0 ? c->k_codes : c->v_codes;
    uint16_t* params = which == 0 ? c->k_params : c->v_params;
#pragma omp parallel for schedule(static) collapse(2)
    for (int b = 0; b < c->B; ++b)
      for (int t = 0; t < n_tokens; ++t) {
        const uint16_t* row = src + (int64_t(b) * n_tokens + t) * stride;
        for (int j = 0; j < nh; ++j) {
          const int64_t slot = (int64_t(b) * nh + j) * c->capacity + pos + t;
          std::vector<uint8_t> q(static_cast<size_t>(hd));
          for (int gi = 0; gi < hd / g; ++gi) {
            uint16_t* p = params + 2 * (slot * (hd / g) + gi);
            quantize_group(row + int64_t(j) * hd + gi * g, 1, g, q.data() + gi * g, p, p + 1);
          }
          orc_pack_nibbles(q.data(), 1, hd, codes + slot * (hd / 2));
        }
      }
  }
  return 0;
}

// One query per sequence over cached positions 0..S-1: q fp16 rows (row b at q + b*q_stride,
// h values), out fp16 [B][h].  Keys and values are the exact code values (D4); scores
// (K_t . q) / sqrt(hd), float64 softmax, output sum_t p_t V_t.
void orc_decode_attention(const uint16_t* q, int64_t q_stride, const orc_cache* c, int S, uint16_t* out) {
  const int nh = c->n_heads, hd = c->head_dim, g = c->group;
  const int64_t h = int64_t(nh) * hd;
  const double scale = 1.0 / std::sqrt(double(hd));
#pragma omp parallel for schedule(dynamic) collapse(2)
  for (int b = 0; b < c->B; ++b)
    for (int j = 0; j < nh; ++j) {
      const int64_t row0 = (int64_t(b) * nh + j) * c->capacity;
      std::vector<double> K(size_t(S) * hd), V(size_t(S) * hd), sc(static_cast<size_t>(S)), o(size_t(hd), 0.0);
      orc_code_values(c->k_codes + row0 * (hd / 2), c->k_params + 2 * row0 * (hd / g), S, hd, g, K.data());
      orc_code_values(c->v_codes + row0 * (hd / 2), c->v_params + 2 * row0 * (hd / g), S, hd, g, V.data());
      const uint16_t* qb = q + int64_t(b) * q_stride + int64_t(j) * hd;
      double m = -INFINITY;
      for (int t = 0; t < S; ++t) {
        double dot = 0.0;
        for (int d = 0; d < hd; ++d) dot += K[size_t(t) * hd + d] * h2d(qb[d]);
        sc[t] = dot * scale;
        if (sc[t] > m) m = sc[t];
      }
      double z = 0.0;
      for (int t = 0; t < S; ++t) {
        sc[t] = std::exp(sc[t] - m);
        z += sc[t];
      }
      for (int t = 0; t < S; ++t) {
        const double p = sc[t] / z;
        for (int d = 0; d < hd; ++d) o[d] += p * V[size_t(t) * hd + d];
      }
      for (int d = 0; d < hd; ++d) out[int64_t(b) * h + int64_t(j) * hd + d] = d2h(o[d]);
    }
}

// ------------------------------------------------------------------ layers (D1-D4)
struct orc_linear_w {
  const uint16_t* w;     // fp16 [K][N]: W_hat (the dequantized 4-bit weight) or W itself
  const uint16_t* bias;  // fp16 [N] or NULL
  int K, N;
};
struct orc_layer {
  const uint16_t *ln1_g, *ln1_b, *ln2_g, *ln2_b;
  orc_linear_w qkv, out, fc1, fc2;
};

static const double kLnEps = 1e-5;

// One decoder block over a whole prompt: x fp16 [B*L][h] in place; the cache (len 0)
// receives positions 0..L-1.
int orc_prefill_layer(const orc_layer* ly, orc_cache* c, uint16_t* x, int B, int L) {
  const int nh = c->n_heads, hd = c->head_dim;
  const int h = nh * hd, F = ly->fc1.N;
  const int64_t BL = int64_t(B) * L;
  std::vector<uint16_t> h1(size_t(BL) * h), qkv(size_t(BL) * 3 * h), att(size_t(BL) * h), x1(size_t(BL) * h),
      f(size_t(BL) * F);
  orc_layernorm(x, BL, h, ly->ln1_g, ly->ln1_b, kLnEps, h1.data());
  orc_linear(h1.data(), BL, h, ly->qkv.w, h, 3 * h, ly->qkv.bias, 0, nullptr, qkv.data());
  if (orc_kv_append(c, qkv.data() + h, qkv.data() + 2 * h, 3 * h, L, 0)) return -1;
  c->len = L;
  orc_prefill_attention(qkv.data(), B, L, nh, hd, att.data());
  orc_linear(att.data(), BL, h, ly->out.w, h, h, ly->out.bias, 0, x, x1.data());
  orc_layernorm(x1.data(), BL, h, ly->ln2_g, ly->ln2_b, kLnEps, h1.data());
  orc_linear(h1.data(), BL, h, ly->fc1.w, h, F, ly->fc1.bias, 1, nullptr, f.data());
  orc_linear(f.data(), BL, F, ly->fc2.w, F, h, ly->fc2.bias, 0, x1.data(), x);
  return 0;
}

// One decoder block for one new token per sequence: x_in, x_out fp16 [B][h] (may alias);
// appends the token at position len, attends over 0..len, advances len.
int orc_decode_layer(const orc_layer* ly, orc_cache* c, const uint16_t* x_in, uint16_t* x_out, int B) {
  const int nh = c->n_heads, hd = c->head_dim;
  const int h = nh * hd, F = ly->fc1.N;
  std::vector<uint16_t> xin(x_in, x_in + size_t(B) * h), h1(size_t(B) * h), qkv(size_t(B) * 3 * h),
      att(size_t(B) * h), x1(size_t(B) * h), f(size_t(B) * F);
  orc_layernorm(xin.data(), B, h, ly->ln1_g, ly->ln1_b, kLnEps, h1.data());
  orc_linear(h1.data(), B, h, ly->qkv.w, h, 3 * h, ly->qkv.bias, 0, nullptr, qkv.data());
  const int pos = c->len;
  if (orc_kv_append(c, qkv.data() + h, qkv.data() + 2 * h, 3 * h, 1, pos)) return -1;
  c->len = pos + 1;
  orc_decode_attention(qkv.data(), 3 * h, c, pos + 1, att.data());
  orc_linear(att.data(), B, h, ly->out.w, h, h, ly->out.bias, 0, xin.data(), x1.data());
  orc_layernorm(x1.data(), B, h, ly->ln2_g, ly->ln2_b, kLnEps, h1.data());
  orc_linear(h1.data(), B, h, ly->fc1.w, h, F, ly->fc1.bias, 1, nullptr, f.data());
  orc_linear(f.data(), B, F, ly->fc2.w, F, h, ly->fc2.bias, 0, x1.data(), x_out);
  return 0;
}

// ------------------------------------------------------------------ model (D5-D7)
struct orc_model {
  int n_layers, hidden, n_heads, head_dim, ffn, vocab, max_pos, group;
  const uint16_t* embed;      // fp16 [vocab][hidden], also the tied LM head
  const uint16_t* pos_embed;  // fp16 [max_pos][hidden]
  const uint16_t *lnf_g, *lnf_b;
  const orc_layer* layers;    // [n_layers]
};

// x[b*T + t] = fp16(E[ids[b*T + t]] + P[pos0 + t]) (one rounding of the exact sum).
void orc_embed(const orc_model* m, const int32_t* ids, int B, int T, int pos0, uint16_t* x) {
  const int h = m->hidden;
  for (int64_t r = 0; r < int64_t(B) * T; ++r) {
    const int t = int(r % T);
    const uint16_t* e = m->embed + int64_t(ids[r]) * h;
    const uint16_t* p = m->pos_embed + int64_t(pos0 + t) * h;
    for (int i = 0; i < h; ++i) x[r * h + i] = d2h(h2d(e[i]) + h2d(p[i]));
  }
}

// Final LayerNorm, tied LM head and greedy argmax for rows x [B][h]; logits [B][vocab].
void orc_lm_head_argmax(const orc_model* m, const uint16_t* x, int B, double* logits, int32_t* tok) {
  std::vector<uint16_t> xn(size_t(B) * m->hidden);
  orc_layernorm(x, B, m->hidden, m->lnf_g, m->lnf_b, kLnEps, xn.data());
  orc_linear_nk(xn.data(), B, m->embed, m->vocab, m->hidden, logits);
  orc_argmax(logits, B, m->vocab, tok);
}

// Greedy generation: the prompt pass over ids [B][L] yields token 1, then T-1 decode steps;
// out [B][T]; caches [n_layers] (capacity >= L + T); all_logits [T][B][vocab] or NULL.
int orc_generate(const orc_model* m, const int32_t* ids, int B, int L, int T, int32_t* out, orc_cache* caches,
                 double* all_logits) {
  const int h = m->hidden, V = m->vocab;
  std::vector<uint16_t> x(size_t(B) * L * h), xd(size_t(B) * h);
  std::vector<double> logits(size_t(B) * V);
  std::vector<int32_t> tok(static_cast<size_t>(B)), prev(static_cast<size_t>(B));
  for (int l = 0; l < m->n_layers; ++l) caches[l].len = 0;
  orc_embed(m, ids, B, L, 0, x.data());
  for (int l = 0; l < m->n_layers; ++l)
    if (orc_prefill_layer(&m->layers[l], &caches[l], x.data(), B, L)) return -1;
  for (int b = 0; b < B; ++b)
    std::memcpy(xd.data() + size_t(b) * h, x.data() + (size_t(b) * L + L - 1) * h, size_t(h) * 2);
  orc_lm_head_argmax(m, xd.data(), B, logits.data(), tok.data());
  for (int step = 0; step < T; ++step) {
    if (step > 0) {
      for (int b = 0; b < B; ++b) prev[b] = out[b * T + step - 1];
      orc_embed(m, prev.data(), B, 1, L + step - 1, xd.data());  // token j-1 sits at position L+j-1
      for (int l = 0; l < m->n_layers; ++l)
        if (orc_decode_layer(&m->layers[l], &caches[l], xd.data(), xd.data(), B)) return -1;
      orc_lm_head_argmax(m, xd.data(), B, logits.data(), tok.data());
    }
    for (int b = 0; b < B; ++b) out[b * T + step] = tok[b];
    if (all_logits) std::memcpy(all_logits + size_t(step) * B * V, logits.data(), sizeof(double) * B * V);
  }
  return 0;
}

}  // extern "C"
