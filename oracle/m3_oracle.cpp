// m3_oracle.cpp -- plain, slow, obviously-correct CPU oracle of the per-frame
// autoregressive decode step of MiniMax Music 3's Qwen3-style "Global LLM"
// and of its RVQ depth decoder.
//
// THIS IS TEST INFRASTRUCTURE.  Only the test-suite, the package smoke check
// and the benchmark's CPU-baseline leg may load it.  It shares no code,
// header, table or constant generator with the CUDA library; the two agree
// only because both follow the same written definitions.
//
// Sources (page title, section):
//  * "MiniMax Music 3 on Metal" (TensorFold PR), section "Precision is the
//    reference's": bf16 activations with bf16 roundings where torch rounds,
//    fp32 norms / softmax / rope / attention sums; int8 weight-only with one
//    scale per row (body, lm_head) or per group of 128 (depth decoder),
//    quantised at load.
//  * "MiniMax-Music3 ... DiffSynth-Studio" (Chinese article), sections
//    "各子模型的结构要点" (Qwen3ForCausalLM: hidden 4096, 36 layers, 32 heads,
//    8 KV heads, rope_theta 1e6; depth decoder 4 layers, 16 heads, 7 residual
//    codebooks) and "第二阶段" (vocab mask to the audio codes, CFG
//    guided = uncond + c*(cond - uncond), depth codes drawn one by one).
//  * "MiniMax Music 3 modular pipeline: 2.9x consumer-GPU speedup" (diffusers
//    issue), finding 3: lm_head sliced to the sampleable rows is identical to
//    masking the others to -inf; softmax+multinomial replaced by
//    Gumbel-argmax, which draws from the same distribution.
//
// Arithmetic rules (so that a reader can check them by eye):
//  * every dot product / sum is a sequential fp32 loop in index order;
//  * bf16(v) is round-to-nearest-even of the fp32 value v;
//  * build with -ffp-contract=off: no multiply-add is fused unless written
//    as std::fma;
//  * the Gumbel noise is computed in fp64 with an ln() written from the
//    atanh series (ln m = 2 atanh((m-1)/(m+1))), so that it is reproducible
//    bit for bit by any IEEE-754 implementation of +,-,*,/ and fma.
//
// Parity pins for every function live in tests/test_oracle_*.py.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <cstdlib>
#include <vector>
#include <algorithm>
#include <limits>

#ifdef _OPENMP
#include <omp.h>
#endif

typedef uint16_t bf16_t;   // raw bf16 bits
typedef uint16_t f16_t;    // raw IEEE binary16 bits

// ---------------------------------------------------------------- numbers --

static inline float bf2f(bf16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

static inline bf16_t f2bf(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (bf16_t)((u >> 16) | 0x40);  // quiet NaN
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;  // round to nearest, ties to even
  return (bf16_t)(u >> 16);
}

static inline float rbf(float f) { return bf2f(f2bf(f)); }  // fp32 -> bf16 -> fp32

static inline f16_t f2h(float f) {
  _Float16 h = (_Float16)f;  // IEEE RNE conversion (compiler / F16C)
  f16_t b;
  std::memcpy(&b, &h, 2);
  return b;
}

static inline float h2f(f16_t b) {
  _Float16 h;
  std::memcpy(&h, &b, 2);
  return (float)h;
}

extern "C" {

uint16_t ora_f2bf(float f) { return f2bf(f); }
float ora_bf2f(uint16_t h) { return bf2f(h); }
uint16_t ora_f2h(float f) { return f2h(f); }
float ora_h2f(uint16_t h) { return h2f(h); }

// ------------------------------------------------------- Gumbel noise ------
// Counter-based generator: the SplitMix64 output function of Steele, Lea and
// Flood ("Fast splittable pseudorandom number generators", OOPSLA 2014), in
// the public-domain form by S. Vigna; mix(z) is one SplitMix64 step applied
// to state z.
uint64_t ora_mix64(uint64_t z) {
  z += 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// 64 random bits for (seed, frame, row, index).
uint64_t ora_noise_bits(uint64_t seed, uint64_t frame, uint64_t row, uint64_t index) {
  uint64_t b = ora_mix64(seed);
  b = ora_mix64(b ^ frame);
  b = ora_mix64(b ^ row);
  b = ora_mix64(b ^ index);
  return b;
}

// Uniform in the open interval (0, 1): the top 24 bits, centred in their cell.
double ora_uniform(uint64_t bits) {
  return ((double)(bits >> 40) + 0.5) * 0x1p-24;
}

// Natural logarithm of a positive, normal double from the series
//   ln m = 2 * sum_{k>=0} t^(2k+1) / (2k+1),  t = (m-1)/(m+1)
// with x = m * 2^e, m in [1/sqrt2, sqrt2), so |t| <= 0.1716 and 13 terms
// leave a truncation error below 1e-19.
double ora_ln(double x) {
  uint64_t bits;
  std::memcpy(&bits, &x, 8);
  int e = (int)((bits >> 52) & 0x7FF) - 1023;
  uint64_t mb = (bits & 0x000FFFFFFFFFFFFFull) | 0x3FF0000000000000ull;  // m in [1, 2)
  double m;
  std::memcpy(&m, &mb, 8);
  if (m >= 1.4142135623730951) {  // sqrt(2), correctly rounded
    m = m * 0.5;
    e += 1;
  }
  double t = (m - 1.0) / (m + 1.0);
  double t2 = t * t;
  double p = 1.0 / 25.0;  // k = 12
  for (int k = 11; k >= 0; --k) p = std::fma(p, t2, 1.0 / (double)(2 * k + 1));
  double lnm = (2.0 * t) * p;
  const double LN2 = 0.6931471805599453;  // 0x3FE62E42FEFA39EF
  return std::fma((double)e, LN2, lnm);
}

// Standard Gumbel sample G = -ln(-ln u), rounded to fp32.
float ora_gumbel(uint64_t seed, uint64_t frame, uint64_t row, uint64_t index) {
  double u = ora_uniform(ora_noise_bits(seed, frame, row, index));
  double a = -ora_ln(u);
  double g = -ora_ln(a);
  return (float)g;
}

// G(seed, frame, row, index0 + i) for i < n.
void ora_gumbel_fill(uint64_t seed, uint64_t frame, uint64_t row, uint64_t index0, int64_t n,
                     float* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = ora_gumbel(seed, frame, row, index0 + (uint64_t)i);
}

// ---------------------------------------------------- int8 quantiser -------
// One symmetric scale per group of `group` consecutive elements of a row
// (group == cols gives one scale per row):
//   s = absmax / 127 (fp32), q = clamp(rint(w / s), -127, 127); s == 0 -> q = 0.
void ora_quantize(const bf16_t* w, int64_t rows, int64_t cols, int64_t group,
                  int8_t* q, float* s) {
  int64_t ng = cols / group;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t g = 0; g < ng; ++g) {
      const bf16_t* src = w + r * cols + g * group;
      float amax = 0.0f;
      for (int64_t i = 0; i < group; ++i) amax = std::max(amax, std::fabs(bf2f(src[i])));
      float sc = amax / 127.0f;
      s[r * ng + g] = sc;
      int8_t* dst = q + r * cols + g * group;
      for (int64_t i = 0; i < group; ++i) {
        if (sc == 0.0f) {
          dst[i] = 0;
        } else {
          float v = std::rint(bf2f(src[i]) / sc);
          v = std::min(127.0f, std::max(-127.0f, v));
          dst[i] = (int8_t)v;
        }
      }
    }
  }
}

// ------------------------------------------------------------ GEMV ---------
// y[o] = sum_i W[o,i] * x[i], sequential fp32 sum.  Weight formats:
//   wfmt 0: bf16 W;  wfmt 1: int8 q with one scale per row, y = s_o * sum q x;
//   wfmt 2: int8 q with one scale per group of 128, y = sum_g s_og * (sum_{i in g} q x).
struct OraMat {
  const bf16_t* w;   // bf16 [rows, cols] (wfmt 0)
  const int8_t* q;   // int8 [rows, cols] (wfmt 1, 2)
  const float* s;    // fp32 [rows] or [rows, cols/128]
  int wfmt;
};

// The summation-order comparator: with g_acc64 set, every GEMV sum runs in
// fp64 (each product exact, one rounding to fp32 at the end) instead of the
// sequential fp32 loop.  It is the same definition computed with a different
// (more accurate) summation, used by the tests to measure how far two
// correct summation orders of the same frame drift apart after many layers.
static int g_acc64 = 0;

static void gemv64(const OraMat& m, int64_t rows, int64_t cols, const float* x, float* y) {
#pragma omp parallel for schedule(static)
  for (int64_t o = 0; o < rows; ++o) {
    double tot = 0.0;
    if (m.wfmt == 0) {
      const bf16_t* wr = m.w + o * cols;
      for (int64_t i = 0; i < cols; ++i) tot += (double)bf2f(wr[i]) * (double)x[i];
    } else if (m.wfmt == 1) {
      const int8_t* qr = m.q + o * cols;
      for (int64_t i = 0; i < cols; ++i) tot += (double)qr[i] * (double)x[i];
      tot *= (double)m.s[o];
    } else {
      const int8_t* qr = m.q + o * cols;
      int64_t ng = cols / 128;
      for (int64_t g = 0; g < ng; ++g) {
        double acc = 0.0;
        for (int64_t i = g * 128; i < g * 128 + 128; ++i) acc += (double)qr[i] * (double)x[i];
        tot += (double)m.s[o * ng + g] * acc;
      }
    }
    y[o] = (float)tot;
  }
}

static void gemv(const OraMat& m, int64_t rows, int64_t cols, const float* x, float* y) {
  if (g_acc64) {
    gemv64(m, rows, cols, x, y);
    return;
  }
#pragma omp parallel for schedule(static)
  for (int64_t o = 0; o < rows; ++o) {
    if (m.wfmt == 0) {
      const bf16_t* wr = m.w + o * cols;
      float acc = 0.0f;
      for (int64_t i = 0; i < cols; ++i) acc = acc + bf2f(wr[i]) * x[i];
      y[o] = acc;
    } else if (m.wfmt == 1) {
      const int8_t* qr = m.q + o * cols;
      float acc = 0.0f;
      for (int64_t i = 0; i < cols; ++i) acc = acc + (float)qr[i] * x[i];
      y[o] = m.s[o] * acc;
    } else {
      const int8_t* qr = m.q + o * cols;
      int64_t ng = cols / 128;
      float tot = 0.0f;
      for (int64_t g = 0; g < ng; ++g) {
        float acc = 0.0f;
        for (int64_t i = g * 128; i < g * 128 + 128; ++i) acc = acc + (float)qr[i] * x[i];
        tot = tot + m.s[o * ng + g] * acc;
      }
      y[o] = tot;
    }
  }
}

void ora_gemv(const bf16_t* w, const int8_t* q, const float* s, int wfmt, int64_t rows,
              int64_t cols, const float* x, float* y) {
  OraMat m{w, q, s, wfmt};
  gemv(m, rows, cols, x, y);
}

// 0: sequential fp32 GEMV sums (the oracle's definition); 1: fp64 sums.
void ora_set_accum64(int on) { g_acc64 = on ? 1 : 0; }

// ------------------------------------------------------------ norms --------
// RMSNorm as torch's Qwen3RMSNorm computes it on a bf16 tensor:
//   r = 1 / sqrt(mean(x^2) + eps)   (fp32)
//   out = bf16( gamma * bf16(x * r) )
void ora_rmsnorm(const float* x, const bf16_t* gamma, int64_t n, float eps, float* out) {
  float ss = 0.0f;
  for (int64_t i = 0; i < n; ++i) ss = ss + x[i] * x[i];
  float r = 1.0f / std::sqrt(ss / (float)n + eps);
  for (int64_t i = 0; i < n; ++i) out[i] = rbf(bf2f(gamma[i]) * rbf(x[i] * r));
}

// --------------------------------------------------------------- RoPE ------
// Half-rotation ("rotate_half") rotary embedding over a head of size d:
// pairs (i, i + d/2), angle pos * theta^(-2i/d) in fp64, rotation in fp32.
void ora_rope(float* v, int d, int64_t pos, double theta) {
  int h = d / 2;
  for (int i = 0; i < h; ++i) {
    double ang = (double)pos * std::pow(theta, -2.0 * (double)i / (double)d);
    float c = (float)std::cos(ang);
    float s = (float)std::sin(ang);
    float a = v[i], b = v[i + h];
    v[i] = a * c - b * s;
    v[i + h] = b * c + a * s;
  }
}

// ---------------------------------------------------------- attention ------
// One query head against n cached positions (keys/values already decoded to
// fp32): s_j = (q . k_j) / sqrt(d); p = softmax(s); out = sum_j p_j v_j.
void ora_attention(const float* q, const float* k, const float* v, int64_t n, int d,
                   float* out) {
  std::vector<float> s(n);
  float scale = 1.0f / std::sqrt((float)d);
  float m = -std::numeric_limits<float>::infinity();
  for (int64_t j = 0; j < n; ++j) {
    float acc = 0.0f;
    for (int i = 0; i < d; ++i) acc = acc + q[i] * k[j * d + i];
    s[j] = acc * scale;
    m = std::max(m, s[j]);
  }
  float l = 0.0f;
  for (int64_t j = 0; j < n; ++j) {
    s[j] = std::exp(s[j] - m);
    l = l + s[j];
  }
  for (int i = 0; i < d; ++i) {
    float acc = 0.0f;
    for (int64_t j = 0; j < n; ++j) acc = acc + s[j] * v[j * d + i];
    out[i] = acc / l;
  }
}

static inline float silu(float g) { return g / (1.0f + std::exp(-g)); }

// --------------------------------------------------------- the frame -------
struct OraCfg {
  int hidden, n_layers, n_q_heads, n_kv_heads, head_dim, ffn;
  int slice_start, slice_len;  // sampleable vocab rows [slice_start, +slice_len)
  double rope_theta;
  float rms_eps;
  int wfmt;    // 0 bf16, 1 int8 per row
  int kv_f16;  // 0 bf16 cache, 1 f16 cache
  // The end token (DiffSynth-Studio article, "第二阶段": the vocab mask
  // leaves the audio codes and the end token sampleable): with has_end the
  // lm_head holds slice_len + 1 rows, the last being vocab row end_token,
  // drawn as slice-relative code slice_len.
  int has_end;
  int end_token;
};

struct OraLayer {
  const bf16_t* attn_norm;  // [H]
  OraMat wq, wk, wv;        // [Hq*d, H], [Hkv*d, H], [Hkv*d, H]
  const bf16_t* q_norm;     // [d]
  const bf16_t* k_norm;     // [d]
  OraMat wo;                // [H, Hq*d]
  const bf16_t* mlp_norm;   // [H]
  OraMat wg, wu;            // [I, H]
  OraMat wd;                // [H, I]
};

static inline float kv_load(const uint16_t* p, int f16) { return f16 ? h2f(*p) : bf2f(*p); }
static inline uint16_t kv_store(float v, int f16) { return f16 ? f2h(v) : f2bf(v); }

// One decoder layer for one row.  x: [H] fp32 holding bf16 values (updated).
// kc / vc: this row's cache for this layer, [max_pos, Hkv, d].
static void layer_row(const OraCfg& c, const OraLayer& L, float* x, uint16_t* kc, uint16_t* vc,
                      int64_t pos) {
  const int H = c.hidden, d = c.head_dim, Hq = c.n_q_heads, Hkv = c.n_kv_heads, I = c.ffn;
  const int grp = Hq / Hkv;
  std::vector<float> n(H), q(Hq * d), k(Hkv * d), v(Hkv * d), o(Hq * d), t(H);
  ora_rmsnorm(x, L.attn_norm, H, c.rms_eps, n.data());
  gemv(L.wq, Hq * d, H, n.data(), q.data());
  gemv(L.wk, Hkv * d, H, n.data(), k.data());
  gemv(L.wv, Hkv * d, H, n.data(), v.data());
  for (auto& e : q) e = rbf(e);
  for (auto& e : k) e = rbf(e);
  for (auto& e : v) e = rbf(e);
  std::vector<float> tmp(d);
  for (int h = 0; h < Hq; ++h) {
    ora_rmsnorm(&q[h * d], L.q_norm, d, c.rms_eps, tmp.data());
    ora_rope(tmp.data(), d, pos, c.rope_theta);
    for (int i = 0; i < d; ++i) q[h * d + i] = rbf(tmp[i]);
  }
  for (int g = 0; g < Hkv; ++g) {
    ora_rmsnorm(&k[g * d], L.k_norm, d, c.rms_eps, tmp.data());
    ora_rope(tmp.data(), d, pos, c.rope_theta);
    for (int i = 0; i < d; ++i) k[g * d + i] = rbf(tmp[i]);
  }
  for (int g = 0; g < Hkv; ++g)
    for (int i = 0; i < d; ++i) {
      kc[(pos * Hkv + g) * d + i] = kv_store(k[g * d + i], c.kv_f16);
      vc[(pos * Hkv + g) * d + i] = kv_store(v[g * d + i], c.kv_f16);
    }
  int64_t n_ctx = pos + 1;
  std::vector<float> K(n_ctx * d), V(n_ctx * d);
  for (int h = 0; h < Hq; ++h) {
    int g = h / grp;
    for (int64_t j = 0; j < n_ctx; ++j)
      for (int i = 0; i < d; ++i) {
        K[j * d + i] = kv_load(&kc[(j * Hkv + g) * d + i], c.kv_f16);
        V[j * d + i] = kv_load(&vc[(j * Hkv + g) * d + i], c.kv_f16);
      }
    ora_attention(&q[h * d], K.data(), V.data(), n_ctx, d, &o[h * d]);
    for (int i = 0; i < d; ++i) o[h * d + i] = rbf(o[h * d + i]);
  }
  gemv(L.wo, H, Hq * d, o.data(), t.data());
  for (int i = 0; i < H; ++i) x[i] = rbf(x[i] + rbf(t[i]));
  ora_rmsnorm(x, L.mlp_norm, H, c.rms_eps, n.data());
  std::vector<float> gg(I), uu(I), a(I);
  gemv(L.wg, I, H, n.data(), gg.data());
  gemv(L.wu, I, H, n.data(), uu.data());
  for (int j = 0; j < I; ++j) a[j] = rbf(rbf(silu(rbf(gg[j]))) * rbf(uu[j]));
  gemv(L.wd, H, I, a.data(), t.data());
  for (int i = 0; i < H; ++i) x[i] = rbf(x[i] + rbf(t[i]));
}

// Gumbel-argmax draw over `n` guided logits g (fp32), noise keyed by
// (seed, frame, key_row, index_base | i).  Returns the smallest i holding the
// maximum of z_i = g_i / T + G_i.
static int64_t gumbel_argmax(const float* g, int64_t n, float temperature, uint64_t seed,
                             uint64_t frame, uint64_t key_row, uint64_t index_base,
                             float* zmax_out) {
  int64_t best = -1;
  float bz = -std::numeric_limits<float>::infinity();
  for (int64_t i = 0; i < n; ++i) {
    float z = g[i] / temperature + ora_gumbel(seed, frame, key_row, index_base + (uint64_t)i);
    if (best < 0 || z > bz) {
      bz = z;
      best = i;
    }
  }
  if (zmax_out) *zmax_out = bz;
  return best;
}

// Top-k filtering before the draw (the AR sampler's "CFG 1.5, top-k 50,
// multinomial" in the DiffSynth-Studio article, "第二阶段"): keep the k
// largest guided logits -- ties at the k-th value broken towards the lower
// index -- and draw among them by Gumbel-argmax; k <= 0 or k >= n keeps all.
// The kept indices, ascending.
static std::vector<int64_t> topk_set(const float* g, int64_t n, int64_t k) {
  std::vector<int64_t> idx(n);
  for (int64_t i = 0; i < n; ++i) idx[i] = i;
  std::stable_sort(idx.begin(), idx.end(), [&](int64_t a, int64_t b) { return g[a] > g[b]; });
  idx.resize(k);
  std::sort(idx.begin(), idx.end());
  return idx;
}

// Noise index of candidate i of a draw: index_base + i, except candidate
// end_i (the end token, when the draw has one), whose index is end_index.
struct NoiseIndex {
  uint64_t base;
  int64_t end_i;  // -1: none
  uint64_t end_index;
  uint64_t at(int64_t i) const { return i == end_i ? end_index : base + (uint64_t)i; }
};

// The draw over the kept set; margin_out (nullable): best minus second-best z
// over the kept set.
static int64_t topk_gumbel_argmax(const float* g, int64_t n, int64_t k, float temperature,
                                  uint64_t seed, uint64_t frame, uint64_t key_row,
                                  NoiseIndex index, float* margin_out) {
  std::vector<int64_t> keep;
  if (k > 0 && k < n) {
    keep = topk_set(g, n, k);
  } else {
    keep.resize(n);
    for (int64_t i = 0; i < n; ++i) keep[i] = i;
  }
  int64_t best = -1;
  float b1 = -INFINITY, b2 = -INFINITY;
  for (int64_t i : keep) {
    float z = g[i] / temperature + ora_gumbel(seed, frame, key_row, index.at(i));
    if (best < 0 || z > b1) {
      b2 = b1;
      b1 = z;
      best = i;
    } else if (z > b2) {
      b2 = z;
    }
  }
  if (margin_out) *margin_out = b1 - b2;
  return best;
}

// One top-k draw from given guided logits g [n] (the sampler's decision on
// another implementation's logits).
int32_t ora_topk_draw(const float* g, int64_t n, int64_t k, float temperature, uint64_t seed,
                      uint64_t frame, uint64_t key_row, uint64_t index_base) {
  return (int32_t)topk_gumbel_argmax(g, n, k, temperature, seed, frame, key_row,
                                     NoiseIndex{index_base, -1, 0}, nullptr);
}

// Repeated top-k draws from fixed logits (frame = frame0 + t, key_row 0).
void ora_topk_draws(const float* logits, int64_t n, int64_t k, float temperature, uint64_t seed,
                    uint64_t frame0, int64_t ndraws, int32_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < ndraws; ++t)
    out[t] = (int32_t)topk_gumbel_argmax(logits, n, k, temperature, seed, frame0 + (uint64_t)t, 0,
                                         NoiseIndex{0, -1, 0}, nullptr);
}

// The draw on given per-row logits [rows, n] (another implementation's
// logits): with cfg_scale > 0 the rows are (cond, uncond) pairs and
// g = l_u + c (l_c - l_u) is drawn once per pair with key_row = pair index
// (both rows get the code); else g = l with key_row = row.  Candidate i has
// noise index index_base + i, except candidate end_i (>= 0), whose index is
// end_index.  margin (nullable): per row the gap between the best and the
// second-best z.  Returns -1 when cfg_scale > 0 and rows is odd.
int ora_draw(const float* logits, int rows, int64_t n, float cfg_scale, float temperature,
             int top_k, uint64_t seed, uint64_t frame, uint64_t index_base, int64_t end_i,
             uint64_t end_index, int32_t* codes, float* margin) {
  if (cfg_scale > 0.0f && (rows % 2)) return -1;
  const NoiseIndex ni{index_base, end_i, end_index};
  const int npick = cfg_scale > 0.0f ? rows / 2 : rows;
  std::vector<float> g(n);
  for (int p = 0; p < npick; ++p) {
    if (cfg_scale > 0.0f) {
      const float* lc = logits + (size_t)(2 * p) * n;
      const float* lu = logits + (size_t)(2 * p + 1) * n;
      for (int64_t i = 0; i < n; ++i) g[i] = lu[i] + cfg_scale * (lc[i] - lu[i]);
    } else {
      std::memcpy(g.data(), logits + (size_t)p * n, sizeof(float) * n);
    }
    float mg = 0.0f;
    const int64_t best = topk_gumbel_argmax(g.data(), n, top_k, temperature, seed, frame,
                                            (uint64_t)p, ni, &mg);
    const int rr[2] = {cfg_scale > 0.0f ? 2 * p : p, cfg_scale > 0.0f ? 2 * p + 1 : -1};
    for (int q = 0; q < 2; ++q) {
      if (rr[q] < 0) continue;
      codes[rr[q]] = (int32_t)best;
      if (margin) margin[rr[q]] = mg;
    }
  }
  return 0;
}

// Repeated draws from fixed logits: draw t uses frame = frame0 + t and
// key_row 0.  Used to check the draw against the categorical distribution.
void ora_gumbel_argmax_draws(const float* logits, int64_t n, float temperature, uint64_t seed,
                             uint64_t frame0, int64_t ndraws, int32_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < ndraws; ++t)
    out[t] = (int32_t)gumbel_argmax(logits, n, temperature, seed, frame0 + (uint64_t)t, 0, 0,
                                    nullptr);
}

// The sampler on given final hidden states hf [rows, H] (bf16 bits):
// logits l = W_lm[slice] hf in fp32 (not rounded); if cfg_scale > 0 the rows
// are (cond, uncond) pairs and g = l_u + c (l_c - l_u) is drawn once per pair
// with key_row = pair index, both rows receiving the code; else g = l with
// key_row = row.  Codes are slice-relative.  Noise index = slice_start + i.
// With the end token (cfg->has_end) there are S + 1 candidates, the last one
// being the end token (code S, noise index end_token); ties between it and a
// code go to the code.
// logits (nullable) receives the raw per-row logits [rows, S (+1)];
// margin (nullable) receives per row the gap between the best and second-best z.
int ora_sample(const OraCfg* cfg, OraMat lm, int rows, const bf16_t* hf, uint64_t seed,
               uint64_t frame, float cfg_scale, float temperature, int top_k, int32_t* codes,
               float* logits, float* margin) {
  const int H = cfg->hidden, S = cfg->slice_len + (cfg->has_end ? 1 : 0);
  const NoiseIndex ni{(uint64_t)cfg->slice_start, cfg->has_end ? (int64_t)cfg->slice_len : -1,
                      (uint64_t)cfg->end_token};
  if (cfg_scale > 0.0f && (rows % 2)) return -1;
  std::vector<float> L((size_t)rows * S), h(H);
  for (int r = 0; r < rows; ++r) {
    for (int i = 0; i < H; ++i) h[i] = bf2f(hf[(size_t)r * H + i]);
    gemv(lm, S, H, h.data(), &L[(size_t)r * S]);
  }
  if (logits) std::memcpy(logits, L.data(), sizeof(float) * L.size());
  int npick = cfg_scale > 0.0f ? rows / 2 : rows;
  std::vector<float> g(S), z(S);
  for (int p = 0; p < npick; ++p) {
    if (cfg_scale > 0.0f) {
      const float* lc = &L[(size_t)(2 * p) * S];
      const float* lu = &L[(size_t)(2 * p + 1) * S];
      for (int i = 0; i < S; ++i) g[i] = lu[i] + cfg_scale * (lc[i] - lu[i]);
    } else {
      std::memcpy(g.data(), &L[(size_t)p * S], sizeof(float) * S);
    }
    float mg = 0.0f;
    int64_t best = topk_gumbel_argmax(g.data(), S, top_k, temperature, seed, frame, (uint64_t)p,
                                      ni, &mg);
    if (margin) {
      if (cfg_scale > 0.0f) { margin[2 * p] = mg; margin[2 * p + 1] = mg; }
      else margin[p] = mg;
    }
    if (cfg_scale > 0.0f) {
      codes[2 * p] = (int32_t)best;
      codes[2 * p + 1] = (int32_t)best;
    } else {
      codes[p] = (int32_t)best;
    }
  }
  return 0;
}

// The same draw over the FULL vocabulary [vocab, H] with every row outside the
// slice -- other than the end token, when there is one -- masked to -inf (the
// unsliced reference form), top-k over the whole guided vector.  Returns codes
// relative to slice_start (the end token as slice_len) so they are directly
// comparable with ora_sample.
int ora_sample_full_masked(const OraCfg* cfg, const bf16_t* lm_full, int vocab, int rows,
                           const bf16_t* hf, uint64_t seed, uint64_t frame, float cfg_scale,
                           float temperature, int top_k, int32_t* codes) {
  const int H = cfg->hidden;
  if (cfg_scale > 0.0f && (rows % 2)) return -1;
  OraMat lm{lm_full, nullptr, nullptr, 0};
  std::vector<float> L((size_t)rows * vocab), h(H);
  for (int r = 0; r < rows; ++r) {
    for (int i = 0; i < H; ++i) h[i] = bf2f(hf[(size_t)r * H + i]);
    gemv(lm, vocab, H, h.data(), &L[(size_t)r * vocab]);
    for (int i = 0; i < vocab; ++i) {
      const bool in_slice = i >= cfg->slice_start && i < cfg->slice_start + cfg->slice_len;
      const bool is_end = cfg->has_end && i == cfg->end_token;
      if (!in_slice && !is_end) L[(size_t)r * vocab + i] = -INFINITY;
    }
  }
  int npick = cfg_scale > 0.0f ? rows / 2 : rows;
  std::vector<float> g(vocab);
  for (int p = 0; p < npick; ++p) {
    for (int i = 0; i < vocab; ++i) {
      if (cfg_scale > 0.0f) {
        float lc = L[(size_t)(2 * p) * vocab + i], lu = L[(size_t)(2 * p + 1) * vocab + i];
        g[i] = (std::isinf(lc) && std::isinf(lu)) ? -INFINITY : lu + cfg_scale * (lc - lu);
      } else {
        g[i] = L[(size_t)p * vocab + i];
      }
    }
    int64_t best = topk_gumbel_argmax(g.data(), vocab, top_k, temperature, seed, frame,
                                      (uint64_t)p, NoiseIndex{0, -1, 0}, nullptr);
    int32_t rel = (cfg->has_end && best == cfg->end_token) ? (int32_t)cfg->slice_len
                                                            : (int32_t)(best - cfg->slice_start);
    if (cfg_scale > 0.0f) { codes[2 * p] = rel; codes[2 * p + 1] = rel; }
    else codes[p] = rel;
  }
  return 0;
}

// One frame of the Global LLM for `rows` independent rows.
//   kcache / vcache: [rows, n_layers, max_pos, Hkv, d] raw bf16 or f16 bits;
//   positions[r]: the position this frame writes (attends 0..positions[r]);
//   x_in: [rows, H] bf16; codes: [rows] slice-relative;
//   h_out (nullable): [rows, H] bf16 final-normed hidden state;
//   logits (nullable): [rows, slice_len (+1 with the end token)] fp32.
int ora_decode_frame(const OraCfg* cfg, const OraLayer* layers, const bf16_t* final_norm,
                     OraMat lm, int rows, int64_t max_pos, uint16_t* kcache, uint16_t* vcache,
                     const int32_t* positions, uint64_t seed, uint64_t frame, const bf16_t* x_in,
                     float cfg_scale, float temperature, int top_k, int32_t* codes,
                     bf16_t* h_out, float* logits) {
  const int H = cfg->hidden, d = cfg->head_dim, Hkv = cfg->n_kv_heads;
  for (int r = 0; r < rows; ++r)
    if (positions[r] < 0 || positions[r] >= max_pos) return -5;
  std::vector<bf16_t> hf((size_t)rows * H);
  std::vector<float> x(H), t(H);
  const size_t layer_stride = (size_t)max_pos * Hkv * d;
  for (int r = 0; r < rows; ++r) {
    for (int i = 0; i < H; ++i) x[i] = bf2f(x_in[(size_t)r * H + i]);
    for (int l = 0; l < cfg->n_layers; ++l) {
      size_t off = ((size_t)r * cfg->n_layers + l) * layer_stride;
      layer_row(*cfg, layers[l], x.data(), kcache + off, vcache + off, positions[r]);
    }
    ora_rmsnorm(x.data(), final_norm, H, cfg->rms_eps, t.data());
    for (int i = 0; i < H; ++i) hf[(size_t)r * H + i] = f2bf(t[i]);
  }
  if (h_out) std::memcpy(h_out, hf.data(), sizeof(bf16_t) * hf.size());
  return ora_sample(cfg, lm, rows, hf.data(), seed, frame, cfg_scale, temperature, top_k, codes,
                    logits, nullptr);
}

// Only the layers (no sampler): used by tests that pin the residual wiring.
int ora_body(const OraCfg* cfg, const OraLayer* layers, int rows, int64_t max_pos,
             uint16_t* kcache, uint16_t* vcache, const int32_t* positions, const bf16_t* x_in,
             bf16_t* x_out) {
  const int H = cfg->hidden, d = cfg->head_dim, Hkv = cfg->n_kv_heads;
  std::vector<float> x(H);
  const size_t layer_stride = (size_t)max_pos * Hkv * d;
  for (int r = 0; r < rows; ++r) {
    for (int i = 0; i < H; ++i) x[i] = bf2f(x_in[(size_t)r * H + i]);
    for (int l = 0; l < cfg->n_layers; ++l) {
      size_t off = ((size_t)r * cfg->n_layers + l) * layer_stride;
      layer_row(*cfg, layers[l], x.data(), kcache + off, vcache + off, positions[r]);
    }
    for (int i = 0; i < H; ++i) x_out[(size_t)r * H + i] = f2bf(x[i]);
  }
  return 0;
}

// ---------------------------------------------------- depth decoder --------
// The RVQ depth decoder that follows each semantic code (DiffSynth-Studio
// article, "第二阶段"): a 4-layer, 16-head block of the body's kind, run over
// 8 frame-local positions:
//   position 0: proj(h_frame)              (4096 -> 1024)
//   position j (1..7): E_{j-1}[c_{j-1}]     (c_0 = the semantic code)
// after position j >= 1 the final norm and head_j give 1024 logits, and c_j is
// drawn by Gumbel-argmax with noise index (j << 32) | i.
// All GEMV weights are int8 with one scale per group of 128.
struct OraDepth {
  int hidden, n_layers, n_heads, head_dim, ffn, codebooks, vocab, in_hidden;
  double rope_theta;
  float rms_eps;
  const OraLayer* layers;   // n_kv_heads == n_heads
  OraMat proj;              // [hidden, in_hidden]
  const bf16_t* const* emb; // codebooks tables: emb[0] [sem_vocab, hidden], emb[j] [vocab, hidden]
  const bf16_t* final_norm; // [hidden]
  const OraMat* heads;      // codebooks heads [vocab, hidden]
  int sem_vocab;            // rows of emb[0]; code0 == sem_vocab (the end token's
                            // code) feeds a zero vector at position 1
};

// codes_out: [rows, codebooks]; forced (nullable): [rows, codebooks] codes to
// feed forward instead of the drawn ones (teacher forcing); logits (nullable):
// [rows, codebooks, vocab] raw per-row logits.
int ora_depth_decode(const OraDepth* D, int rows, const bf16_t* h_frame, const int32_t* code0,
                     uint64_t seed, uint64_t frame, float cfg_scale, float temperature,
                     const int32_t* forced, int32_t* codes_out, float* logits) {
  const int H = D->hidden, d = D->head_dim, nh = D->n_heads, NC = D->codebooks, V = D->vocab;
  if (cfg_scale > 0.0f && (rows % 2)) return -1;
  OraCfg c{};
  c.hidden = H; c.n_layers = D->n_layers; c.n_q_heads = nh; c.n_kv_heads = nh; c.head_dim = d;
  c.ffn = D->ffn; c.rope_theta = D->rope_theta; c.rms_eps = D->rms_eps; c.wfmt = 2; c.kv_f16 = 0;
  const int P = NC + 1;  // positions per frame
  const size_t lstride = (size_t)P * nh * d;
  std::vector<uint16_t> kc((size_t)rows * D->n_layers * lstride), vc(kc.size());
  std::vector<float> x((size_t)rows * H), hin(D->in_hidden), t(H), L((size_t)rows * V), g(V);
  std::vector<int32_t> prev(rows);
  for (int r = 0; r < rows; ++r) {
    for (int i = 0; i < D->in_hidden; ++i) hin[i] = bf2f(h_frame[(size_t)r * D->in_hidden + i]);
    gemv(D->proj, H, D->in_hidden, hin.data(), &x[(size_t)r * H]);
    for (int i = 0; i < H; ++i) x[(size_t)r * H + i] = rbf(x[(size_t)r * H + i]);
    prev[r] = code0[r];
  }
  for (int j = 0; j < P; ++j) {
    for (int r = 0; r < rows; ++r) {
      float* xr = &x[(size_t)r * H];
      if (j > 0) {
        if (j == 1 && prev[r] == D->sem_vocab) {
          for (int i = 0; i < H; ++i) xr[i] = 0.0f;
        } else {
          const bf16_t* e = D->emb[j - 1] + (size_t)prev[r] * H;
          for (int i = 0; i < H; ++i) xr[i] = bf2f(e[i]);
        }
      }
      for (int l = 0; l < D->n_layers; ++l) {
        size_t off = ((size_t)r * D->n_layers + l) * lstride;
        layer_row(c, D->layers[l], xr, kc.data() + off, vc.data() + off, j);
      }
      if (j > 0) {
        std::vector<float> hf(H);
        ora_rmsnorm(xr, D->final_norm, H, D->rms_eps, hf.data());
        gemv(D->heads[j - 1], V, H, hf.data(), &L[(size_t)r * V]);
        if (logits) std::memcpy(&logits[((size_t)r * NC + (j - 1)) * V], &L[(size_t)r * V],
                                sizeof(float) * V);
      }
    }
    if (j == 0) continue;
    int npick = cfg_scale > 0.0f ? rows / 2 : rows;
    for (int p = 0; p < npick; ++p) {
      if (cfg_scale > 0.0f) {
        for (int i = 0; i < V; ++i) {
          float lc = L[(size_t)(2 * p) * V + i], lu = L[(size_t)(2 * p + 1) * V + i];
          g[i] = lu + cfg_scale * (lc - lu);
        }
      } else {
        std::memcpy(g.data(), &L[(size_t)p * V], sizeof(float) * V);
      }
      int64_t best = gumbel_argmax(g.data(), V, temperature, seed, frame, (uint64_t)p,
                                   (uint64_t)j << 32, nullptr);
      int rr[2] = {cfg_scale > 0.0f ? 2 * p : p, cfg_scale > 0.0f ? 2 * p + 1 : -1};
      for (int q = 0; q < 2; ++q) {
        if (rr[q] < 0) continue;
        codes_out[(size_t)rr[q] * NC + (j - 1)] = (int32_t)best;
        prev[rr[q]] = forced ? forced[(size_t)rr[q] * NC + (j - 1)] : (int32_t)best;
      }
    }
  }
  return 0;
}

// ------------------------------------------------- the multi-frame loop ----
// The autoregressive loop of the Global LLM (DiffSynth-Studio article,
// "第二阶段": each frame's codes are embedded back as the next input and the
// loop stops early at the end token, an error if no frame came out;
// "MiniMax Music 3 on Metal": position, step and count advance frame by
// frame).  Frame f = 0, 1, ... runs every row at position positions[r] + f
// with noise frame frame0 + f:
//   1. the Global LLM frame gives code0 per row and its final hidden state hf;
//   2. with a depth decoder (D non-null), its NC residual codes from (hf, code0);
//   3. the next input (the article's embed_audio_frame): the token embedding
//      of code0 plus the residual codebooks' audio embeddings, scaled by
//      (1 + NC)^-0.5 -- the article's 8^-0.5 for its 8 codebooks:
//        x = bf16(s * (tok_emb[code0] + audio_emb[0][code_1] + ... + audio_emb[NC-1][code_NC]))
//      with the sum in fp32 in that order and s = fp32(1 / sqrt(1 + NC)).
// A key (a CFG pair, or a row without CFG) stops at the first frame whose
// code0 is the end token (code slice_len); its count is the number of frames
// before that one.  The loop ends once every key has stopped, or after
// max_frames frames.  A stopped key's rows keep being computed, on a zero
// input, as rows of a lockstep batch are.
//   tok_emb [slice_len, H] bf16: embed_tokens rows slice_start..;
//   audio_emb: NC tables [D->vocab, H] bf16 (unused without D);
//   forced (nullable) [max_frames, rows, 1 + NC]: teacher forcing -- these
//     codes are fed forward (and stopped on) instead of the drawn ones; a
//     negative entry (as in this loop's own -1 fill) stands for the drawn
//     semantic code, or for residual code 0 (only ever read for rows whose
//     output is not recorded);
//   codes_out [max_frames, rows, 1 + NC]: the drawn code0 and residual codes
//     of every frame a row's key runs; on its end frame the residual entries
//     are -1; -1 everywhere after that;
//   h_hist (nullable) [max_frames, rows, H] bf16: hf of every frame a row's
//     key runs (end frame included), zeros after;
//   n_frames [keys].
// Returns 0; -1 on bad arguments or a fed code out of range; -5 if a
// position would reach max_pos; -8 if some key stopped at frame 0.
int ora_generate(const OraCfg* cfg, const OraLayer* layers, const bf16_t* final_norm, OraMat lm,
                 const OraDepth* D, const bf16_t* tok_emb, const bf16_t* const* audio_emb,
                 int rows, int64_t max_pos, uint16_t* kcache, uint16_t* vcache,
                 const int32_t* positions, uint64_t seed, uint64_t frame0, const bf16_t* x_in,
                 float cfg_scale, float temperature, int top_k, int max_frames,
                 const int32_t* forced, int32_t* codes_out, bf16_t* h_hist, int32_t* n_frames) {
  const int H = cfg->hidden, S = cfg->slice_len;
  const int NC = D ? D->codebooks : 0, W = 1 + NC;
  const bool cfg_on = cfg_scale > 0.0f;
  if (rows < 1 || max_frames < 0 || (cfg_on && (rows % 2))) return -1;
  const int keys = cfg_on ? rows / 2 : rows;
  for (int r = 0; r < rows; ++r)
    if (positions[r] < 0 || (int64_t)positions[r] + max_frames > max_pos) return -5;
  const float sc = (float)(1.0 / std::sqrt((double)(1 + NC)));
  std::vector<bf16_t> x(x_in, x_in + (size_t)rows * H), hf((size_t)rows * H);
  std::vector<int32_t> pos(rows), code0(rows), c0(rows), fed((size_t)rows * W);
  std::vector<int32_t> dcodes((size_t)rows * (NC ? NC : 1)), fz((size_t)rows * (NC ? NC : 1));
  std::vector<int> active(keys, 1);
  for (int k = 0; k < keys; ++k) n_frames[k] = 0;
  for (size_t i = 0; i < (size_t)max_frames * rows * W; ++i) codes_out[i] = -1;
  if (h_hist) std::memset(h_hist, 0, sizeof(bf16_t) * (size_t)max_frames * rows * H);
  for (int f = 0; f < max_frames; ++f) {
    bool any = false;
    for (int k = 0; k < keys; ++k) any = any || active[k];
    if (!any) break;
    const uint64_t frame = frame0 + (uint64_t)f;
    for (int r = 0; r < rows; ++r) pos[r] = positions[r] + f;
    int rc = ora_decode_frame(cfg, layers, final_norm, lm, rows, max_pos, kcache, vcache,
                              pos.data(), seed, frame, x.data(), cfg_scale, temperature, top_k,
                              code0.data(), hf.data(), nullptr);
    if (rc) return rc;
    const int32_t* fr = forced ? forced + (size_t)f * rows * W : nullptr;
    for (int r = 0; r < rows; ++r)
      c0[r] = fr && fr[(size_t)r * W] >= 0 ? fr[(size_t)r * W] : code0[r];
    if (NC) {
      for (int r = 0; r < rows; ++r)
        for (int j = 0; j < NC; ++j)
          fz[(size_t)r * NC + j] = fr && fr[(size_t)r * W + 1 + j] > 0 ? fr[(size_t)r * W + 1 + j] : 0;
      rc = ora_depth_decode(D, rows, hf.data(), c0.data(), seed, frame, cfg_scale, temperature,
                            fr ? fz.data() : nullptr, dcodes.data(), nullptr);
      if (rc) return rc;
    }
    for (int r = 0; r < rows; ++r) {
      fed[(size_t)r * W] = c0[r];
      for (int j = 0; j < NC; ++j)
        fed[(size_t)r * W + 1 + j] = fr ? fz[(size_t)r * NC + j] : dcodes[(size_t)r * NC + j];
    }
    // this frame's record, for the rows whose key still runs
    for (int r = 0; r < rows; ++r) {
      if (!active[cfg_on ? r / 2 : r]) continue;
      const bool ends = cfg->has_end && fed[(size_t)r * W] == S;
      int32_t* out = codes_out + ((size_t)f * rows + r) * W;
      out[0] = code0[r];
      for (int j = 0; j < NC; ++j) out[1 + j] = ends ? -1 : dcodes[(size_t)r * NC + j];
      if (h_hist)
        std::memcpy(h_hist + ((size_t)f * rows + r) * H, &hf[(size_t)r * H], sizeof(bf16_t) * H);
    }
    // the stop rule and the counts
    for (int k = 0; k < keys; ++k) {
      if (!active[k]) continue;
      const int r = cfg_on ? 2 * k : k;
      if (cfg->has_end && fed[(size_t)r * W] == S) active[k] = 0;
      else n_frames[k] += 1;
    }
    // the next frame's input
    for (int r = 0; r < rows; ++r) {
      bf16_t* xr = &x[(size_t)r * H];
      if (!active[cfg_on ? r / 2 : r]) {
        for (int i = 0; i < H; ++i) xr[i] = 0;
        continue;
      }
      const int32_t* cr = &fed[(size_t)r * W];
      if (cr[0] < 0 || cr[0] >= S) return -1;
      for (int j = 0; j < NC; ++j)
        if (cr[1 + j] < 0 || cr[1 + j] >= D->vocab) return -1;
      for (int i = 0; i < H; ++i) {
        float t = bf2f(tok_emb[(size_t)cr[0] * H + i]);
        for (int j = 0; j < NC; ++j) t += bf2f(audio_emb[j][(size_t)cr[1 + j] * H + i]);
        xr[i] = f2bf(t * sc);
      }
    }
  }
  for (int k = 0; k < keys; ++k)
    if (n_frames[k] == 0) return -8;
  return 0;
}

int ora_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void ora_set_num_threads(int n) {
#ifdef _OPENMP
  omp_set_num_threads(n);
#else
  (void)n;
#endif
}

}  // extern "C"
