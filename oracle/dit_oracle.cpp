// dit_oracle.cpp -- plain, slow, obviously-correct CPU oracle of one
// chunk-denoise step of MiniMax Music 3's flow-matching DiT (the second
// workload of the build, next to the autoregressive decode of m3_oracle.cpp).
//
// THIS IS TEST INFRASTRUCTURE.  Only the test-suite and the benchmark's
// CPU-baseline leg may load it.  It shares no code with the CUDA library.
//
// Sources (page title, section):
//  * "MiniMax-Music3 ... DiffSynth-Studio" (Chinese article):
//    - "各子模型的结构要点": the DiT is a 36-layer Transformer with 32 heads of
//      64 and an FFN of 8192; its input concatenates the noisy latent and the
//      condition, 2*128 + 2048 = 2304 channels; partial rotary position
//      embedding and a Fourier timestep embedding;
//    - "第三阶段": chunks of 200 frames; latents (1, 128, condition length);
//      flow matching with 1000 training timesteps; each step predicts with the
//      condition and with an all-zero condition, guides
//      velocity = uncond + cfg_scale * (cond - uncond), then steps the
//      scheduler; "推理参数详解": cfg_scale 1.7, 30 steps.
//  * "MiniMax Music 3 modular pipeline" (diffusers issue), finding 3: the
//    conditional and unconditional predictions as ONE batch-2 forward, which
//    is formula-identical to two batch-1 forwards.
//  * "MiniMax Music 3 on Metal", "Precision is the reference's": fp16 in the
//    DiT with fp16 roundings and fp32 sums; its kernel list names LayerNorm,
//    the timestep MLP, the guided velocity, the Euler step, q/k RoPE and a
//    GLU, and attention with fp16 probabilities for P V.
//
// Readings where the pages are silent (each also listed in the design notes):
//  * input h_in = [x_t (128) | context latent (128) | condition (2048)], the
//    second 128 being the chunk's context latent (previous chunk over the
//    overlap, zeros elsewhere); the unconditional branch zeroes the
//    condition channels only;
//  * no bias in any linear layer; LayerNorm with gain and bias, eps 1e-5,
//    one fp16 rounding at its output (fp32 statistics);
//  * timestep t = 1000 * sigma; Fourier features [cos(t f_k), sin(t f_k)],
//    f_k = 10000^(-k/half), half = temb/2; MLP W_t2 silu(W_t1 feat); the
//    embedding is added to every token after the input projection;
//  * pre-norm blocks: h += W_o attn(LN1 h); h += W_d (silu(W_g n) * W_u n),
//    n = LN2 h; final LN and W_out (2048 -> 128) give the velocity;
//  * partial RoPE: the first rope_dims (32) of each q / k head rotated by
//    half-rotation pairs (i, i + rope_dims/2) at the token's index in its
//    chunk, angle pos * theta^(-2i/rope_dims) (fp64), theta 10000;
//  * attention bidirectional over the chunk, per batch element and head;
//    scores fp32, e_j = exp(s_j - max) fp32, l = sum e_j, o = sum f16(e_j) v_j / l;
//  * Euler step x <- x + (sigma_next - sigma) v in fp32 (the scheduler's
//    first-order step); x kept in fp32.
//
// Arithmetic rules: f16(v) is round-to-nearest-even of the fp32 value v;
// every dot product is a sequential fp32 loop in index order (a product of
// two fp16 values is exact in fp32); built with -ffp-contract=off.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

typedef uint16_t f16_t;  // raw IEEE binary16 bits

namespace {

inline f16_t to_h(float f) {
  _Float16 h = (_Float16)f;  // IEEE RNE conversion
  f16_t b;
  std::memcpy(&b, &h, 2);
  return b;
}
inline float from_h(f16_t b) {
  _Float16 h;
  std::memcpy(&h, &b, 2);
  return (float)h;
}
inline float rh(float f) { return from_h(to_h(f)); }  // fp32 -> f16 -> fp32

}  // namespace

extern "C" {

struct OraDitCfg {
  int width;      // W = heads * head_dim (2048)
  int n_layers;   // 36
  int n_heads;    // 32
  int head_dim;   // 64
  int ffn;        // 8192
  int latent;     // 128 latent channels
  int cond;       // 2048 condition channels
  int temb;       // Fourier feature count (256)
  int rope_dims;  // rotated dims per head (32)
  double rope_theta;
  float ln_eps;
};

struct OraDitLayer {
  const f16_t *ln1_g, *ln1_b;  // [W]
  const f16_t* wqkv;           // [3W, W]: q rows, k rows, v rows (head-major)
  const f16_t* wo;             // [W, W]
  const f16_t *ln2_g, *ln2_b;  // [W]
  const f16_t *wg, *wu;        // [F, W]
  const f16_t* wd;             // [W, F]
};

struct OraDitWeights {
  const f16_t* w_in;   // [W, 2*latent + cond]
  const f16_t* w_t1;   // [W, temb]
  const f16_t* w_t2;   // [W, W]
  const OraDitLayer* layers;
  const f16_t *lnf_g, *lnf_b;  // [W]
  const f16_t* w_out;  // [latent, W]
};

// y[t][o] = f16(sum_k W[o][k] x[t][k]) for rows t < n, W [N, K]; x holds f16 values.
static void linear(const f16_t* W, int64_t N, int64_t K, const float* x, int64_t n, float* y) {
#pragma omp parallel for collapse(2) schedule(static)
  for (int64_t t = 0; t < n; ++t)
    for (int64_t o = 0; o < N; ++o) {
      const f16_t* w = W + o * K;
      const float* xr = x + t * K;
      float acc = 0.0f;
      for (int64_t k = 0; k < K; ++k) acc = acc + from_h(w[k]) * xr[k];
      y[t * N + o] = rh(acc);
    }
}

// LayerNorm of one row: mean and variance in fp32 (two passes, sequential),
// out = f16(((x - mean) * r) * g + b), r = 1 / sqrt(var + eps).
void ora_dit_layernorm(const float* x, const f16_t* g, const f16_t* b, int64_t n, float eps,
                       float* out) {
  float s = 0.0f;
  for (int64_t i = 0; i < n; ++i) s = s + x[i];
  const float mean = s / (float)n;
  float v = 0.0f;
  for (int64_t i = 0; i < n; ++i) v = v + (x[i] - mean) * (x[i] - mean);
  const float var = v / (float)n;
  const float r = 1.0f / std::sqrt(var + eps);
  for (int64_t i = 0; i < n; ++i) out[i] = rh(((x[i] - mean) * r) * from_h(g[i]) + from_h(b[i]));
}

// Partial rotary embedding of one head: dims i < rot/2 pair with i + rot/2,
// angle pos * theta^(-2i/rot) in fp64, rotation in fp32, results f16; dims
// >= rot unchanged.
void ora_dit_rope(float* v, int rot, int64_t pos, double theta) {
  const int h = rot / 2;
  for (int i = 0; i < h; ++i) {
    const double ang = (double)pos * std::pow(theta, -2.0 * (double)i / (double)rot);
    const float c = (float)std::cos(ang), s = (float)std::sin(ang);
    const float a = v[i], b = v[i + h];
    v[i] = rh(a * c - b * s);
    v[i + h] = rh(b * c + a * s);
  }
}

// One head over T tokens (bidirectional): q, k, v [T, d] f16 values;
// s_j = (q . k_j) * (1 / sqrt(d)); e_j = exp(s_j - max_j s_j); l = sum_j e_j;
// out_i = f16(sum_j f16(e_j) v_j / l), sums sequential fp32.
void ora_dit_attention(const float* q, const float* k, const float* v, int64_t T, int d,
                       float* out) {
  const float scale = 1.0f / std::sqrt((float)d);
  std::vector<float> s(T), e(T);
  for (int64_t t = 0; t < T; ++t) {
    const float* qt = q + t * d;
    float m = -INFINITY;
    for (int64_t j = 0; j < T; ++j) {
      float acc = 0.0f;
      for (int i = 0; i < d; ++i) acc = acc + qt[i] * k[j * d + i];
      s[j] = acc * scale;
      m = s[j] > m ? s[j] : m;
    }
    float l = 0.0f;
    for (int64_t j = 0; j < T; ++j) {
      e[j] = std::exp(s[j] - m);
      l = l + e[j];
    }
    for (int i = 0; i < d; ++i) {
      float acc = 0.0f;
      for (int64_t j = 0; j < T; ++j) acc = acc + rh(e[j]) * v[j * d + i];
      out[t * d + i] = rh(acc / l);
    }
  }
}

// Fourier timestep features of t (fp32): feat[k] = f16(cos(t f_k)),
// feat[half + k] = f16(sin(t f_k)), f_k = 10000^(-k/half) -- in fp64, then fp32.
void ora_dit_time_features(float t, int temb, float* feat) {
  const int half = temb / 2;
  for (int k = 0; k < half; ++k) {
    const double f = std::exp(-std::log(10000.0) * (double)k / (double)half);
    const double a = (double)t * f;
    feat[k] = rh((float)std::cos(a));
    feat[half + k] = rh((float)std::sin(a));
  }
}

static inline float silu(float g) { return g / (1.0f + std::exp(-g)); }

// The DiT layers on h [B, T, W] (f16 bits, updated in place).
int ora_dit_layers(const OraDitCfg* c, const OraDitLayer* layers, int n_layers, int B, int T,
                   f16_t* h_bits) {
  const int W = c->width, d = c->head_dim, nh = c->n_heads, F = c->ffn;
  if (nh * d != W || c->rope_dims > d || c->rope_dims % 2) return -1;
  const int64_t n = (int64_t)B * T;
  std::vector<float> h(n * W), x(n * W), qkv(n * 3 * W), o(n * W), t(n * W), g(n * F), u(n * F);
  for (int64_t i = 0; i < n * W; ++i) h[i] = from_h(h_bits[i]);
  for (int l = 0; l < n_layers; ++l) {
    const OraDitLayer& L = layers[l];
    for (int64_t r = 0; r < n; ++r)
      ora_dit_layernorm(&h[r * W], L.ln1_g, L.ln1_b, W, c->ln_eps, &x[r * W]);
    linear(L.wqkv, 3 * W, W, x.data(), n, qkv.data());
    // partial RoPE of q and k at the token's index in its chunk
    for (int64_t r = 0; r < n; ++r)
      for (int hd = 0; hd < nh; ++hd) {
        ora_dit_rope(&qkv[r * 3 * W + hd * d], c->rope_dims, r % T, c->rope_theta);
        ora_dit_rope(&qkv[r * 3 * W + W + hd * d], c->rope_dims, r % T, c->rope_theta);
      }
    // attention per batch element and head
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
      for (int hd = 0; hd < nh; ++hd) {
        std::vector<float> q(T * d), k(T * d), v(T * d), oh(T * d);
        for (int j = 0; j < T; ++j)
          for (int i = 0; i < d; ++i) {
            const float* row = &qkv[((int64_t)b * T + j) * 3 * W];
            q[j * d + i] = row[hd * d + i];
            k[j * d + i] = row[W + hd * d + i];
            v[j * d + i] = row[2 * W + hd * d + i];
          }
        ora_dit_attention(q.data(), k.data(), v.data(), T, d, oh.data());
        for (int j = 0; j < T; ++j)
          for (int i = 0; i < d; ++i) o[((int64_t)b * T + j) * W + hd * d + i] = oh[j * d + i];
      }
    linear(L.wo, W, W, o.data(), n, t.data());
    for (int64_t i = 0; i < n * W; ++i) h[i] = rh(h[i] + t[i]);
    for (int64_t r = 0; r < n; ++r)
      ora_dit_layernorm(&h[r * W], L.ln2_g, L.ln2_b, W, c->ln_eps, &x[r * W]);
    linear(L.wg, F, W, x.data(), n, g.data());
    linear(L.wu, F, W, x.data(), n, u.data());
    for (int64_t i = 0; i < n * F; ++i) g[i] = rh(rh(silu(g[i])) * u[i]);
    linear(L.wd, W, F, g.data(), n, t.data());
    for (int64_t i = 0; i < n * W; ++i) h[i] = rh(h[i] + t[i]);
  }
  for (int64_t i = 0; i < n * W; ++i) h_bits[i] = to_h(h[i]);
  return 0;
}

// The whole DiT forward for B batch elements of T tokens each:
//   h_in [B, T, 2*latent + cond] f16 bits; t = 1000 * sigma;
//   v_out [B, T, latent] f16 bits (the velocity prediction);
//   h_last (nullable) [B, T, W]: the residual stream after the last layer.
int ora_dit_forward(const OraDitCfg* c, const OraDitWeights* w, int B, int T, const f16_t* h_in,
                    float t, f16_t* v_out, f16_t* h_last) {
  const int W = c->width, Cin = 2 * c->latent + c->cond, Lt = c->latent;
  const int64_t n = (int64_t)B * T;
  std::vector<float> xin(n * Cin), h(n * W), feat(c->temb), a1(W), temb(W), x(n * W), v(n * Lt);
  for (int64_t i = 0; i < n * Cin; ++i) xin[i] = from_h(h_in[i]);
  linear(w->w_in, W, Cin, xin.data(), n, h.data());
  ora_dit_time_features(t, c->temb, feat.data());
  linear(w->w_t1, W, c->temb, feat.data(), 1, a1.data());
  for (int i = 0; i < W; ++i) a1[i] = rh(silu(a1[i]));
  linear(w->w_t2, W, W, a1.data(), 1, temb.data());
  for (int64_t r = 0; r < n; ++r)
    for (int i = 0; i < W; ++i) h[r * W + i] = rh(h[r * W + i] + temb[i]);
  std::vector<f16_t> hb(n * W);
  for (int64_t i = 0; i < n * W; ++i) hb[i] = to_h(h[i]);
  const int rc = ora_dit_layers(c, w->layers, c->n_layers, B, T, hb.data());
  if (rc) return rc;
  if (h_last) std::memcpy(h_last, hb.data(), sizeof(f16_t) * hb.size());
  for (int64_t i = 0; i < n * W; ++i) h[i] = from_h(hb[i]);
  for (int64_t r = 0; r < n; ++r)
    ora_dit_layernorm(&h[r * W], w->lnf_g, w->lnf_b, W, c->ln_eps, &x[r * W]);
  linear(w->w_out, Lt, W, x.data(), n, v.data());
  for (int64_t i = 0; i < n * Lt; ++i) v_out[i] = to_h(v[i]);
  return 0;
}

// The guided velocity and the Euler step, per element:
//   vg = vu + cfg_scale * (vc - vu)          (fp32, from the f16 predictions)
//   x_next = x + (sigma_next - sigma) * vg   (fp32)
void ora_dit_guide_step(int64_t n, const float* x, const f16_t* vc, const f16_t* vu,
                        float cfg_scale, float sigma, float sigma_next, float* x_next,
                        float* vg) {
  const float dt = sigma_next - sigma;
  for (int64_t i = 0; i < n; ++i) {
    const float u = from_h(vu[i]), cc = from_h(vc[i]);
    const float g = u + cfg_scale * (cc - u);
    if (vg) vg[i] = g;
    x_next[i] = x[i] + dt * g;
  }
}

// One denoising step of one chunk (T latent frames): the batch-2 forward on
// [x_t | ctx | cond] (cond) and [x_t | ctx | 0] (uncond), the guided
// velocity, the Euler step.  x, x_next [T, latent] fp32; ctx [T, latent] and
// cond [T, cond] f16 bits; v_pair (nullable) [2, T, latent] f16 bits (cond
// then uncond prediction); vg (nullable) [T, latent] fp32.
int ora_dit_step(const OraDitCfg* c, const OraDitWeights* w, int T, const float* x,
                 const f16_t* ctx, const f16_t* cond, float sigma, float sigma_next,
                 float cfg_scale, float* x_next, float* vg, f16_t* v_pair) {
  const int Lt = c->latent, C = c->cond, Cin = 2 * Lt + C;
  std::vector<f16_t> hin((size_t)2 * T * Cin), v((size_t)2 * T * Lt);
  for (int b = 0; b < 2; ++b)
    for (int j = 0; j < T; ++j) {
      f16_t* row = &hin[((size_t)b * T + j) * Cin];
      for (int i = 0; i < Lt; ++i) row[i] = to_h(x[(size_t)j * Lt + i]);
      for (int i = 0; i < Lt; ++i) row[Lt + i] = ctx[(size_t)j * Lt + i];
      for (int i = 0; i < C; ++i) row[2 * Lt + i] = b == 0 ? cond[(size_t)j * C + i] : (f16_t)0;
    }
  const int rc = ora_dit_forward(c, w, 2, T, hin.data(), sigma * 1000.0f, v.data(), nullptr);
  if (rc) return rc;
  if (v_pair) std::memcpy(v_pair, v.data(), sizeof(f16_t) * v.size());
  ora_dit_guide_step((int64_t)T * Lt, x, v.data(), v.data() + (size_t)T * Lt, cfg_scale, sigma,
                     sigma_next, x_next, vg);
  return 0;
}

}  // extern "C"
