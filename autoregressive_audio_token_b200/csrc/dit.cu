// dit.cu -- runtime of the DiT chunk-denoise step (include/m3_dit.h):
// weights, activation buffers, the per-T CUDA graph of one step.
//
// One step of a chunk of T latent frames, batch 2 (cond, uncond) as one
// forward (the diffusers issue, finding 3), rows = 2T tokens:
//   assemble [x_t | ctx | cond or 0] -> W_in GEMM (+ timestep embedding)
//   -> 36 x { LayerNorm -> QKV GEMM (+ partial RoPE) -> attention
//             -> O GEMM (+ residual) -> LayerNorm -> gate/up GEMM (+ GLU)
//             -> down GEMM (+ residual) }
//   -> LayerNorm -> W_out GEMM -> guided velocity and Euler step.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <map>
#include <string>
#include <vector>

#include "dit_gemm.cuh"
#include "dit_kernels.cuh"
#include "m3_dit.h"

namespace m3 {
int set_error(int code, const std::string& msg);
}

using namespace m3;

namespace {

int fail(int code, const std::string& msg) { return set_error(code, msg); }

#define DCK(call)                                                                        \
  do {                                                                                   \
    cudaError_t e_ = (call);                                                             \
    if (e_ != cudaSuccess)                                                               \
      return fail(e_ == cudaErrorMemoryAllocation ? M3_ENOMEM : M3_ECUDA,                \
                  std::string(#call) + ": " + cudaGetErrorString(e_));                   \
  } while (0)

#define DCKR(expr)              \
  do {                          \
    int r_ = (expr);            \
    if (r_ != M3_OK) return r_; \
  } while (0)

struct DitLayer {
  __half *ln1_g = nullptr, *ln1_b = nullptr, *wqkv = nullptr, *wo = nullptr;
  __half *ln2_g = nullptr, *ln2_b = nullptr, *wgu = nullptr, *wd = nullptr;
};

}  // namespace

struct m3_dit {
  m3_dit_config cfg{};
  cudaStream_t user_st = nullptr, st = nullptr;
  cudaEvent_t ev_in = nullptr, ev_out = nullptr;
  int dev = 0, nsm = 148;
  std::vector<void*> allocs;
  // weights
  __half *w_in = nullptr, *w_t1 = nullptr, *w_t2 = nullptr;
  __half *lnf_g = nullptr, *lnf_b = nullptr, *w_out = nullptr;
  std::vector<DitLayer> L;
  std::vector<char> loaded;
  bool outer_loaded = false;
  // activations, 2 * max_tokens rows
  __half *hin = nullptr, *h = nullptr, *n = nullptr, *qkv = nullptr, *o = nullptr, *a = nullptr;
  __half *v = nullptr, *feat = nullptr, *a1 = nullptr, *temb = nullptr;
  float *x = nullptr, *vg = nullptr;        // [max_tokens][latent]
  __half *ctx = nullptr, *cond = nullptr;   // step inputs
  float2* rope = nullptr;                   // [max_tokens][rope_dims / 2]
  DitParams* params = nullptr;
  int* err = nullptr;
  std::map<int, cudaGraphExec_t> graphs;    // one step per T
};

namespace {

int dalloc(m3_dit* d, void** p, size_t bytes) {
  DCK(cudaMalloc(p, bytes < 256 ? 256 : bytes));
  d->allocs.push_back(*p);
  return M3_OK;
}

template <typename T>
int dalloc_t(m3_dit* d, T** p, size_t count) {
  void* q = nullptr;
  DCKR(dalloc(d, &q, sizeof(T) * count));
  *p = static_cast<T*>(q);
  return M3_OK;
}

int enter(m3_dit* d) {
  DCK(cudaSetDevice(d->dev));
  DCK(cudaEventRecord(d->ev_in, d->user_st));
  DCK(cudaStreamWaitEvent(d->st, d->ev_in, 0));
  return M3_OK;
}

int leave(m3_dit* d) {
  DCK(cudaEventRecord(d->ev_out, d->st));
  DCK(cudaStreamWaitEvent(d->user_st, d->ev_out, 0));
  return M3_OK;
}

bool valid_cfg(const m3_dit_config* c, std::string& why) {
  const int W = c->width;
  if (c->head_dim != 64) return why = "head_dim must be 64", false;
  if (c->rope_dims != 32) return why = "rope_dims must be 32", false;
  if (c->n_heads * c->head_dim != W) return why = "width != n_heads * head_dim", false;
  if (W != 256 && W != 512 && W != 1024 && W != 2048) return why = "width not in 256..2048", false;
  if (c->ffn < 64 || c->ffn % 64) return why = "ffn not a multiple of 64", false;
  if (c->latent < 32 || c->latent % 32 || c->cond < 0 || (2 * c->latent + c->cond) % 64)
    return why = "2*latent + cond not a multiple of 64 (latent a multiple of 32)", false;
  if (c->temb < 8 || c->temb % 8) return why = "temb not a multiple of 8", false;
  if (c->n_layers < 1 || c->max_tokens < 1 || c->max_tokens > 65536)
    return why = "n_layers / max_tokens", false;
  if (!(c->ln_eps > 0.0f) || !(c->rope_theta > 0.0)) return why = "ln_eps / rope_theta", false;
  return true;
}

cudaError_t launch_layernorm(const m3_dit* d, const __half* x, const __half* g, const __half* b,
                             int rows, __half* out) {
  const dim3 grid((rows + 7) / 8), block(256);
  switch (d->cfg.width) {
    case 256: dit_layernorm_kernel<256><<<grid, block, 0, d->st>>>(x, g, b, rows, d->cfg.ln_eps, out); break;
    case 512: dit_layernorm_kernel<512><<<grid, block, 0, d->st>>>(x, g, b, rows, d->cfg.ln_eps, out); break;
    case 1024: dit_layernorm_kernel<1024><<<grid, block, 0, d->st>>>(x, g, b, rows, d->cfg.ln_eps, out); break;
    default: dit_layernorm_kernel<2048><<<grid, block, 0, d->st>>>(x, g, b, rows, d->cfg.ln_eps, out); break;
  }
  return cudaGetLastError();
}

// One GEMM of the step: out = epilogue(X W^T), X [M][ldx].
int gemm(m3_dit* d, const __half* X, int ldx, const __half* W, int M, int N, int K, __half* out,
         int ldo, int epi, int T = 1) {
  DitGemmArgs g{};
  g.M = M;
  g.N = N;
  g.K = K;
  g.out = out;
  g.ldo = ldo;
  g.vec = d->temb;
  g.rope = d->rope;
  g.rope_T = T;
  g.rope_cols = 2 * d->cfg.width;
  g.head_dim = d->cfg.head_dim;
  g.rope_half = d->cfg.rope_dims / 2;
  g.err = d->err;
  DCK(launch_dit_gemm(X, ldx, W, g, epi, d->nsm, d->st));
  return M3_OK;
}

// Blocks first .. first + n - 1 on d->h ([B*T][W]).
int record_blocks(m3_dit* d, int B, int T, int first, int nl) {
  const m3_dit_config& c = d->cfg;
  const int W = c.width, M = B * T;
  for (int l = first; l < first + nl; ++l) {
    const DitLayer& L = d->L[l];
    DCK(launch_layernorm(d, d->h, L.ln1_g, L.ln1_b, M, d->n));
    DCKR(gemm(d, d->n, W, L.wqkv, M, 3 * W, W, d->qkv, 3 * W, DIT_EPI_ROPE, T));
    dit_attention_kernel<<<dim3((T + kDaQ - 1) / kDaQ, c.n_heads, B), kDaWarps * 32, kDaSmem,
                           d->st>>>(d->qkv, T, W, d->o);
    DCK(cudaGetLastError());
    DCKR(gemm(d, d->o, W, L.wo, M, W, W, d->h, W, DIT_EPI_RESID));
    DCK(launch_layernorm(d, d->h, L.ln2_g, L.ln2_b, M, d->n));
    DCKR(gemm(d, d->n, W, L.wgu, M, 2 * c.ffn, W, d->a, c.ffn, DIT_EPI_GLU));
    DCKR(gemm(d, d->a, c.ffn, L.wd, M, W, c.ffn, d->h, W, DIT_EPI_RESID));
  }
  return M3_OK;
}

// The forward on d->hin ([B*T][Cin]) with t from d->params -> d->v ([B*T][latent]).
int record_forward(m3_dit* d, int B, int T) {
  const m3_dit_config& c = d->cfg;
  const int W = c.width, M = B * T, Cin = 2 * c.latent + c.cond;
  dit_time_features_kernel<<<1, 128, 0, d->st>>>(d->params, c.temb, d->feat);
  DCK(cudaGetLastError());
  dit_gemv_kernel<<<(W + 7) / 8, 256, 0, d->st>>>(d->w_t1, d->feat, W, c.temb, 1, d->a1);
  DCK(cudaGetLastError());
  dit_gemv_kernel<<<(W + 7) / 8, 256, 0, d->st>>>(d->w_t2, d->a1, W, W, 0, d->temb);
  DCK(cudaGetLastError());
  DCKR(gemm(d, d->hin, Cin, d->w_in, M, W, Cin, d->h, W, DIT_EPI_TEMB));
  DCKR(record_blocks(d, B, T, 0, c.n_layers));
  DCK(launch_layernorm(d, d->h, d->lnf_g, d->lnf_b, M, d->n));
  DCKR(gemm(d, d->n, W, d->w_out, M, c.latent, W, d->v, c.latent, DIT_EPI_STORE));
  return M3_OK;
}

int record_step(m3_dit* d, int T) {
  const m3_dit_config& c = d->cfg;
  dit_assemble_kernel<<<2 * T, 256, 0, d->st>>>(d->x, d->ctx, d->cond, T, c.latent, c.cond,
                                                d->hin);
  DCK(cudaGetLastError());
  DCKR(record_forward(d, 2, T));
  const int n = T * c.latent;
  dit_guide_step_kernel<<<(n + 255) / 256, 256, 0, d->st>>>(d->params, d->v, n, d->x, d->vg);
  DCK(cudaGetLastError());
  return M3_OK;
}

int ready(const m3_dit* d) {
  if (!d->outer_loaded) return fail(M3_ESTATE, "DiT input / time / output weights not loaded");
  for (size_t l = 0; l < d->loaded.size(); ++l)
    if (!d->loaded[l]) return fail(M3_ESTATE, "DiT block " + std::to_string(l) + " not loaded");
  return M3_OK;
}

int run_step_graph(m3_dit* d, int T) {
  auto it = d->graphs.find(T);
  if (it == d->graphs.end()) {
    cudaGraph_t graph = nullptr;
    DCK(cudaStreamBeginCapture(d->st, cudaStreamCaptureModeThreadLocal));
    const int rc = record_step(d, T);
    const cudaError_t e = cudaStreamEndCapture(d->st, &graph);
    if (rc != M3_OK) {
      if (graph) cudaGraphDestroy(graph);
      return rc;
    }
    if (e != cudaSuccess) return fail(M3_ECUDA, std::string("graph capture: ") + cudaGetErrorString(e));
    cudaGraphExec_t exec = nullptr;
    const cudaError_t e2 = cudaGraphInstantiate(&exec, graph, 0);
    cudaGraphDestroy(graph);
    if (e2 != cudaSuccess)
      return fail(M3_ECUDA, std::string("graph instantiate: ") + cudaGetErrorString(e2));
    it = d->graphs.emplace(T, exec).first;
  }
  DCK(cudaGraphLaunch(it->second, d->st));
  return M3_OK;
}

int put(m3_dit* d, __half** dst, const void* src, size_t count, int mem) {
  if (!src) return M3_OK;
  if (!*dst) DCKR(dalloc_t(d, dst, count));
  DCK(cudaMemcpyAsync(*dst, src, count * 2,
                      mem == M3_MEM_DEVICE ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice,
                      d->st));
  return M3_OK;
}

}  // namespace

extern "C" int m3_dit_create(const m3_dit_config* cfg, void* cuda_stream, m3_dit** out) {
  if (!cfg || !out) return fail(M3_EINVAL, "null argument");
  std::string why;
  if (!valid_cfg(cfg, why)) return fail(M3_EINVAL, "m3_dit_config: " + why);
  m3_dit* d = new m3_dit();
  d->cfg = *cfg;
  d->user_st = static_cast<cudaStream_t>(cuda_stream);
  auto bail = [&](int rc) { m3_dit_destroy(d); return rc; };
  if (cudaGetDevice(&d->dev) != cudaSuccess) return bail(fail(M3_ECUDA, "cudaGetDevice"));
  if (cudaDeviceGetAttribute(&d->nsm, cudaDevAttrMultiProcessorCount, d->dev) != cudaSuccess)
    return bail(fail(M3_ECUDA, "SM count"));
  if (cudaStreamCreateWithFlags(&d->st, cudaStreamNonBlocking) != cudaSuccess ||
      cudaEventCreateWithFlags(&d->ev_in, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&d->ev_out, cudaEventDisableTiming) != cudaSuccess)
    return bail(fail(M3_ECUDA, "stream/event creation"));
  const m3_dit_config& c = d->cfg;
  const size_t R = 2 * (size_t)c.max_tokens, W = c.width, Cin = 2 * c.latent + c.cond;
  d->L.resize(c.n_layers);
  d->loaded.assign(c.n_layers, 0);
  int rc = M3_OK;
  if ((rc = dalloc_t(d, &d->hin, R * Cin)) || (rc = dalloc_t(d, &d->h, R * W)) ||
      (rc = dalloc_t(d, &d->n, R * W)) || (rc = dalloc_t(d, &d->qkv, R * 3 * W)) ||
      (rc = dalloc_t(d, &d->o, R * W)) || (rc = dalloc_t(d, &d->a, R * c.ffn)) ||
      (rc = dalloc_t(d, &d->v, R * c.latent)) || (rc = dalloc_t(d, &d->feat, (size_t)c.temb)) ||
      (rc = dalloc_t(d, &d->a1, W)) || (rc = dalloc_t(d, &d->temb, W)) ||
      (rc = dalloc_t(d, &d->x, (size_t)c.max_tokens * c.latent)) ||
      (rc = dalloc_t(d, &d->vg, (size_t)c.max_tokens * c.latent)) ||
      (rc = dalloc_t(d, &d->ctx, (size_t)c.max_tokens * c.latent)) ||
      (rc = dalloc_t(d, &d->cond, (size_t)c.max_tokens * (c.cond > 0 ? c.cond : 1))) ||
      (rc = dalloc_t(d, &d->rope, (size_t)c.max_tokens * (c.rope_dims / 2))) ||
      (rc = dalloc_t(d, &d->params, 1)) || (rc = dalloc_t(d, &d->err, 1)))
    return bail(rc);
  if (cudaMemset(d->err, 0, sizeof(int)) != cudaSuccess) return bail(fail(M3_ECUDA, "memset"));
  if (const cudaError_t e = prepare_dit_gemm())
    return bail(fail(M3_ECUDA, std::string("GEMM set-up: ") + cudaGetErrorString(e)));
  dit_rope_table_kernel<<<64, 256>>>(c.max_tokens, c.rope_dims, c.rope_theta, d->rope);
  if (cudaGetLastError() != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess)
    return bail(fail(M3_ECUDA, "RoPE table"));
  *out = d;
  return M3_OK;
}

extern "C" void m3_dit_destroy(m3_dit* d) {
  if (!d) return;
  cudaSetDevice(d->dev);
  if (d->st) cudaStreamSynchronize(d->st);
  for (auto& kv : d->graphs) cudaGraphExecDestroy(kv.second);
  for (void* p : d->allocs) cudaFree(p);
  if (d->ev_in) cudaEventDestroy(d->ev_in);
  if (d->ev_out) cudaEventDestroy(d->ev_out);
  if (d->st) cudaStreamDestroy(d->st);
  delete d;
}

extern "C" int m3_dit_load(m3_dit* d, const m3_dit_src* s) {
  if (!d || !s) return fail(M3_EINVAL, "null argument");
  const m3_dit_config& c = d->cfg;
  if (s->mem != M3_MEM_HOST && s->mem != M3_MEM_DEVICE) return fail(M3_EINVAL, "mem");
  if (s->n_layers < 0 || s->first_layer < 0 || s->first_layer + s->n_layers > c.n_layers ||
      (s->n_layers > 0 && !s->layers))
    return fail(M3_EINVAL, "layer range");
  const bool any_outer = s->w_in || s->w_t1 || s->w_t2 || s->lnf_g || s->lnf_b || s->w_out;
  if (any_outer && !(s->w_in && s->w_t1 && s->w_t2 && s->lnf_g && s->lnf_b && s->w_out))
    return fail(M3_EINVAL, "the outer tensors come together");
  const size_t W = c.width, F = c.ffn, Cin = 2 * c.latent + c.cond;
  DCKR(enter(d));
  const cudaMemcpyKind kind = s->mem == M3_MEM_DEVICE ? cudaMemcpyDeviceToDevice
                                                      : cudaMemcpyHostToDevice;
  for (int i = 0; i < s->n_layers; ++i) {
    const m3_dit_layer_src& ls = s->layers[i];
    if (!ls.ln1_g || !ls.ln1_b || !ls.wqkv || !ls.wo || !ls.ln2_g || !ls.ln2_b || !ls.wg ||
        !ls.wu || !ls.wd)
      return fail(M3_EINVAL, "null block tensor");
    DitLayer& L = d->L[s->first_layer + i];
    DCKR(put(d, &L.ln1_g, ls.ln1_g, W, s->mem));
    DCKR(put(d, &L.ln1_b, ls.ln1_b, W, s->mem));
    DCKR(put(d, &L.wqkv, ls.wqkv, 3 * W * W, s->mem));
    DCKR(put(d, &L.wo, ls.wo, W * W, s->mem));
    DCKR(put(d, &L.ln2_g, ls.ln2_g, W, s->mem));
    DCKR(put(d, &L.ln2_b, ls.ln2_b, W, s->mem));
    DCKR(put(d, &L.wd, ls.wd, W * F, s->mem));
    // gate row j -> row 2j, up row j -> row 2j + 1 of one [2F][W] matrix
    if (!L.wgu) DCKR(dalloc_t(d, &L.wgu, 2 * F * W));
    DCK(cudaMemcpy2DAsync(L.wgu, 2 * W * 2, ls.wg, W * 2, W * 2, F, kind, d->st));
    DCK(cudaMemcpy2DAsync(L.wgu + W, 2 * W * 2, ls.wu, W * 2, W * 2, F, kind, d->st));
    d->loaded[s->first_layer + i] = 1;
  }
  if (any_outer) {
    DCKR(put(d, &d->w_in, s->w_in, W * Cin, s->mem));
    DCKR(put(d, &d->w_t1, s->w_t1, W * c.temb, s->mem));
    DCKR(put(d, &d->w_t2, s->w_t2, W * W, s->mem));
    DCKR(put(d, &d->lnf_g, s->lnf_g, W, s->mem));
    DCKR(put(d, &d->lnf_b, s->lnf_b, W, s->mem));
    DCKR(put(d, &d->w_out, s->w_out, (size_t)c.latent * W, s->mem));
    d->outer_loaded = true;
  }
  if (s->mem == M3_MEM_HOST) DCK(cudaStreamSynchronize(d->st));
  return leave(d);
}

static int check_T(const m3_dit* d, int T) {
  if (T < 1 || T > d->cfg.max_tokens) return fail(M3_EINVAL, "T out of 1..max_tokens");
  return M3_OK;
}

// Inputs into the library's buffers, the step parameters, then the graph.
static int stage_inputs(m3_dit* d, int T, const float* x, const void* ctx, const void* cond) {
  const m3_dit_config& c = d->cfg;
  DCK(cudaMemcpyAsync(d->x, x, sizeof(float) * T * c.latent, cudaMemcpyDeviceToDevice, d->st));
  DCK(cudaMemcpyAsync(d->ctx, ctx, 2 * (size_t)T * c.latent, cudaMemcpyDeviceToDevice, d->st));
  if (c.cond > 0)
    DCK(cudaMemcpyAsync(d->cond, cond, 2 * (size_t)T * c.cond, cudaMemcpyDeviceToDevice, d->st));
  return M3_OK;
}

static int set_params(m3_dit* d, float sigma, float sigma_next, float cfg_scale) {
  DitParams p{sigma, sigma_next, cfg_scale, sigma * 1000.0f};
  dit_set_params_kernel<<<1, 32, 0, d->st>>>(d->params, p);
  DCK(cudaGetLastError());
  return M3_OK;
}

extern "C" int m3_dit_step(m3_dit* d, int T, float* x, const void* ctx, const void* cond,
                           float sigma, float sigma_next, float cfg_scale, float* v_guided,
                           void* v_pair) {
  if (!d || !x || !ctx || (!cond && d->cfg.cond > 0)) return fail(M3_EINVAL, "null argument");
  DCKR(check_T(d, T));
  DCKR(ready(d));
  const m3_dit_config& c = d->cfg;
  DCKR(enter(d));
  DCKR(stage_inputs(d, T, x, ctx, cond));
  DCKR(set_params(d, sigma, sigma_next, cfg_scale));
  DCKR(run_step_graph(d, T));
  DCK(cudaMemcpyAsync(x, d->x, sizeof(float) * T * c.latent, cudaMemcpyDeviceToDevice, d->st));
  if (v_guided)
    DCK(cudaMemcpyAsync(v_guided, d->vg, sizeof(float) * T * c.latent, cudaMemcpyDeviceToDevice,
                        d->st));
  if (v_pair)
    DCK(cudaMemcpyAsync(v_pair, d->v, 2 * (size_t)2 * T * c.latent, cudaMemcpyDeviceToDevice,
                        d->st));
  return leave(d);
}

extern "C" int m3_dit_denoise(m3_dit* d, int T, float* x, const void* ctx, const void* cond,
                              const float* sigmas, int steps, float cfg_scale) {
  if (!d || !x || !ctx || !sigmas || (!cond && d->cfg.cond > 0))
    return fail(M3_EINVAL, "null argument");
  if (steps < 1) return fail(M3_EINVAL, "steps < 1");
  DCKR(check_T(d, T));
  DCKR(ready(d));
  DCKR(enter(d));
  DCKR(stage_inputs(d, T, x, ctx, cond));
  for (int i = 0; i < steps; ++i) {
    DCKR(set_params(d, sigmas[i], sigmas[i + 1], cfg_scale));
    DCKR(run_step_graph(d, T));
  }
  DCK(cudaMemcpyAsync(x, d->x, sizeof(float) * T * d->cfg.latent, cudaMemcpyDeviceToDevice,
                      d->st));
  return leave(d);
}

extern "C" int m3_dit_forward(m3_dit* d, int B, int T, const void* h_in, float t, void* v) {
  if (!d || !h_in || !v) return fail(M3_EINVAL, "null argument");
  if (B < 1 || B > 2) return fail(M3_EINVAL, "B must be 1 or 2");
  DCKR(check_T(d, T));
  DCKR(ready(d));
  const m3_dit_config& c = d->cfg;
  const size_t Cin = 2 * c.latent + c.cond;
  DCKR(enter(d));
  DCK(cudaMemcpyAsync(d->hin, h_in, 2 * (size_t)B * T * Cin, cudaMemcpyDeviceToDevice, d->st));
  DitParams p{t / 1000.0f, 0.0f, 0.0f, t};
  dit_set_params_kernel<<<1, 32, 0, d->st>>>(d->params, p);
  DCK(cudaGetLastError());
  DCKR(record_forward(d, B, T));
  DCK(cudaMemcpyAsync(v, d->v, 2 * (size_t)B * T * c.latent, cudaMemcpyDeviceToDevice, d->st));
  return leave(d);
}

extern "C" int m3_dit_blocks(m3_dit* d, int B, int T, void* h, int first, int n) {
  if (!d || !h) return fail(M3_EINVAL, "null argument");
  if (B < 1 || B > 2) return fail(M3_EINVAL, "B must be 1 or 2");
  DCKR(check_T(d, T));
  if (first < 0 || n < 1 || first + n > d->cfg.n_layers) return fail(M3_EINVAL, "block range");
  for (int l = first; l < first + n; ++l)
    if (!d->loaded[l]) return fail(M3_ESTATE, "DiT block " + std::to_string(l) + " not loaded");
  const size_t bytes = 2 * (size_t)B * T * d->cfg.width;
  DCKR(enter(d));
  DCK(cudaMemcpyAsync(d->h, h, bytes, cudaMemcpyDeviceToDevice, d->st));
  DCKR(record_blocks(d, B, T, first, n));
  DCK(cudaMemcpyAsync(h, d->h, bytes, cudaMemcpyDeviceToDevice, d->st));
  return leave(d);
}

extern "C" int m3_dit_time_gemm(m3_dit* d, int which, int T, int iters, float* avg_ms,
                                double* flops) {
  if (!d || !avg_ms || !flops) return fail(M3_EINVAL, "null argument");
  if (which < 0 || which > 3 || iters < 1) return fail(M3_EINVAL, "which / iters");
  DCKR(check_T(d, T));
  DCKR(ready(d));
  const m3_dit_config& c = d->cfg;
  const int W = c.width, M = 2 * T, F = c.ffn;
  DCKR(enter(d));
  cudaEvent_t e0, e1;
  DCK(cudaEventCreate(&e0));
  DCK(cudaEventCreate(&e1));
  auto one = [&](int i) -> int {
    const DitLayer& L = d->L[i % c.n_layers];
    switch (which) {
      case 0: return gemm(d, d->n, W, L.wqkv, M, 3 * W, W, d->qkv, 3 * W, DIT_EPI_ROPE, T);
      case 1: return gemm(d, d->o, W, L.wo, M, W, W, d->h, W, DIT_EPI_RESID);
      case 2: return gemm(d, d->n, W, L.wgu, M, 2 * F, W, d->a, F, DIT_EPI_GLU);
      default: return gemm(d, d->a, F, L.wd, M, W, F, d->h, W, DIT_EPI_RESID);
    }
  };
  int rc = one(0);  // warm
  if (rc == M3_OK) {
    cudaEventRecord(e0, d->st);
    for (int i = 0; i < iters && rc == M3_OK; ++i) rc = one(i);
    cudaEventRecord(e1, d->st);
  }
  cudaError_t e = cudaEventSynchronize(e1);
  float ms = 0.0f;
  if (rc == M3_OK && e == cudaSuccess) e = cudaEventElapsedTime(&ms, e0, e1);
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  if (rc != M3_OK) return rc;
  DCK(e);
  const double N = which == 0 ? 3.0 * W : which == 2 ? 2.0 * F : (double)W;
  const double K = which == 3 ? (double)F : (double)W;
  *avg_ms = ms / iters;
  *flops = 2.0 * M * N * K;
  return leave(d);
}

extern "C" int m3_dit_sync_status(m3_dit* d) {
  if (!d) return fail(M3_EINVAL, "null argument");
  DCK(cudaSetDevice(d->dev));
  DCK(cudaStreamSynchronize(d->st));
  DCK(cudaStreamSynchronize(d->user_st));
  int e = 0;
  DCK(cudaMemcpy(&e, d->err, sizeof(int), cudaMemcpyDeviceToHost));
  if (e != 0) {
    DCK(cudaMemset(d->err, 0, sizeof(int)));
    if (e == kErrTimeout) return fail(M3_ETIMEOUT, "a device-side wait gave up");
    return fail(M3_EDEVICE, "a kernel recorded an error word");
  }
  return M3_OK;
}
