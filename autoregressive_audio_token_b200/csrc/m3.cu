// m3.cu -- host runtime behind the C ABI of include/m3.h: context, weight
// store (upload, GPU quantisation, gate/up interleave), paged KV cache with
// bucketed growth, one CUDA graph per (rows, KV bucket count) for the frame
// and per (rows, teacher forcing) for the depth decoder, error plumbing.
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <map>
#include <string>
#include <tuple>
#include <vector>

#include "m3.h"
#include "launch.cuh"
#include "misc.cuh"
#include "gemv_tile.cuh"
#include "dit_gemm.cuh"
#include "depth.cuh"

using namespace m3;
typedef __nv_bfloat16 bf16;

// ------------------------------------------------------------------ errors --
static thread_local std::string g_err;

static int fail(int code, const std::string& msg) {
  g_err = msg;
  return code;
}

namespace m3 {
// The same thread-local message for the library's other translation units.
int set_error(int code, const std::string& msg) { return fail(code, msg); }
}  // namespace m3

#define CK(call)                                                                        \
  do {                                                                                  \
    cudaError_t e_ = (call);                                                            \
    if (e_ != cudaSuccess)                                                              \
      return fail(e_ == cudaErrorMemoryAllocation ? M3_ENOMEM : M3_ECUDA,               \
                  std::string(#call) + ": " + cudaGetErrorString(e_));                  \
  } while (0)

#define CKR(expr)             \
  do {                        \
    int r_ = (expr);          \
    if (r_ != M3_OK) return r_; \
  } while (0)

// ------------------------------------------------------------------- state --
struct DMat {
  void* w = nullptr;   // [N][K] bf16 or int8: row-major, or tiled (gemv_tile.cuh)
  float* s = nullptr;  // int8 scales
  int N = 0, K = 0, wf = WF_BF16;
  bool tiled = false;  // bf16 and int8-row matrices of the tensor-core GEMV
};

struct DLayer {
  DMat qkv, o, gu, d;
  bf16 *attn_norm = nullptr, *mlp_norm = nullptr, *q_norm = nullptr, *k_norm = nullptr;
};

struct Acts {  // activation buffers of one stack (body or depth)
  bf16 *x = nullptr, *qkv = nullptr, *o = nullptr, *act = nullptr;
};

// Counter pairs of the dynamically scheduled GEMV: far more than the
// launches a stream can have in flight (a frame has ~5 per layer).
constexpr int kTileCtrPairs = 4096;

struct m3_ctx {
  m3_config cfg{};
  cudaStream_t user_st = nullptr;  // caller's stream
  cudaStream_t st = nullptr;       // internal stream (capturable)
  cudaEvent_t ev_in = nullptr, ev_out = nullptr;
  int dev = 0, nsm = 148;
  bool use_graphs = true;
  std::vector<void*> allocs;

  // body
  int wdtype = -1;
  std::vector<DLayer> L;
  std::vector<char> loaded;
  bf16* final_norm = nullptr;
  DMat lm;
  bool head_loaded = false;
  double* inv_freq = nullptr;

  // depth decoder
  bool depth_loaded = false;
  std::vector<DLayer> DL;
  DMat dproj;
  std::vector<bf16*> demb;
  std::vector<int> demb_rows;
  std::vector<DMat> dheads;
  bf16* dfinal = nullptr;
  double* dinv_freq = nullptr;
  float2* drope = nullptr;  // (cos, sin) of the depth decoder's positions [codebooks + 1][hd / 2]

  // KV cache
  int kv_rows = 0, kv_max_pos = 0, kv_f16 = 0, bucket = 256, max_pages = 0, n_buckets = 0;
  std::vector<void*> buckets;
  unsigned long long* d_pages = nullptr;
  std::vector<unsigned long long> h_pages;
  size_t bucket_bytes = 0;

  // per-frame buffers
  Acts A, DA;
  bf16* h = nullptr;
  float* logits = nullptr;
  int* codes = nullptr;
  float* spz = nullptr;
  int* spi = nullptr;
  unsigned* scnt = nullptr;
  FrameParams* fp = nullptr;
  int* err = nullptr;
  int max_splits = kAttnMaxSplits;
  int attn_per_sm[2] = {0, 0};  // attention CTAs an SM holds (bf16 / f16 cache)
  // depth buffers
  bf16* dh = nullptr;
  int* dcodes = nullptr;
  int* dprev = nullptr;
  int* dforced = nullptr;
  float* dlogits = nullptr;
  unsigned long long* d_dpages = nullptr;
  void* dkv = nullptr;
  // the persistent depth kernel: its tagged-word buffers (residual stream,
  // qkv, attention output, SwiGLU output, frame-local K/V) and argmax
  // partials (one per SM)
  uint32_t* dwords = nullptr;
  size_t dwords_bytes = 0;
  unsigned long long* dpart = nullptr;

  std::map<std::pair<int, int>, cudaGraphExec_t> graphs;
  std::map<std::pair<int, int>, cudaGraphExec_t> dgraphs;

  // tiled GEMV: ring geometry and the launch plan per (N, K, rows, format, epilogue)
  // ring stages (0: by weight format, measured: 3 for bf16, 2 for int8) and
  // those of the O projection alone (0: the same)
  int tile_sb = 65536, tile_ns = 0;
  int tile_ns_o = 0;
  bool tile_dyn = true;  // dynamic unit claiming where it applies
  // ... for the epilogues whose bit is set (-1: by weight format, measured:
  // bf16 leaves the residual projections, O and down, to the cluster-split
  // kernel, which balances them better; int8 claims everywhere)
  int tile_dyn_mask = -1;
  int tile_lazy = 1;      // dynamic GEMV: claim ahead only once the consumers run
  std::map<std::tuple<int, int, int, int, int>, TileLaunch> tile_plans;
  // {claim, done} counter pairs of the dynamically scheduled GEMV, one per
  // launch in flight: launches take pairs round-robin, the last CTA of a
  // launch zeroes its pair
  unsigned* tile_ctrs = nullptr;
  unsigned tile_ctr_next = 0;
  // RMSNorm partials of the residual stream between a residual-add launch
  // and the normalising launch after it (recording a frame only): two
  // [max_rows][units] buffers used alternately; ssq_cur is the one that
  // holds the current stream's partials, or null
  float* ssq_buf[2] = {nullptr, nullptr};
  float* ssq_cur = nullptr;
  int ssq_n = 0;
  bool ssq_track = false;
  float2* rope = nullptr;  // this frame's RoPE (cos, sin) [max_rows][head_dim / 2]
  int top_k = 0;           // the frame draw keeps the top_k guided logits (0: all)
  // generation loop: feedback tables, device state, its host copy, graphs
  bf16* fb_tok = nullptr;          // [slice_len][H]
  std::vector<bf16*> fb_aud;       // depth_codebooks tables [depth_vocab][H]
  bf16** d_fb_aud = nullptr;       // device array of the fb_aud pointers
  LoopState* loop = nullptr;
  unsigned long long* d_vpages = nullptr;  // prefill: every row -> one sequence's pages
  // prefill on the tensor-core GEMM, prompt chunks of pf_chunk tokens:
  // 1 always, 0 never, -1 for bf16 weights only (int8 streams faster through
  // the decode GEMVs, whose tiles convert in registers without a ring)
  int prefill_tc = -1;
  // 0 until the first GEMM prefill: then 2048 on the TMA-fed GEMM (bf16
  // weights; a large M keeps its tiles' rounds full and reads the weights
  // once per 2048 tokens), else 256
  int pf_chunk = 0;
  bf16 *pf_x = nullptr, *pf_n = nullptr, *pf_qkv = nullptr, *pf_o = nullptr, *pf_act = nullptr;
  float2* pf_rope = nullptr;       // [pf_chunk][head_dim / 2]
  // the prefill GEMM's operands: a row-major copy of each bf16 layer's
  // projections (qkv | o | gate/up interleaved | down), made at the first
  // GEMM prefill from the tiled weights; stale once the layer is reloaded
  std::vector<bf16*> pf_rm;
  std::vector<char> pf_rm_ok;
  LoopState* h_loop = nullptr;     // pinned
  int* h_err = nullptr;            // pinned
  std::map<std::pair<int, int>, cudaGraphExec_t> lgraphs;
  float* gbuf = nullptr;   // the guided logits of the top-k draw [max_rows][candidates]
  // host-side fault injection (m3_inject_fault, environment M3_FAULT): the
  // fault_left-th next call of kind fault_kind fails as its CUDA call would
  int fault_kind = 0;
  long long fault_left = 0;
  // device address of the allocation-free sampler's static scratch on this
  // context's device (looked up once, at m3_create)
  unsigned char* noalloc_scratch = nullptr;
};

// Is this call of `kind` the one scheduled to fail?  (Counts down, then
// clears the schedule: one injected failure per m3_inject_fault.)
static bool fault_due(m3_ctx* c, int kind) {
  if (!c || c->fault_kind != kind) return false;
  if (--c->fault_left > 0) return false;
  c->fault_kind = M3_FAULT_NONE;
  return true;
}

template <typename T>
static int dalloc(m3_ctx* c, T** p, size_t bytes) {
  void* q = nullptr;
  if (fault_due(c, M3_FAULT_ALLOC)) return fail(M3_ENOMEM, "injected device allocation failure");
  CK(cudaMalloc(&q, bytes < 256 ? 256 : bytes));
  c->allocs.push_back(q);
  *p = static_cast<T*>(q);
  return M3_OK;
}

static int dzalloc(m3_ctx* c, void** p, size_t bytes) {
  CKR(dalloc(c, p, bytes));
  CK(cudaMemset(*p, 0, bytes < 256 ? 256 : bytes));
  return M3_OK;
}

// Order the internal stream after the caller's stream, and back.
static int enter(m3_ctx* c) {
  CK(cudaSetDevice(c->dev));
  CK(cudaEventRecord(c->ev_in, c->user_st));
  CK(cudaStreamWaitEvent(c->st, c->ev_in, 0));
  return M3_OK;
}

static int leave(m3_ctx* c) {
  CK(cudaEventRecord(c->ev_out, c->st));
  CK(cudaStreamWaitEvent(c->user_st, c->ev_out, 0));
  return M3_OK;
}

static void drop_graphs(m3_ctx* c) {
  for (auto& kv : c->graphs) cudaGraphExecDestroy(kv.second);
  c->graphs.clear();
  for (auto& kv : c->dgraphs) cudaGraphExecDestroy(kv.second);
  c->dgraphs.clear();
  for (auto& kv : c->lgraphs) cudaGraphExecDestroy(kv.second);
  c->lgraphs.clear();
}

static double* make_inv_freq(m3_ctx* c, int d, double theta, int* rc) {
  std::vector<double> h(d / 2);
  for (int i = 0; i < d / 2; ++i) h[i] = std::pow(theta, -2.0 * (double)i / (double)d);
  double* p = nullptr;
  *rc = dalloc(c, &p, sizeof(double) * h.size());
  if (*rc != M3_OK) return nullptr;
  if (cudaMemcpy(p, h.data(), sizeof(double) * h.size(), cudaMemcpyHostToDevice) != cudaSuccess)
    *rc = fail(M3_ECUDA, "inv_freq upload");
  return p;
}

static int alloc_acts(m3_ctx* c, Acts& A, int rows, int H, int Hq, int Hkv, int d, int ffn) {
  CKR(dalloc(c, &A.x, sizeof(bf16) * rows * H));
  CKR(dalloc(c, &A.qkv, sizeof(bf16) * rows * (Hq + 2 * Hkv) * d));
  CKR(dalloc(c, &A.o, sizeof(bf16) * rows * Hq * d));
  CKR(dalloc(c, &A.act, sizeof(bf16) * rows * ffn));
  return M3_OK;
}

// Rows of the lm_head the draw chooses among: the code block, and the end
// token after it when the config has one.
static inline int n_cand(const m3_config& g) { return g.slice_len + (g.has_end_token ? 1 : 0); }

// ------------------------------------------------------------- validation --
static bool valid_cfg(const m3_config* g, std::string& why) {
  if (g->hidden <= 0 || g->n_layers <= 0 || g->n_q_heads <= 0 || g->n_kv_heads <= 0 ||
      g->ffn <= 0) { why = "non-positive dimension"; return false; }
  if (g->head_dim != 64 && g->head_dim != 128) { why = "head_dim must be 64 or 128"; return false; }
  if (g->n_q_heads % g->n_kv_heads || g->n_q_heads / g->n_kv_heads > kAttnWarps) {
    why = "n_q_heads / n_kv_heads must be an integer <= 4"; return false; }
  if (g->hidden % 16 || g->ffn % 16 || (g->n_q_heads * g->head_dim) % 16) {
    why = "hidden, ffn and n_q_heads*head_dim must be multiples of 16"; return false; }
  if (g->max_rows < 1 || g->max_rows > kMaxRows) { why = "max_rows must be in 1..16"; return false; }
  if (g->slice_len <= 0 || g->slice_start < 0) { why = "bad vocab slice"; return false; }
  if (g->has_end_token && (g->end_token < 0 || (g->end_token >= g->slice_start &&
                                                g->end_token < g->slice_start + g->slice_len))) {
    why = "end_token must be a vocab row outside the slice"; return false; }
  if (g->depth_layers > 0) {
    if (g->depth_head_dim != 64 && g->depth_head_dim != 128) { why = "depth_head_dim"; return false; }
    if (g->depth_hidden % 128 || g->depth_ffn % 128 || g->hidden % 128 ||
        (g->depth_heads * g->depth_head_dim) % 128) {
      why = "depth dimensions (and hidden) must be multiples of 128 (int8 groups)"; return false; }
    if (g->depth_codebooks < 1 || g->depth_codebooks > 31 || g->depth_codebooks + 1 > 32) {
      why = "depth_codebooks must be in 1..31"; return false; }
    if (g->depth_vocab <= 0) { why = "depth_vocab"; return false; }
  }
  return true;
}

// ------------------------------------------- allocation-free sampler -------
// Scratch of m3_sample_noalloc: the frame-parameter block, the cross-CTA
// argmax ticket and the per-CTA partial argmaxes live in this file-scope
// device array instead of context-owned buffers.  Every GPU that loads the
// library holds it (about 129 KB) until the process exits.
namespace {
constexpr int kNoAllocMaxCtas = 1024;
constexpr size_t kNoAllocParamsOff = 0;
constexpr size_t kNoAllocCounterOff = 256;
constexpr size_t kNoAllocPartZOff = 512;
constexpr size_t kNoAllocPartIOff = kNoAllocPartZOff + sizeof(float) * kNoAllocMaxCtas * kMaxRows;
constexpr size_t kNoAllocBytes = kNoAllocPartIOff + sizeof(int) * kNoAllocMaxCtas * kMaxRows;
static_assert(sizeof(FrameParams) <= 256, "frame params fit their slot");
}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

// ------------------------------------------------------------------ create --
extern "C" int m3_create(const m3_config* cfg, void* cuda_stream, m3_ctx** out) {
  if (!cfg || !out) return fail(M3_EINVAL, "null argument");
  std::string why;
  if (!valid_cfg(cfg, why)) return fail(M3_EINVAL, "m3_config: " + why);
  m3_ctx* c = new m3_ctx();
  c->cfg = *cfg;
  c->user_st = static_cast<cudaStream_t>(cuda_stream);
  auto bail = [&](int rc) { m3_destroy(c); return rc; };
  if (cudaGetDevice(&c->dev) != cudaSuccess) return bail(fail(M3_ECUDA, "cudaGetDevice"));
  if (cudaDeviceGetAttribute(&c->nsm, cudaDevAttrMultiProcessorCount, c->dev) != cudaSuccess)
    return bail(fail(M3_ECUDA, "SM count"));
  {
    // the host-side name of the static scratch is not a device address: look
    // the address up on this device now, before any stream capture
    void* sp = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&sp, g_noalloc_scratch);
    if (e != cudaSuccess)
      return bail(fail(M3_ECUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e)));
    c->noalloc_scratch = static_cast<unsigned char*>(sp);
  }
  if (const char* e = getenv("M3_FAULT")) {
    // "alloc:N", "h2d:N" or "graph:N": the N-th such call from here on fails
    const char* colon = strchr(e, ':');
    const long long n = colon ? atoll(colon + 1) : 0;
    const size_t len = colon ? (size_t)(colon - e) : 0;
    const int kind = (len == 5 && !strncmp(e, "alloc", 5)) ? M3_FAULT_ALLOC
                   : (len == 3 && !strncmp(e, "h2d", 3))   ? M3_FAULT_H2D
                   : (len == 5 && !strncmp(e, "graph", 5)) ? M3_FAULT_GRAPH
                                                           : M3_FAULT_NONE;
    if (kind == M3_FAULT_NONE || n < 1) {
      delete c;
      return fail(M3_EINVAL, "M3_FAULT must be alloc:N, h2d:N or graph:N with N >= 1");
    }
    c->fault_kind = kind;
    c->fault_left = n;
  }
  if (const char* e = getenv("M3_NO_GRAPH")) c->use_graphs = (e[0] == '0');
  if (const char* e = getenv("M3_GEMV_STAGE_KB")) c->tile_sb = atoi(e) * 1024;
  if (const char* e = getenv("M3_GEMV_STAGES")) c->tile_ns = atoi(e);
  if (const char* e = getenv("M3_GEMV_STAGES_O")) c->tile_ns_o = atoi(e);
  if (const char* e = getenv("M3_GEMV_DYN")) c->tile_dyn = (e[0] == '1');
  if (const char* e = getenv("M3_GEMV_DYN_MASK")) c->tile_dyn_mask = atoi(e);
  if (const char* e = getenv("M3_ATTN_MAX_SPLITS")) {
    const int v = atoi(e);
    if (v >= 1 && v <= kAttnMaxSplits) c->max_splits = v;
  }
  if (const char* e = getenv("M3_PREFILL_TC")) c->prefill_tc = (e[0] == '1') ? 1 : 0;
  if (const char* e = getenv("M3_PREFILL_CHUNK")) {
    const int v = atoi(e);
    if (v >= 16 && v <= 4096) c->pf_chunk = v;
  }
  if (const char* e = getenv("M3_GEMV_LAZY")) c->tile_lazy = atoi(e);
  if (cudaStreamCreateWithFlags(&c->st, cudaStreamNonBlocking) != cudaSuccess ||
      cudaEventCreateWithFlags(&c->ev_in, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&c->ev_out, cudaEventDisableTiming) != cudaSuccess)
    return bail(fail(M3_ECUDA, "stream/event creation"));
  const m3_config& g = c->cfg;
  const int R = g.max_rows;
  c->attn_per_sm[0] = attn_ctas_per_sm(g.head_dim, 0);
  c->attn_per_sm[1] = attn_ctas_per_sm(g.head_dim, 1);
  c->L.resize(g.n_layers);
  c->loaded.assign(g.n_layers, 0);
  int rc = M3_OK;
  c->inv_freq = make_inv_freq(c, g.head_dim, g.rope_theta, &rc);
  if (rc) return bail(rc);
  if ((rc = alloc_acts(c, c->A, R, g.hidden, g.n_q_heads, g.n_kv_heads, g.head_dim, g.ffn)))
    return bail(rc);
  void* p = nullptr;
  if ((rc = dalloc(c, &c->h, sizeof(bf16) * R * g.hidden)) ||
      (rc = dalloc(c, &c->logits, sizeof(float) * R * n_cand(g))) ||
      (rc = dalloc(c, &c->codes, sizeof(int) * R)) ||
      (rc = dalloc(c, &c->spz, sizeof(float) * 1024 * kMaxRows)) ||
      (rc = dalloc(c, &c->spi, sizeof(int) * 1024 * kMaxRows)) ||
      (rc = dzalloc(c, &p, sizeof(unsigned) * 64)) )
    return bail(rc);
  c->scnt = static_cast<unsigned*>(p);
  if ((rc = dzalloc(c, &p, sizeof(unsigned) * 2 * kTileCtrPairs))) return bail(rc);
  c->tile_ctrs = static_cast<unsigned*>(p);
  for (int i = 0; i < 2; ++i)
    if ((rc = dalloc(c, &c->ssq_buf[i], sizeof(float) * R * ((g.hidden + kUnitRows - 1) / kUnitRows))))
      return bail(rc);
  if ((rc = dalloc(c, &c->rope, sizeof(float2) * R * (g.head_dim / 2)))) return bail(rc);
  if ((rc = dalloc(c, &c->gbuf, sizeof(float) * R * n_cand(g)))) return bail(rc);
  if ((rc = dzalloc(c, &p, sizeof(FrameParams)))) return bail(rc);
  c->fp = static_cast<FrameParams*>(p);
  if ((rc = dzalloc(c, &p, sizeof(int)))) return bail(rc);
  c->err = static_cast<int*>(p);
  if (g.depth_layers > 0) {
    const int Dh = g.depth_hidden, NC = g.depth_codebooks;
    c->DL.resize(g.depth_layers);
    c->dinv_freq = make_inv_freq(c, g.depth_head_dim, g.depth_rope_theta, &rc);
    if (rc) return bail(rc);
    {
      const int half = g.depth_head_dim / 2, npos = NC + 1;
      if ((rc = dalloc(c, &c->drope, sizeof(float2) * npos * half))) return bail(rc);
      rope_positions_kernel<<<1, 256>>>(c->dinv_freq, half, 0, npos, c->drope);
      if (cudaGetLastError() != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess)
        return bail(fail(M3_ECUDA, "depth RoPE table"));
    }
    if ((rc = alloc_acts(c, c->DA, R, Dh, g.depth_heads, g.depth_heads, g.depth_head_dim,
                         g.depth_ffn)) ||
        (rc = dalloc(c, &c->dh, sizeof(bf16) * R * g.hidden)) ||
        (rc = dalloc(c, &c->dcodes, sizeof(int) * R * NC)) ||
        (rc = dalloc(c, &c->dprev, sizeof(int) * R)) ||
        (rc = dalloc(c, &c->dforced, sizeof(int) * R * NC)) ||
        (rc = dalloc(c, &c->dlogits, sizeof(float) * R * NC * g.depth_vocab)))
      return bail(rc);
    // depth KV: one 32-position page per (row, layer), bf16
    const size_t page = (size_t)2 * g.depth_heads * 32 * g.depth_head_dim * 2;
    if ((rc = dzalloc(c, &c->dkv, page * R * g.depth_layers))) return bail(rc);
    std::vector<unsigned long long> hp((size_t)R * g.depth_layers);
    for (size_t i = 0; i < hp.size(); ++i)
      hp[i] = (unsigned long long)(static_cast<char*>(c->dkv) + i * page);
    if ((rc = dalloc(c, &c->d_dpages, sizeof(unsigned long long) * hp.size()))) return bail(rc);
    if (cudaMemcpy(c->d_dpages, hp.data(), sizeof(unsigned long long) * hp.size(),
                   cudaMemcpyHostToDevice) != cudaSuccess)
      return bail(fail(M3_ECUDA, "depth page table"));
    const size_t qn = (size_t)g.depth_heads * g.depth_head_dim;
    const size_t words = (size_t)R * (Dh + 3 * qn + qn + g.depth_ffn) +
                         (size_t)R * g.depth_layers * (NC + 1) * 2 * qn;
    c->dwords_bytes = sizeof(uint32_t) * words;
    if ((rc = dzalloc(c, reinterpret_cast<void**>(&c->dwords), c->dwords_bytes)) ||
        (rc = dzalloc(c, reinterpret_cast<void**>(&c->dpart),
                      sizeof(unsigned long long) * c->nsm * kMaxRows)))
      return bail(rc);
  }
  *out = c;
  return M3_OK;
}

extern "C" void m3_destroy(m3_ctx* c) {
  if (!c) return;
  cudaSetDevice(c->dev);
  if (c->st) cudaStreamSynchronize(c->st);
  drop_graphs(c);
  for (void* p : c->buckets) cudaFree(p);
  for (void* p : c->allocs) cudaFree(p);
  if (c->h_loop) cudaFreeHost(c->h_loop);
  if (c->h_err) cudaFreeHost(c->h_err);
  if (c->ev_in) cudaEventDestroy(c->ev_in);
  if (c->ev_out) cudaEventDestroy(c->ev_out);
  if (c->st) cudaStreamDestroy(c->st);
  delete c;
}

extern "C" const char* m3_last_error(void) { return g_err.c_str(); }

extern "C" int m3_set_top_k(m3_ctx* c, int top_k) {
  if (!c) return fail(M3_EINVAL, "null ctx");
  if (top_k < 0) return fail(M3_EINVAL, "top_k < 0");
  c->top_k = top_k >= n_cand(c->cfg) ? 0 : top_k;  // keeping every logit is no filter
  return M3_OK;
}

// ----------------------------------------------------------------- weights --
// Copy a bf16 [rows, cols] source into device staging memory (or use it as is).
static int stage_src(m3_ctx* c, const void* src, size_t bytes, int mem, const void** dev,
                     void** owned) {
  *owned = nullptr;
  if (mem == M3_MEM_DEVICE) {
    *dev = src;
    return M3_OK;
  }
  if (fault_due(c, M3_FAULT_ALLOC)) return fail(M3_ENOMEM, "injected device allocation failure");
  CK(cudaMallocAsync(owned, bytes, c->st));
  const cudaError_t e = fault_due(c, M3_FAULT_H2D)
                            ? cudaErrorUnknown
                            : cudaMemcpyAsync(*owned, src, bytes, cudaMemcpyHostToDevice, c->st);
  if (e != cudaSuccess) {
    cudaFreeAsync(*owned, c->st);
    *owned = nullptr;
    return fail(M3_ECUDA, std::string("host-to-device copy of a source: ") +
                              (e == cudaErrorUnknown ? "injected failure" : cudaGetErrorString(e)));
  }
  *dev = *owned;
  return M3_OK;
}

// Place a [rows, cols] bf16 source at rows dst_row0, dst_row0 + row_step, ...
// of matrix M, quantising on the GPU when M is int8.
static int put_rows(m3_ctx* c, DMat& M, const void* src, int mem, int rows, int dst_row0,
                    int row_step) {
  if (!src) return fail(M3_EINVAL, "null weight pointer");
  const int cols = M.K;
  const size_t bytes = sizeof(bf16) * (size_t)rows * cols;
  const void* dsrc = nullptr;
  void* owned = nullptr;
  CKR(stage_src(c, src, bytes, mem, &dsrc, &owned));
  const unsigned tgrid = (unsigned)(c->nsm * 8);
  if (M.wf == WF_BF16 && M.tiled) {
    tile_rows_kernel<uint16_t><<<tgrid, 256, 0, c->st>>>(
        static_cast<const uint16_t*>(dsrc), rows, cols, static_cast<uint8_t*>(M.w), dst_row0,
        row_step);
    CK(cudaGetLastError());
  } else if (M.wf == WF_BF16) {
    CK(cudaMemcpy2DAsync(static_cast<bf16*>(M.w) + (size_t)dst_row0 * cols,
                         sizeof(bf16) * cols * row_step, dsrc, sizeof(bf16) * cols,
                         sizeof(bf16) * cols, rows, cudaMemcpyDeviceToDevice, c->st));
  } else if (M.wf == WF_I8ROW) {
    // quantise row-major (into a staging buffer when the matrix is tiled)
    void* q = nullptr;
    if (M.tiled) CK(cudaMallocAsync(&q, (size_t)rows * cols, c->st));
    int8_t* qdst = M.tiled ? static_cast<int8_t*>(q) : static_cast<int8_t*>(M.w) + (size_t)dst_row0 * cols;
    const int64_t q_ld = M.tiled ? cols : (int64_t)cols * row_step;
    quantize_rows_kernel<<<dim3(1, rows), 256, 0, c->st>>>(static_cast<const bf16*>(dsrc), cols,
                                                           cols, qdst, q_ld, M.s + dst_row0,
                                                           row_step);
    CK(cudaGetLastError());
    if (M.tiled) {
      tile_rows_kernel<int8_t><<<tgrid, 256, 0, c->st>>>(static_cast<const int8_t*>(q), rows, cols,
                                                         static_cast<uint8_t*>(M.w), dst_row0,
                                                         row_step);
      CK(cudaGetLastError());
      CK(cudaFreeAsync(q, c->st));
    }
  } else {
    const int ng = cols / 128;
    const int64_t warps = (int64_t)rows * ng;
    quantize_g128_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, c->st>>>(
        static_cast<const bf16*>(dsrc), rows, cols,
        static_cast<int8_t*>(M.w) + (size_t)dst_row0 * cols, (int64_t)cols * row_step,
        M.s + (size_t)dst_row0 * ng, (int64_t)ng * row_step);
    CK(cudaGetLastError());
  }
  if (owned) CK(cudaFreeAsync(owned, c->st));
  return M3_OK;
}

static int alloc_mat(m3_ctx* c, DMat& M, int N, int K, int wf) {
  M.N = N;
  M.K = K;
  M.wf = wf;
  M.tiled = wf != WF_I8G128;
  const size_t esz = wf == WF_BF16 ? 2 : 1;
  // tiled: rows padded to whole 16-row units with zeros
  const size_t rows = M.tiled ? (size_t)(N + kUnitRows - 1) / kUnitRows * kUnitRows : (size_t)N;
  CKR(dalloc(c, &M.w, esz * rows * K));
  // padding rows: zeros (int8 is stored biased: 0x80 is q = 0)
  if (M.tiled && rows != (size_t)N) CK(cudaMemset(M.w, wf == WF_I8ROW ? 0x80 : 0, esz * rows * K));
  if (wf == WF_I8ROW) CKR(dalloc(c, &M.s, sizeof(float) * N));
  if (wf == WF_I8G128) CKR(dalloc(c, &M.s, sizeof(float) * (size_t)N * (K / 128)));
  return M3_OK;
}

static int put_vec(m3_ctx* c, bf16** dst, const void* src, int n, int mem) {
  if (!src) return fail(M3_EINVAL, "null norm pointer");
  if (!*dst) CKR(dalloc(c, dst, sizeof(bf16) * n));
  CK(cudaMemcpyAsync(*dst, src, sizeof(bf16) * n,
                     mem == M3_MEM_DEVICE ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice,
                     c->st));
  return M3_OK;
}

static int load_layer(m3_ctx* c, DLayer& L, const m3_layer_src& s, int mem, int wf, int H,
                      int Hq, int Hkv, int d, int ffn) {
  const int nq = Hq * d, nkv = Hkv * d;
  if (!L.qkv.w) {
    CKR(alloc_mat(c, L.qkv, nq + 2 * nkv, H, wf));
    CKR(alloc_mat(c, L.o, H, nq, wf));
    CKR(alloc_mat(c, L.gu, 2 * ffn, H, wf));
    CKR(alloc_mat(c, L.d, H, ffn, wf));
  }
  CKR(put_rows(c, L.qkv, s.wq, mem, nq, 0, 1));
  CKR(put_rows(c, L.qkv, s.wk, mem, nkv, nq, 1));
  CKR(put_rows(c, L.qkv, s.wv, mem, nkv, nq + nkv, 1));
  CKR(put_rows(c, L.o, s.wo, mem, H, 0, 1));
  CKR(put_rows(c, L.gu, s.wg, mem, ffn, 0, 2));  // gate rows at 2j
  CKR(put_rows(c, L.gu, s.wu, mem, ffn, 1, 2));  // up rows at 2j+1
  CKR(put_rows(c, L.d, s.wd, mem, ffn == 0 ? 0 : H, 0, 1));
  CKR(put_vec(c, &L.attn_norm, s.attn_norm, H, mem));
  CKR(put_vec(c, &L.mlp_norm, s.mlp_norm, H, mem));
  CKR(put_vec(c, &L.q_norm, s.q_norm, d, mem));
  CKR(put_vec(c, &L.k_norm, s.k_norm, d, mem));
  return M3_OK;
}

extern "C" int m3_load_weights(m3_ctx* c, const m3_weight_src* src, int wdtype) {
  if (!c || !src) return fail(M3_EINVAL, "null argument");
  if (wdtype != M3_W_BF16 && wdtype != M3_W_INT8) return fail(M3_EINVAL, "wdtype");
  if (c->wdtype >= 0 && c->wdtype != wdtype) return fail(M3_ESTATE, "wdtype differs from first load");
  const m3_config& g = c->cfg;
  if (src->n_layers < 0 || src->first_layer < 0 || src->first_layer + src->n_layers > g.n_layers)
    return fail(M3_EINVAL, "layer range");
  if (src->n_layers > 0 && !src->layers) return fail(M3_EINVAL, "null layers");
  c->wdtype = wdtype;
  const int wf = wdtype == M3_W_INT8 ? WF_I8ROW : WF_BF16;
  CKR(enter(c));
  for (int i = 0; i < src->n_layers; ++i) {
    const int l = src->first_layer + i;
    CKR(load_layer(c, c->L[l], src->layers[i], src->mem, wf, g.hidden, g.n_q_heads, g.n_kv_heads,
                   g.head_dim, g.ffn));
    c->loaded[l] = 1;
    if ((size_t)l < c->pf_rm_ok.size()) c->pf_rm_ok[l] = 0;  // the prefill copy is stale
  }
  if (src->final_norm) CKR(put_vec(c, &c->final_norm, src->final_norm, g.hidden, src->mem));
  if (src->lm_head) {
    if (g.has_end_token && !src->lm_end_row)
      return fail(M3_EINVAL, "the config has an end token: lm_end_row is needed with lm_head");
    if (!c->lm.w) CKR(alloc_mat(c, c->lm, n_cand(g), g.hidden, wf));
    CKR(put_rows(c, c->lm, src->lm_head, src->mem, g.slice_len, 0, 1));
    if (g.has_end_token) CKR(put_rows(c, c->lm, src->lm_end_row, src->mem, 1, g.slice_len, 1));
    c->head_loaded = true;
  }
  CK(cudaStreamSynchronize(c->st));  // sources may be freed on return
  return leave(c);
}

extern "C" int m3_load_depth_weights(m3_ctx* c, const m3_depth_src* src) {
  if (!c || !src) return fail(M3_EINVAL, "null argument");
  const m3_config& g = c->cfg;
  if (g.depth_layers <= 0) return fail(M3_ESTATE, "config has no depth decoder");
  if (!src->layers || !src->proj || !src->emb || !src->final_norm || !src->heads)
    return fail(M3_EINVAL, "null depth weight pointer");
  CKR(enter(c));
  const int Dh = g.depth_hidden;
  for (int l = 0; l < g.depth_layers; ++l)
    CKR(load_layer(c, c->DL[l], src->layers[l], src->mem, WF_I8G128, Dh, g.depth_heads,
                   g.depth_heads, g.depth_head_dim, g.depth_ffn));
  if (!c->dproj.w) CKR(alloc_mat(c, c->dproj, Dh, g.hidden, WF_I8G128));
  CKR(put_rows(c, c->dproj, src->proj, src->mem, Dh, 0, 1));
  c->demb.resize(g.depth_codebooks, nullptr);
  c->demb_rows.resize(g.depth_codebooks);
  c->dheads.resize(g.depth_codebooks);
  for (int j = 0; j < g.depth_codebooks; ++j) {
    const int n = j == 0 ? g.slice_len : g.depth_vocab;
    c->demb_rows[j] = n;
    if (!src->emb[j] || !src->heads[j]) return fail(M3_EINVAL, "null depth table");
    if (!c->demb[j]) CKR(dalloc(c, &c->demb[j], sizeof(bf16) * (size_t)n * Dh));
    CK(cudaMemcpyAsync(c->demb[j], src->emb[j], sizeof(bf16) * (size_t)n * Dh,
                       src->mem == M3_MEM_DEVICE ? cudaMemcpyDeviceToDevice
                                                 : cudaMemcpyHostToDevice,
                       c->st));
    if (!c->dheads[j].w) CKR(alloc_mat(c, c->dheads[j], g.depth_vocab, Dh, WF_I8G128));
    CKR(put_rows(c, c->dheads[j], src->heads[j], src->mem, g.depth_vocab, 0, 1));
  }
  CKR(put_vec(c, &c->dfinal, src->final_norm, Dh, src->mem));
  CK(cudaStreamSynchronize(c->st));
  c->depth_loaded = true;
  return leave(c);
}

extern "C" int m3_quantize_int8(const void* w, int64_t rows, int64_t cols, int64_t group,
                                int8_t* q, float* scales, void* cuda_stream) {
  if (!w || !q || !scales || rows <= 0 || cols <= 0) return fail(M3_EINVAL, "bad argument");
  if (group != cols && group != 128) return fail(M3_EINVAL, "group must be cols or 128");
  if (cols % group) return fail(M3_EINVAL, "cols % group != 0");
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  if (group == cols) {
    quantize_rows_kernel<<<dim3(1, (unsigned)rows), 256, 0, st>>>(static_cast<const bf16*>(w),
                                                                  cols, cols, q, cols, scales, 1);
  } else {
    const int64_t warps = rows * (cols / 128);
    quantize_g128_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, st>>>(
        static_cast<const bf16*>(w), rows, cols, q, cols, scales, cols / 128);
  }
  CK(cudaGetLastError());
  return M3_OK;
}

// which: 0 wq 1 wk 2 wv 3 wo 4 wg 5 wu 6 wd 7 lm_head; 8.. the same for depth
// layers; 16 depth proj; 17 + j depth head j.
extern "C" int m3_export_weight(m3_ctx* c, int which, int layer, void* q_host, float* s_host) {
  if (!c || !q_host) return fail(M3_EINVAL, "null argument");
  const m3_config& g = c->cfg;
  const DMat* M = nullptr;
  int row0 = 0, rows = 0, step = 1;
  const bool depth = which >= 8;
  const int w = depth && which < 16 ? which - 8 : which;
  if (which == 16) {
    M = &c->dproj;
    rows = M->N;
  } else if (which >= 17) {
    if (which - 17 >= (int)c->dheads.size()) return fail(M3_EINVAL, "depth head index");
    M = &c->dheads[which - 17];
    rows = M->N;
  } else if (w == 7) {
    if (depth) return fail(M3_EINVAL, "which");
    M = &c->lm;
    rows = M->N;
  } else {
    const std::vector<DLayer>& LL = depth ? c->DL : c->L;
    if (layer < 0 || layer >= (int)LL.size()) return fail(M3_EINVAL, "layer");
    const DLayer& L = LL[layer];
    const int hq = depth ? g.depth_heads : g.n_q_heads, hkv = depth ? g.depth_heads : g.n_kv_heads;
    const int d = depth ? g.depth_head_dim : g.head_dim;
    switch (w) {
      case 0: M = &L.qkv; row0 = 0; rows = hq * d; break;
      case 1: M = &L.qkv; row0 = hq * d; rows = hkv * d; break;
      case 2: M = &L.qkv; row0 = (hq + hkv) * d; rows = hkv * d; break;
      case 3: M = &L.o; rows = M->N; break;
      case 4: M = &L.gu; row0 = 0; step = 2; rows = M->N / 2; break;
      case 5: M = &L.gu; row0 = 1; step = 2; rows = M->N / 2; break;
      case 6: M = &L.d; rows = M->N; break;
      default: return fail(M3_EINVAL, "which");
    }
  }
  if (!M || !M->w) return fail(M3_ESTATE, "weight not loaded");
  CK(cudaStreamSynchronize(c->st));
  const size_t esz = M->wf == WF_BF16 ? 2 : 1;
  const size_t rb = esz * M->K;
  if (M->tiled) {
    // whole tiled matrix to the host, then the requested rows back to row-major
    std::vector<uint8_t> t(esz * (size_t)(M->N + kUnitRows - 1) / kUnitRows * kUnitRows * M->K);
    CK(cudaMemcpy(t.data(), M->w, t.size(), cudaMemcpyDeviceToHost));
    uint8_t* q = static_cast<uint8_t*>(q_host);
    for (int r = 0; r < rows; ++r)
      for (int k = 0; k < M->K; ++k)
        memcpy(q + (size_t)r * rb + k * esz,
               t.data() + tile_byte_offset(row0 + r * step, k, M->K, (int)esz), esz);
    if (M->wf == WF_I8ROW)  // tiled int8 is stored biased (q + 128)
      for (size_t i = 0; i < (size_t)rows * rb; ++i) q[i] ^= 0x80u;
  } else {
    CK(cudaMemcpy2D(q_host, rb, static_cast<const char*>(M->w) + (size_t)row0 * rb, rb * step, rb,
                    rows, cudaMemcpyDeviceToHost));
  }
  if (M->wf != WF_BF16 && s_host) {
    const int ns = M->wf == WF_I8ROW ? 1 : M->K / 128;
    CK(cudaMemcpy2D(s_host, sizeof(float) * ns, M->s + (size_t)row0 * ns,
                    sizeof(float) * ns * step, sizeof(float) * ns, rows, cudaMemcpyDeviceToHost));
  }
  return M3_OK;
}

// ---------------------------------------------------------------- KV cache --
extern "C" int m3_kv_alloc(m3_ctx* c, int rows, int max_positions, int kvdtype, int bucket) {
  if (!c) return fail(M3_EINVAL, "null ctx");
  if (rows < 1 || rows > c->cfg.max_rows) return fail(M3_EINVAL, "rows out of 1..max_rows");
  if (max_positions < 1) return fail(M3_EINVAL, "max_positions");
  if (bucket < 32 || bucket % 32) return fail(M3_EINVAL, "bucket must be a multiple of 32");
  if (kvdtype != M3_KV_BF16 && kvdtype != M3_KV_F16) return fail(M3_EINVAL, "kvdtype");
  CKR(enter(c));
  CK(cudaStreamSynchronize(c->st));
  drop_graphs(c);
  for (void* p : c->buckets) cudaFree(p);
  c->buckets.clear();
  const m3_config& g = c->cfg;
  c->kv_rows = rows;
  c->kv_max_pos = max_positions;
  c->kv_f16 = kvdtype == M3_KV_F16;
  c->bucket = bucket;
  c->max_pages = (max_positions + bucket - 1) / bucket;
  c->n_buckets = 0;
  c->bucket_bytes = (size_t)rows * g.n_layers * 2 * g.n_kv_heads * bucket * g.head_dim * 2;
  c->h_pages.assign((size_t)rows * g.n_layers * c->max_pages, 0ull);
  if (c->d_pages) {
    cudaFree(c->d_pages);
    for (auto it = c->allocs.begin(); it != c->allocs.end(); ++it)
      if (*it == c->d_pages) { c->allocs.erase(it); break; }
    c->d_pages = nullptr;
  }
  CKR(dalloc(c, &c->d_pages, sizeof(unsigned long long) * c->h_pages.size()));
  CK(cudaMemset(c->d_pages, 0, sizeof(unsigned long long) * c->h_pages.size()));
  if (c->d_vpages) {  // the prefill table is sized by max_pages too
    cudaFree(c->d_vpages);
    for (auto it = c->allocs.begin(); it != c->allocs.end(); ++it)
      if (*it == c->d_vpages) { c->allocs.erase(it); break; }
    c->d_vpages = nullptr;
  }
  return leave(c);
}

// Make sure buckets cover positions [0, npos).  New buckets are zeroed, so a
// row that skips positions reads zeros there.
static int ensure_pages(m3_ctx* c, int npos) {
  const int need = (npos + c->bucket - 1) / c->bucket;
  if (need <= c->n_buckets) return M3_OK;
  if (need > c->max_pages) return fail(M3_ECAPACITY, "KV capacity exceeded");
  CK(cudaStreamSynchronize(c->st));
  const m3_config& g = c->cfg;
  const size_t page_bytes = (size_t)2 * g.n_kv_heads * c->bucket * g.head_dim * 2;
  for (int b = c->n_buckets; b < need; ++b) {
    void* p = nullptr;
    if (fault_due(c, M3_FAULT_ALLOC)) return fail(M3_ENOMEM, "injected KV bucket allocation failure");
    CK(cudaMalloc(&p, c->bucket_bytes));
    c->buckets.push_back(p);  // owned from here on, even if what follows fails
    CK(cudaMemset(p, 0, c->bucket_bytes));
    for (int r = 0; r < c->kv_rows; ++r)
      for (int l = 0; l < g.n_layers; ++l)
        c->h_pages[((size_t)r * g.n_layers + l) * c->max_pages + b] =
            (unsigned long long)(static_cast<char*>(p) + ((size_t)r * g.n_layers + l) * page_bytes);
  }
  c->n_buckets = need;
  CK(cudaMemcpy(c->d_pages, c->h_pages.data(), sizeof(unsigned long long) * c->h_pages.size(),
                cudaMemcpyHostToDevice));
  CK(cudaDeviceSynchronize());
  return M3_OK;
}

extern "C" int m3_kv_set(m3_ctx* c, int row, int n_positions, const void* k, const void* v, int mem) {
  if (!c || !k || !v) return fail(M3_EINVAL, "null argument");
  if (!c->d_pages) return fail(M3_ESTATE, "m3_kv_alloc first");
  if (row < 0 || row >= c->kv_rows) return fail(M3_EINVAL, "row");
  if (n_positions < 0 || n_positions > c->kv_max_pos) return fail(M3_ECAPACITY, "n_positions");
  if (n_positions == 0) return M3_OK;
  CKR(enter(c));
  CKR(ensure_pages(c, n_positions));
  const m3_config& g = c->cfg;
  const size_t bytes = sizeof(bf16) * (size_t)g.n_layers * n_positions * g.n_kv_heads * g.head_dim;
  const void *dk = nullptr, *dv = nullptr;
  void *ok = nullptr, *ov = nullptr;
  CKR(stage_src(c, k, bytes, mem, &dk, &ok));
  if (const int rc = stage_src(c, v, bytes, mem, &dv, &ov)) {
    if (ok) cudaFreeAsync(ok, c->st);
    return rc;
  }
  kv_set_kernel<<<c->nsm * 4, 256, 0, c->st>>>(
      static_cast<const bf16*>(dk), static_cast<const bf16*>(dv),
      c->d_pages + (size_t)row * g.n_layers * c->max_pages, g.n_layers, c->max_pages, c->bucket,
      n_positions, g.n_kv_heads, g.head_dim, c->kv_f16);
  CK(cudaGetLastError());
  if (ok) CK(cudaFreeAsync(ok, c->st));
  if (ov) CK(cudaFreeAsync(ov, c->st));
  CK(cudaStreamSynchronize(c->st));
  return leave(c);
}

extern "C" int m3_kv_get(m3_ctx* c, int row, int n_positions, void* k_host, void* v_host) {
  if (!c || !k_host || !v_host) return fail(M3_EINVAL, "null argument");
  if (!c->d_pages) return fail(M3_ESTATE, "m3_kv_alloc first");
  if (row < 0 || row >= c->kv_rows) return fail(M3_EINVAL, "row");
  if (n_positions < 0 || n_positions > c->n_buckets * c->bucket)
    return fail(M3_ECAPACITY, "n_positions beyond the allocated buckets");
  if (n_positions == 0) return M3_OK;
  CKR(enter(c));
  const m3_config& g = c->cfg;
  const size_t n = (size_t)g.n_layers * n_positions * g.n_kv_heads * g.head_dim;
  void *dk = nullptr, *dv = nullptr;
  CK(cudaMallocAsync(&dk, n * 2, c->st));
  CK(cudaMallocAsync(&dv, n * 2, c->st));
  kv_get_kernel<<<c->nsm * 4, 256, 0, c->st>>>(
      static_cast<uint16_t*>(dk), static_cast<uint16_t*>(dv),
      c->d_pages + (size_t)row * g.n_layers * c->max_pages, g.n_layers, c->max_pages, c->bucket,
      n_positions, g.n_kv_heads, g.head_dim);
  CK(cudaGetLastError());
  CK(cudaMemcpyAsync(k_host, dk, n * 2, cudaMemcpyDeviceToHost, c->st));
  CK(cudaMemcpyAsync(v_host, dv, n * 2, cudaMemcpyDeviceToHost, c->st));
  CK(cudaFreeAsync(dk, c->st));
  CK(cudaFreeAsync(dv, c->st));
  CK(cudaStreamSynchronize(c->st));
  return leave(c);
}

// ------------------------------------------------------------ the frame ----
static int attn_splits(const m3_ctx* c, int rows, int nb) {
  // as many splits as keep every (row, KV head) pair's CTAs resident at
  // once: a second, partial wave of CTAs would run at a fraction of the SMs
  const int pairs = rows * c->cfg.n_kv_heads;
  const int per_sm = c->attn_per_sm[c->kv_f16 ? 1 : 0];
  int s = (c->nsm * (per_sm > 0 ? per_sm : 2)) / pairs;
  const int tiles = nb * c->bucket / kAttnTile;
  if (s > tiles) s = tiles;
  if (s > c->max_splits) s = c->max_splits;
  return s < 1 ? 1 : s;
}

// A GEMV over all `rows` batch rows: one launch of the tiled tensor-core
// kernel, or launches of at most 4 rows of the CUDA-core kernel (int8 with
// group-128 scales).
static int ring_stages(const m3_ctx* c, int wf) {
  return c->tile_ns > 0 ? c->tile_ns : (wf == WF_I8ROW ? 2 : 3);
}

static int dyn_mask(const m3_ctx* c, int wf) {
  if (c->tile_dyn_mask >= 0) return c->tile_dyn_mask;
  return wf == WF_I8ROW ? ~0 : (1 << EPI_STORE) | (1 << EPI_SWIGLU);
}

static int gemv_rows(m3_ctx* c, const DMat& M, int epi, int rows, const bf16* x, int ldx,
                     const bf16* gamma, bf16* out, int ldo, const SampleArgs* smp, bool& pdl,
                     const FrameParams* fp = nullptr, bool cache_plan = true, int ring_ns = 0,
                     int max_grid = 0) {
  const int ns = ring_ns > 0 ? ring_ns : ring_stages(c, M.wf);
  const int step = M.tiled ? rows : 4;
  for (int r0 = 0; r0 < rows; r0 += step) {
    GemvArgs a{};
    a.w = M.w;
    a.scales = M.s;
    a.N = M.N;
    a.K = M.K;
    a.row0 = r0;
    a.mr = rows - r0 < step ? rows - r0 : step;
    a.x = x + (size_t)r0 * ldx;
    a.ldx = ldx;
    a.gamma = gamma;
    a.eps = c->cfg.rms_eps;
    a.out = out ? out + (size_t)r0 * ldo : nullptr;
    a.ldo = ldo;
    a.fp = fp ? fp : c->fp;
    if (smp) a.smp = *smp;
    a.err = c->err;
    if (M.tiled) {
      const auto key = std::make_tuple(M.N, M.K, a.mr, M.wf, epi * 16 + ns);
      auto it = c->tile_plans.find(key);
      TileLaunch L;
      if (it != c->tile_plans.end()) {
        L = it->second;
      } else {
        // the preferred ring and kernel; when the activations of many rows
        // leave no room for that ring, two stages, then dynamic claiming
        const bool dyn_ok = c->tile_dyn && a.ldx % 8 == 0;
        cudaError_t pe = plan_gemv_tile(M.N, M.K, a.mr, M.wf, epi, c->nsm, c->tile_sb, ns,
                                        dyn_ok && ((dyn_mask(c, M.wf) >> epi) & 1), &L);
        if (pe == cudaErrorInvalidConfiguration && ns > 2)
          pe = plan_gemv_tile(M.N, M.K, a.mr, M.wf, epi, c->nsm, c->tile_sb, 2,
                              dyn_ok && ((dyn_mask(c, M.wf) >> epi) & 1), &L);
        if (pe == cudaErrorInvalidConfiguration)
          pe = plan_gemv_tile(M.N, M.K, a.mr, M.wf, epi, c->nsm, c->tile_sb, 2, dyn_ok, &L);
        CK(pe);
        if (cache_plan) c->tile_plans.emplace(key, L);
      }
      // a caller's fixed-size scratch (part_z / part_i) bounds the CTAs
      if (max_grid > 0 && L.grid > max_grid)
        return fail(M3_EINVAL, "the launch needs more CTAs than the static scratch holds");
      if (L.dyn) {
        a.ctr = c->tile_ctrs + 2 * (c->tile_ctr_next % kTileCtrPairs);
        a.lazy_claim = c->tile_lazy;
        ++c->tile_ctr_next;
      }
      float* ssq_written = nullptr;
      if (c->ssq_track) {
        if (gamma && c->ssq_cur) {
          a.ssq_in = c->ssq_cur;
          a.ssq_n = c->ssq_n;
        }
        if (epi == EPI_RESID && M.N == c->cfg.hidden) {
          ssq_written = c->ssq_cur == c->ssq_buf[0] ? c->ssq_buf[1] : c->ssq_buf[0];
          a.ssq_out = ssq_written;
        }
      }
      CK(launch_gemv_tile(a, M.wf, epi, L, c->st, pdl));
      if (epi == EPI_RESID) {
        c->ssq_cur = ssq_written;  // a residual add without partials invalidates them
        c->ssq_n = (M.N + kUnitRows - 1) / kUnitRows;
      }
    } else {
      if (max_grid > 0) return fail(M3_EINVAL, "static scratch needs the tiled GEMV");
      CK(launch_gemv(a, M.wf, epi, c->st, pdl, c->nsm));
    }
    pdl = true;
  }
  return M3_OK;
}

// prefill: the rows are tokens of one sequence whose page-table rows all
// point at its pages; the attention first appends every row's K/V, then
// attends from the cache (causal through the positions).
static int record_layer(m3_ctx* c, const DLayer& L, Acts& A, int rows, int H, int Hq, int Hkv,
                        int d, int ffn, const unsigned long long* pages, int layer, int n_layers,
                        int max_pages, int page_size, int kv_f16, int splits, int fixed_pos,
                        const double* inv_freq, const float2* rope, bool& pdl,
                        bool prefill = false) {
  const int ldqkv = (Hq + 2 * Hkv) * d;
  CKR(gemv_rows(c, L.qkv, EPI_STORE, rows, A.x, H, L.attn_norm, A.qkv, ldqkv, nullptr, pdl));
  AttnArgs at{};
  at.qkv = A.qkv;
  at.ldqkv = ldqkv;
  at.q_norm = L.q_norm;
  at.k_norm = L.k_norm;
  at.eps = c->cfg.rms_eps;
  at.inv_freq = inv_freq;
  at.rope = rope;
  at.rope_ld = fixed_pos >= 0 ? 0 : d / 2;  // a fixed position: one row of the table
  at.pages = pages;
  at.layer = layer;
  at.n_layers = n_layers;
  at.max_pages = max_pages;
  at.page_size = page_size;
  at.Hq = Hq;
  at.Hkv = Hkv;
  at.out = A.o;
  at.fp = c->fp;
  at.fixed_pos = fixed_pos;
  at.err = c->err;
  if (prefill) {
    at.mode = 1;
    CK(launch_attn(at, d, kv_f16, 1, rows, c->st, true));
    // the cached tiles are fetched before a PDL wait: take a full dependency
    at.mode = 2;
    CK(launch_attn(at, d, kv_f16, splits, rows, c->st, false));
  } else {
    CK(launch_attn(at, d, kv_f16, splits, rows, c->st, true));
  }
  // the projection after attention: a ring small enough for its CTAs to
  // sit beside the attention CTAs and stream while attention runs
  CKR(gemv_rows(c, L.o, EPI_RESID, rows, A.o, Hq * d, nullptr, A.x, H, nullptr, pdl, nullptr,
                true, fixed_pos < 0 ? c->tile_ns_o : 0));
  CKR(gemv_rows(c, L.gu, EPI_SWIGLU, rows, A.x, H, L.mlp_norm, A.act, ffn, nullptr, pdl));
  CKR(gemv_rows(c, L.d, EPI_RESID, rows, A.act, ffn, nullptr, A.x, H, nullptr, pdl));
  return M3_OK;
}

static int record_frame(m3_ctx* c, int rows, int nb) {
  const m3_config& g = c->cfg;
  const int splits = attn_splits(c, rows, nb);
  bool pdl = false;  // the first kernel follows the parameter block in plain stream order
  // the frame's input was copied in: no partials for the first norm
  c->ssq_cur = nullptr;
  c->ssq_track = true;
  struct Untrack {
    m3_ctx* c;
    ~Untrack() {
      c->ssq_track = false;
      c->ssq_cur = nullptr;
    }
  } untrack{c};
  for (int l = 0; l < g.n_layers; ++l)
    CKR(record_layer(c, c->L[l], c->A, rows, g.hidden, g.n_q_heads, g.n_kv_heads, g.head_dim,
                     g.ffn, c->d_pages, l, g.n_layers, c->max_pages, c->bucket, c->kv_f16, splits,
                     -1, c->inv_freq, c->rope, pdl));
  SampleArgs sa{};
  sa.logits = c->logits;
  sa.logits_ld = n_cand(g);
  sa.codes = c->codes;
  sa.code_stride = 1;
  sa.index_base = (unsigned long long)g.slice_start;
  sa.end_row1 = g.has_end_token ? g.slice_len + 1 : 0;
  sa.end_index = (unsigned long long)g.end_token;
  sa.part_z = c->spz;
  sa.part_i = c->spi;
  sa.counter = c->scnt;
  sa.h_out = c->h;
  sa.gbuf = c->gbuf;
  CKR(gemv_rows(c, c->lm, EPI_SAMPLE, rows, c->A.x, g.hidden, c->final_norm, nullptr, 0, &sa, pdl));
  return M3_OK;
}

// Run `record` either directly or through a cached graph keyed by `key`.
template <typename F>
static int run_graph(m3_ctx* c, std::map<std::pair<int, int>, cudaGraphExec_t>& cache,
                     std::pair<int, int> key, F record) {
  if (!c->use_graphs) return record();
  auto it = cache.find(key);
  if (it == cache.end()) {
    cudaGraph_t graph = nullptr;
    if (fault_due(c, M3_FAULT_GRAPH)) return fail(M3_ECUDA, "injected graph capture failure");
    CK(cudaStreamBeginCapture(c->st, cudaStreamCaptureModeThreadLocal));
    int rc = record();
    cudaError_t e = cudaStreamEndCapture(c->st, &graph);
    if (rc != M3_OK) {
      if (graph) cudaGraphDestroy(graph);
      return rc;
    }
    if (e != cudaSuccess) return fail(M3_ECUDA, std::string("graph capture: ") + cudaGetErrorString(e));
    cudaGraphExec_t exec = nullptr;
    e = cudaGraphInstantiate(&exec, graph, 0);
    cudaGraphDestroy(graph);
    if (e != cudaSuccess) return fail(M3_ECUDA, std::string("graph instantiate: ") + cudaGetErrorString(e));
    it = cache.emplace(key, exec).first;
  }
  CK(cudaGraphLaunch(it->second, c->st));
  return M3_OK;
}

extern "C" int m3_decode_frame(m3_ctx* c, int rows, const int32_t* positions, uint64_t seed,
                               uint64_t frame, const void* x_in, float cfg_scale,
                               float temperature, int32_t* codes, void* h_out, float* logits) {
  if (!c || !positions || !x_in || !codes) return fail(M3_EINVAL, "null argument");
  const m3_config& g = c->cfg;
  if (!c->d_pages) return fail(M3_ESTATE, "m3_kv_alloc first");
  for (int l = 0; l < g.n_layers; ++l)
    if (!c->loaded[l]) return fail(M3_ESTATE, "layer " + std::to_string(l) + " not loaded");
  if (!c->head_loaded || !c->final_norm) return fail(M3_ESTATE, "lm_head / final norm not loaded");
  if (rows < 1 || rows > c->kv_rows) return fail(M3_EINVAL, "rows out of 1..cache rows");
  if (!(cfg_scale >= 0.0f) || !(temperature > 0.0f)) return fail(M3_EINVAL, "cfg_scale / temperature");
  if (cfg_scale > 0.0f && rows % 2) return fail(M3_EINVAL, "cfg_scale > 0 needs (cond, uncond) row pairs");
  FrameParams fp{};
  fp.rows = rows;
  fp.cfg_on = cfg_scale > 0.0f;
  fp.cfg_scale = cfg_scale;
  fp.temperature = temperature;
  fp.seed = seed;
  fp.frame = frame;
  fp.top_k = c->top_k;
  int maxpos = 0;
  for (int r = 0; r < rows; ++r) {
    if (positions[r] < 0 || positions[r] >= c->kv_max_pos)
      return fail(M3_ECAPACITY, "position " + std::to_string(positions[r]) + " outside the KV capacity");
    fp.pos[r] = positions[r];
    maxpos = positions[r] > maxpos ? positions[r] : maxpos;
  }
  CKR(enter(c));
  CKR(ensure_pages(c, maxpos + 1));
  CK(cudaMemcpyAsync(c->A.x, x_in, sizeof(bf16) * rows * g.hidden, cudaMemcpyDeviceToDevice, c->st));
  set_frame_params_kernel<<<1, 32, 0, c->st>>>(c->fp, fp);
  CK(cudaGetLastError());
  rope_table_kernel<<<rows, 64, 0, c->st>>>(c->fp, c->inv_freq, g.head_dim / 2, c->rope);
  CK(cudaGetLastError());
  CKR(run_graph(c, c->graphs, {rows, c->n_buckets},
                [&] { return record_frame(c, rows, c->n_buckets); }));
  CK(cudaMemcpyAsync(codes, c->codes, sizeof(int) * rows, cudaMemcpyDeviceToDevice, c->st));
  if (h_out)
    CK(cudaMemcpyAsync(h_out, c->h, sizeof(bf16) * rows * g.hidden, cudaMemcpyDeviceToDevice, c->st));
  if (logits)
    CK(cudaMemcpyAsync(logits, c->logits, sizeof(float) * rows * n_cand(g),
                       cudaMemcpyDeviceToDevice, c->st));
  return leave(c);
}

// --------------------------------------------------------- depth decoder ---

// Arguments of the persistent depth kernel (depth.cu) for `rows` rows.
static void fill_depth_args(const m3_ctx* c, int rows, bool forced, const bf16* hin, DepthArgs* a) {
  const m3_config& g = c->cfg;
  *a = DepthArgs{};
  a->rows = rows;
  a->Dh = g.depth_hidden;
  a->nh = g.depth_heads;
  a->hd = g.depth_head_dim;
  a->F = g.depth_ffn;
  a->NC = g.depth_codebooks;
  a->V = g.depth_vocab;
  a->Hin = g.hidden;
  a->n_layers = g.depth_layers;
  a->eps = g.rms_eps;
  auto mat = [](const DMat& M) { return DepthMat{static_cast<const int8_t*>(M.w), M.s}; };
  for (int l = 0; l < g.depth_layers && l < kDepthMaxLayers; ++l) {
    const DLayer& L = c->DL[l];
    a->L[l] = DepthLayerW{mat(L.qkv), mat(L.o), mat(L.gu), mat(L.d),
                          L.attn_norm, L.mlp_norm, L.q_norm, L.k_norm};
  }
  a->proj = mat(c->dproj);
  for (int j = 0; j < g.depth_codebooks && j < kDepthMaxCodebooks; ++j) {
    if (j < (int)c->dheads.size()) a->heads[j] = mat(c->dheads[j]);
    if (j < (int)c->demb.size()) {
      a->emb[j] = c->demb[j];
      a->emb_rows[j] = c->demb_rows[j];
    }
  }
  a->final_norm = c->dfinal;
  a->rope = c->drope;
  a->h_in = hin;
  a->code0 = c->dprev;
  a->forced = forced ? c->dforced : nullptr;
  // the end token's code (slice_len) has no semantic embedding: a zero input
  a->zero_code = g.has_end_token ? g.slice_len : INT_MIN;
  a->codes = c->dcodes;
  a->prev = c->dprev;
  a->logits = c->dlogits;
  a->fp = c->fp;
  const size_t R = g.max_rows, qn = (size_t)g.depth_heads * g.depth_head_dim;
  a->words = c->dwords;
  a->words_bytes = c->dwords_bytes;
  a->xw = c->dwords;
  a->qkvw = a->xw + R * g.depth_hidden;
  a->attw = a->qkvw + R * 3 * qn;
  a->actw = a->attw + R * qn;
  a->kvw = a->actw + R * g.depth_ffn;
  a->part = c->dpart;
  a->err = c->err;
}

// Whether the persistent kernel takes `rows` rows of this decoder (its
// shape limits and shared memory): then *smem its shared memory.
static int depth_persistent_plan(const m3_ctx* c, DepthArgs* a, size_t* smem, bool* ok) {
  const m3_config& g = c->cfg;
  *ok = false;
  if (g.depth_layers > kDepthMaxLayers || g.depth_codebooks > kDepthMaxCodebooks) return M3_OK;
  const cudaError_t e = depth_plan(a, c->nsm, smem);
  if (e == cudaErrorInvalidConfiguration) {
    (void)cudaGetLastError();
    return M3_OK;
  }
  CK(e);
  *ok = true;
  return M3_OK;
}

// hin: the frame's final-normed hidden state [rows][hidden]; the semantic
// code is in dprev.
static int record_depth(m3_ctx* c, int rows, bool forced, const bf16* hin) {
  const m3_config& g = c->cfg;
  const int Dh = g.depth_hidden, NC = g.depth_codebooks, V = g.depth_vocab;
  {  // the whole decoder as one persistent launch where its shape allows
    DepthArgs a;
    fill_depth_args(c, rows, forced, hin, &a);
    size_t smem = 0;
    bool ok = false;
    CKR(depth_persistent_plan(c, &a, &smem, &ok));
    if (ok) {
      CK(launch_depth(a, c->nsm, smem, c->st));
      return M3_OK;
    }
  }
  // separate launches per position and layer
  bool pdl = false;
  CKR(gemv_rows(c, c->dproj, EPI_STORE, rows, hin, g.hidden, nullptr, c->DA.x, Dh, nullptr, pdl));
  for (int j = 0; j <= NC; ++j) {
    if (j >= 1) {
      // the end token's code (slice_len) has no semantic embedding: a zero input
      const int zero_code = j == 1 && g.has_end_token ? g.slice_len : INT_MIN;
      CK(launch_ex(embed_kernel, dim3(rows), dim3(128), 0, c->st, true, (const int*)c->dprev,
                   (const bf16*)c->demb[j - 1], c->demb_rows[j - 1], 0, Dh, c->DA.x, c->err,
                   zero_code));
    }
    for (int l = 0; l < g.depth_layers; ++l)
      CKR(record_layer(c, c->DL[l], c->DA, rows, Dh, g.depth_heads, g.depth_heads,
                       g.depth_head_dim, g.depth_ffn, c->d_dpages, l, g.depth_layers, 1, 32, 0, 1,
                       j, c->dinv_freq, c->drope + (size_t)j * (g.depth_head_dim / 2), pdl));
    if (j >= 1) {
      SampleArgs sa{};
      sa.logits = c->dlogits + (size_t)(j - 1) * V;
      sa.logits_ld = NC * V;
      sa.codes = c->dcodes + (j - 1);
      sa.code_stride = NC;
      sa.prev = c->dprev;
      sa.forced = forced ? c->dforced + (j - 1) : nullptr;
      sa.forced_stride = NC;
      sa.index_base = (unsigned long long)j << 32;
      sa.part_z = c->spz;
      sa.part_i = c->spi;
      sa.counter = c->scnt + 1;
      CKR(gemv_rows(c, c->dheads[j - 1], EPI_SAMPLE, rows, c->DA.x, Dh, c->dfinal, nullptr, 0, &sa, pdl));
    }
  }
  return M3_OK;
}

extern "C" int m3_depth_decode(m3_ctx* c, int rows, const void* h_frame, const int32_t* code0,
                               uint64_t seed, uint64_t frame, float cfg_scale, float temperature,
                               const int32_t* forced, int32_t* codes, float* logits) {
  if (!c || !h_frame || !code0 || !codes) return fail(M3_EINVAL, "null argument");
  const m3_config& g = c->cfg;
  if (!c->depth_loaded) return fail(M3_ESTATE, "depth decoder not loaded");
  if (rows < 1 || rows > g.max_rows) return fail(M3_EINVAL, "rows out of 1..max_rows");
  if (!(cfg_scale >= 0.0f) || !(temperature > 0.0f)) return fail(M3_EINVAL, "cfg_scale / temperature");
  if (cfg_scale > 0.0f && rows % 2) return fail(M3_EINVAL, "cfg_scale > 0 needs (cond, uncond) row pairs");
  const int NC = g.depth_codebooks;
  FrameParams fp{};
  fp.rows = rows;
  fp.cfg_on = cfg_scale > 0.0f;
  fp.cfg_scale = cfg_scale;
  fp.temperature = temperature;
  fp.seed = seed;
  fp.frame = frame;
  CKR(enter(c));
  CK(cudaMemcpyAsync(c->dh, h_frame, sizeof(bf16) * rows * g.hidden, cudaMemcpyDeviceToDevice, c->st));
  CK(cudaMemcpyAsync(c->dprev, code0, sizeof(int) * rows, cudaMemcpyDeviceToDevice, c->st));
  if (forced)
    CK(cudaMemcpyAsync(c->dforced, forced, sizeof(int) * rows * NC, cudaMemcpyDeviceToDevice, c->st));
  set_frame_params_kernel<<<1, 32, 0, c->st>>>(c->fp, fp);
  CK(cudaGetLastError());
  const bool f = forced != nullptr;
  CKR(run_graph(c, c->dgraphs, {rows, f ? 1 : 0}, [&] { return record_depth(c, rows, f, c->dh); }));
  CK(cudaMemcpyAsync(codes, c->dcodes, sizeof(int) * rows * NC, cudaMemcpyDeviceToDevice, c->st));
  if (logits)
    CK(cudaMemcpyAsync(logits, c->dlogits, sizeof(float) * rows * NC * g.depth_vocab,
                       cudaMemcpyDeviceToDevice, c->st));
  return leave(c);
}

// ----------------------------------------------------------- prefill ----
// One layer over a prompt chunk of T tokens at positions p0 .. p0 + T - 1
// with the tensor-core GEMM: the norms over all T rows, the four projections
// as GEMMs, and the attention appending every token's K/V, then attending
// from the cache (causal through the positions).
// Elements of each projection in a layer's row-major prefill copy, in order.
static void pf_rm_sizes(const m3_config& g, size_t (&n)[4]) {
  const size_t H = g.hidden, q = (size_t)(g.n_q_heads + 2 * g.n_kv_heads) * g.head_dim;
  const size_t hq = (size_t)g.n_q_heads * g.head_dim, F = g.ffn;
  n[0] = q * H;       // qkv
  n[1] = H * hq;      // o
  n[2] = 2 * F * H;   // gate/up, interleaved rows
  n[3] = H * F;       // down
}

// The row-major bf16 copies the prefill GEMM reads, for every layer whose
// copy is missing or stale (untiled on the GPU from the decode layout).
static int ensure_prefill_copies(m3_ctx* c) {
  const m3_config& g = c->cfg;
  if (c->pf_rm.size() != (size_t)g.n_layers) {
    c->pf_rm.assign(g.n_layers, nullptr);
    c->pf_rm_ok.assign(g.n_layers, 0);
  }
  size_t n[4];
  pf_rm_sizes(g, n);
  CK(prepare_dit_gemm());  // the GEMM kernels' shared-memory limit, the tensor-map encoder
  for (int l = 0; l < g.n_layers; ++l) {
    if (c->pf_rm_ok[l]) continue;
    if (!c->pf_rm[l]) CKR(dalloc(c, &c->pf_rm[l], sizeof(bf16) * (n[0] + n[1] + n[2] + n[3])));
    const DLayer& L = c->L[l];
    bf16* dst = c->pf_rm[l];
    const DMat* mats[4] = {&L.qkv, &L.o, &L.gu, &L.d};
    for (int m = 0; m < 4; ++m) {
      untile_rows_kernel<<<c->nsm * 8, 256, 0, c->st>>>(static_cast<const uint8_t*>(mats[m]->w),
                                                          mats[m]->N, mats[m]->K, dst);
      CK(cudaGetLastError());
      dst += n[m];
    }
    c->pf_rm_ok[l] = 1;
  }
  return M3_OK;
}

static int record_prefill_layer(m3_ctx* c, const DLayer& L, int T, int p0, int layer) {
  const m3_config& g = c->cfg;
  const int H = g.hidden, d = g.head_dim, ldqkv = (g.n_q_heads + 2 * g.n_kv_heads) * d;
  const int hq = g.n_q_heads * d;
  // bf16 weights with their row-major copy: the TMA-fed tcgen05 GEMM
  const bf16* rm = (size_t)layer < c->pf_rm_ok.size() && c->pf_rm_ok[layer] ? c->pf_rm[layer]
                                                                           : nullptr;
  size_t nrm[4];
  pf_rm_sizes(g, nrm);
  auto gemm = [&](const DMat& M, int epi, const bf16* x, int ldx, bf16* out, int ldo) -> int {
    if (rm) {
      const bf16* w = rm + (&M == &L.qkv ? 0 : &M == &L.o ? nrm[0]
                                           : &M == &L.gu ? nrm[0] + nrm[1]
                                                         : nrm[0] + nrm[1] + nrm[2]);
      DitGemmArgs a{};
      a.M = T;
      a.N = M.N;
      a.K = M.K;
      a.out = out;
      a.ldo = ldo;
      a.err = c->err;
      const int de = epi == EPI_STORE ? DIT_EPI_STORE : epi == EPI_RESID ? DIT_EPI_RESID
                                                                         : DIT_EPI_GLU;
      CK(launch_dit_gemm(x, ldx, w, a, de, c->nsm, c->st, true));
      return M3_OK;
    }
    GemmTcArgs a{};
    a.w = static_cast<const uint8_t*>(M.w);
    a.scales = M.s;
    a.N = M.N;
    a.K = M.K;
    a.x = x;
    a.ldx = ldx;
    a.T = T;
    a.out = out;
    a.ldo = ldo;
    a.err = c->err;
    CK(launch_gemm_tc(a, M.wf, epi, c->st));
    return M3_OK;
  };
  rmsnorm_rows_kernel<<<T, 256, 0, c->st>>>(c->pf_x, L.attn_norm, g.rms_eps, H, c->pf_n);
  CK(cudaGetLastError());
  CKR(gemm(L.qkv, EPI_STORE, c->pf_n, H, c->pf_qkv, ldqkv));
  AttnArgs at{};
  at.qkv = c->pf_qkv;
  at.ldqkv = ldqkv;
  at.q_norm = L.q_norm;
  at.k_norm = L.k_norm;
  at.eps = g.rms_eps;
  at.inv_freq = c->inv_freq;
  at.rope = c->pf_rope;
  at.rope_ld = d / 2;
  at.pages = c->d_vpages;
  at.layer = layer;
  at.n_layers = g.n_layers;
  at.max_pages = c->max_pages;
  at.page_size = c->bucket;
  at.Hq = g.n_q_heads;
  at.Hkv = g.n_kv_heads;
  at.out = c->pf_o;
  at.fp = c->fp;
  at.fixed_pos = p0;
  at.pos_stride = 1;
  at.err = c->err;
  const int grp = g.n_q_heads / g.n_kv_heads;
  if ((d == 64 || d == 128) && 16 % grp == 0 && c->bucket % 32 == 0) {
    // the chunk's K/V appended, then the tiled causal attention in which the
    // chunk's tokens share every K/V tile
    CK(launch_attn_prefill(at, d, c->kv_f16, T, c->st));
  } else {
    at.mode = 1;
    CK(launch_attn(at, d, c->kv_f16, 1, T, c->st, false));
    at.mode = 2;
    CK(launch_attn(at, d, c->kv_f16, attn_splits(c, T, c->n_buckets), T, c->st, false));
  }
  CKR(gemm(L.o, EPI_RESID, c->pf_o, hq, c->pf_x, H));
  rmsnorm_rows_kernel<<<T, 256, 0, c->st>>>(c->pf_x, L.mlp_norm, g.rms_eps, H, c->pf_n);
  CK(cudaGetLastError());
  CKR(gemm(L.gu, EPI_SWIGLU, c->pf_n, H, c->pf_act, g.ffn));
  CKR(gemm(L.d, EPI_RESID, c->pf_act, g.ffn, c->pf_x, H));
  return M3_OK;
}

// Shapes the TMA GEMM takes: every K a multiple of 64, every N of 32.
static bool prefill_gemm_shapes_ok(const m3_config& g) {
  const int q = (g.n_q_heads + 2 * g.n_kv_heads) * g.head_dim, hq = g.n_q_heads * g.head_dim;
  return g.hidden % 64 == 0 && hq % 64 == 0 && g.ffn % 64 == 0 && q % 32 == 0;
}

static bool prefill_tc_ok(const m3_ctx* c) {
  if (c->prefill_tc == 0) return false;
  const m3_config& g = c->cfg;
  if (g.hidden % 16 || g.ffn % 16 || (g.n_q_heads * g.head_dim) % 16) return false;
  for (int l = 0; l < g.n_layers; ++l) {
    const DLayer& L = c->L[l];
    for (const DMat* M : {&L.qkv, &L.o, &L.gu, &L.d})
      if (!M->tiled || (M->wf != WF_BF16 && M->wf != WF_I8ROW) ||
          (c->prefill_tc < 0 && M->wf != WF_BF16))
        return false;
  }
  return true;
}

extern "C" int m3_prefill(m3_ctx* c, int row, int start, int n_tokens, const void* x,
                          void* h_last) {
  if (!c || !x) return fail(M3_EINVAL, "null argument");
  const m3_config& g = c->cfg;
  if (!c->d_pages) return fail(M3_ESTATE, "m3_kv_alloc first");
  for (int l = 0; l < g.n_layers; ++l)
    if (!c->loaded[l]) return fail(M3_ESTATE, "layer " + std::to_string(l) + " not loaded");
  if (h_last && !c->final_norm) return fail(M3_ESTATE, "final norm not loaded");
  if (row < 0 || row >= c->kv_rows) return fail(M3_EINVAL, "row");
  if (n_tokens < 1 || start < 0) return fail(M3_EINVAL, "start / n_tokens");
  if ((long long)start + n_tokens > c->kv_max_pos)
    return fail(M3_ECAPACITY, "start + n_tokens outside the KV capacity");
  const int R = g.max_rows;
  const bool tc = prefill_tc_ok(c);
  if (c->pf_chunk == 0)
    c->pf_chunk = c->wdtype == M3_W_BF16 && prefill_gemm_shapes_ok(g) ? 2048 : 256;
  const int P = c->pf_chunk;
  const int Rv = tc && P > R ? P : R;  // rows of the page table that map to the sequence
  CKR(enter(c));
  CKR(ensure_pages(c, start + n_tokens));
  // every token row of a chunk reads and writes the sequence's pages
  const size_t per_row = (size_t)g.n_layers * c->max_pages;
  if (!c->d_vpages) CKR(dalloc(c, &c->d_vpages, sizeof(unsigned long long) * (P > R ? P : R) * per_row));
  std::vector<unsigned long long> vp((size_t)Rv * per_row);
  for (int r = 0; r < Rv; ++r)
    std::memcpy(&vp[(size_t)r * per_row], &c->h_pages[(size_t)row * per_row],
                sizeof(unsigned long long) * per_row);
  CK(cudaMemcpyAsync(c->d_vpages, vp.data(), sizeof(unsigned long long) * vp.size(),
                     cudaMemcpyHostToDevice, c->st));
  CK(cudaStreamSynchronize(c->st));  // the host staging of the page table
  const bf16* xs = static_cast<const bf16*>(x);
  if (tc) {
    const int H = g.hidden, d = g.head_dim, ldqkv = (g.n_q_heads + 2 * g.n_kv_heads) * d;
    if (!c->pf_x) {
      CKR(dalloc(c, &c->pf_x, sizeof(bf16) * P * H));
      CKR(dalloc(c, &c->pf_n, sizeof(bf16) * P * H));
      CKR(dalloc(c, &c->pf_qkv, sizeof(bf16) * P * ldqkv));
      CKR(dalloc(c, &c->pf_o, sizeof(bf16) * P * g.n_q_heads * d));
      CKR(dalloc(c, &c->pf_act, sizeof(bf16) * P * g.ffn));
      CKR(dalloc(c, &c->pf_rope, sizeof(float2) * P * (d / 2)));
    }
    if (c->wdtype == M3_W_BF16 && prefill_gemm_shapes_ok(g)) CKR(ensure_prefill_copies(c));
    for (int c0 = 0; c0 < n_tokens; c0 += P) {
      const int T = n_tokens - c0 < P ? n_tokens - c0 : P;
      const int p0 = start + c0;
      CK(cudaMemcpyAsync(c->pf_x, xs + (size_t)c0 * H, sizeof(bf16) * T * H,
                         cudaMemcpyDeviceToDevice, c->st));
      rope_positions_kernel<<<(T * (d / 2) + 255) / 256, 256, 0, c->st>>>(c->inv_freq, d / 2, p0,
                                                                         T, c->pf_rope);
      CK(cudaGetLastError());
      for (int l = 0; l < g.n_layers; ++l) CKR(record_prefill_layer(c, c->L[l], T, p0, l));
      if (h_last && c0 + T == n_tokens) {
        rmsnorm_rows_kernel<<<1, 256, 0, c->st>>>(c->pf_x + (size_t)(T - 1) * H, c->final_norm,
                                                  g.rms_eps, H, static_cast<bf16*>(h_last));
        CK(cudaGetLastError());
      }
    }
    return leave(c);
  }
  for (int c0 = 0; c0 < n_tokens; c0 += R) {
    const int cn = n_tokens - c0 < R ? n_tokens - c0 : R;
    FrameParams fp{};
    fp.rows = cn;
    fp.temperature = 1.0f;
    for (int r = 0; r < cn; ++r) fp.pos[r] = start + c0 + r;
    CK(cudaMemcpyAsync(c->A.x, xs + (size_t)c0 * g.hidden, sizeof(bf16) * cn * g.hidden,
                       cudaMemcpyDeviceToDevice, c->st));
    set_frame_params_kernel<<<1, 32, 0, c->st>>>(c->fp, fp);
    CK(cudaGetLastError());
    rope_table_kernel<<<cn, 64, 0, c->st>>>(c->fp, c->inv_freq, g.head_dim / 2, c->rope);
    CK(cudaGetLastError());
    const int splits = attn_splits(c, cn, c->n_buckets);
    bool pdl = false;
    c->ssq_cur = nullptr;  // the chunk's input was copied in
    c->ssq_track = true;
    int rc = M3_OK;
    for (int l = 0; l < g.n_layers && rc == M3_OK; ++l)
      rc = record_layer(c, c->L[l], c->A, cn, g.hidden, g.n_q_heads, g.n_kv_heads, g.head_dim,
                        g.ffn, c->d_vpages, l, g.n_layers, c->max_pages, c->bucket, c->kv_f16,
                        splits, -1, c->inv_freq, c->rope, pdl, true);
    c->ssq_track = false;
    c->ssq_cur = nullptr;
    if (rc != M3_OK) return rc;
    if (h_last && c0 + cn == n_tokens) {
      rmsnorm_rows_kernel<<<1, 256, 0, c->st>>>(c->A.x + (size_t)(cn - 1) * g.hidden,
                                                c->final_norm, g.rms_eps, g.hidden,
                                                static_cast<bf16*>(h_last));
      CK(cudaGetLastError());
    }
  }
  return leave(c);
}

// ------------------------------------------------------ generation loop ----
constexpr int kLoopChunk = 16;  // frames between reads of the loop state

extern "C" int m3_load_feedback(m3_ctx* c, const void* tok_emb, const void* const* audio_emb,
                                int mem) {
  if (!c || !tok_emb) return fail(M3_EINVAL, "null argument");
  const m3_config& g = c->cfg;
  const int nc = g.depth_layers > 0 ? g.depth_codebooks : 0;
  if (nc && !audio_emb) return fail(M3_EINVAL, "the depth decoder's codebooks need audio_emb");
  for (int j = 0; j < nc; ++j)
    if (!audio_emb[j]) return fail(M3_EINVAL, "null audio_emb table");
  const cudaMemcpyKind kind = mem == M3_MEM_DEVICE ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice;
  CKR(enter(c));
  const size_t tb = sizeof(bf16) * (size_t)g.slice_len * g.hidden;
  if (!c->fb_tok) CKR(dalloc(c, &c->fb_tok, tb));
  CK(cudaMemcpyAsync(c->fb_tok, tok_emb, tb, kind, c->st));
  if (nc) {
    const size_t ab = sizeof(bf16) * (size_t)g.depth_vocab * g.hidden;
    c->fb_aud.resize(nc, nullptr);
    for (int j = 0; j < nc; ++j) {
      if (!c->fb_aud[j]) CKR(dalloc(c, &c->fb_aud[j], ab));
      CK(cudaMemcpyAsync(c->fb_aud[j], audio_emb[j], ab, kind, c->st));
    }
    if (!c->d_fb_aud) CKR(dalloc(c, &c->d_fb_aud, sizeof(bf16*) * nc));
    CK(cudaMemcpyAsync(c->d_fb_aud, c->fb_aud.data(), sizeof(bf16*) * nc, cudaMemcpyHostToDevice,
                       c->st));
  }
  CK(cudaStreamSynchronize(c->st));  // sources may be freed on return
  return leave(c);
}

// One frame of the loop: RoPE table from the device positions, the frame,
// the depth decoder, the feedback input and the loop state's advance.
static int record_loop_frame(m3_ctx* c, int rows, int nb, bool depth) {
  const m3_config& g = c->cfg;
  rope_table_kernel<<<rows, 64, 0, c->st>>>(c->fp, c->inv_freq, g.head_dim / 2, c->rope);
  CK(cudaGetLastError());
  CKR(record_frame(c, rows, nb));
  const int nc = depth ? g.depth_codebooks : 0;
  if (depth) {
    CK(cudaMemcpyAsync(c->dprev, c->codes, sizeof(int) * rows, cudaMemcpyDeviceToDevice, c->st));
    CKR(record_depth(c, rows, false, c->h));
  }
  LoopArgs la{};
  la.fp = c->fp;
  la.ls = c->loop;
  la.codes = c->codes;
  la.dcodes = c->dcodes;
  la.h = c->h;
  la.tok = c->fb_tok;
  la.aud = c->d_fb_aud;
  la.x = c->A.x;
  la.err = c->err;
  la.nc = nc;
  la.V = g.depth_vocab;
  la.H = g.hidden;
  la.S = g.slice_len;
  la.has_end = g.has_end_token ? 1 : 0;
  la.scale = (float)(1.0 / std::sqrt((double)(1 + nc)));
  loop_feedback_kernel<<<rows, 128, 0, c->st>>>(la);
  CK(cudaGetLastError());
  loop_advance_kernel<<<1, 32, 0, c->st>>>(la);
  CK(cudaGetLastError());
  return M3_OK;
}

extern "C" int m3_generate(m3_ctx* c, int rows, const int32_t* positions, uint64_t seed,
                           uint64_t frame0, const void* x_in, float cfg_scale, float temperature,
                           int max_frames, int32_t* codes, void* h_hist, int32_t* n_frames) {
  if (!c || !positions || !x_in || !codes || !n_frames) return fail(M3_EINVAL, "null argument");
  const m3_config& g = c->cfg;
  if (!c->d_pages) return fail(M3_ESTATE, "m3_kv_alloc first");
  for (int l = 0; l < g.n_layers; ++l)
    if (!c->loaded[l]) return fail(M3_ESTATE, "layer " + std::to_string(l) + " not loaded");
  if (!c->head_loaded || !c->final_norm) return fail(M3_ESTATE, "lm_head / final norm not loaded");
  if (!c->fb_tok) return fail(M3_ESTATE, "m3_load_feedback first");
  const bool depth = c->depth_loaded;
  if (depth && !c->d_fb_aud) return fail(M3_ESTATE, "m3_load_feedback without audio tables");
  if (rows < 1 || rows > c->kv_rows) return fail(M3_EINVAL, "rows out of 1..cache rows");
  if (max_frames < 1) return fail(M3_EINVAL, "max_frames < 1");
  if (!(cfg_scale >= 0.0f) || !(temperature > 0.0f)) return fail(M3_EINVAL, "cfg_scale / temperature");
  if (cfg_scale > 0.0f && rows % 2) return fail(M3_EINVAL, "cfg_scale > 0 needs (cond, uncond) row pairs");
  FrameParams fp{};
  fp.rows = rows;
  fp.cfg_on = cfg_scale > 0.0f;
  fp.cfg_scale = cfg_scale;
  fp.temperature = temperature;
  fp.seed = seed;
  fp.frame = frame0;
  fp.top_k = c->top_k;
  int maxpos = 0;
  for (int r = 0; r < rows; ++r) {
    if (positions[r] < 0 || (long long)positions[r] + max_frames > c->kv_max_pos)
      return fail(M3_ECAPACITY, "positions[" + std::to_string(r) + "] + max_frames outside the KV capacity");
    fp.pos[r] = positions[r];
    maxpos = positions[r] > maxpos ? positions[r] : maxpos;
  }
  const int nc = depth ? g.depth_codebooks : 0;
  const int keys = fp.cfg_on ? rows / 2 : rows;
  LoopState ls{};
  ls.keys = keys;
  for (int k = 0; k < keys; ++k) ls.active[k] = 1;
  ls.codes_out = codes;
  ls.h_hist = static_cast<bf16*>(h_hist);
  if (!c->loop) {
    void* p = nullptr;
    CKR(dzalloc(c, &p, sizeof(LoopState)));
    c->loop = static_cast<LoopState*>(p);
  }
  if (!c->h_loop) CK(cudaMallocHost(&c->h_loop, sizeof(LoopState)));
  if (!c->h_err) CK(cudaMallocHost(&c->h_err, sizeof(int)));
  CKR(enter(c));
  CK(cudaMemcpyAsync(c->A.x, x_in, sizeof(bf16) * rows * g.hidden, cudaMemcpyDeviceToDevice, c->st));
  CK(cudaMemsetAsync(codes, 0xFF, sizeof(int32_t) * (size_t)max_frames * rows * (1 + nc), c->st));
  if (h_hist) CK(cudaMemsetAsync(h_hist, 0, sizeof(bf16) * (size_t)max_frames * rows * g.hidden, c->st));
  set_frame_params_kernel<<<1, 32, 0, c->st>>>(c->fp, fp);
  CK(cudaGetLastError());
  loop_init_kernel<<<1, 32, 0, c->st>>>(c->loop, ls);
  CK(cudaGetLastError());
  for (int s0 = 0; s0 < max_frames; s0 += kLoopChunk) {
    const int n = max_frames - s0 < kLoopChunk ? max_frames - s0 : kLoopChunk;
    CKR(ensure_pages(c, maxpos + s0 + n));
    for (int i = 0; i < n; ++i)
      CKR(run_graph(c, c->lgraphs, {rows, 2 * c->n_buckets + (depth ? 1 : 0)},
                    [&] { return record_loop_frame(c, rows, c->n_buckets, depth); }));
    CK(cudaMemcpyAsync(c->h_loop, c->loop, sizeof(LoopState), cudaMemcpyDeviceToHost, c->st));
    CK(cudaMemcpyAsync(c->h_err, c->err, sizeof(int), cudaMemcpyDeviceToHost, c->st));
    CK(cudaStreamSynchronize(c->st));
    if (*c->h_err) break;
    bool any = false;
    for (int k = 0; k < keys; ++k) any = any || c->h_loop->active[k];
    if (!any) break;
  }
  for (int k = 0; k < keys; ++k) n_frames[k] = c->h_loop->count[k];
  CKR(leave(c));
  if (*c->h_err) return m3_sync_status(c);
  for (int k = 0; k < keys; ++k)
    if (n_frames[k] == 0) return fail(M3_EEMPTY, "key " + std::to_string(k) + " drew the end token at its first frame");
  return M3_OK;
}

// ------------------------------------------------------------- the rest ----
extern "C" int m3_embed(m3_ctx* c, int rows, const int32_t* codes, const void* table, int offset,
                        void* x_out) {
  if (!c || !codes || !table || !x_out) return fail(M3_EINVAL, "null argument");
  if (rows < 1 || rows > c->cfg.max_rows) return fail(M3_EINVAL, "rows");
  CKR(enter(c));
  CK(launch_ex(embed_kernel, dim3(rows), dim3(128), 0, c->st, false, codes,
               static_cast<const bf16*>(table), 0x7fffffff, offset, c->cfg.hidden,
               static_cast<bf16*>(x_out), c->err, INT_MIN));
  return leave(c);
}

extern "C" int m3_frame_kernels(const m3_ctx* c, int rows) {
  if (!c || rows < 1 || rows > c->cfg.max_rows) return fail(M3_EINVAL, "rows");
  if (c->L.empty() || !c->loaded[0]) return fail(M3_ESTATE, "weights not loaded");
  int n = 2 + 1;  // parameter block, RoPE table; the sampler
  for (int l = 0; l < c->cfg.n_layers; ++l) {
    n += 1;  // attention
    for (const DMat* M : {&c->L[l].qkv, &c->L[l].o, &c->L[l].gu, &c->L[l].d})
      n += M->tiled ? 1 : (rows + 3) / 4;
  }
  return n;
}

extern "C" int m3_depth_kernels(const m3_ctx* c, int rows) {
  if (!c || rows < 1 || rows > c->cfg.max_rows) return fail(M3_EINVAL, "rows");
  if (!c->depth_loaded) return fail(M3_ESTATE, "depth decoder not loaded");
  const m3_config& g = c->cfg;
  DepthArgs a;
  fill_depth_args(c, rows, false, c->dh, &a);
  size_t smem = 0;
  bool ok = false;
  CKR(depth_persistent_plan(c, &a, &smem, &ok));
  if (ok) return 1;
  // separate launches: the projections in launches of 4 rows (the CUDA-core
  // group-128 GEMV), embeddings, attention per position and layer
  const int P = g.depth_codebooks + 1, per4 = (rows + 3) / 4;
  return (1 + P * g.depth_layers * 4 + g.depth_codebooks) * per4 + g.depth_codebooks +
         P * g.depth_layers;
}

extern "C" double m3_frame_bytes(const m3_ctx* c, int rows, int ctx_len) {
  if (!c) return 0.0;
  const m3_config& g = c->cfg;
  const double esz = c->wdtype == M3_W_INT8 ? 1.0 : 2.0;
  const double H = g.hidden, d = g.head_dim;
  const double per_layer = H * (g.n_q_heads + 2.0 * g.n_kv_heads) * d + H * g.n_q_heads * d +
                           3.0 * H * g.ffn;
  double w = g.n_layers * per_layer * esz + (double)n_cand(g) * H * esz;
  if (c->wdtype == M3_W_INT8)
    w += 4.0 * (g.n_layers * ((g.n_q_heads + 2.0 * g.n_kv_heads) * d + H + 2.0 * g.ffn + H) +
                n_cand(g));
  w += 2.0 * (g.n_layers * (2.0 * H + 2.0 * d) + H);  // norm gains
  const double kv = (double)rows * (ctx_len + 1.0) * g.n_layers * 2.0 * g.n_kv_heads * d * 2.0;
  return w + kv;
}

extern "C" int m3_time_gemv(m3_ctx* c, int which, int rows, int iters, float* avg_ms,
                            double* bytes_per_launch) {
  if (!c || !avg_ms || !bytes_per_launch) return fail(M3_EINVAL, "null argument");
  const m3_config& g = c->cfg;
  if (which < 0 || which > 4 || iters < 1) return fail(M3_EINVAL, "which / iters");
  if (rows < 1 || rows > g.max_rows) return fail(M3_EINVAL, "rows");
  for (int l = 0; l < g.n_layers; ++l)
    if (!c->loaded[l]) return fail(M3_ESTATE, "weights not loaded");
  if (which == 4 && (!c->head_loaded || !c->final_norm)) return fail(M3_ESTATE, "lm_head not loaded");
  CKR(enter(c));
  // a neutral frame block (positions 0, no CFG) for the sampler's reads
  FrameParams fp{};
  fp.rows = rows;
  fp.temperature = 1.0f;
  set_frame_params_kernel<<<1, 32, 0, c->st>>>(c->fp, fp);
  CK(cudaGetLastError());
  cudaEvent_t e0, e1;
  CK(cudaEventCreate(&e0));
  CK(cudaEventCreate(&e1));
  const int H = g.hidden, ld = (g.n_q_heads + 2 * g.n_kv_heads) * g.head_dim;
  double bytes = 0.0;
  bool pdl = false;
  auto one = [&](int l) -> int {
    const DLayer& L = c->L[l];
    const DMat* M = nullptr;
    switch (which) {
      case 0: M = &L.qkv; CKR(gemv_rows(c, L.qkv, EPI_STORE, rows, c->A.x, H, L.attn_norm, c->A.qkv, ld, nullptr, pdl)); break;
      case 1: M = &L.o; CKR(gemv_rows(c, L.o, EPI_RESID, rows, c->A.o, g.n_q_heads * g.head_dim, nullptr, c->A.x, H, nullptr, pdl, nullptr, true, c->tile_ns_o)); break;
      case 2: M = &L.gu; CKR(gemv_rows(c, L.gu, EPI_SWIGLU, rows, c->A.x, H, L.mlp_norm, c->A.act, g.ffn, nullptr, pdl)); break;
      case 3: M = &L.d; CKR(gemv_rows(c, L.d, EPI_RESID, rows, c->A.act, g.ffn, nullptr, c->A.x, H, nullptr, pdl)); break;
      default: {
        M = &c->lm;
        SampleArgs sa{};
        sa.logits = c->logits;
        sa.logits_ld = n_cand(g);
        sa.codes = c->codes;
        sa.code_stride = 1;
        sa.index_base = (unsigned long long)g.slice_start;
        sa.end_row1 = g.has_end_token ? g.slice_len + 1 : 0;
        sa.end_index = (unsigned long long)g.end_token;
        sa.part_z = c->spz;
        sa.part_i = c->spi;
        sa.counter = c->scnt;
        sa.h_out = c->h;
        CKR(gemv_rows(c, c->lm, EPI_SAMPLE, rows, c->A.x, H, c->final_norm, nullptr, 0, &sa, pdl));
      }
    }
    const double esz = M->wf == WF_BF16 ? 2.0 : 1.0;
    const double nsc = M->wf == WF_I8ROW ? 1.0 : (M->wf == WF_I8G128 ? M->K / 128.0 : 0.0);
    const double outs = which == 2 ? M->N / 2.0 : (which == 4 ? M->N * 2.0 : M->N);  // fp32 logits
    bytes = (double)M->N * M->K * esz + 4.0 * M->N * nsc + 2.0 * rows * M->K + 2.0 * rows * outs +
            (which == 1 || which == 3 ? 2.0 * rows * M->N : 0.0);
    return M3_OK;
  };
  for (int i = 0; i < 3; ++i) CKR(one(i % g.n_layers));  // warm-up
  CK(cudaEventRecord(e0, c->st));
  for (int i = 0; i < iters; ++i) CKR(one(i % g.n_layers));
  CK(cudaEventRecord(e1, c->st));
  CK(cudaEventSynchronize(e1));
  float ms = 0.0f;
  CK(cudaEventElapsedTime(&ms, e0, e1));
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  *avg_ms = ms / iters;
  *bytes_per_launch = bytes;
  return leave(c);
}

// ------------------------------------------------------ checking hooks -----
extern "C" int m3_gumbel_fill(uint64_t seed, uint64_t frame, uint64_t row, uint64_t index0,
                              int64_t n, float* out, void* cuda_stream) {
  if (n < 0 || (n > 0 && !out)) return fail(M3_EINVAL, "n < 0 or null output");
  if (n == 0) return M3_OK;
  const long long blocks = (n + 255) / 256;
  gumbel_fill_kernel<<<(unsigned)(blocks < 4096 ? blocks : 4096), 256, 0,
                       static_cast<cudaStream_t>(cuda_stream)>>>(seed, frame, row, index0,
                                                                 (long long)n, out);
  CK(cudaGetLastError());
  return M3_OK;
}

extern "C" int m3_inject_fault(m3_ctx* c, int kind, int64_t nth) {
  if (!c) return fail(M3_EINVAL, "null ctx");
  if (kind == M3_FAULT_NONE) {
    c->fault_kind = M3_FAULT_NONE;
    c->fault_left = 0;
    return M3_OK;
  }
  if (kind < M3_FAULT_ALLOC || kind > M3_FAULT_GRAPH || nth < 1)
    return fail(M3_EINVAL, "kind must be M3_FAULT_ALLOC / _H2D / _GRAPH and nth >= 1");
  c->fault_kind = kind;
  c->fault_left = nth;
  return M3_OK;
}

extern "C" int m3_stalled_wait(m3_ctx* c, int64_t polls) {
  if (!c) return fail(M3_EINVAL, "null ctx");
  if (polls < 1 || polls > kSpinLimit) return fail(M3_EINVAL, "polls out of 1..2^22");
  CKR(enter(c));
  stalled_wait_kernel<<<1, 32, 0, c->st>>>(c->err, (long long)polls);
  CK(cudaGetLastError());
  return leave(c);
}

extern "C" int m3_sync_status(m3_ctx* c) {
  if (!c) return fail(M3_EINVAL, "null ctx");
  CK(cudaSetDevice(c->dev));
  CK(cudaStreamSynchronize(c->st));
  CK(cudaStreamSynchronize(c->user_st));
  int e = 0;
  CK(cudaMemcpy(&e, c->err, sizeof(int), cudaMemcpyDeviceToHost));
  if (e != 0) {
    CK(cudaMemset(c->err, 0, sizeof(int)));
    // a launch that gave up may have left its claim counters set
    CK(cudaMemset(c->tile_ctrs, 0, sizeof(unsigned) * 2 * kTileCtrPairs));
    if (e == kErrTimeout) return fail(M3_ETIMEOUT, "a device-side wait gave up");
    return fail(M3_EDEVICE, "a kernel recorded an out-of-range index");
  }
  return M3_OK;
}

extern "C" int m3_sample_noalloc(m3_ctx* c, int rows, const void* h, uint64_t seed,
                                 uint64_t frame, float cfg_scale, float temperature,
                                 int32_t* codes, float* logits) {
  if (!c || !h || !codes) return fail(M3_EINVAL, "null argument");
  const m3_config& g = c->cfg;
  if (!c->head_loaded) return fail(M3_ESTATE, "lm_head not loaded");
  if (rows < 1 || rows > kMaxRows || rows > g.max_rows)
    return fail(M3_EINVAL, "rows must be in 1..min(16, max_rows)");
  if (!(cfg_scale >= 0.0f) || !(temperature > 0.0f)) return fail(M3_EINVAL, "cfg_scale / temperature");
  if (cfg_scale > 0.0f && rows % 2) return fail(M3_EINVAL, "cfg_scale > 0 needs (cond, uncond) row pairs");
  unsigned char* scratch = c->noalloc_scratch;
  CKR(enter(c));
  FrameParams fp{};
  fp.rows = rows;
  fp.cfg_on = cfg_scale > 0.0f;
  fp.cfg_scale = cfg_scale;
  fp.temperature = temperature;
  fp.seed = seed;
  fp.frame = frame;
  FrameParams* dfp = reinterpret_cast<FrameParams*>(scratch + kNoAllocParamsOff);
  unsigned* counter = reinterpret_cast<unsigned*>(scratch + kNoAllocCounterOff);
  set_frame_params_kernel<<<1, 32, 0, c->st>>>(dfp, fp);
  CK(cudaGetLastError());
  CK(cudaMemsetAsync(counter, 0, sizeof(unsigned), c->st));  // the ticket starts at zero
  SampleArgs sa{};
  sa.logits = logits;
  sa.logits_ld = n_cand(g);
  sa.codes = codes;
  sa.code_stride = 1;
  sa.index_base = (unsigned long long)g.slice_start;
  sa.end_row1 = g.has_end_token ? g.slice_len + 1 : 0;
  sa.end_index = (unsigned long long)g.end_token;
  sa.part_z = reinterpret_cast<float*>(scratch + kNoAllocPartZOff);
  sa.part_i = reinterpret_cast<int*>(scratch + kNoAllocPartIOff);
  sa.counter = counter;
  bool pdl = false;
  // h is already the final-normed hidden state: no gain; launch plans are
  // looked up, not cached, so this call allocates nothing on the host either
  CKR(gemv_rows(c, c->lm, EPI_SAMPLE, rows, static_cast<const bf16*>(h), g.hidden, nullptr,
                nullptr, 0, &sa, pdl, dfp, false, 0, kNoAllocMaxCtas));
  return leave(c);
}
