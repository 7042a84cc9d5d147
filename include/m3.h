/*
 * m3.h -- C ABI of the B200 (sm_100a) per-frame autoregressive decode of
 * MiniMax Music 3's Qwen3-style 8B "Global LLM" and of its RVQ depth decoder.
 *
 * The operation and its sources (page title, section):
 *  - One frame of the Global LLM: RMSNorm, fused QKV projection, per-head
 *    q/k RMSNorm and RoPE (theta 1e6), GQA attention over the KV cache,
 *    O projection + residual, RMSNorm, SwiGLU MLP + residual, over all
 *    layers; then the final norm, the lm_head restricted to the sampleable
 *    vocabulary rows, optional classifier-free guidance over (cond, uncond)
 *    row pairs and a Gumbel-argmax draw.
 *      "MiniMax-Music3 ... DiffSynth-Studio" (Chinese article), sections
 *      "各子模型的结构要点" (Qwen3ForCausalLM, vocab 200000, hidden 4096,
 *      36 layers, 32 heads / 8 KV heads, rope_theta 1e6) and "第二阶段"
 *      (audio-code vocab mask, guided = uncond + c*(cond - uncond), depth
 *      codes drawn one codebook at a time, 25 frames/s, 9000-frame cap).
 *      "MiniMax Music 3 modular pipeline: 2.9x consumer-GPU speedup"
 *      (diffusers issue), findings 2-4: static graph inputs, lm_head sliced
 *      to the sampleable rows, Gumbel-argmax instead of softmax+multinomial,
 *      K variations decoded in lockstep as 2K rows.
 *  - Precision: bf16 activations rounded where torch rounds; fp32 norms,
 *    softmax, rope and attention sums; int8 weight-only with one fp32 scale
 *    per row (body, lm_head) or per group of 128 (depth decoder), quantised
 *    on the GPU at load.
 *      "MiniMax Music 3 on Metal" (TensorFold PR), section "Precision is
 *      the reference's".
 *  - Bucketed KV growth and an f16 KV cache option.
 *      "MiniMax Music 3, local" (portfolio page), section "Where the time went".
 *
 * Conventions common to every call:
 *  - Every call returns an m3_status; no exception crosses the ABI.  On a
 *    non-zero status m3_last_error() returns a thread-local message.
 *  - Calls are asynchronous on the context's CUDA stream (the stream given
 *    to m3_create, as a cudaStream_t cast to void*).  Device output buffers
 *    are written in stream order; the caller keeps them alive until the
 *    stream has passed them.
 *  - "dev" pointers are device memory; "host" pointers are host memory;
 *    a `mem` argument (M3_MEM_HOST / M3_MEM_DEVICE) says which for a source.
 *  - Weights and KV cache are owned by the library and freed by m3_destroy.
 *  - Raw bf16 / f16 values are passed as 16-bit patterns (uint16_t).
 */
#ifndef M3_H_
#define M3_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define M3_API __attribute__((visibility("default")))
#else
#define M3_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct m3_ctx m3_ctx;

typedef enum {
  M3_OK = 0,
  M3_EINVAL = -1,     /* bad argument (null, size, shape, alignment)      */
  M3_ENOMEM = -2,     /* device or host allocation failed                 */
  M3_ECUDA = -3,      /* a CUDA runtime call failed                       */
  M3_ESTATE = -4,     /* call out of order (no weights, no KV cache ...)  */
  M3_ECAPACITY = -5,  /* a position is outside the KV cache capacity      */
  M3_ETIMEOUT = -6,   /* a bounded device-side wait gave up               */
  M3_EDEVICE = -7,    /* a kernel recorded an error word on the device    */
  M3_EEMPTY = -8      /* m3_generate: a key drew the end token at its first
                         frame, so nothing was generated for it           */
} m3_status;

enum { M3_W_BF16 = 0, M3_W_INT8 = 1 };   /* weight storage of the body + lm_head */
enum { M3_KV_BF16 = 0, M3_KV_F16 = 1 };  /* KV cache element type               */
enum { M3_MEM_HOST = 0, M3_MEM_DEVICE = 1 };

/* Model shape.  depth_layers == 0 means no depth decoder. */
typedef struct {
  int hidden;          /* H: 4096 for the 8B                                  */
  int n_layers;        /* 36                                                  */
  int n_q_heads;       /* 32                                                  */
  int n_kv_heads;      /* 8 (GQA group n_q_heads / n_kv_heads)                */
  int head_dim;        /* 128 (64 also supported)                             */
  int ffn;             /* SwiGLU intermediate, 12288                          */
  int vocab;           /* full vocabulary, 200000 (informational)             */
  int slice_start;     /* first sampleable vocab row, e.g. 151675             */
  int slice_len;       /* number of sampleable rows, e.g. 16384               */
  double rope_theta;   /* 1e6                                                 */
  float rms_eps;       /* 1e-6                                                */
  int max_rows;        /* largest `rows` any call will use, 1..16             */
  int depth_layers;    /* 4, or 0                                             */
  int depth_hidden;    /* 1024                                                */
  int depth_heads;     /* 16 (MHA)                                            */
  int depth_head_dim;  /* 64                                                  */
  int depth_ffn;       /* 2816                                                */
  int depth_codebooks; /* 7 residual codebooks                                */
  int depth_vocab;     /* 1024 entries per residual codebook                  */
  double depth_rope_theta;
  int has_end_token;   /* 1: the end token is sampleable besides the code block */
  int end_token;       /* its vocab row, e.g. 151670 (outside the slice)        */
} m3_config;

/* One decoder layer's source tensors, bf16, row-major [out, in]. */
typedef struct {
  const void* attn_norm; /* [H]                 */
  const void* wq;        /* [Hq*d, H]           */
  const void* wk;        /* [Hkv*d, H]          */
  const void* wv;        /* [Hkv*d, H]          */
  const void* q_norm;    /* [d]                 */
  const void* k_norm;    /* [d]                 */
  const void* wo;        /* [H, Hq*d]           */
  const void* mlp_norm;  /* [H]                 */
  const void* wg;        /* [ffn, H]            */
  const void* wu;        /* [ffn, H]            */
  const void* wd;        /* [H, ffn]            */
} m3_layer_src;

/* Body weights.  layers[i] goes to layer first_layer + i, so a caller can
 * load a model layer by layer.  final_norm [H] and lm_head [slice_len, H]
 * (rows slice_start.. of the full lm_head) may be null to skip them; with
 * cfg.has_end_token, lm_end_row [H] (row end_token of the full lm_head) must
 * come with lm_head. */
typedef struct {
  int first_layer;
  int n_layers;
  const m3_layer_src* layers;
  const void* final_norm;
  const void* lm_head;
  int mem; /* M3_MEM_HOST or M3_MEM_DEVICE for every pointer here */
  const void* lm_end_row;
} m3_weight_src;

/* Depth-decoder weights, bf16 (quantised to int8, one scale per group of
 * 128, on the GPU at load).  emb[0] is [slice_len, depth_hidden] (indexed by
 * the slice-relative semantic code); emb[j], j>=1, and heads[j] are
 * [depth_vocab, depth_hidden]; proj is [depth_hidden, hidden]. */
typedef struct {
  const m3_layer_src* layers; /* depth_layers entries, MHA shapes */
  const void* proj;
  const void* const* emb;     /* depth_codebooks tables */
  const void* final_norm;     /* [depth_hidden] */
  const void* const* heads;   /* depth_codebooks heads */
  int mem;
} m3_depth_src;

/* Create a context bound to the current CUDA device and `cuda_stream`
 * (cudaStream_t, may be 0 for the legacy default stream).  Allocates only
 * the small per-frame activation buffers (sized by cfg->max_rows: the 2K
 * rows of K lockstep variations, "MiniMax Music 3 modular pipeline",
 * finding 4; the model shape of "MiniMax-Music3 ... DiffSynth-Studio",
 * "各子模型的结构要点"). */
M3_API int m3_create(const m3_config* cfg, void* cuda_stream, m3_ctx** out);

/* Copy (and, for M3_W_INT8, quantise on the GPU: one fp32 scale per row,
 * "MiniMax Music 3 on Metal", "Precision is the reference's") body weights
 * into library-owned device memory.  The first call fixes wdtype; the source
 * may be freed once the call returns (host sources are copied
 * synchronously; device sources in stream order before the call returns). */
M3_API int m3_load_weights(m3_ctx* ctx, const m3_weight_src* src, int wdtype);

/* Copy and quantise (int8, one fp32 scale per 128 inputs) the depth decoder. */
M3_API int m3_load_depth_weights(m3_ctx* ctx, const m3_depth_src* src);

/* Set up the paged KV cache ("MiniMax Music 3, local", "Where the time
 * went": the cache grows in buckets; an f16 cache option; the 9000-frame
 * cap of "MiniMax-Music3 ... DiffSynth-Studio", "推理参数详解"): `rows`
 * independent rows, each with capacity `max_positions` (<= 9000 for the
 * 8B; any value fits memory).
 * Pages of `bucket` positions (a multiple of 32; 256 recommended) are
 * allocated lazily, one bucket for all rows and layers at a time, as frames
 * reach them -- the cache grows without copying.  kvdtype M3_KV_BF16 or
 * M3_KV_F16.  Replaces any previous cache. */
M3_API int m3_kv_alloc(m3_ctx* ctx, int rows, int max_positions, int kvdtype, int bucket);

/* Fill positions [0, n_positions) of `row` (prefill).  k, v: bf16
 * [n_layers, n_positions, Hkv, d]; stored converted to the cache type
 * (f16 by round-to-nearest-even).  Values are taken as already rotated. */
M3_API int m3_kv_set(m3_ctx* ctx, int row, int n_positions, const void* k, const void* v, int mem);

/* Read positions [0, n_positions) of `row` back in the m3_kv_set layout, as
 * raw cache-type bits (bf16 or f16).  Synchronises the stream. */
M3_API int m3_kv_get(m3_ctx* ctx, int row, int n_positions, void* k_host, void* v_host);

/* Prompt prefill of one cache row (the prompt embedder's tokens, DiffSynth-
 * Studio article "第一阶段", ahead of the autoregressive frames): token t of
 * x (dev bf16 [n_tokens, H]) runs through every layer at position start + t,
 * attending to positions 0..start + t of the row (causal), and its K/V land
 * in the row's cache -- the same result as decoding the tokens one by one.
 * With bf16 weights the tokens go in chunks of 2048 (environment
 * M3_PREFILL_CHUNK, 16..4096), each chunk one pass of the layers whose
 * projections are tcgen05 GEMMs over the chunk's tokens, both operands
 * brought in by TMA tensor maps: the weights from a row-major bf16 copy of
 * every layer's projections (about 0.39 GB per 8B layer, 14 GB for 36),
 * made on the device at the first prefill and again for a layer that
 * m3_load_weights has replaced since.  With int8 weights (or
 * M3_PREFILL_TC=0) the tokens go in chunks of up to max_rows as the batch
 * rows of the decode projections; M3_PREFILL_TC=1 takes a GEMM over the
 * tiled int8 weights (chunks of 256) instead.
 *  h_last (dev bf16 [H], nullable): the final-normed hidden state of the last
 *    token.
 * start + n_tokens must be <= max_positions (M3_ECAPACITY).  May allocate KV
 * buckets and, at the first GEMM prefill, the weight copies and chunk-sized
 * activation buffers (M3_ENOMEM when they do not fit); synchronises the
 * stream once. */
M3_API int m3_prefill(m3_ctx* ctx, int row, int start, int n_tokens, const void* x, void* h_last);

/* The end token.  With cfg.has_end_token the draw of m3_decode_frame chooses
 * among slice_len + 1 candidates: the code block and, as slice-relative code
 * slice_len, the end token (noise index end_token); the vocabulary mask of
 * "第二阶段" in the DiffSynth-Studio article, which leaves the audio codes and
 * the end token sampleable.  Ties between the end token and a code go to the
 * code.  Logit buffers are then slice_len + 1 wide. */

/* Top-k filter of the frame draw (the AR sampler's "CFG 1.5, top-k 50,
 * multinomial", DiffSynth-Studio article, "第二阶段"): m3_decode_frame keeps
 * the top_k largest guided logits per key -- ties at the k-th value going to
 * the lower index -- and draws among them by Gumbel-argmax.  0 (the default)
 * or top_k >= slice_len keeps every logit.  Applies to the calls that follow;
 * the depth decoder and m3_sample_noalloc always keep every logit; the
 * generation loop (m3_generate) keeps the setting.
 * Returns M3_EINVAL for top_k < 0. */
M3_API int m3_set_top_k(m3_ctx* ctx, int top_k);

/* Decode one frame for rows 0..rows-1 (rows <= cache rows and <= max_rows):
 * the per-frame step of "MiniMax-Music3 ... DiffSynth-Studio", "第二阶段"
 * (the Global LLM's forward, the guided draw over the audio-code rows), with
 * the static graph inputs, sliced lm_head and Gumbel-argmax draw of
 * "MiniMax Music 3 modular pipeline", findings 2-3.
 *  positions (HOST, [rows]): the position each row writes this frame; the
 *    row attends to positions 0..positions[r] inclusive.  Every position must
 *    be < max_positions or the call returns M3_ECAPACITY before any launch.
 *  x_in (dev bf16 [rows, H]): the frame's input embedding per row; copied
 *    into a library-owned graph-input buffer before the launch.
 *  cfg_scale > 0: rows are (cond, uncond) pairs (rows must be even); the
 *    guided logits uncond + cfg_scale*(cond - uncond) are drawn once per pair
 *    with noise row key = pair index, and both rows receive the code.
 *    cfg_scale == 0: each row draws from its own logits, row key = row.
 *  temperature > 0: z_i = g_i / temperature + Gumbel(seed, frame, key, slice_start + i).
 *  codes (dev int32 [rows]): slice-relative code (0..slice_len-1; slice_len
 *    is the end token when the config has one).
 *  h_out (dev bf16 [rows, H], nullable): final-normed hidden state.
 *  logits (dev fp32 [rows, slice_len (+1 with the end token)], nullable):
 *    raw per-row logits.
 * The whole frame runs as one CUDA graph per (rows, KV bucket count),
 * captured on first use.  May allocate a new KV bucket (synchronising). */
M3_API int m3_decode_frame(m3_ctx* ctx, int rows, const int32_t* positions, uint64_t seed,
                    uint64_t frame, const void* x_in, float cfg_scale, float temperature,
                    int32_t* codes, void* h_out, float* logits);

/* The 7 residual codes of one frame from the depth decoder.
 *  h_frame (dev bf16 [rows, H]): the frame's final-normed hidden state
 *    (m3_decode_frame's h_out), projected to depth_hidden at position 0;
 *  code0 (dev int32 [rows]): the frame's semantic code (slice-relative),
 *    embedded with emb[0] at position 1 (the end token's code, slice_len,
 *    gives a zero vector there);
 *  position j (1..7) yields codebook j's logits from heads[j-1], drawn with
 *    noise index (j << 32) | i, and E_j[code_j] is the input of position j+1;
 *  forced (dev int32 [rows, codebooks], nullable): teacher forcing -- feed
 *    these codes forward instead of the drawn ones;
 *  codes (dev int32 [rows, codebooks]); logits (dev fp32
 *    [rows, codebooks, depth_vocab], nullable).
 * cfg_scale / temperature as in m3_decode_frame. */
M3_API int m3_depth_decode(m3_ctx* ctx, int rows, const void* h_frame, const int32_t* code0,
                    uint64_t seed, uint64_t frame, float cfg_scale, float temperature,
                    const int32_t* forced, int32_t* codes, float* logits);

/* Tables of the generation loop's feedback embedding (the DiffSynth-Studio
 * article's embed_audio_frame, "第二阶段"), copied into library memory:
 *  tok_emb [slice_len, H] bf16: embed_tokens rows slice_start.. (the code
 *    block's token embeddings);
 *  audio_emb: depth_codebooks tables [depth_vocab, H] bf16, the residual
 *    codebooks' audio embeddings; null when the config has no depth decoder.
 * Returns M3_EINVAL for a null table the config needs. */
M3_API int m3_load_feedback(m3_ctx* ctx, const void* tok_emb, const void* const* audio_emb,
                            int mem);

/* The autoregressive generation loop on the GPU: frame f = 0, 1, ... runs
 * every row at position positions[r] + f with noise frame frame0 + f, as
 * m3_decode_frame; with the depth decoder loaded, m3_depth_decode follows on
 * the frame's hidden state and code.  The next frame's input is, per row,
 *   x = bf16((tok_emb[c0] + audio_emb[0][c1] + ... + audio_emb[NC-1][cNC]) * (1 + NC)^-0.5)
 * (fp32 sum in that order; NC = depth_codebooks, or 0 without the depth
 * decoder: x = tok_emb[c0]; the article's 8^-0.5 for its 8 codebooks).
 * A key (a CFG pair, or a row without CFG) stops at the first frame whose
 * code is the end token (slice_len; needs cfg.has_end_token); its count is
 * the frames before that one.  Positions, the noise frame, the step and the
 * counts advance on the GPU; the host reads the loop state every 16 frames
 * and stops once every key has stopped, or after max_frames.  Rows of a
 * stopped key keep being computed, on a zero input.
 *  positions (HOST, [rows]): each row's first position; positions[r] +
 *    max_frames must be <= max_positions, else M3_ECAPACITY before any launch.
 *  x_in (dev bf16 [rows, H]): the first frame's input.
 *  cfg_scale, temperature: as in m3_decode_frame; the top-k setting applies.
 *  codes (dev int32 [max_frames, rows, 1 + NC]): per frame and row the semantic
 *    code and the residual codes while the row's key runs; on its end frame
 *    the semantic code is slice_len and the residual entries -1; -1 after.
 *  h_hist (dev bf16 [max_frames, rows, H], nullable): each frame's
 *    final-normed hidden state while the row's key runs; zeros after.
 *  n_frames (HOST int32 [keys]): frames generated per key.
 * Synchronises the stream (every 16 frames and at the end).  Returns
 * M3_EEMPTY, with every output written, when some key drew the end token at
 * its first frame; a device-side error as m3_sync_status reports it. */
M3_API int m3_generate(m3_ctx* ctx, int rows, const int32_t* positions, uint64_t seed,
                       uint64_t frame0, const void* x_in, float cfg_scale, float temperature,
                       int max_frames, int32_t* codes, void* h_hist, int32_t* n_frames);

/* Frame feedback by table lookup: x_out[r] = table[offset + codes[r]].
 * table (dev bf16 [n, H]), codes (dev int32 [rows]), x_out (dev bf16 [rows, H]). */
M3_API int m3_embed(m3_ctx* ctx, int rows, const int32_t* codes, const void* table, int offset,
             void* x_out);

/* Stateless int8 weight-only quantiser on the GPU.  w (dev bf16 [rows, cols]);
 * group = cols (one scale per row) or 128 (cols % group == 0);
 * s = absmax/127 in fp32, q = clamp(rint(w/s), -127, 127), s == 0 -> q = 0.
 * q (dev int8 [rows, cols]); scales (dev fp32 [rows, cols/group]). */
M3_API int m3_quantize_int8(const void* w, int64_t rows, int64_t cols, int64_t group, int8_t* q,
                     float* scales, void* cuda_stream);

/* Export a loaded, possibly quantised weight in its source layout, to host
 * memory (synchronises).  which: 0 wq 1 wk 2 wv 3 wo 4 wg 5 wu 6 wd 7 lm_head,
 * 8 + same for the depth decoder's layers, 16 depth proj, 17 + j depth head j.
 * For int8, q_host gets int8 [rows, cols] and s_host fp32 scales; for bf16
 * q_host gets the bf16 bits and s_host is ignored. */
M3_API int m3_export_weight(m3_ctx* ctx, int which, int layer, void* q_host, float* s_host);

/* Kernels one m3_decode_frame of `rows` rows launches, for launch
 * accounting: the parameter block, the RoPE table, QKV, attention, O,
 * gate/up and down per layer (the int8 group-128 projections in launches of
 * 4 rows) and the sampler.  A negative m3_status on bad arguments or before
 * the weights are loaded. */
M3_API int m3_frame_kernels(const m3_ctx* ctx, int rows);

/* Kernels one m3_depth_decode of `rows` rows launches, for launch
 * accounting: 1 where the decoder runs as one persistent kernel (its shape
 * and shared memory allow), else its separate launches.  A negative
 * m3_status on bad arguments or before the depth weights are loaded. */
M3_API int m3_depth_kernels(const m3_ctx* ctx, int rows);

/* Algorithmic HBM bytes of one frame: weights read once per frame plus the
 * KV cache read for `rows` rows at context length ctx (positions 0..ctx). */
M3_API double m3_frame_bytes(const m3_ctx* ctx, int rows, int ctx_len);

/* Time one kind of the frame's GEMVs in isolation, for roofline accounting:
 * which = 0 fused QKV, 1 O projection, 2 gate/up + SwiGLU, 3 down, 4 lm_head
 * + sampler.  Launch i (i < iters) uses layer i % n_layers, so consecutive
 * launches stream different weights (layers beyond L2); launches follow each
 * other with programmatic dependent launch as inside a frame.  The region is
 * bracketed by CUDA events on the context's stream (synchronises).  Writes
 * the mean milliseconds per launch and the algorithmic bytes per launch
 * (weights, scales and activations read plus outputs written). */
M3_API int m3_time_gemv(m3_ctx* ctx, int which, int rows, int iters, float* avg_ms,
                        double* bytes_per_launch);

/* The lm_head + CFG + Gumbel-argmax draw of m3_decode_frame on a given
 * final-normed hidden state, for callers that must not allocate GPU memory
 * on the decode thread (a real-time audio callback, a host thread that runs
 * while a CUDA graph is being captured elsewhere, an embedder whose memory
 * is budgeted up front): it calls no cudaMalloc / cudaFree and no
 * allocating library routine.  The pages have no counterpart of this call.
 *  h (dev bf16 [rows, H]): final-normed hidden state (m3_decode_frame's h_out);
 *  rows <= 16 and <= max_rows, else M3_EINVAL; seed, frame, cfg_scale,
 *  temperature, codes, logits as in m3_decode_frame (logits nullable).
 * Its scratch (parameter block, argmax partials, ticket; about 129 KB) is a
 * file-scope __device__ array that every GPU loading the library holds
 * until exit.  m3_create looks up that array's device address on the
 * context's device (so this call does no lookup and takes no lock); a
 * cudaDeviceReset invalidates it together with the context.  All calls
 * share the array and keep the last call's contents (the ticket is cleared
 * by each call): calls that overlap on the GPU -- on different streams or
 * contexts of one device -- race and must be ordered by the caller.  A
 * launch plan needing more than 1024 CTAs is rejected with M3_EINVAL. */
M3_API int m3_sample_noalloc(m3_ctx* ctx, int rows, const void* h, uint64_t seed, uint64_t frame,
                             float cfg_scale, float temperature, int32_t* codes, float* logits);

/* The Gumbel noise of the draws, written out: out[i] (dev fp32 [n]) =
 * G(seed, frame, row, index0 + i), computed by the same device function the
 * samplers use, so that the noise can be compared bit for bit with another
 * implementation of its definition (the diffusers issue "MiniMax Music 3
 * modular pipeline", finding 3: Gumbel-argmax in place of softmax +
 * multinomial; definition: SplitMix64 counters, u = ((b >> 40) + 0.5) 2^-24,
 * G = -ln(-ln u) in fp64 with a series ln, rounded to fp32).  Stateless;
 * asynchronous on cuda_stream.  M3_EINVAL for n < 0 or a null output. */
M3_API int m3_gumbel_fill(uint64_t seed, uint64_t frame, uint64_t row, uint64_t index0,
                          int64_t n, float* out, void* cuda_stream);

/* Host-side fault injection, for testing the error paths: the nth (>= 1) next
 * device allocation (M3_FAULT_ALLOC, the call then returns M3_ENOMEM), host-
 * to-device copy of a host source (M3_FAULT_H2D, M3_ECUDA) or CUDA-graph
 * capture (M3_FAULT_GRAPH, M3_ECUDA) made by this context fails as if the
 * CUDA call had; the context stays usable, and the same call made again
 * succeeds.  One failure per injection; M3_FAULT_NONE cancels.  The
 * environment variable M3_FAULT = alloc:N | h2d:N | graph:N, read by
 * m3_create, schedules the same from the context's creation on.  No GPU
 * fault is involved: the CUDA call is simply not made. */
enum { M3_FAULT_NONE = 0, M3_FAULT_ALLOC = 1, M3_FAULT_H2D = 2, M3_FAULT_GRAPH = 3 };
M3_API int m3_inject_fault(m3_ctx* ctx, int kind, int64_t nth);

/* Launch, on the context's stream, one kernel that waits on an mbarrier no
 * thread ever arrives on, with at most `polls` (1..2^22) polls: the bounded
 * wait gives up and records the timeout error word, which the next
 * m3_sync_status returns as M3_ETIMEOUT (and clears).  This is the path every
 * device-side wait of the library takes when the copy or the CTA it waits
 * for never comes; the kernel returns normally and the context stays usable. */
M3_API int m3_stalled_wait(m3_ctx* ctx, int64_t polls);

/* Synchronise the stream and return the first error a kernel recorded on
 * the device (M3_ETIMEOUT / M3_EDEVICE), clearing it, or M3_OK. */
M3_API int m3_sync_status(m3_ctx* ctx);

/* Thread-local message for the last failing call on this thread. */
M3_API const char* m3_last_error(void);

M3_API void m3_destroy(m3_ctx* ctx);

#ifdef __cplusplus
}
#endif

#endif /* M3_H_ */
