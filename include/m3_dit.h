/*
 * m3_dit.h -- C ABI of the B200 (sm_100a) chunk-denoise step of MiniMax
 * Music 3's flow-matching DiT, the acoustic stage that follows the
 * autoregressive decode of m3.h (same library, libm3.so).
 *
 * The operation and its sources (page title, section):
 *  - "MiniMax-Music3 ... DiffSynth-Studio" (Chinese article):
 *      "各子模型的结构要点": a 36-layer Transformer, 32 heads of 64, FFN 8192;
 *      input = noisy latent and condition concatenated, 2*128 + 2048 = 2304
 *      channels; partial rotary position embedding; Fourier time embedding.
 *      "第三阶段": chunks of 200 frames (hop 100, overlap 172 latent frames),
 *      latents of 128 channels over the condition's length, flow matching
 *      with 1000 training timesteps; every step predicts with the condition
 *      and with an all-zero condition and guides
 *      velocity = uncond + cfg_scale * (cond - uncond), then steps the
 *      scheduler.  "推理参数详解": cfg_scale 1.7, 30 steps per chunk.
 *  - "MiniMax Music 3 modular pipeline" (diffusers issue), finding 3: the
 *    cond / uncond pair as ONE batch-2 forward.
 *  - "MiniMax Music 3 on Metal", "Precision is the reference's": fp16 in
 *    the DiT with fp16 roundings and fp32 sums; "Next steps": the DiT's
 *    GEMMs are its long pole.
 *
 * Readings where the pages are silent (the library follows them exactly):
 *  - input row = [x_t (latent) | context latent (latent) | condition (cond)];
 *    the unconditional branch zeroes the condition channels only;
 *  - no linear biases; LayerNorm (gain, bias, eps) with one fp16 rounding;
 *  - t = 1000 * sigma; features [cos(t f_k), sin(t f_k)], f_k = 10000^(-k/half);
 *    temb = W_t2 silu(W_t1 features), added to every token after W_in;
 *  - pre-norm blocks h += W_o attn(LN1 h), h += W_d (silu(W_g n) * W_u n),
 *    n = LN2 h; v = W_out LN_f h;
 *  - partial RoPE on the first rope_dims of each q / k head, half-rotation
 *    pairs, angle pos * theta^(-2i/rope_dims), pos = the token's index in
 *    its chunk; attention bidirectional per batch element;
 *  - Euler step x += (sigma_next - sigma) * v_guided in fp32.
 *
 * Conventions as in m3.h: every call returns an m3_status (m3.h); calls are
 * asynchronous on the context's stream; "dev" pointers are device memory;
 * fp16 values are raw 16-bit patterns; weights are library-owned.
 */
#ifndef M3_DIT_H_
#define M3_DIT_H_

#include <stdint.h>

#include "m3.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct m3_dit m3_dit;

typedef struct {
  int width;        /* W = n_heads * head_dim: 2048                           */
  int n_layers;     /* 36                                                     */
  int n_heads;      /* 32                                                     */
  int head_dim;     /* 64 (the only supported value)                          */
  int ffn;          /* 8192                                                   */
  int latent;       /* 128 latent channels                                    */
  int cond;         /* 2048 condition channels                                */
  int temb;         /* 256 Fourier features                                   */
  int rope_dims;    /* 32 rotated dims per head (the only supported value)    */
  double rope_theta;/* 1e4                                                    */
  float ln_eps;     /* 1e-5                                                   */
  int max_tokens;   /* largest T (latent frames per chunk) any call uses: 689 */
} m3_dit_config;

/* One block's fp16 source tensors, row-major [out, in]. */
typedef struct {
  const void *ln1_g, *ln1_b; /* [W]          */
  const void* wqkv;          /* [3W, W]: q rows, k rows, v rows (head-major) */
  const void* wo;            /* [W, W]       */
  const void *ln2_g, *ln2_b; /* [W]          */
  const void *wg, *wu;       /* [ffn, W]     */
  const void* wd;            /* [W, ffn]     */
} m3_dit_layer_src;

/* Weights.  layers[i] goes to block first_layer + i; the outer tensors may
 * be null to skip them.  mem: M3_MEM_HOST or M3_MEM_DEVICE for every pointer. */
typedef struct {
  int first_layer, n_layers;
  const m3_dit_layer_src* layers;
  const void* w_in;          /* [W, 2*latent + cond] */
  const void* w_t1;          /* [W, temb]            */
  const void* w_t2;          /* [W, W]               */
  const void *lnf_g, *lnf_b; /* [W]                  */
  const void* w_out;         /* [latent, W]          */
  int mem;
} m3_dit_src;

/* A context on the current device and `cuda_stream`; allocates the
 * activation buffers for 2 * max_tokens rows.  M3_EINVAL for shapes the
 * kernels do not support: head_dim != 64, rope_dims != 32, width not in
 * {256, 512, 1024, 2048}, width / ffn / 2*latent + cond not multiples of 64,
 * latent not a multiple of 32, temb not a multiple of 8. */
M3_API int m3_dit_create(const m3_dit_config* cfg, void* cuda_stream, m3_dit** out);

/* Copy weights into library memory (gate and up rows interleaved there, so
 * the GLU pairs sit side by side in one GEMM).  Synchronises for host sources. */
M3_API int m3_dit_load(m3_dit* dit, const m3_dit_src* src);

/* One denoising step of one chunk of T latent frames (T <= max_tokens):
 *  x (dev fp32 [T, latent]): the noisy latent x_t, replaced by
 *    x_t + (sigma_next - sigma) * v_guided;
 *  ctx (dev fp16 [T, latent]): the context latent; cond (dev fp16 [T, cond]);
 *  v_guided (dev fp32 [T, latent], nullable); v_pair (dev fp16
 *    [2, T, latent], nullable): the cond and uncond predictions.
 * The step runs as one CUDA graph per T (captured on first use); inputs are
 * copied into library buffers first. */
M3_API int m3_dit_step(m3_dit* dit, int T, float* x, const void* ctx, const void* cond,
                       float sigma, float sigma_next, float cfg_scale, float* v_guided,
                       void* v_pair);

/* `steps` denoising steps with sigmas[i] -> sigmas[i + 1] (HOST fp32
 * [steps + 1]); x as in m3_dit_step, written once at the end. */
M3_API int m3_dit_denoise(m3_dit* dit, int T, float* x, const void* ctx, const void* cond,
                          const float* sigmas, int steps, float cfg_scale);

/* The forward alone on B (1 or 2) batch elements of T tokens each, for
 * parity checks: h_in (dev fp16 [B*T, 2*latent + cond]); t = 1000 * sigma;
 * v (dev fp16 [B*T, latent]). */
M3_API int m3_dit_forward(m3_dit* dit, int B, int T, const void* h_in, float t, void* v);

/* Blocks first .. first + n - 1 on h (dev fp16 [B*T, W], in place). */
M3_API int m3_dit_blocks(m3_dit* dit, int B, int T, void* h, int first, int n);

/* Time one kind of the block GEMMs at T tokens per batch element (B = 2):
 * which = 0 QKV (+ RoPE), 1 O (+ residual), 2 gate/up (+ GLU), 3 down
 * (+ residual); launch i uses block i % n_layers.  Writes the mean
 * milliseconds per launch and the FLOPs of one launch (2 M N K). */
M3_API int m3_dit_time_gemm(m3_dit* dit, int which, int T, int iters, float* avg_ms,
                            double* flops);

/* Synchronise and return the device error word as a status (as m3_sync_status). */
M3_API int m3_dit_sync_status(m3_dit* dit);

M3_API void m3_dit_destroy(m3_dit* dit);

#ifdef __cplusplus
}
#endif

#endif /* M3_DIT_H_ */
