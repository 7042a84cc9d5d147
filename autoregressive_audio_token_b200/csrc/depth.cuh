// depth.cuh -- the RVQ depth decoder of one frame as ONE persistent,
// cooperative kernel.
//
// The depth decoder ("第二阶段" of the DiffSynth-Studio article on
// MiniMax-Music3: after each semantic code a 4-layer, 16-head decoder draws
// the 7 residual codes one codebook at a time) runs 8 frame-local positions
// x 4 layers of small GEMVs (hidden 1024, int8 weights with one scale per
// group of 128) whose ~60 MB of weights stay in L2.  As separate kernels its
// ~175 launches cost far more than their bytes; here every CTA of the grid
// walks the same sequence of phases, separated by grid-wide barriers:
//   proj            x = bf16(W_p h)                                 (once)
//   per position j = 0..7 (x = E_{j-1}[c_{j-1}] for j >= 1) and layer l:
//     A  n1 = norm(x) (each CTA, into shared memory); qkv = bf16(W_qkv n1)
//     B  per (row, head): q/k norm + RoPE at position j, K/V of position j
//        stored, attention over positions 0..j -> att
//     C  x = bf16(x + bf16(W_o att))
//     D  n2 = norm(x); act = bf16(bf16(silu(bf16(W_g n2))) * bf16(W_u n2))
//     E  x = bf16(x + bf16(W_d act))
//   per position j >= 1: logits = W_head_j norm_f(x) (fp32), guided over CFG
//     pairs, z = g / T + Gumbel(seed, frame, key, (j << 32) | i), the code
//     of the largest z (lowest index on ties) -- per-CTA winners, a barrier,
//     then every CTA reduces them in the same order.
// The grid barrier is a counter + generation in global memory, spun on with
// a bound: a CTA that gives up records kErrTimeout and raises an abort word
// after which no CTA waits again, so a failure ends the kernel instead of
// hanging it.  The launch is cooperative (all CTAs resident).
// Measured on B200 this form is slower than the separate launches (about
// 9 us per phase and 2 us per barrier over 168 barriers), so it is opt-in:
// the context uses it when M3_DEPTH_FUSED=1.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "gemv.cuh"

namespace m3 {

constexpr int kDepthThreads = 256;
constexpr int kDepthWarps = kDepthThreads / 32;
constexpr int kDepthMaxLayers = 8;
constexpr int kDepthMaxCB = 32;
constexpr long long kDepthSpinLimit = 1ll << 22;

struct DepthMat {
  const int8_t* q;  // [N][K] row-major
  const float* s;   // [N][K / 128]
};

struct DepthLayerW {
  DepthMat qkv, o, gu, d;  // gu: gate row 2i, up row 2i + 1
  const __nv_bfloat16 *attn_norm, *mlp_norm, *q_norm, *k_norm;
};

struct DepthArgs {
  DepthLayerW L[kDepthMaxLayers];
  DepthMat proj;                                 // [Dh][Hin]
  DepthMat heads[kDepthMaxCB];                   // [V][Dh]
  const __nv_bfloat16* emb[kDepthMaxCB];         // emb[0] [S][Dh], emb[j] [V][Dh]
  int emb_rows[kDepthMaxCB];
  const __nv_bfloat16* final_norm;               // [Dh]
  const double* inv_freq;                        // [hd / 2]
  int n_layers, Dh, nh, hd, F, NC, V, Hin, rows;
  int zero_code;                                 // code0 with a zero embedding (end token)
  float eps;
  const FrameParams* fp;                         // cfg, scale, temperature, seed, frame
  const __nv_bfloat16* h_in;                     // [rows][Hin]
  const int* code0;                              // [rows]
  const int* forced;                             // nullable [rows][NC]
  int* codes;                                    // [rows][NC]
  float* logits;                                 // nullable [rows][NC][V]
  // global scratch
  __nv_bfloat16* x;                              // [rows][Dh] residual stream
  __nv_bfloat16* qkv;                            // [rows][3 nh hd]
  __nv_bfloat16* att;                            // [rows][nh hd]
  __nv_bfloat16* act;                            // [rows][F]
  __nv_bfloat16* kv;                             // [rows][layers][NC + 1][2][nh][hd]
  unsigned long long* part;                      // [grid][kMaxRows] argmax winners
  unsigned* bar;                                 // [3] count, generation, abort
  int* err;
};

}  // namespace m3
