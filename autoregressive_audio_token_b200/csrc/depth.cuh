// depth.cuh -- arguments of the persistent depth-decoder kernel (depth.cu).
//
// The RVQ depth decoder that follows each semantic code (DiffSynth-Studio
// article "MiniMax-Music3 ... DiffSynth-Studio", "第二阶段": 7 residual codes
// per frame, drawn one after another by a 4-layer block of 16 heads over 8
// frame-local positions) is a chain of about 170 small dependent steps whose
// weights (53 MB of int8 with group-128 scales, "MiniMax Music 3 on Metal",
// "Precision is the reference's") stay in L2 across the positions. As
// separate launches it is bound by launch latency; this kernel runs the whole
// chain with one CTA per SM, each step waiting only for the tagged words of
// its own inputs.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "gemv.cuh"

namespace m3 {

constexpr int kDepthThreads = 512;
constexpr int kDepthWarps = kDepthThreads / 32;
constexpr int kDepthMaxLayers = 8;
constexpr int kDepthMaxCodebooks = 31;
constexpr int kDepthMaxTiles = kDepthWarps;  // 16-row weight tiles of one CTA per projection

struct DepthMat {
  const int8_t* q;  // [N][K] row-major int8
  const float* s;   // [N][K / 128] group scales
};

struct DepthLayerW {
  DepthMat qkv, o, gu, d;  // qkv rows [q | k | v]; gu rows interleaved (gate 2i, up 2i + 1)
  const __nv_bfloat16 *attn_norm, *mlp_norm, *q_norm, *k_norm;
};

struct DepthArgs {
  int rows, Dh, nh, hd, F, NC, V, Hin, n_layers;
  float eps;
  int merge_attn;  // 1: every CTA of the O projection computes the attention itself
  int wb_bytes;    // shared memory of the weight slices (two consecutive projections)
  int xs_bytes;    // shared memory of the staged activations
  int max_tiles;   // most 16-row tiles any CTA holds in one projection
  int side_bytes;  // static vectors copied with a slice (norm gains, q/k gains + a RoPE row)
  int own_tiles;   // most tiles of the residual stream one CTA owns
  DepthLayerW L[kDepthMaxLayers];
  DepthMat proj;                              // [Dh][Hin]
  DepthMat heads[kDepthMaxCodebooks];         // [V][Dh]
  const __nv_bfloat16* emb[kDepthMaxCodebooks];  // emb[j]: [emb_rows[j]][Dh]
  int emb_rows[kDepthMaxCodebooks];
  const __nv_bfloat16* final_norm;
  const float2* rope;          // [NC + 1][hd / 2] (cos, sin) of positions 0..NC
  const __nv_bfloat16* h_in;   // [rows][Hin] the frame's final-normed hidden state
  const int* code0;            // [rows] semantic codes
  const int* forced;           // nullable [rows][NC]: codes fed forward instead of the drawn
  int zero_code;               // a code0 equal to it feeds a zero vector (INT_MIN: none)
  int* codes;                  // [rows][NC]
  int* prev;                   // [rows] the last code fed forward
  float* logits;               // [rows][NC][V] raw per-row logits
  const FrameParams* fp;
  // Step outputs that other CTAs read, as tagged 32-bit words: the bf16
  // value in the low half, the tag of the step that wrote it in the high
  // half; a reader polls each word until it carries the tag it expects, so
  // no grid-wide barrier is needed (every reader of a buffer is upstream of
  // the buffer's next writer). All of them lie in [words, words +
  // words_bytes), cleared before each launch.
  uint32_t* words;
  size_t words_bytes;
  uint32_t* xw;    // [rows][Dh] residual stream
  uint32_t* qkvw;  // [rows][3 nh hd]
  uint32_t* attw;  // [rows][nh hd]
  uint32_t* actw;  // [rows][F]
  uint32_t* kvw;   // [rows][n_layers][NC + 1][2][nh hd] normed/rotated keys, values
  unsigned long long* part;  // [grid][kMaxRows] per-CTA argmax keys, tag in the low 16 bits
  int* err;
};

// Bytes of one CTA's slice of a projection: nt tiles of 16 rows of K int8
// (rows padded by 64 bytes against bank conflicts), their group scales, then
// `side` bytes of the step's static vectors.
__host__ __device__ __forceinline__ int depth_slice_bytes(int nt, int K, int side) {
  const int b = 16 * nt * (K + 64) + 16 * nt * (K / 128) * 4 + side;
  return (b + 127) & ~127;
}

// Shape checks and the shared-memory carve for `grid` CTAs; fills
// a->wb_bytes, xs_bytes, max_tiles, side_bytes, own_tiles, merge_attn.
// cudaErrorInvalidConfiguration when the shape does not suit the kernel (the
// caller then takes the per-launch path).
cudaError_t depth_plan(DepthArgs* a, int grid, size_t* smem);
cudaError_t launch_depth(const DepthArgs& a, int grid, size_t smem, cudaStream_t st);

}  // namespace m3
