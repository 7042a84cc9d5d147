// dit_gemm.cuh -- the DiT's projections as persistent GEMMs on the
// 5th-generation tensor cores, operands brought in by TMA tensor maps.
//
// Y[t][o] = sum_k X[t][k] W[o][k] with X the tokens (fp16, [M][K] row-major)
// and W an nn.Linear weight (fp16, [N][K] row-major): both operands are
// K-major, which is what tcgen05.mma reads directly.
//   * tile = 128 tokens (MMA M, the accumulator's TMEM lanes) x 256 outputs
//     (MMA N, 256 fp32 TMEM columns); K in stages of 64 = one 128-byte row of
//     the 128-byte swizzle, so one 2-D tensor-map copy per operand and stage
//     lands in the canonical K-major SWIZZLE_128B layout (8-row atoms of
//     1024 bytes); the four K = 16 MMAs of a stage advance the descriptor's
//     start address by 32 bytes;
//   * persistent CTAs (one per SM) walk the tiles output-block-major, so the
//     CTAs that run at the same time share a weight block through L2;
//   * warp-specialised: warp 0 issues the TMA copies of a 4-stage ring,
//     warp 1 issues the MMAs (one thread) and owns the tensor memory, warps
//     2-5 drain the accumulator -- double-buffered in TMEM (2 x 256 columns),
//     so the epilogue of one tile overlaps the MMAs of the next;
//   * fused epilogues with the fp16 roundings of the reference: store
//     f16(y); add a per-output vector (the timestep embedding) after
//     rounding; partial RoPE of the q / k heads; residual x = f16(x + f16(y));
//     GLU over interleaved (gate, up) output pairs.
// Every mbarrier wait is bounded; a timeout records kErrTimeout, the MMA
// thread waits (bounded) for its own MMAs, and tensor memory is freed.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace m3 {

enum : int {
  DIT_EPI_STORE = 0,  // y16 = f16(acc)
  DIT_EPI_TEMB = 1,   // y16 = f16(f16(acc) + vec[o])
  DIT_EPI_ROPE = 2,   // y16 = f16(acc), then partial RoPE on the q / k heads
  DIT_EPI_RESID = 3,  // out = f16(out + f16(acc))
  DIT_EPI_GLU = 4     // out[o/2] = f16(f16(silu(f16(acc_gate))) * f16(acc_up))
};

struct DitGemmArgs {
  int M, N, K;           // tokens, outputs, inputs
  void* out;             // [M][ldo] of the operand type; for the GLU [M][N/2]
  int ldo;
  const __half* vec;     // DIT_EPI_TEMB: [N]
  const float2* rope;    // DIT_EPI_ROPE: (cos, sin) [rope_T][rope_half]
  int rope_T;            // tokens per batch element: row t sits at position t % rope_T
  int rope_cols;         // output columns < rope_cols are q / k heads
  int head_dim;          // 64
  int rope_half;         // rotated pairs per head (rope_dims / 2 = 16)
  int* err;
};

// Once per device before the first launch (and before any stream capture):
// the kernels' shared-memory limit and the tensor-map encoder.
cudaError_t prepare_dit_gemm();

// One GEMM on the stream: X [M][ldx] and W [N][K], both fp16 or (bf16 =
// true, the prompt prefill of the decode body: store, residual and GLU
// epilogues with bf16 roundings) both bf16 (ldx >= K, both 16-byte aligned,
// K a multiple of 64, ldx a multiple of 8).
cudaError_t launch_dit_gemm(const void* X, int ldx, const void* W, const DitGemmArgs& a,
                            int epi, int nsm, cudaStream_t st, bool bf16 = false);

}  // namespace m3
