// launch.cuh -- host-side launchers of the decode kernels (one definition per
// weight format lives in gemv_<format>.cu so they compile in parallel).
#pragma once

#include <cuda_runtime.h>

#include "attention.cuh"
#include "gemv.cuh"

namespace m3 {

// Launch `kernel` with cudaLaunchKernelEx; with pdl the launch may begin
// while the previous kernel in the stream is still running
// (programmatic stream serialization); the kernel orders itself with
// griddepcontrol.wait before touching that kernel's outputs.
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                      cudaStream_t st, bool pdl, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = pdl ? attr : nullptr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Threads per output row for a GEMV over K inputs: one 16-byte chunk each
// (8 bf16 or 16 int8 inputs), the fewest threads covering min(K, 4096);
// K > 4096 streams in segments of 4096.
inline int gemv_tpr(int K, int esz) {
  const int ept = 16 / esz;
  const int target = K < 4096 ? K : 4096;
  int tpr = 32;
  while (tpr * ept < target && tpr < 512) tpr *= 2;
  return tpr;
}

cudaError_t launch_gemv_bf16(const GemvArgs& a, int epi, cudaStream_t st, bool pdl, int nsm);
cudaError_t launch_gemv_i8row(const GemvArgs& a, int epi, cudaStream_t st, bool pdl, int nsm);
cudaError_t launch_gemv_i8g128(const GemvArgs& a, int epi, cudaStream_t st, bool pdl, int nsm);

inline cudaError_t launch_gemv(const GemvArgs& a, int wf, int epi, cudaStream_t st, bool pdl,
                               int nsm) {
  if (wf == WF_BF16) return launch_gemv_bf16(a, epi, st, pdl, nsm);
  if (wf == WF_I8ROW) return launch_gemv_i8row(a, epi, st, pdl, nsm);
  return launch_gemv_i8g128(a, epi, st, pdl, nsm);
}

// The tiled tensor-core GEMV (gemv_tile.cuh): its launch plan and launcher.
struct TileLaunch {
  int C = 1, grid = 0, sb = 0, ns = 0;
  size_t smem = 0;
  bool dyn = false;  // dynamic unit claiming (gemv_dyn.cuh): needs a counter pair
};
cudaError_t plan_gemv_tile(int N, int K, int mr, int wf, int epi, int nsm, int sb, int ns,
                           bool dyn, TileLaunch* out);
cudaError_t launch_gemv_tile(const GemvArgs& a, int wf, int epi, const TileLaunch& L,
                             cudaStream_t st, bool pdl);

// Attention CTAs one SM holds at once (0 if the query fails).
int attn_ctas_per_sm(int D, int kv_f16);
cudaError_t launch_attn(const AttnArgs& a, int D, int kv_f16, int splits, int rows,
                        cudaStream_t st, bool pdl);
// The causal attention of a prompt chunk of T tokens at positions
// a.fixed_pos .. + T - 1 (attn_prefill.cuh): their K/V appended to the row's
// cache, then the tiled attention.
cudaError_t launch_attn_prefill(const AttnArgs& a, int D, int kv_f16, int T, cudaStream_t st);

// The prefill's tensor-core GEMM (gemm_tc.cu, tcgen05 with tensor-memory
// accumulators): Y[t][o] = sum_k W[o][k] X[t][k] for T tokens, W in the tiled
// layout of gemv_tile.cuh (bf16, or int8 with one scale per row).
struct GemmTcArgs {
  const uint8_t* w;        // tiled weights, rows padded to 16
  const float* scales;     // int8: [N] row scales; else null
  int N, K;                // output rows, inputs (K a multiple of 16)
  const __nv_bfloat16* x;  // [T][ldx] activations (16-byte aligned rows)
  int ldx, T;
  __nv_bfloat16* out;      // STORE: out[t][o]; RESID: out[t][o] += y; SWIGLU: out[t][o / 2]
  int ldo;
  int* err;
};
cudaError_t launch_gemm_tc(const GemmTcArgs& a, int wf, int epi, cudaStream_t st);


}  // namespace m3
