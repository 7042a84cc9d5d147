// frame.cu -- instantiation and cooperative launcher of the persistent
// whole-frame kernel (frame.cuh).
#include "frame.cuh"
#include "launch.cuh"

namespace m3 {

template <int MR, int WF, int KVF16>
static cudaError_t launch_frame_t(const FrameArgs& a, int rows_cta_max, int grid,
                                  cudaStream_t st) {
  const size_t smem = frame_smem_bytes<MR, WF>(rows_cta_max);
  auto kern = frame_kernel<MR, WF, KVF16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kFrameThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // all CTAs co-resident (grid barriers)
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

size_t frame_smem(int mr, int wf, int rows_cta_max) {
  if (mr <= 2) return wf == WF_BF16 ? frame_smem_bytes<2, WF_BF16>(rows_cta_max)
                                    : frame_smem_bytes<2, WF_I8ROW>(rows_cta_max);
  return wf == WF_BF16 ? frame_smem_bytes<4, WF_BF16>(rows_cta_max)
                       : frame_smem_bytes<4, WF_I8ROW>(rows_cta_max);
}

cudaError_t launch_frame(const FrameArgs& a, int wf, int kv_f16, int rows_cta_max, int grid,
                         cudaStream_t st) {
  if (a.mr <= 2) {
    if (wf == WF_BF16)
      return kv_f16 ? launch_frame_t<2, WF_BF16, 1>(a, rows_cta_max, grid, st)
                    : launch_frame_t<2, WF_BF16, 0>(a, rows_cta_max, grid, st);
    return kv_f16 ? launch_frame_t<2, WF_I8ROW, 1>(a, rows_cta_max, grid, st)
                  : launch_frame_t<2, WF_I8ROW, 0>(a, rows_cta_max, grid, st);
  }
  if (wf == WF_BF16)
    return kv_f16 ? launch_frame_t<4, WF_BF16, 1>(a, rows_cta_max, grid, st)
                  : launch_frame_t<4, WF_BF16, 0>(a, rows_cta_max, grid, st);
  return kv_f16 ? launch_frame_t<4, WF_I8ROW, 1>(a, rows_cta_max, grid, st)
                : launch_frame_t<4, WF_I8ROW, 0>(a, rows_cta_max, grid, st);
}

}  // namespace m3
