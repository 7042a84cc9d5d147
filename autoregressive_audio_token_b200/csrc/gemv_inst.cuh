// gemv_inst.cuh -- the launcher body shared by gemv_<format>.cu: picks the
// row-batch template (2 or 4 rows), the threads per row from K, sizes the grid
// to the SM count and the dynamic shared memory to the CTA's row block.
#pragma once

#include "launch.cuh"

namespace m3 {

template <int MR, int WF, int EPI, int TPR>
cudaError_t launch_gemv_t(const GemvArgs& a, cudaStream_t st, bool pdl, int nsm) {
  constexpr int ESZ = WF == WF_BF16 ? 2 : 1;
  using S = GemvShape<TPR, ESZ>;
  constexpr int UNIT = EPI == EPI_SWIGLU ? 2 : 1;
  if (EPI == EPI_SAMPLE && a.K > S::KC) return cudaErrorInvalidValue;  // one segment per row
  const int units = a.N / UNIT;
  const int grid = units < nsm ? units : nsm;
  const int per = (units + grid - 1) / grid * UNIT;
  const int rows_cta_max = (per + S::R - 1) / S::R * S::R;
  const size_t smem = gemv_smem_bytes<MR, TPR, ESZ>(rows_cta_max);
  auto kern = gemv_kernel<MR, WF, EPI, TPR>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_ex(kern, dim3(grid), dim3(kGemvThreads), smem, st, pdl, a);
}

template <int WF, int EPI, int TPR>
cudaError_t launch_gemv_mr(const GemvArgs& a, cudaStream_t st, bool pdl, int nsm) {
  if (a.mr <= 2) return launch_gemv_t<2, WF, EPI, TPR>(a, st, pdl, nsm);
  return launch_gemv_t<4, WF, EPI, TPR>(a, st, pdl, nsm);
}

template <int WF, int EPI>
cudaError_t launch_gemv_k(const GemvArgs& a, cudaStream_t st, bool pdl, int nsm) {
  constexpr int ESZ = WF == WF_BF16 ? 2 : 1;
  switch (gemv_tpr(a.K, ESZ)) {
    case 32: return launch_gemv_mr<WF, EPI, 32>(a, st, pdl, nsm);
    case 64: return launch_gemv_mr<WF, EPI, 64>(a, st, pdl, nsm);
    case 128: return launch_gemv_mr<WF, EPI, 128>(a, st, pdl, nsm);
    case 256: return launch_gemv_mr<WF, EPI, 256>(a, st, pdl, nsm);
    default:
      if constexpr (ESZ == 2) return launch_gemv_mr<WF, EPI, 512>(a, st, pdl, nsm);
      return cudaErrorInvalidValue;
  }
}

template <int WF>
cudaError_t launch_gemv_wf(const GemvArgs& a, int epi, cudaStream_t st, bool pdl, int nsm) {
  switch (epi) {
    case EPI_STORE: return launch_gemv_k<WF, EPI_STORE>(a, st, pdl, nsm);
    case EPI_RESID: return launch_gemv_k<WF, EPI_RESID>(a, st, pdl, nsm);
    case EPI_SWIGLU: return launch_gemv_k<WF, EPI_SWIGLU>(a, st, pdl, nsm);
    default: return launch_gemv_k<WF, EPI_SAMPLE>(a, st, pdl, nsm);
  }
}

}  // namespace m3
