// gemv_bf16.cu -- instantiation of the weight-streaming GEMV for one weight format.
#include "gemv_inst.cuh"

namespace m3 {
cudaError_t launch_gemv_bf16(const GemvArgs& a, int epi, cudaStream_t st, bool pdl, int nsm) {
  return launch_gemv_wf<WF_BF16>(a, epi, st, pdl, nsm);
}
}  // namespace m3
