// gemv_i8g128.cu -- instantiation of the weight-streaming GEMV for one weight format.
#include "gemv_inst.cuh"

namespace m3 {
cudaError_t launch_gemv_i8g128(const GemvArgs& a, int epi, cudaStream_t st, bool pdl, int nsm) {
  return launch_gemv_wf<WF_I8G128>(a, epi, st, pdl, nsm);
}
}  // namespace m3
