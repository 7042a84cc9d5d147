// gemv_i8row.cu -- instantiation of the weight-streaming GEMV for one weight format.
#include "gemv_inst.cuh"

namespace m3 {
cudaError_t launch_gemv_i8row(const GemvArgs& a, int epi, cudaStream_t st, bool pdl, int nsm) {
  return launch_gemv_wf<WF_I8ROW>(a, epi, st, pdl, nsm);
}
}  // namespace m3
