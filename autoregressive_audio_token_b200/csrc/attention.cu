// attention.cu -- instantiation and launcher of the split-K decode attention.
#include "launch.cuh"

namespace m3 {

template <int D, int KVF16>
static cudaError_t launch_attn_t(const AttnArgs& a, int splits, int rows, cudaStream_t st,
                                 bool pdl) {
  constexpr size_t smem = attn_smem_bytes<D>();
  auto kern = attn_decode_kernel<D, KVF16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_ex(kern, dim3(splits, a.Hkv, rows), dim3(kAttnWarps * 32), smem, st, pdl, a);
}

cudaError_t launch_attn(const AttnArgs& a, int D, int kv_f16, int splits, int rows,
                        cudaStream_t st, bool pdl) {
  if (D == 128) return kv_f16 ? launch_attn_t<128, 1>(a, splits, rows, st, pdl)
                              : launch_attn_t<128, 0>(a, splits, rows, st, pdl);
  if (D == 64) return kv_f16 ? launch_attn_t<64, 1>(a, splits, rows, st, pdl)
                             : launch_attn_t<64, 0>(a, splits, rows, st, pdl);
  return cudaErrorInvalidValue;
}

}  // namespace m3
