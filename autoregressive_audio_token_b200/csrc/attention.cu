// attention.cu -- instantiation and launcher of the split-K decode attention.
#include "attn_prefill.cuh"
#include "launch.cuh"

namespace m3 {

template <int D, int KVF16>
static cudaError_t launch_attn_t(const AttnArgs& a, int splits, int rows, cudaStream_t st,
                                 bool pdl) {
  constexpr size_t smem = attn_smem_bytes<D>();
  auto kern = attn_decode_kernel<D, KVF16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // the whole unified L1 as shared memory, so that the next kernel's CTA
  // fits beside this one
  e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  if (splits < 1 || splits > kAttnMaxSplits) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(splits, a.Hkv, rows);
  cfg.blockDim = dim3(kAttnWarps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = splits;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

template <int D, int KVF16>
static int attn_resident_t() {
  constexpr size_t smem = attn_smem_bytes<D>();
  auto kern = attn_decode_kernel<D, KVF16>;
  int n = 0;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
          cudaSuccess ||
      cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kAttnWarps * 32, smem) !=
          cudaSuccess)
    return 0;
  return n;
}

int attn_ctas_per_sm(int D, int kv_f16) {
  if (D == 128) return kv_f16 ? attn_resident_t<128, 1>() : attn_resident_t<128, 0>();
  if (D == 64) return kv_f16 ? attn_resident_t<64, 1>() : attn_resident_t<64, 0>();
  return 0;
}

template <int D, int KVF16>
static cudaError_t launch_attn_prefill_t(const AttnArgs& a, int T, cudaStream_t st) {
  constexpr size_t smem = attn_prefill_smem<D>();
  auto kern = attn_prefill_kernel<D, KVF16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int tpw = 16 / (a.Hq / a.Hkv);
  const int per = kApWarps * tpw;
  kern<<<dim3((T + per - 1) / per, a.Hkv), kApWarps * 32, smem, st>>>(a, T);
  return cudaGetLastError();
}

cudaError_t launch_attn_prefill(const AttnArgs& a, int D, int kv_f16, int T, cudaStream_t st) {
  if (T < 1 || a.Hkv < 1 || a.Hq % a.Hkv || 16 % (a.Hq / a.Hkv) || a.fixed_pos < 0 ||
      a.page_size % kApKT)
    return cudaErrorInvalidValue;
  {  // the chunk's K/V first
    const dim3 grid((unsigned)((T * a.Hkv + 7) / 8));
    if (D == 128) {
      if (kv_f16) kv_append_kernel<128, 1><<<grid, 256, 0, st>>>(a, T);
      else kv_append_kernel<128, 0><<<grid, 256, 0, st>>>(a, T);
    } else if (D == 64) {
      if (kv_f16) kv_append_kernel<64, 1><<<grid, 256, 0, st>>>(a, T);
      else kv_append_kernel<64, 0><<<grid, 256, 0, st>>>(a, T);
    }
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (D == 128) return kv_f16 ? launch_attn_prefill_t<128, 1>(a, T, st)
                              : launch_attn_prefill_t<128, 0>(a, T, st);
  if (D == 64) return kv_f16 ? launch_attn_prefill_t<64, 1>(a, T, st)
                             : launch_attn_prefill_t<64, 0>(a, T, st);
  return cudaErrorInvalidValue;
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
