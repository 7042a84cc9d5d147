// gemv_tile.cu -- launch planning and launchers of the tiled tensor-core GEMV
// (gemv_tile.cuh): cluster size (K split) and grid from the SM count and the
// co-resident cluster capacity, shared-memory ring size.
#include <cuda_runtime.h>

#include <cstdlib>

#include "gemv_dyn.cuh"
#include "gemv_tile.cuh"
#include "launch.cuh"

namespace m3 {

namespace {

template <int WF, int EPI>
cudaError_t launch_tile_t(const GemvArgs& a0, const TileLaunch& L, cudaStream_t st, bool pdl) {
  GemvArgs a = a0;
  a.tc = L.C;
  a.tsb = L.sb;
  a.tns = L.ns;
  auto kern = a.mr > 8 ? gemv_tile_kernel<WF, EPI, true> : gemv_tile_kernel<WF, EPI, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.smem);
  if (e != cudaSuccess) return e;
  // the whole unified L1 as shared memory, so that the next kernel's CTA
  // fits beside this one
  e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(L.grid);
  cfg.blockDim = dim3(kTThreads);
  cfg.dynamicSmemBytes = L.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = L.C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

template <int WF, int EPI>
cudaError_t max_clusters_t(int C, size_t smem, int* n) {
  auto kern = gemv_tile_kernel<WF, EPI, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // the whole unified L1 as shared memory, so that the next kernel's CTA
  // fits beside this one
  e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C);
  cfg.blockDim = dim3(kTThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaOccupancyMaxActiveClusters(n, kern, &cfg);
}

template <int WF, int EPI>
cudaError_t launch_dyn_t(const GemvArgs& a0, const TileLaunch& L, cudaStream_t st, bool pdl) {
  GemvArgs a = a0;
  a.tc = 1;
  a.tsb = L.sb;
  a.tns = L.ns;
  auto kern = gemv_dyn_kernel<WF, EPI>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.smem);
  if (e != cudaSuccess) return e;
  // the whole unified L1 as shared memory, so that the next kernel's CTA
  // fits beside this one
  e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  return launch_ex(kern, dim3(L.grid), dim3(kDThreads), L.smem, st, pdl, a);
}

template <int WF>
cudaError_t dispatch_epi(const GemvArgs& a, int epi, const TileLaunch& L, cudaStream_t st, bool pdl) {
  if (L.dyn) {
    if (!a.ctr) return cudaErrorInvalidValue;
    switch (epi) {
      case EPI_STORE: return launch_dyn_t<WF, EPI_STORE>(a, L, st, pdl);
      case EPI_RESID: return launch_dyn_t<WF, EPI_RESID>(a, L, st, pdl);
      case EPI_SWIGLU: return launch_dyn_t<WF, EPI_SWIGLU>(a, L, st, pdl);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (epi) {
    case EPI_STORE: return launch_tile_t<WF, EPI_STORE>(a, L, st, pdl);
    case EPI_RESID: return launch_tile_t<WF, EPI_RESID>(a, L, st, pdl);
    case EPI_SWIGLU: return launch_tile_t<WF, EPI_SWIGLU>(a, L, st, pdl);
    default: return launch_tile_t<WF, EPI_SAMPLE>(a, L, st, pdl);
  }
}

template <int WF>
cudaError_t clusters_epi(int epi, int C, size_t smem, int* n) {
  switch (epi) {
    case EPI_STORE: return max_clusters_t<WF, EPI_STORE>(C, smem, n);
    case EPI_RESID: return max_clusters_t<WF, EPI_RESID>(C, smem, n);
    case EPI_SWIGLU: return max_clusters_t<WF, EPI_SWIGLU>(C, smem, n);
    default: return max_clusters_t<WF, EPI_SAMPLE>(C, smem, n);
  }
}

cudaError_t max_clusters(int wf, int epi, int C, size_t smem, int* n) {
  return wf == WF_BF16 ? clusters_epi<WF_BF16>(epi, C, smem, n)
                       : clusters_epi<WF_I8ROW>(epi, C, smem, n);
}

}  // namespace

// Shared memory that still lets a second CTA of this kernel (the next
// launch's, prefetching) sit on the same SM: 228 KB per SM, 1 KB reserved
// per CTA.
constexpr size_t kTCoresidentSmem = 113 * 1024;

cudaError_t plan_gemv_tile(int N, int K, int mr, int wf, int epi, int nsm, int sb, int ns,
                           bool dyn, TileLaunch* out) {
  if (K % 16 || N < 1 || mr < 1 || mr > kMaxRows) return cudaErrorInvalidValue;
  const int esz = wf == WF_BF16 ? 2 : 1;
  if (sb % (256 * esz)) return cudaErrorInvalidValue;
  const int T = K / 16, U = (N + kUnitRows - 1) / kUnitRows;
  // dynamic claiming: whole K per CTA, up to 8 rows, not the sampler
  if (epi != EPI_SAMPLE && mr <= kDMaxRows && dyn) {
    const DynPlan d = dyn_plan(K, esz, sb, sb * ns);
    const size_t smem = dyn_smem_bytes(d, mr);
    if (d.slots >= 2 && smem <= 227 * 1024) {
      out->C = 1;
      out->grid = nsm;
      out->sb = sb;
      out->ns = ns;
      out->smem = smem;
      out->dyn = true;
      return cudaSuccess;
    }
  }
  // the static partition: the cluster size (K split) whose busiest CTA
  // streams the fewest tiles, for stage bytes sbt
  auto search = [&](int sbt, TileLaunch* best, double* best_cost) -> cudaError_t {
    bool found = false;
    // M3_GEMV_CLUSTER: only this cluster size (tuning)
    int force_c = 0;
    if (const char* e = getenv("M3_GEMV_CLUSTER")) force_c = atoi(e);
    for (int C = 1; C <= 8; C *= 2) {
      if (T % C || C > nsm) continue;
      if (force_c > 0 && C != force_c) continue;
      int ncl = nsm / C;
      if (ncl > U) ncl = U;
      TilePlan p = tile_plan(N, K, esz, C, ncl, sbt, sbt * ns);
      if (p.slots < 2) continue;
      size_t smem = tile_smem_bytes(p, mr);
      if (smem > 227 * 1024) continue;
      int cap = 0;
      cudaError_t e = max_clusters(wf, epi, C, smem, &cap);
      if (e != cudaSuccess) return e;
      if (cap < 1) continue;
      if (ncl > cap) {
        ncl = cap;
        p = tile_plan(N, K, esz, C, ncl, sbt, sbt * ns);
        smem = tile_smem_bytes(p, mr);
      }
      // time ~ the busiest CTA's tiles; a cluster reduction and a footprint
      // that rules out co-residency cost a little extra
      double cost = (double)p.nu_max * p.Tr * (1.0 + (C > 1 ? 0.01 : 0.0));
      if (smem > kTCoresidentSmem) cost *= 1.05;
      if (!found || cost < *best_cost) {
        found = true;
        *best_cost = cost;
        best->C = C;
        best->grid = ncl * C;
        best->sb = sbt;
        best->ns = ns;
        best->smem = smem;
        best->dyn = false;
      }
    }
    return found ? cudaSuccess : cudaErrorInvalidConfiguration;
  };
  double cost = 0.0;
  cudaError_t e = search(sb, out, &cost);
  if (e != cudaSuccess && e != cudaErrorInvalidConfiguration) return e;
  // more than 8 rows: their activations crowd the shared memory, and half
  // stages can admit a smaller cluster that runs on more SMs (16 rows of
  // gate/up: 74 clusters of 2 instead of 33 of 4); taken when the busiest
  // CTA's share drops by more than 5 % (where the full stages fit no ring at
  // all, the caller's next try is fewer full stages, measured better)
  if (e == cudaSuccess && mr > 8 && sb / 2 >= 4096 && (sb / 2) % (256 * esz) == 0) {
    TileLaunch h;
    double hc = 0.0;
    const cudaError_t eh = search(sb / 2, &h, &hc);
    if (eh != cudaSuccess && eh != cudaErrorInvalidConfiguration) return eh;
    if (eh == cudaSuccess && hc < 0.95 * cost) *out = h;
  }
  return e;
}

cudaError_t launch_gemv_tile(const GemvArgs& a, int wf, int epi, const TileLaunch& L,
                             cudaStream_t st, bool pdl) {
  if (wf == WF_BF16) return dispatch_epi<WF_BF16>(a, epi, L, st, pdl);
  if (wf == WF_I8ROW) return dispatch_epi<WF_I8ROW>(a, epi, L, st, pdl);
  return cudaErrorInvalidValue;
}

}  // namespace m3
