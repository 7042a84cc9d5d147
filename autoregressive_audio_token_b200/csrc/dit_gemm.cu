// dit_gemm.cu -- persistent tcgen05 GEMM of the DiT (see dit_gemm.cuh).
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "dit_gemm.cuh"

namespace m3 {

namespace {

constexpr int kGM = 128;                         // tokens per tile (MMA M = TMEM lanes)
constexpr int kGN = 256;                         // outputs per tile (MMA N = TMEM columns)
constexpr int kGK = 64;                          // K per stage: 64 fp16 = 128 bytes
constexpr int kGStages = 4;
constexpr int kGThreads = 192;                   // TMA warp, MMA warp, 4 epilogue warps
constexpr uint32_t kABytes = kGM * kGK * 2;      // 16 KB
constexpr uint32_t kBBytes = kGN * kGK * 2;      // 32 KB
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr uint32_t kAccCols = kGN;               // fp32 columns of one accumulator
constexpr uint32_t kTmemCols = 2 * kAccCols;     // two accumulators: all 512 columns
constexpr size_t kGSmem = (size_t)kGStages * kStageBytes + 1024 /* align */ + 256 /* bars */;

// kind::f16 instruction descriptor: D fp32 (bits 4-5 = 1), A and B fp16
// (bits 7-9, 10-12 = 0) or both bf16 (= 1), both K-major (bits 15, 16 = 0),
// N >> 3 at bit 17, M >> 4 at bit 24.
template <int BF>
constexpr uint32_t idesc_1() {
  return (1u << 4) | ((uint32_t)BF << 7) | ((uint32_t)BF << 10) | ((uint32_t)(kGN >> 3) << 17) |
         ((uint32_t)(kGM >> 4) << 24);
}

// Shared-memory matrix descriptor of a K-major operand in the 128-byte swizzle:
// start address >> 4 (bits 0-13), leading byte offset (unused by swizzled
// K-major layouts: 16 bytes) at bit 16, stride byte offset 1024 (8 rows of
// 128 bytes) >> 4 at bit 32, version 1 at bit 46, swizzle mode 2 (128 B) at
// bit 61.  The tile bases are 1024-byte aligned, so the base offset is 0.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

template <int BF>
__device__ __forceinline__ void tc_mma_f16(uint32_t tmem_d, uint64_t a, uint64_t b,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
      ::"r"(tmem_d), "l"(a), "l"(b), "r"(idesc_1<BF>()), "r"(accumulate), "r"(0u), "r"(0u),
        "r"(0u), "r"(0u)
      : "memory");
}

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// 32 consecutive fp32 columns of this thread's accumulator lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 2-D tiled tensor-map copy global -> this CTA's shared memory (no multicast).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* tm, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, "
      "{%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* tm) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tm)) : "memory");
}

// Two fp32 -> the output type's packed pair (round to nearest even); one fp32
// through the output type; a packed pair of the output type -> fp32.
template <int BF>
__device__ __forceinline__ uint32_t h2pack(float lo, float hi) {
  if constexpr (BF) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
  } else {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
  }
}

template <int BF>
__device__ __forceinline__ float rh(float v) {
  if constexpr (BF) return __bfloat162float(__float2bfloat16_rn(v));
  else return __half2float(__float2half_rn(v));
}

template <int BF>
__device__ __forceinline__ float2 unpack2(uint32_t w) {
  if constexpr (BF) return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w));
  else return __half22float2(*reinterpret_cast<const __half2*>(&w));
}

// The epilogue of 32 accumulator columns o0..o0+31 of token row t.
template <int EPI, int BF>
__device__ __forceinline__ void epilogue_chunk(const DitGemmArgs& a, int t, int o0,
                                               float (&v)[32]) {
  typedef uint16_t elem_t;  // the output type's bits (fp16 or bf16)
  elem_t* const out = static_cast<elem_t*>(a.out);
  if (t >= a.M) return;
  if constexpr (EPI == DIT_EPI_GLU) {
    // columns (2j, 2j+1) are (gate, up) of GLU output o0/2 + j
    float y[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float g = rh<BF>(v[2 * j]), u = rh<BF>(v[2 * j + 1]);
      const float s = rh<BF>(__fdiv_rn(g, __fadd_rn(1.0f, expf(-g))));
      y[j] = __fmul_rn(s, u);
    }
    uint4* q = reinterpret_cast<uint4*>(out + (size_t)t * a.ldo + (o0 >> 1));
#pragma unroll
    for (int c = 0; c < 2; ++c)
      q[c] = make_uint4(h2pack<BF>(y[8 * c], y[8 * c + 1]), h2pack<BF>(y[8 * c + 2], y[8 * c + 3]),
                        h2pack<BF>(y[8 * c + 4], y[8 * c + 5]), h2pack<BF>(y[8 * c + 6], y[8 * c + 7]));
  } else {
  float y[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) y[j] = rh<BF>(v[j]);
  elem_t* p = out + (size_t)t * a.ldo + o0;  // N is a multiple of 32: whole chunks only
  if constexpr (EPI == DIT_EPI_TEMB) {
    const uint4* q = reinterpret_cast<const uint4*>(a.vec + o0);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 w = q[c];
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = unpack2<BF>(ws[k]);
        y[8 * c + 2 * k] = __fadd_rn(y[8 * c + 2 * k], f.x);
        y[8 * c + 2 * k + 1] = __fadd_rn(y[8 * c + 2 * k + 1], f.y);
      }
    }
  } else if constexpr (EPI == DIT_EPI_ROPE) {
    // the first 2 * rope_half dims of every q / k head: pairs (i, i + rope_half)
    if (o0 < a.rope_cols && (o0 % a.head_dim) == 0 && a.rope_half == 16) {
      const float2* cs = a.rope + (size_t)(t % a.rope_T) * 16;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float2 r = cs[i];
        const float x0 = y[i], x1 = y[i + 16];
        y[i] = __fsub_rn(__fmul_rn(x0, r.x), __fmul_rn(x1, r.y));
        y[i + 16] = __fadd_rn(__fmul_rn(x1, r.x), __fmul_rn(x0, r.y));
      }
    }
  } else if constexpr (EPI == DIT_EPI_RESID) {
    const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 w = q[c];
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = unpack2<BF>(ws[k]);
        y[8 * c + 2 * k] = __fadd_rn(f.x, y[8 * c + 2 * k]);
        y[8 * c + 2 * k + 1] = __fadd_rn(f.y, y[8 * c + 2 * k + 1]);
      }
    }
  }
  uint4* q = reinterpret_cast<uint4*>(p);
#pragma unroll
  for (int c = 0; c < 4; ++c)
    q[c] = make_uint4(h2pack<BF>(y[8 * c], y[8 * c + 1]), h2pack<BF>(y[8 * c + 2], y[8 * c + 3]),
                      h2pack<BF>(y[8 * c + 4], y[8 * c + 5]), h2pack<BF>(y[8 * c + 6], y[8 * c + 7]));
  }
}

template <int EPI, int BF>
__global__ void __launch_bounds__(kGThreads, 1)
    dit_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const DitGemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kGStages * kStageBytes);
  uint64_t* empty = full + kGStages;
  uint64_t* tfull = empty + kGStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* counts = reinterpret_cast<int*>(tmem_slot + 1);  // [0] issued, [1] consumed

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_m = (a.M + kGM - 1) / kGM, num_n = (a.N + kGN - 1) / kGN;
  const int ntiles = num_m * num_n;
  const int KB = a.K / kGK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4);  // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
    counts[0] = counts[1] = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA --
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        const int m0 = (tile % num_m) * kGM, n0 = (tile / num_m) * kGN;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % kGStages, use = it / kGStages;
          if (use > 0 && !(ok = mbar_wait(&empty[s], (uint32_t)(use - 1) & 1u, a.err))) break;
          uint8_t* sa = smem + (size_t)s * kStageBytes;
          mbar_arrive_expect_tx(&full[s], kStageBytes);
          tma_load_2d(sa, &tmA, kb * kGK, m0, &full[s]);
          tma_load_2d(sa + kABytes, &tmB, kb * kGK, n0, &full[s]);
        }
      }
      counts[0] = it;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA --
    if (lane == 0) {
      int it = 0, lt = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++lt) {
        const int acc = lt & 1, use_a = lt >> 1;
        if (use_a > 0 && !(ok = mbar_wait(&tempty[acc], (uint32_t)(use_a - 1) & 1u, a.err))) break;
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)acc * kAccCols;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % kGStages, use = it / kGStages;
          if (!(ok = mbar_wait(&full[s], (uint32_t)use & 1u, a.err))) break;
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + (size_t)s * kStageBytes), sb = sa + kABytes;
#pragma unroll
          for (int ks = 0; ks < kGK / 16; ++ks)
            tc_mma_f16<BF>(d, sw128_desc(sa + ks * 32), sw128_desc(sb + ks * 32),
                       (kb > 0 || ks > 0) ? 1u : 0u);
          tc_commit(&empty[s]);
        }
        if (ok) tc_commit(&tfull[acc]);
      }
      counts[1] = it;
      if (!ok) {  // let this thread's MMAs finish before the memory goes away
        tc_commit(drain);
        for (long long i = 0; i < kSpinLimit && !mbar_try_wait(drain, 0); ++i) {
        }
      }
    }
  } else {
    // ------------------------------------------------------- epilogue --
    const int q = warp & 3;  // TMEM lanes 32q..32q+31 (the warp's access window)
    int lt = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++lt) {
      const int acc = lt & 1, use_a = lt >> 1;
      if (!mbar_wait(&tfull[acc], (uint32_t)use_a & 1u, a.err)) break;
      tc_fence_after();
      const int m0 = (tile % num_m) * kGM, n0 = (tile / num_m) * kGN;
      const int t = m0 + q * 32 + lane;
      const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)acc * kAccCols;
#pragma unroll 1
      for (int c = 0; c < kGN / 32; ++c) {
        if (n0 + c * 32 >= a.N) break;  // the last output block may be narrower (uniform)
        float v[32];
        tmem_ld32(taddr + (uint32_t)(c * 32), v);
        epilogue_chunk<EPI, BF>(a, t, n0 + c * 32, v);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
  }

  __syncthreads();
  if (threadIdx.x == 0) {
    // copies issued but never consumed (only after a failed wait): let them land
    for (int it = counts[1]; it < counts[0]; ++it) {
      const int s = it % kGStages;
      for (long long i = 0; i < kSpinLimit && !mbar_try_wait(&full[s], (uint32_t)(it / kGStages) & 1u);
           ++i) {
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

// --------------------------------------------------- CTA-pair variant ----
// Two CTAs of a cluster compute one 256 x 256 tile with tcgen05.mma
// cta_group::2: CTA r holds the tokens m0 + 128 r .. + 127 of A (and their
// 128 accumulator rows in its own tensor memory) and the outputs
// n0 + 128 r .. + 127 of B, and the MMA issued by rank 0 reads the A half
// and both B halves of the pair.  Each SM then moves 32 KB per 64-wide K
// stage for the same MMA work as the one-CTA kernel's 48 KB, so the ring
// (6 stages) covers more L2 latency.  Both CTAs' copies complete on rank
// 0's "full" barrier; rank 0's commits arrive on both CTAs' "empty" and
// "accumulator full" barriers (commit multicast within the pair; no
// multicast loads); both CTAs' epilogue warps arrive on rank 0's
// "accumulator empty" barrier.
constexpr int kPStages = 6;
constexpr uint32_t kPHalfBytes = 128 * kGK * 2;  // 16 KB: one operand half of a stage
constexpr uint32_t kPStageBytes = 2 * kPHalfBytes;
constexpr size_t kPSmem = (size_t)kPStages * kPStageBytes + 1024 + 256;
// M = 256 (the pair), N = 256
template <int BF>
constexpr uint32_t idesc_2() {
  return (1u << 4) | ((uint32_t)BF << 7) | ((uint32_t)BF << 10) | ((uint32_t)(kGN >> 3) << 17) |
         ((uint32_t)(256 >> 4) << 24);
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

// The shared::cluster address of the same shared-memory object in CTA `rank`.
__device__ __forceinline__ uint32_t map_rank(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}

__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}

template <int BF>
__device__ __forceinline__ void tc_mma_f16_pair(uint32_t tmem_d, uint64_t a, uint64_t b,
                                                uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8, %9, %10, %11, %12}, "
      "p;\n\t}" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc_2<BF>()), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u), "r"(0u),
      "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}

// Arrive (once each) on `bar` in both CTAs of the pair when this thread's
// MMAs have completed.
__device__ __forceinline__ void tc_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 "
      "[%0], %1;" ::"r"(smem_u32(bar)),
      "h"((uint16_t)3)
      : "memory");
}

// A pair copy: lands in this CTA's shared memory, completes on rank 0's barrier.
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* tm, int x, int y,
                                                 uint32_t bar_rank0) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(bar_rank0)
      : "memory");
}

template <int EPI, int BF>
__global__ void __launch_bounds__(kGThreads, 1)
    dit_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                         const __grid_constant__ CUtensorMap tmB, const DitGemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kPStages * kPStageBytes);
  uint64_t* empty = full + kPStages;
  uint64_t* tfull = empty + kPStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* counts = reinterpret_cast<int*>(tmem_slot + 1);  // [0] issued, [1] consumed

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int num_m = (a.M + 255) / 256, num_n = (a.N + kGN - 1) / kGN;
  const int ntiles = num_m * num_n;
  const int KB = a.K / kGK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 8);  // one arrival per epilogue warp of the pair
    }
    mbar_init(drain, 1);
    counts[0] = counts[1] = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers exist before any copy or commit reaches them
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA --
    if (lane == 0) {
      const uint32_t full0 = map_rank(full, 0);  // rank 0's full[0]
      int it = 0;
      bool ok = true;
      for (int tile = pair; tile < ntiles && ok; tile += npairs) {
        const int m0 = (tile % num_m) * 256 + (int)rank * 128;
        const int n0 = (tile / num_m) * kGN + (int)rank * 128;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % kPStages, use = it / kPStages;
          if (use > 0 && !(ok = mbar_wait(&empty[s], (uint32_t)(use - 1) & 1u, a.err))) break;
          uint8_t* sa = smem + (size_t)s * kPStageBytes;
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * kPStageBytes);  // both CTAs' bytes
          const uint32_t fb = full0 + (uint32_t)(s * sizeof(uint64_t));
          tma_load_2d_pair(sa, &tmA, kb * kGK, m0, fb);
          tma_load_2d_pair(sa + kPHalfBytes, &tmB, kb * kGK, n0, fb);
        }
      }
      counts[0] = it;
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA (rank 0 only) --
    if (lane == 0 && rank == 0) {
      int it = 0, lt = 0;
      bool ok = true;
      for (int tile = pair; tile < ntiles && ok; tile += npairs, ++lt) {
        const int acc = lt & 1, use_a = lt >> 1;
        if (use_a > 0 && !(ok = mbar_wait(&tempty[acc], (uint32_t)(use_a - 1) & 1u, a.err))) break;
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)acc * kAccCols;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % kPStages, use = it / kPStages;
          if (!(ok = mbar_wait(&full[s], (uint32_t)use & 1u, a.err))) break;
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + (size_t)s * kPStageBytes), sb = sa + kPHalfBytes;
#pragma unroll
          for (int ks = 0; ks < kGK / 16; ++ks)
            tc_mma_f16_pair<BF>(d, sw128_desc(sa + ks * 32), sw128_desc(sb + ks * 32),
                            (kb > 0 || ks > 0) ? 1u : 0u);
          tc_commit_pair(&empty[s]);
        }
        if (ok) tc_commit_pair(&tfull[acc]);
      }
      counts[1] = it;
      if (!ok) {  // let this thread's MMAs finish before the memory goes away
        tc_commit_pair(drain);
        for (long long i = 0; i < kSpinLimit && !mbar_try_wait(drain, 0); ++i) {
        }
      }
    }
  } else {
    // ------------------------------------------------------- epilogue --
    const int q = warp & 3;  // TMEM lanes 32q..32q+31 (the warp's access window)
    const uint32_t tempty0 = map_rank(tempty, 0);
    int lt = 0;
    for (int tile = pair; tile < ntiles; tile += npairs, ++lt) {
      const int acc = lt & 1, use_a = lt >> 1;
      if (!mbar_wait(&tfull[acc], (uint32_t)use_a & 1u, a.err)) break;
      tc_fence_after();
      const int m0 = (tile % num_m) * 256 + (int)rank * 128, n0 = (tile / num_m) * kGN;
      const int t = m0 + q * 32 + lane;
      const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)acc * kAccCols;
#pragma unroll 1
      for (int c = 0; c < kGN / 32; ++c) {
        if (n0 + c * 32 >= a.N) break;  // the last output block may be narrower (uniform)
        float v[32];
        tmem_ld32(taddr + (uint32_t)(c * 32), v);
        epilogue_chunk<EPI, BF>(a, t, n0 + c * 32, v);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(tempty0 + (uint32_t)(acc * sizeof(uint64_t)));
    }
  }

  __syncthreads();
  if (threadIdx.x == 0 && rank == 0) {
    // copies issued but never consumed (only after a failed wait): let them land
    for (int it = counts[1]; it < counts[0]; ++it) {
      const int s = it % kPStages;
      for (long long i = 0; i < kSpinLimit && !mbar_try_wait(&full[s], (uint32_t)(it / kPStages) & 1u);
           ++i) {
      }
    }
  }
  tc_fence_before();
  cluster_sync_all();  // no CTA leaves while its peer may still signal its barriers
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// A [rows][ld] fp16 or bf16 row-major matrix as a tensor map of
// (box_rows x 64) boxes in the 128-byte swizzle.
cudaError_t make_map(CUtensorMap* tm, const void* base, int rows, int cols, int ld,
                     int box_rows, bool bf16) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)kGK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(tm, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                        2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int EPI, int BF>
cudaError_t set_attr() {
  const cudaError_t e = cudaFuncSetAttribute(
      dit_gemm_kernel<EPI, BF>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGSmem);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(dit_gemm_pair_kernel<EPI, BF>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPSmem);
}

template <int EPI, int BF>
cudaError_t launch_pair_t(const CUtensorMap& ta, const CUtensorMap& tb, const DitGemmArgs& a,
                          int nsm, cudaStream_t st) {
  const int ntiles = ((a.M + 255) / 256) * ((a.N + kGN - 1) / kGN);
  const int pairs = ntiles < nsm / 2 ? ntiles : nsm / 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(kGThreads);
  cfg.dynamicSmemBytes = kPSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, dit_gemm_pair_kernel<EPI, BF>, ta, tb, a);
}

template <int EPI, int BF>
cudaError_t launch_t(const CUtensorMap& ta, const CUtensorMap& tb, const DitGemmArgs& a, int nsm,
                     cudaStream_t st) {
  const int ntiles = ((a.M + kGM - 1) / kGM) * ((a.N + kGN - 1) / kGN);
  const int grid = ntiles < nsm ? ntiles : nsm;
  dit_gemm_kernel<EPI, BF><<<grid, kGThreads, kGSmem, st>>>(ta, tb, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t prepare_dit_gemm() {
  if (!encode_fn()) return cudaErrorNotSupported;
  cudaError_t e = set_attr<DIT_EPI_STORE, 0>();
  if (e == cudaSuccess) e = set_attr<DIT_EPI_TEMB, 0>();
  if (e == cudaSuccess) e = set_attr<DIT_EPI_ROPE, 0>();
  if (e == cudaSuccess) e = set_attr<DIT_EPI_RESID, 0>();
  if (e == cudaSuccess) e = set_attr<DIT_EPI_GLU, 0>();
  if (e == cudaSuccess) e = set_attr<DIT_EPI_STORE, 1>();
  if (e == cudaSuccess) e = set_attr<DIT_EPI_RESID, 1>();
  if (e == cudaSuccess) e = set_attr<DIT_EPI_GLU, 1>();
  return e;
}

cudaError_t launch_dit_gemm(const void* X, int ldx, const void* W, const DitGemmArgs& a,
                            int epi, int nsm, cudaStream_t st, bool bf16) {
  if (!X || !W || !a.out || a.M < 1 || a.N < 1 || a.K < kGK || a.K % kGK || ldx < a.K ||
      ldx % 8 || (reinterpret_cast<uintptr_t>(X) & 15) || (reinterpret_cast<uintptr_t>(W) & 15) ||
      (reinterpret_cast<uintptr_t>(a.out) & 15) || a.ldo % 8 || nsm < 1)
    return cudaErrorInvalidValue;
  // whole 32-column chunks in the epilogue; 16-byte aligned vector accesses
  if (a.N % 32 || (epi == DIT_EPI_GLU ? a.ldo < a.N / 2 : a.ldo < a.N)) return cudaErrorInvalidValue;
  if (epi == DIT_EPI_TEMB && (reinterpret_cast<uintptr_t>(a.vec) & 15)) return cudaErrorInvalidValue;
  if (epi == DIT_EPI_TEMB && !a.vec) return cudaErrorInvalidValue;
  if (epi == DIT_EPI_ROPE && (!a.rope || a.rope_T < 1 || a.head_dim % 32 || a.rope_half != 16))
    return cudaErrorInvalidValue;
  // bf16 operands: the epilogues of the prompt prefill (store, residual, GLU)
  if (bf16 && epi != DIT_EPI_STORE && epi != DIT_EPI_RESID && epi != DIT_EPI_GLU)
    return cudaErrorInvalidValue;
  // CTA pairs or single CTAs: a pair tile streams about 12 % faster per SM
  // (32 instead of 48 KB of operands per stage, measured on the chunk's
  // GEMMs), but its 256-token blocks pad a ragged M more and its tiles come
  // in half as many slots; take the pairs when their rounds of tiles, so
  // discounted, end first
  const long long n_blk = (a.N + kGN - 1) / kGN;
  const long long rounds1 = ((a.M + 127) / 128 * n_blk + nsm - 1) / nsm;
  const long long rounds2 = nsm >= 2 ? ((a.M + 255) / 256 * n_blk + nsm / 2 - 1) / (nsm / 2) : 0;
  const bool pair = a.M >= 256 && nsm >= 2 && rounds2 * 88 < rounds1 * 100;
  CUtensorMap ta, tb;
  cudaError_t e = make_map(&ta, X, a.M, a.K, ldx, kGM, bf16);
  if (e == cudaSuccess) e = make_map(&tb, W, a.N, a.K, a.K, pair ? 128 : kGN, bf16);
  if (e != cudaSuccess) return e;
  if (bf16) {
    if (pair) {
      switch (epi) {
        case DIT_EPI_STORE: return launch_pair_t<DIT_EPI_STORE, 1>(ta, tb, a, nsm, st);
        case DIT_EPI_RESID: return launch_pair_t<DIT_EPI_RESID, 1>(ta, tb, a, nsm, st);
        default: return launch_pair_t<DIT_EPI_GLU, 1>(ta, tb, a, nsm, st);
      }
    }
    switch (epi) {
      case DIT_EPI_STORE: return launch_t<DIT_EPI_STORE, 1>(ta, tb, a, nsm, st);
      case DIT_EPI_RESID: return launch_t<DIT_EPI_RESID, 1>(ta, tb, a, nsm, st);
      default: return launch_t<DIT_EPI_GLU, 1>(ta, tb, a, nsm, st);
    }
  }
  if (pair) {
    switch (epi) {
      case DIT_EPI_STORE: return launch_pair_t<DIT_EPI_STORE, 0>(ta, tb, a, nsm, st);
      case DIT_EPI_TEMB: return launch_pair_t<DIT_EPI_TEMB, 0>(ta, tb, a, nsm, st);
      case DIT_EPI_ROPE: return launch_pair_t<DIT_EPI_ROPE, 0>(ta, tb, a, nsm, st);
      case DIT_EPI_RESID: return launch_pair_t<DIT_EPI_RESID, 0>(ta, tb, a, nsm, st);
      case DIT_EPI_GLU: return launch_pair_t<DIT_EPI_GLU, 0>(ta, tb, a, nsm, st);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (epi) {
    case DIT_EPI_STORE: return launch_t<DIT_EPI_STORE, 0>(ta, tb, a, nsm, st);
    case DIT_EPI_TEMB: return launch_t<DIT_EPI_TEMB, 0>(ta, tb, a, nsm, st);
    case DIT_EPI_ROPE: return launch_t<DIT_EPI_ROPE, 0>(ta, tb, a, nsm, st);
    case DIT_EPI_RESID: return launch_t<DIT_EPI_RESID, 0>(ta, tb, a, nsm, st);
    case DIT_EPI_GLU: return launch_t<DIT_EPI_GLU, 0>(ta, tb, a, nsm, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace m3
