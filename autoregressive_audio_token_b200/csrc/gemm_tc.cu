// gemm_tc.cu -- the prompt prefill's projections as GEMMs on the
// 5th-generation tensor cores (tcgen05, accumulators in tensor memory).
//
// The first stage of the DiffSynth-Studio article on MiniMax-Music3 runs the
// prompt (about 300 tokens per CFG row, at most 5000) through the same
// Qwen3-style body before the first frame.  With T tokens at once every
// projection is a dense contraction Y[t][o] = sum_k W[o][k] X[t][k], so here
// it is a tensor-core GEMM rather than the decode path's GEMV:
//   * A = a 128-row block of W (the MMA's M = 128 accumulator lanes),
//     B = 128 tokens of X (N = 128 fp32 columns of tensor memory), K in
//     stages of 64, four tcgen05.mma of K = 16 per stage;
//   * both operands sit in shared memory in the canonical K-major layout
//     without swizzle: "core matrices" of 8 rows x 16 bytes (128 contiguous
//     bytes), K-adjacent core matrices 128 bytes apart (the descriptor's
//     leading byte offset), 8-row groups 1024 bytes apart (its stride byte
//     offset);
//   * W stays in the decode path's tiled fragment layout (gemv_tile.cuh):
//     one lane's 16 bytes of a 16x16 tile are four 4-byte pairs that land in
//     the same (row, word) slot of four core matrices, so a warp stores each
//     core matrix as 128 contiguous bytes.  int8 weights (stored q + 128)
//     become bf16 q exactly on the way in; the row scale is applied in the
//     epilogue, y = s * sum q x, as the int8 definition states;
//   * bf16: a 6-stage ring filled by cp.async (4-byte copies of W straight
//     into their core-matrix slots, 16-byte copies of X), five stages in
//     flight; int8: a 4-stage ring staged through registers (the bytes are
//     converted on the way).  Every thread fences its generic-proxy writes for
//     the async proxy before the CTA barrier; one thread then issues the
//     MMAs and commits them to the stage's "empty" mbarrier;
//   * the epilogue reads the accumulator with tcgen05.ld (warp w owns lanes
//     32w..32w+31, one output row per thread) and applies the projection's
//     rounding: store bf16(y); residual x = bf16(x + bf16(y)); SwiGLU on the
//     interleaved (gate, up) row pairs.
// Every wait is bounded; a timeout records kErrTimeout and the kernel still
// frees its tensor memory.
#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"
#include "gemv.cuh"
#include "launch.cuh"

namespace m3 {

namespace {

constexpr int kBM = 128;     // weight rows per CTA (MMA M, TMEM lanes)
constexpr int kBN = 128;     // tokens per CTA (MMA N, TMEM columns)
constexpr int kBK = 64;      // K per stage
constexpr int kMmaK = 16;    // K per tcgen05.mma (bf16)
constexpr int kStagesBF16 = 6;   // cp.async ring: 5 stages of loads in flight
constexpr int kStagesI8 = 4;     // register-staged ring (the int8 -> bf16 conversion)
constexpr int kThreads = 128;
constexpr int kOpBytes = kBM * kBK * 2;          // one operand of one stage: 16 KB
constexpr int kStageBytes = 2 * kOpBytes;
constexpr int kCoreBytes = 128;                  // 8 rows x 16 bytes
constexpr int kLBO = kCoreBytes;                 // K-adjacent core matrices
constexpr int kSBO = (kBK / 8) * kCoreBytes;     // 8-row groups: 1024 bytes
constexpr size_t smem_bytes(int stages) { return (size_t)stages * kStageBytes + 1024 + 256; }
constexpr int kTmemCols = kBN;                   // fp32 accumulator, one column per token

static_assert(kBM == 128 && kBN % 16 == 0 && kBN >= 16 && kBN <= 256, "tcgen05 M=128 shape");
static_assert(kThreads == kBM, "one epilogue thread per accumulator lane");

// Instruction descriptor of kind::f16: D fp32 (bits 4-5 = 1), A and B bf16
// (bits 7-9, 10-12 = 1), both K-major (bits 15, 16 = 0), N >> 3 at bit 17,
// M >> 4 at bit 24.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kBN >> 3) << 17) |
                            ((uint32_t)(kBM >> 4) << 24);

// Shared-memory matrix descriptor: start address >> 4 (bits 0-13), leading
// byte offset >> 4 (16-29), stride byte offset >> 4 (32-45), descriptor
// version 1 (bits 46-47), no swizzle (bits 61-63 = 0).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)(kLBO >> 4) << 16) |
         ((uint64_t)(kSBO >> 4) << 32) | (1ull << 46);
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
      ::"r"(tmem_d), "l"(a), "l"(b), "r"(kIdesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u),
        "r"(0u)
      : "memory");
}

// Arrive on `bar` once every tcgen05.mma this thread issued has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// A bounded wait on the kernel's own MMAs (no early exit on other launches'
// error words: tensor memory and shared memory stay in use until they end).
__device__ __forceinline__ bool own_wait(uint64_t* bar, uint32_t parity, int* err) {
  for (long long i = 0; i < kSpinLimit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  record_error(err, kErrTimeout);
  return false;
}

__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, bool ok) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src),
               "r"(ok ? 4 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool ok) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(ok ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// One bf16 stage by cp.async: each lane's 16-byte fragment of a W tile as
// four 4-byte copies into its four core matrices; X as in store_stage.  An
// operand outside the matrix copies zero bytes (the slot is zero-filled).
__device__ __forceinline__ void issue_stage_bf16(const GemmTcArgs& a, int m0, int n0, int k0,
                                                 uint32_t sa, uint32_t sb) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Kt = a.K >> 4, rt_valid = (a.N + 15) >> 4;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int tl = warp * 8 + i;
    const int rt = tl >> 2, kt = tl & 3;
    const int grt = (m0 >> 4) + rt, gkt = (k0 >> 4) + kt;
    const bool ok = grt < rt_valid && gkt < Kt;
    const uint8_t* src = ok ? a.w + ((size_t)grt * Kt + gkt) * 512 + lane * 16 : a.w;
    const uint32_t d = sa + (2 * rt) * kSBO + (2 * kt) * kLBO + lane * 4;
    cp_async4(d, src, ok);
    cp_async4(d + kSBO, ok ? src + 4 : src, ok);
    cp_async4(d + kLBO, ok ? src + 8 : src, ok);
    cp_async4(d + kSBO + kLBO, ok ? src + 12 : src, ok);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int c = i * kThreads + tid;
    const int tok = n0 + (c >> 6) * 8 + (c & 7);
    const int k = k0 + ((c >> 3) & 7) * 8;
    const bool ok = tok < a.T && k < a.K;
    cp_async16(sb + (uint32_t)c * 16, ok ? a.x + (size_t)tok * a.ldx + k : a.x, ok);
  }
}

// bf16 pair of two biased int8 bytes (q + 128), exact.
__device__ __forceinline__ uint32_t i8pair_to_bf16x2(uint32_t b0, uint32_t b1) {
  const __nv_bfloat162 h =
      __floats2bfloat162_rn((float)((int)b0 - 128), (float)((int)b1 - 128));
  return *reinterpret_cast<const uint32_t*>(&h);
}

// One stage's operands in registers: 8 fragment tiles of W per warp (one
// 16-byte fragment per lane each) and 8 16-byte chunks of X per thread.
struct StageRegs {
  uint4 w[8];
  uint4 x[8];
};

template <int WF>
__device__ __forceinline__ void load_stage(const GemmTcArgs& a, int m0, int n0, int k0,
                                           StageRegs& R) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Kt = a.K >> 4;                   // 16-wide K tiles per row tile
  const int rt_valid = (a.N + 15) >> 4;      // stored row tiles
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int tl = warp * 8 + i;             // tile of the 8 x 4 block: (rt, kt)
    const int rt = tl >> 2, kt = tl & 3;
    const int grt = (m0 >> 4) + rt, gkt = (k0 >> 4) + kt;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (grt < rt_valid && gkt < Kt) {
      const size_t tile = (size_t)grt * Kt + gkt;
      if constexpr (WF == WF_BF16) {
        v = __ldg(reinterpret_cast<const uint4*>(a.w + tile * 512) + lane);
      } else {
        const uint2 q = __ldg(reinterpret_cast<const uint2*>(a.w + tile * 256) + lane);
        v.x = i8pair_to_bf16x2(q.x & 0xFF, (q.x >> 8) & 0xFF);
        v.y = i8pair_to_bf16x2((q.x >> 16) & 0xFF, q.x >> 24);
        v.z = i8pair_to_bf16x2(q.y & 0xFF, (q.y >> 8) & 0xFF);
        v.w = i8pair_to_bf16x2((q.y >> 16) & 0xFF, q.y >> 24);
      }
    }
    R.w[i] = v;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int c = i * kThreads + tid;        // chunk = (token group, k group, token in group)
    const int tok = n0 + (c >> 6) * 8 + (c & 7);
    const int k = k0 + ((c >> 3) & 7) * 8;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (tok < a.T && k < a.K)
      v = __ldg(reinterpret_cast<const uint4*>(a.x + (size_t)tok * a.ldx + k));
    R.x[i] = v;
  }
}

__device__ __forceinline__ void store_stage(uint8_t* sa, uint8_t* sb, const StageRegs& R) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int tl = warp * 8 + i;
    const int rt = tl >> 2, kt = tl & 3;
    // fragment words: (row g, k 2t), (row g+8, k 2t), (row g, k 2t+8),
    // (row g+8, k 2t+8) with g = lane / 4, t = lane % 4 -> word `lane` of
    // core matrices (2rt, 2kt), (2rt+1, 2kt), (2rt, 2kt+1), (2rt+1, 2kt+1)
    uint8_t* base = sa + (2 * rt) * kSBO + (2 * kt) * kLBO + lane * 4;
    *reinterpret_cast<uint32_t*>(base) = R.w[i].x;
    *reinterpret_cast<uint32_t*>(base + kSBO) = R.w[i].y;
    *reinterpret_cast<uint32_t*>(base + kLBO) = R.w[i].z;
    *reinterpret_cast<uint32_t*>(base + kSBO + kLBO) = R.w[i].w;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int c = i * kThreads + tid;
    // (token group c / 64, k group (c / 8) % 8, token c % 8) -> byte 16 c
    *reinterpret_cast<uint4*>(sb + (size_t)c * 16) = R.x[i];
  }
}

template <int WF, int EPI>
__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(const GemmTcArgs a) {
  constexpr int S = WF == WF_BF16 ? kStagesBF16 : kStagesI8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* ops = smem;                                             // [stage][A | B]
  uint64_t* empty = reinterpret_cast<uint64_t*>(smem + S * kStageBytes);
  uint64_t* done = empty + S;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = blockIdx.x * kBN;  // tokens: fastest, so the CTAs of one W block share it in L2
  const int m0 = blockIdx.y * kBM;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) mbar_init(&empty[s], 1);
    mbar_init(done, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
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

  const int KB = (a.K + kBK - 1) / kBK;
  auto issue_mma = [&](int kb) {
    const int s = kb % S;
    tc_fence_after();
    const uint32_t a0 = smem_u32(ops + (size_t)s * kStageBytes), b0 = a0 + kOpBytes;
#pragma unroll
    for (int ks = 0; ks < kBK / kMmaK; ++ks)  // K = 16: two core matrices along K
      tc_mma(tmem, smem_desc(a0 + ks * 2 * kLBO), smem_desc(b0 + ks * 2 * kLBO),
             (kb > 0 || ks > 0) ? 1u : 0u);
    tc_commit(&empty[s]);
  };
  if constexpr (WF == WF_BF16) {
    const uint32_t ops0 = smem_u32(ops);
#pragma unroll 1
    for (int s = 0; s < S - 1; ++s) {
      if (s < KB) issue_stage_bf16(a, m0, n0, s * kBK, ops0 + s * kStageBytes,
                                   ops0 + s * kStageBytes + kOpBytes);
      cp_async_commit();
    }
    bool ok = true;
#pragma unroll 1
    for (int kb = 0; kb < KB; ++kb) {
      cp_async_wait<S - 2>();    // this thread's copies of stage kb have landed
      fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor core
      __syncthreads();
      if (tid == 0) issue_mma(kb);
      const int nk = kb + S - 1;  // refill the slot the MMAs of kb - 1 read
      if (nk < KB) {
        const int s = nk % S;
        if (kb >= 1 && ok) ok = own_wait(&empty[s], (uint32_t)((kb - 1) / S) & 1u, a.err);
        issue_stage_bf16(a, m0, n0, nk * kBK, ops0 + s * kStageBytes,
                         ops0 + s * kStageBytes + kOpBytes);
      }
      cp_async_commit();
    }
  } else {
    StageRegs R;
    load_stage<WF>(a, m0, n0, 0, R);
    bool ok = true;
#pragma unroll 1
    for (int kb = 0; kb < KB; ++kb) {
      const int s = kb % S;
      uint8_t* sa = ops + (size_t)s * kStageBytes;
      uint8_t* sb = sa + kOpBytes;
      if (kb >= S && ok) ok = own_wait(&empty[s], (uint32_t)((kb / S) - 1) & 1u, a.err);
      store_stage(sa, sb, R);
      fence_proxy_async_smem();  // generic-proxy stores -> visible to the tensor core
      __syncthreads();
      if (kb + 1 < KB) load_stage<WF>(a, m0, n0, (kb + 1) * kBK, R);
      if (tid == 0) issue_mma(kb);
    }
  }
  if (tid == 0) tc_commit(done);
  own_wait(done, 0, a.err);
  tc_fence_after();

  // epilogue: thread = accumulator lane = output row o
  const int o = m0 + warp * 32 + lane;
  const bool row_ok = o < a.N;
  float sc = 1.0f;
  if constexpr (WF != WF_BF16) sc = row_ok ? __ldg(a.scales + o) : 0.0f;
  const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
  for (int c0 = 0; c0 < kBN; c0 += 16) {
    float v[16];
    tmem_ld16(trow + (uint32_t)c0, v);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int t = n0 + c0 + j;
      const float y = v[j] * sc;
      if constexpr (EPI == EPI_SWIGLU) {
        const float yu = __shfl_xor_sync(0xffffffffu, y, 1);  // the up row beside each gate row
        if (t < a.T && row_ok && !(o & 1)) {
          const float gb = round_bf16(y), ub = round_bf16(yu);
          a.out[(size_t)t * a.ldo + (o >> 1)] =
              __float2bfloat16_rn(round_bf16(silu_f(gb)) * ub);
        }
      } else if (t < a.T && row_ok) {
        __nv_bfloat16* p = a.out + (size_t)t * a.ldo + o;
        if constexpr (EPI == EPI_RESID)
          *p = __float2bfloat16_rn(__bfloat162float(*p) + round_bf16(y));
        else
          *p = __float2bfloat16_rn(y);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

template <int WF, int EPI>
cudaError_t launch_gemm_tc_t(const GemmTcArgs& a, cudaStream_t st) {
  auto kern = gemm_tc_kernel<WF, EPI>;
  const size_t smem = smem_bytes(WF == WF_BF16 ? kStagesBF16 : kStagesI8);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((a.T + kBN - 1) / kBN, (a.N + kBM - 1) / kBM);
  kern<<<grid, kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_tc(const GemmTcArgs& a, int wf, int epi, cudaStream_t st) {
  // the operand loads need 16-byte rows of X and whole 16-wide weight tiles
  if (!a.w || !a.x || !a.out || a.T < 1 || a.N < 1 || a.K < 16 || a.K % 16 || a.ldx % 8 ||
      a.ldx < a.K || (epi == EPI_SWIGLU && a.N % 2) ||
      (reinterpret_cast<uintptr_t>(a.x) & 15) || (reinterpret_cast<uintptr_t>(a.w) & 15) ||
      a.ldo < (epi == EPI_SWIGLU ? a.N / 2 : a.N) || (wf != WF_BF16 && !a.scales))
    return cudaErrorInvalidValue;
  if (wf == WF_BF16) {
    if (epi == EPI_STORE) return launch_gemm_tc_t<WF_BF16, EPI_STORE>(a, st);
    if (epi == EPI_RESID) return launch_gemm_tc_t<WF_BF16, EPI_RESID>(a, st);
    if (epi == EPI_SWIGLU) return launch_gemm_tc_t<WF_BF16, EPI_SWIGLU>(a, st);
  } else if (wf == WF_I8ROW) {
    if (epi == EPI_STORE) return launch_gemm_tc_t<WF_I8ROW, EPI_STORE>(a, st);
    if (epi == EPI_RESID) return launch_gemm_tc_t<WF_I8ROW, EPI_RESID>(a, st);
    if (epi == EPI_SWIGLU) return launch_gemm_tc_t<WF_I8ROW, EPI_SWIGLU>(a, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace m3
