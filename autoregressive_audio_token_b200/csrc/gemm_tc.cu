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
//   * the MMAs read both operands from shared memory in the canonical
//     K-major layout without swizzle: "core matrices" of 8 rows x 16 bytes
//     (128 contiguous bytes), K-adjacent core matrices 128 bytes apart (the
//     descriptor's leading byte offset), 8-row groups 1024 bytes apart (its
//     stride byte offset);
//   * a producer warp streams each stage with bulk copies (TMA) into a raw
//     4-stage ring: per 16-row tile of W its 4 K-tiles (contiguous in the
//     decode path's tiled layout, gemv_tile.cuh), per token its 64 inputs
//     (rows padded to 144 bytes so the reads below are free of bank
//     conflicts);
//   * four warps rewrite each raw stage into one of two canonical buffers:
//     one lane's 16 bytes of a W tile are four 4-byte (row, k-pair) words
//     that land in the same slot of four core matrices, so each warp store
//     is 128 contiguous bytes; int8 weights (stored q + 128) become bf16 q
//     exactly on the way (the row scale is applied in the epilogue,
//     y = s * sum q x, as the int8 definition states); out-of-range rows,
//     tokens and inputs become zeros.  They fence their generic-proxy writes
//     for the async proxy, synchronise, and one thread issues the MMAs and
//     commits them to the buffer's "empty" mbarrier;
//   * the epilogue reads the accumulator with tcgen05.ld (warp w owns lanes
//     32w..32w+31, one output row per thread) and applies the projection's
//     rounding: store bf16(y); residual x = bf16(x + bf16(y)); SwiGLU on the
//     interleaved (gate, up) row pairs.
// Every wait is bounded; a timeout records kErrTimeout, and the kernel still
// waits for its MMAs (bounded) and frees its tensor memory.
#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"
#include "gemv.cuh"
#include "launch.cuh"

namespace m3 {

namespace {

constexpr int kBM = 128;      // weight rows per CTA (MMA M, TMEM lanes)
constexpr int kBN = 128;      // tokens per CTA (MMA N, TMEM columns)
constexpr int kBK = 64;       // K per stage
constexpr int kMmaK = 16;     // K per tcgen05.mma (bf16)
constexpr int kRawStages = 4; // bulk-copy ring
constexpr int kCanon = 2;     // canonical buffers the MMAs read
constexpr int kConsumers = 128;             // warps 0-3: rewrite + epilogue
constexpr int kThreads = kConsumers + 32;   // + the producer warp
constexpr int kOpBytes = kBM * kBK * 2;     // one canonical operand: 16 KB
constexpr int kCanonBytes = 2 * kOpBytes;
constexpr int kXPitch = 144;                // raw token row: 128 bytes + 16 of padding
constexpr int kRawW = kBM * kBK * 2;        // raw W stage (bf16 size; int8 uses half)
constexpr int kRawBytes = kRawW + kBN * kXPitch;
constexpr int kCoreBytes = 128;             // 8 rows x 16 bytes
constexpr int kLBO = kCoreBytes;            // K-adjacent core matrices
constexpr int kSBO = (kBK / 8) * kCoreBytes;  // 8-row groups: 1024 bytes
constexpr int kBarBytes = 256;
constexpr size_t kSmemBytes =
    (size_t)kCanon * kCanonBytes + (size_t)kRawStages * kRawBytes + kBarBytes + 1024;
constexpr int kTmemCols = kBN;              // fp32 accumulator, one column per token
constexpr int kBarConsumers = 1;            // named barrier of the 128 consumer threads

static_assert(kBM == 128 && kBN % 16 == 0 && kBN >= 16 && kBN <= 256, "tcgen05 M=128 shape");
static_assert(kConsumers == kBM, "one epilogue thread per accumulator lane");
static_assert(kRawBytes % 128 == 0, "raw stages stay 128-byte aligned");
static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");

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

// A bounded wait (no early exit on other launches' error words: shared and
// tensor memory stay in use until this kernel's own copies and MMAs end).
__device__ __forceinline__ bool own_wait(uint64_t* bar, uint32_t parity, int* err) {
  for (long long i = 0; i < kSpinLimit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  record_error(err, kErrTimeout);
  return false;
}

// bf16 pair of two biased int8 bytes (q + 128), exact.
__device__ __forceinline__ uint32_t i8pair_to_bf16x2(uint32_t b0, uint32_t b1) {
  const __nv_bfloat162 h =
      __floats2bfloat162_rn((float)((int)b0 - 128), (float)((int)b1 - 128));
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Producer: stage kb of the raw ring by bulk copies, all completing on
// `full`.  W: per 16-row tile its (up to) 4 K-tiles, one copy; X: per token
// its inputs k0 .. k0 + 63 (fewer at the end of K), one copy.
template <int WF>
__device__ __forceinline__ void produce_stage(const GemmTcArgs& a, int m0, int n0, int kb,
                                              uint8_t* raw, uint64_t* full, int lane) {
  constexpr int TB = WF == WF_BF16 ? 512 : 256;  // bytes of one 16x16 tile
  const int Kt = a.K >> 4, rt_valid = (a.N + 15) >> 4;
  const int gkt0 = kb * (kBK / 16);
  const int nkt = Kt - gkt0 < 4 ? Kt - gkt0 : 4;
  const int nrt = rt_valid - (m0 >> 4) < 8 ? rt_valid - (m0 >> 4) : 8;
  const int ntok = a.T - n0 < kBN ? a.T - n0 : kBN;
  const uint32_t xbytes = (uint32_t)nkt * 32;   // 16 inputs of 2 bytes per K-tile
  const uint32_t bytes = (uint32_t)(nrt * nkt * TB) + (uint32_t)ntok * xbytes;
  if (lane == 0) mbar_arrive_expect_tx(full, bytes);
  __syncwarp();
  if (lane < nrt) {
    const int grt = (m0 >> 4) + lane;
    bulk_g2s_nohint(raw + lane * 4 * TB, a.w + ((size_t)grt * Kt + gkt0) * TB,
                    (uint32_t)(nkt * TB), full);
  }
  uint8_t* rx = raw + kRawW;
  for (int t = lane; t < ntok; t += 32)
    bulk_g2s_nohint(rx + t * kXPitch, a.x + (size_t)(n0 + t) * a.ldx + (size_t)kb * kBK, xbytes,
                    full);
}

// Consumers: raw stage -> canonical buffer (zeros outside the matrices).
template <int WF>
__device__ __forceinline__ void rewrite_stage(const GemmTcArgs& a, int m0, int n0, int kb,
                                              const uint8_t* raw, uint8_t* ca, int tid) {
  constexpr int TB = WF == WF_BF16 ? 512 : 256;
  const int warp = tid >> 5, lane = tid & 31;
  const int Kt = a.K >> 4, rt_valid = (a.N + 15) >> 4;
  const int gkt0 = kb * (kBK / 16);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int tl = warp * 8 + i;  // tile (rt, kt) of the 8 x 4 block
    const int rt = tl >> 2, kt = tl & 3;
    uint4 v = make_uint4(0, 0, 0, 0);
    if ((m0 >> 4) + rt < rt_valid && gkt0 + kt < Kt) {
      const uint8_t* src = raw + (rt * 4 + kt) * TB;
      if constexpr (WF == WF_BF16) {
        v = *reinterpret_cast<const uint4*>(src + lane * 16);
      } else {
        const uint2 q = *reinterpret_cast<const uint2*>(src + lane * 8);
        v.x = i8pair_to_bf16x2(q.x & 0xFF, (q.x >> 8) & 0xFF);
        v.y = i8pair_to_bf16x2((q.x >> 16) & 0xFF, q.x >> 24);
        v.z = i8pair_to_bf16x2(q.y & 0xFF, (q.y >> 8) & 0xFF);
        v.w = i8pair_to_bf16x2((q.y >> 16) & 0xFF, q.y >> 24);
      }
    }
    // fragment words: (row g, k 2t), (row g+8, k 2t), (row g, k 2t+8),
    // (row g+8, k 2t+8) with g = lane / 4, t = lane % 4 -> word `lane` of
    // core matrices (2rt, 2kt), (2rt+1, 2kt), (2rt, 2kt+1), (2rt+1, 2kt+1)
    uint8_t* d = ca + (2 * rt) * kSBO + (2 * kt) * kLBO + lane * 4;
    *reinterpret_cast<uint32_t*>(d) = v.x;
    *reinterpret_cast<uint32_t*>(d + kSBO) = v.y;
    *reinterpret_cast<uint32_t*>(d + kLBO) = v.z;
    *reinterpret_cast<uint32_t*>(d + kSBO + kLBO) = v.w;
  }
  const uint8_t* rx = raw + kRawW;
  uint8_t* cb = ca + kOpBytes;
  const int kin = a.K - kb * kBK;  // inputs of this stage (>= 16)
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    // chunk c = (token group c / 64, k group (c / 8) % 8, token c % 8) -> byte 16 c
    const int c = i * kConsumers + tid;
    const int t = (c >> 6) * 8 + (c & 7), kk = (c >> 3) & 7;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (n0 + t < a.T && kk * 8 < kin) v = *reinterpret_cast<const uint4*>(rx + t * kXPitch + kk * 16);
    *reinterpret_cast<uint4*>(cb + (size_t)c * 16) = v;
  }
}

template <int WF, int EPI>
__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(const GemmTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* canon = smem;                                   // [kCanon][A | B]
  uint8_t* raw = smem + kCanon * kCanonBytes;              // [kRawStages][W | X]
  uint64_t* full = reinterpret_cast<uint64_t*>(raw + kRawStages * kRawBytes);
  uint64_t* rempty = full + kRawStages;
  uint64_t* cempty = rempty + kRawStages;
  uint64_t* done = cempty + kCanon;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = blockIdx.x * kBN;  // tokens: fastest, so the CTAs of one W block share it in L2
  const int m0 = blockIdx.y * kBM;
  const int KB = (a.K + kBK - 1) / kBK;

  if (tid == 0) {
    for (int s = 0; s < kRawStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&rempty[s], 1);
    }
    for (int c = 0; c < kCanon; ++c) mbar_init(&cempty[c], 1);
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
  __syncthreads();  // the last barrier of all 160 threads
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kConsumers / 32) {  // producer warp
    bool ok = true;
    for (int kb = 0; kb < KB && ok; ++kb) {
      const int s = kb % kRawStages;
      if (kb >= kRawStages) ok = own_wait(&rempty[s], (uint32_t)((kb / kRawStages) - 1) & 1u, a.err);
      if (ok) produce_stage<WF>(a, m0, n0, kb, raw + (size_t)s * kRawBytes, &full[s], lane);
    }
    return;
  }

  bool ok = true;
  for (int kb = 0; kb < KB; ++kb) {
    const int s = kb % kRawStages, c = kb % kCanon;
    if (ok) ok = own_wait(&full[s], (uint32_t)(kb / kRawStages) & 1u, a.err);
    if (kb >= kCanon && ok) ok = own_wait(&cempty[c], (uint32_t)((kb / kCanon) - 1) & 1u, a.err);
    uint8_t* ca = canon + (size_t)c * kCanonBytes;
    rewrite_stage<WF>(a, m0, n0, kb, raw + (size_t)s * kRawBytes, ca, tid);
    fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor core
    named_bar_sync(kBarConsumers, kConsumers);
    if (tid == 0) {
      mbar_arrive(&rempty[s]);  // the raw stage is free for the producer
      tc_fence_after();
      const uint32_t a0 = smem_u32(ca), b0 = a0 + kOpBytes;
#pragma unroll
      for (int ks = 0; ks < kBK / kMmaK; ++ks)  // K = 16: two core matrices along K
        tc_mma(tmem, smem_desc(a0 + ks * 2 * kLBO), smem_desc(b0 + ks * 2 * kLBO),
               (kb > 0 || ks > 0) ? 1u : 0u);
      tc_commit(&cempty[c]);
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
  named_bar_sync(kBarConsumers, kConsumers);
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
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const dim3 grid((a.T + kBN - 1) / kBN, (a.N + kBM - 1) / kBM);
  kern<<<grid, kThreads, kSmemBytes, st>>>(a);
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
