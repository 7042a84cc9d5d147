// common.cuh -- small device helpers shared by the sm_100a kernels:
// mbarrier / bulk-copy (TMA) PTX wrappers, programmatic dependent launch,
// bounded waits that record an error word instead of trapping, and bf16
// unpacking.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace m3 {

// Device error words (first one wins; the host reads and clears them).
enum : int { kErrNone = 0, kErrTimeout = 1, kErrBounds = 2 };

// A bounded spin: 2^22 polls of try_wait (each may suspend for up to about
// a microsecond) is far beyond any healthy wait in these kernels, which only
// ever wait for their own bulk copies.
constexpr long long kSpinLimit = 1ll << 22;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void record_error(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

// ---------------------------------------------------------------- mbarrier --
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for phase `parity` of `bar` to complete; false (and an error word)
// if it does not within the spin limit.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* err) {
  for (long long i = 0; i < kSpinLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    // once any wait of the launch has given up, give up at once too, so a
    // failure ends the kernel in one spin limit rather than one per stage
    if ((i & 1023) == 1023 && err && *reinterpret_cast<volatile int*>(err) != 0) return false;
  }
  record_error(err, kErrTimeout);
  return false;
}

// ------------------------------------------------------ bulk copies (TMA) --
// L2 policy for data streamed once per frame (weights): evict first.
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Non-multicast bulk copy global -> this CTA's shared memory, completing
// `bytes` of transaction count on `bar`.  dst, src 16-byte aligned, bytes a
// multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Bulk prefetch of [src, src + bytes) into L2 (no shared memory, no
// completion); src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ void named_bar_arrive(int id, int nthreads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void bulk_g2s_nohint(void* dst, const void* src, uint32_t bytes,
                                                uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ------------------------------------------- programmatic dependent launch --
// Let the next kernel in the stream start (its pre-wait part only touches
// data that no kernel of this frame writes).
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// Wait until the previous kernel in the stream has completed and its
// writes are visible.  A no-op when launched without the PDL attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ------------------------------------------------------------- named barrier
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ----------------------------------------------------------------- numbers --
// Two packed bf16 -> two fp32 (exact).
__device__ __forceinline__ void bf16x2_to_f32(uint32_t w, float& lo, float& hi) {
  lo = __uint_as_float(w << 16);
  hi = __uint_as_float(w & 0xFFFF0000u);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t h) {
  return __uint_as_float(((uint32_t)h) << 16);
}

__device__ __forceinline__ float round_bf16(float v) {
  return __bfloat162float(__float2bfloat16_rn(v));
}

// Four int8 packed in w -> four exact fp32 values, via the 2^23 magic:
// float(0x4B000000 | (b ^ 0x80)) = 2^23 + 128 + q.
__device__ __forceinline__ void s8x4_to_f32(uint32_t w, float* f) {
  const uint32_t x = w ^ 0x80808080u;
  const float bias = 8388736.0f;  // 2^23 + 128
  f[0] = __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7650)) - bias;
  f[1] = __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7651)) - bias;
  f[2] = __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7652)) - bias;
  f[3] = __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7653)) - bias;
}

// ------------------------------------------- packed fp32 pairs (sm_100a) ---
// Two fp32 values in one 64-bit register pair, for the packed f32x2 FMA/ADD
// of sm_100 (one instruction for two lanes of arithmetic).
__device__ __forceinline__ uint64_t pack_u32x2(uint32_t lo, uint32_t hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
  return r;
}

__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
  return pack_u32x2(__float_as_uint(lo), __float_as_uint(hi));
}

__device__ __forceinline__ float2 unpack_f32x2(uint64_t v) {
  uint32_t lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(v));
  return make_float2(__uint_as_float(lo), __uint_as_float(hi));
}

// acc = a * b + acc, elementwise on (lo, hi), each with one rounding.
__device__ __forceinline__ void ffma2(uint64_t& acc, uint64_t a, uint64_t b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}

__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// (bf16 lo, bf16 hi) packed -> the exact fp32 pair
__device__ __forceinline__ uint64_t bf16x2_to_f32x2(uint32_t w) {
  return pack_u32x2(w << 16, w & 0xFFFF0000u);
}

// fp32 pair -> (bf16 lo, bf16 hi) packed, each rounded to nearest even
__device__ __forceinline__ uint32_t f32x2_to_bf16x2(uint64_t v) {
  const float2 f = unpack_f32x2(v);
  const __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);
  return *reinterpret_cast<const uint32_t*>(&b);
}

__device__ __forceinline__ void fadd2(uint64_t& acc, uint64_t b) {
  asm("add.rn.f32x2 %0, %0, %1;" : "+l"(acc) : "l"(b));
}

// Four int8 packed in w -> two exact fp32 pairs (q0, q1), (q2, q3), via the
// 2^23 magic: float(0x4B000000 | (b ^ 0x80)) = 2^23 + 128 + q.
__device__ __forceinline__ void s8x4_to_f32x2(uint32_t w, uint64_t& f01, uint64_t& f23) {
  const uint32_t x = w ^ 0x80808080u;
  const uint64_t nb = pack_f32x2(-8388736.0f, -8388736.0f);  // -(2^23 + 128)
  f01 = pack_u32x2(__byte_perm(x, 0x4B000000u, 0x7650), __byte_perm(x, 0x4B000000u, 0x7651));
  f23 = pack_u32x2(__byte_perm(x, 0x4B000000u, 0x7652), __byte_perm(x, 0x4B000000u, 0x7653));
  fadd2(f01, nb);
  fadd2(f23, nb);
}

// Element offset of (head slot hs, page-local position off, dim d) in a KV
// page laid out [2 * Hkv head slots][page_size][D]: the 16-byte chunk index
// of d is XOR-ed with (off & 7), so that eight consecutive positions' chunk c
// fall in eight different shared-memory bank groups once a tile is copied
// linearly into shared memory (conflict-free ldmatrix).
__host__ __device__ __forceinline__ size_t kv_elem_offset(int hs, int page_size, int off, int D,
                                                         int d) {
  return ((size_t)hs * page_size + off) * D + ((((d >> 3) ^ (off & 7))) << 3) + (d & 7);
}

}  // namespace m3
