// gemv_tile.cuh -- the decode step's weight-streaming GEMV on tensor-core
// fragments (1..16 activation rows, bf16 or int8 weights with a row scale):
// weight layout, launch plan, shared device routines, and the statically
// partitioned kernel (cluster K split; used for the lm_head sampler and for
// more than 8 rows).  gemv_dyn.cuh holds the dynamically scheduled kernel
// that the body projections use.
//
// The AR stage reads every weight once per frame and is HBM bound ("MiniMax
// Music 3 modular pipeline", finding 4).  A CUDA-core GEMV spends about two
// instructions per weight, which leaves no issue slack to absorb the
// dependency bubble at each kernel boundary.  Here the dot products are
// m16n8k16 MMAs with a tile of 16 weight rows x 16 inputs as the A operand
// and the activations as the 8-column B operand (columns beyond the batch
// are zero registers), so one instruction retires 256 weights x up to 8
// rows:
//   * weights are stored tiled: 16 rows x 16 inputs per tile in the exact
//     per-lane order of the A fragment (each lane reads its 16 bytes of a
//     bf16 tile, or 8 of an int8 tile, with one conflict-free load); the
//     tiles of one 16-row unit are contiguous along K;
//   * a producer warp streams tiles through a ring of shared-memory stages
//     with non-multicast bulk copies (TMA engine, mbarrier transaction
//     counts, L2 evict-first), starting before the previous kernel ends
//     (programmatic dependent launch: weights do not depend on it);
//   * 8 consumer warps split each stage's tiles and hold the (normalised)
//     activations in shared memory in B-fragment order;
//   * epilogues: store, residual add, SwiGLU on interleaved gate/up rows,
//     the fused lm_head sampler (fp32 logits, CFG, Gumbel noise, argmax).
// int8 weights run as f16 MMAs: an int8 value is exact in f16 (a two-op
// conversion), and the activation row is scaled by a power of two so its
// largest magnitude stays inside the f16 range (bf16 values keep all their
// bits there); the scale is undone in fp32 in the epilogue.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"
#include "gemv.cuh"
#include "noise.cuh"

namespace m3 {

constexpr int kTW = 8;                     // consumer warps
constexpr int kTThreads = (kTW + 1) * 32;  // + producer warp
constexpr int kTMiscBytes = 1024;          // per-row scalars + argmax keys
constexpr int kTMaxSlots = 16;             // ring slots, at most
constexpr int kUnitRows = 16;              // weight rows per unit (one A tile high)

// ---------------------------------------------------------------- layout --
// Byte offset of weight element (n, k) in the tiled matrix of K inputs.
// Tile (n / 16, k / 16); lane l = 4 g + t of the A fragment holds
//   a0 = (row g, inputs 2t, 2t+1)     a1 = (row g+8, inputs 2t, 2t+1)
//   a2 = (row g, inputs 2t+8, 2t+9)   a3 = (row g+8, inputs 2t+8, 2t+9)
// stored consecutively (16 bytes bf16, 8 bytes int8).
__host__ __device__ __forceinline__ size_t tile_byte_offset(int n, int k, int K, int esz) {
  const int r = n & 15, kk = k & 15;
  const int g = r & 7, hr = r >> 3;
  const int t = (kk & 7) >> 1, hk = kk >> 3, e = kk & 1;
  const size_t tile = (size_t)(n >> 4) * (size_t)(K >> 4) + (size_t)(k >> 4);
  return tile * (size_t)(256 * esz) + (size_t)((g * 4 + t) * 8 * esz) +
         (size_t)((hr + 2 * hk) * 2 * esz) + (size_t)(e * esz);
}

// The static kernel's partition, derived identically on host and device.
// A cluster of C CTAs owns a contiguous range of units; each CTA streams,
// for each unit, its K slice (a "run" of Tr tiles) in ppr parts of at most
// pt tiles; a part is one ring stage, the ring holds `slots` stages.
struct TilePlan {
  int U, T, C, Tr, TB, runb, ppr, pt, stage, slots, nu_max;
};

__host__ __device__ __forceinline__ TilePlan tile_plan(int N, int K, int esz, int C, int ncl,
                                                       int sb, int ring_bytes) {
  TilePlan p;
  p.U = (N + kUnitRows - 1) / kUnitRows;
  p.T = K >> 4;
  p.C = C;
  p.Tr = p.T / C;
  p.TB = 256 * esz;
  p.runb = p.Tr * p.TB;
  p.ppr = (p.runb + sb - 1) / sb;
  p.pt = (p.Tr + p.ppr - 1) / p.ppr;
  p.stage = p.pt * p.TB;
  p.slots = ring_bytes / p.stage;
  if (p.slots > kTMaxSlots) p.slots = kTMaxSlots;
  p.nu_max = (p.U + ncl - 1) / ncl;
  return p;
}

// Dynamic shared memory of one static-kernel CTA (host and device agree).
__host__ __device__ __forceinline__ size_t tile_smem_bytes(const TilePlan& p, int mr) {
  return (size_t)p.slots * p.stage + 2 * kTMaxSlots * sizeof(uint64_t) + kTMiscBytes +
         (size_t)p.Tr * mr * 32 +                                 // activations, B-fragment order
         (size_t)2 * kTW * mr * kUnitRows * sizeof(float) +       // per-warp partials, 2 buffers
         (size_t)p.nu_max * mr * kUnitRows * sizeof(float);       // the CTA's unit sums
}

// ------------------------------------------------------------------ MMAs --
__device__ __forceinline__ void mma_bf16(float* c, uint4 a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16(float* c, uint4 a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b0), "r"(b1));
}

// int8 weights of the tiled GEMVs are stored biased, byte = q + 128 (q ^ 0x80).
// Under the f16 exponent pattern 0x64 a byte b reads as 1024 + b = 1152 + q,
// exact, so four weights become two f16 pairs in two byte permutes; the
// 1152 is taken out again by a second MMA with every A entry -1152, so the
// accumulator holds sum (1152 + q) x - 1152 x = sum q x.
__device__ __forceinline__ void u8x4_to_f16x2_biased(uint32_t w, uint32_t& b0, uint32_t& b1) {
  b0 = __byte_perm(w, 0x64646464u, 0x5140);  // bytes b0, b1 under 0x64
  b1 = __byte_perm(w, 0x64646464u, 0x7362);  // bytes b2, b3 under 0x64
}

// One lane's A fragment of a weight tile in shared memory (int8: 1152 + q).
// Items (16 inputs of one row) a thread stages per batch when there is no
// norm: 8 for bf16; 4 for int8, whose conversion needs more registers (8
// measured slower)
template <int WF>
constexpr int kStageItems = WF == WF_I8ROW ? 4 : 8;

template <int WF>
__device__ __forceinline__ uint4 load_afrag(const uint8_t* p) {
  if constexpr (WF == WF_BF16) {
    return *reinterpret_cast<const uint4*>(p);
  } else {
    const uint2 q = *reinterpret_cast<const uint2*>(p);
    uint4 a;
    u8x4_to_f16x2_biased(q.x, a.x, a.y);
    u8x4_to_f16x2_biased(q.y, a.z, a.w);
    return a;
  }
}

template <int WF>
__device__ __forceinline__ void mma_w(float* c, uint4 a, uint2 b) {
  if constexpr (WF == WF_BF16) {
    mma_bf16(c, a, b.x, b.y);
  } else {
    constexpr uint32_t kMinus1152 = 0xE480E480u;  // f16 pair (-1152, -1152)
    mma_f16(c, a, b.x, b.y);
    mma_f16(c, make_uint4(kMinus1152, kMinus1152, kMinus1152, kMinus1152), b.x, b.y);
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  const __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// C fragment of lane (g, t) -> per-warp partial buffer [m][16]:
// c0 = (weight row g, batch row 2t), c1 = (g, 2t+1), c2 = (g+8, 2t),
// c3 = (g+8, 2t+1); batch rows from m0 on, below mr only.
__device__ __forceinline__ void put_cfrag(float* pb, const float* c, int lane, int m0, int mr) {
  const int g = lane >> 2, m = m0 + 2 * (lane & 3);
  if (m < mr) {
    pb[m * kUnitRows + g] = c[0];
    pb[m * kUnitRows + g + 8] = c[2];
  }
  if (m + 1 < mr) {
    pb[(m + 1) * kUnitRows + g] = c[1];
    pb[(m + 1) * kUnitRows + g + 8] = c[3];
  }
}

// ------------------------------------------------------------ activations --
// 16 consecutive bf16 at p (16-byte aligned) -> fp32.
__device__ __forceinline__ void load16(const __nv_bfloat16* p, uint4& lo, uint4& hi) {
  lo = *reinterpret_cast<const uint4*>(p);
  hi = *reinterpret_cast<const uint4*>(p + 8);
}
__device__ __forceinline__ void unpack16(const uint4& lo, const uint4& hi, float* v) {
  const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) bf16x2_to_f32(w[i], v[2 * i], v[2 * i + 1]);
}

// Per-row reduction of vals[m * n + j] over j < n (sum or max) by warps in a
// fixed order (lane-strided, then a shuffle tree); lane 0 of warp m stores
// f(result).  Deterministic for a given n.
template <bool MAX, typename F>
__device__ __forceinline__ void rows_reduce(const float* vals, int n, int mr, int warp, int nwarps,
                                            int lane, F store) {
  for (int m = warp; m < mr; m += nwarps) {
    float s = 0.0f;
#pragma unroll 8
    for (int j = lane; j < n; j += 32) s = MAX ? fmaxf(s, vals[m * n + j]) : s + vals[m * n + j];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float y = __shfl_xor_sync(0xffffffffu, s, o);
      s = MAX ? fmaxf(s, y) : s + y;
    }
    if (lane == 0) store(m, s);
  }
}

// The consumer threads' setup of one launch (nt threads, named barrier 1),
// which also waits for the previous kernel (after fetching static gains):
// RMSNorm statistics over the whole K (when a.gamma) and the activations of
// tiles [kt0, kt0 + Tr) in B-fragment order, xs[j][m][t] = {(k, k+1),
// (k+8, k+9)} with k = 16 (kt0 + j) + 2t, normalised as
// out = bf16(gamma * bf16(x / rms)).
// The sum of squares comes from a.ssq_in when the previous kernel left
// per-unit partials there ([mr][a.ssq_n], summed here in a fixed order),
// else from a pass over x.  Each thread holds up to NB items (16 inputs of
// one row) in registers, so with the partials the setup is one round trip
// to L2.  `sq` is scratch of T * mr floats that may alias xs.
// int8 weights take f16 activations scaled by 2^-e per row, e >= 0 the
// smallest exponent that keeps the largest staged magnitude of the row below
// 2^15 (rpow[m] = 2^e undoes it on the sums; the CTAs of a cluster stage
// different K ranges, so each scales its own partial sums).  Every row is staged at scale 1
// first; magnitudes >= 2^15 (normally none) are recorded, and only then are
// the exponents set and the rows staged again.  rpow + 16 holds 17 words of
// scratch (row maxima, an any-row flag).
template <int WF, int NB, bool GAMMA>
__device__ __forceinline__ void stage_activations(const GemvArgs& a, int mr, int kt0, int Tr,
                                                  float* rinv, float* rpow, float* sq, uint2* xs,
                                                  __nv_bfloat16* h_out, int tid, int nt) {
  const int K = a.K, T = K >> 4;
  const int warp = tid >> 5, lane = tid & 31, nwarps = nt >> 5;
  const __nv_bfloat16* __restrict__ x = a.x;
  const __nv_bfloat16* __restrict__ gm = GAMMA ? a.gamma : nullptr;
  const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
  unsigned* big = reinterpret_cast<unsigned*>(rpow + 16);  // [16] maxima >= 2^15, [16] flag
  auto set_rinv = [&](int m, float s) { rinv[m] = 1.0f / sqrtf(s / (float)K + a.eps); };
  auto normalise = [&](int m, const uint4& xl, const uint4& xh, const uint4& gl, const uint4& gh,
                       float* v) {
    unpack16(xl, xh, v);
    if (gm) {
      float g[16];
      unpack16(gl, gh, g);
      const float r = rinv[m];
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = round_bf16(g[i] * round_bf16(v[i] * r));
    }
  };
  // the gains are static: their first batch is fetched (from HBM, the
  // slowest load here) before waiting for the previous kernel
  uint4 xl[NB], xh[NB], gl[NB], gh[NB];
  auto load_gamma = [&](int i0) {
#pragma unroll
    for (int q = 0; q < NB; ++q) {
      const int i = i0 + q * nt;
      gl[q] = gh[q] = z4;
      if (gm && i < Tr * mr) load16(gm + 16 * (kt0 + i / mr), gl[q], gh[q]);
    }
  };
  if (WF == WF_I8ROW && tid < 17) {
    big[tid] = 0u;
    if (tid < 16) rpow[tid] = 1.0f;
  }
  load_gamma(tid);
  pdl_wait();  // the activations come from the previous kernel
  if constexpr (WF == WF_I8ROW) named_bar_sync(1, nt);  // the scratch words are zero
  const bool have_ss = gm && a.ssq_in;
  if (gm && !have_ss) {  // sum of squares per (row, 16 inputs), then per row
    for (int i0 = tid; i0 < T * mr; i0 += NB * nt) {
      uint4 xl[NB], xh[NB];
#pragma unroll
      for (int q = 0; q < NB; ++q) {
        const int i = i0 + q * nt;
        xl[q] = xh[q] = z4;
        if (i < T * mr) load16(x + (size_t)(i / T) * a.ldx + 16 * (i % T), xl[q], xh[q]);
      }
#pragma unroll
      for (int q = 0; q < NB; ++q) {
        const int i = i0 + q * nt;
        if (i >= T * mr) continue;
        float v[16];
        unpack16(xl[q], xh[q], v);
        float s = 0.0f;
#pragma unroll
        for (int e = 0; e < 16; ++e) s = fmaf(v[e], v[e], s);
        sq[i] = s;
      }
    }
    named_bar_sync(1, nt);
    rows_reduce<false>(sq, T, mr, warp, nwarps, lane, set_rinv);
    named_bar_sync(1, nt);
  }
  // the slice in B-fragment order, NB items per thread per batch; item i is
  // (tile jj = i / mr, row m = i % mr), so a warp's stores are 32-byte
  // steps and its loads 32-byte sectors
  auto load_x = [&](int i0) {
#pragma unroll
    for (int q = 0; q < NB; ++q) {
      const int i = i0 + q * nt;
      xl[q] = xh[q] = z4;
      if (i < Tr * mr) load16(x + (size_t)(i % mr) * a.ldx + 16 * (kt0 + i / mr), xl[q], xh[q]);
    }
  };
  // first: the first pass (int8 at scale 1, recording large magnitudes)
  auto store_batch = [&](int i0, bool first) {
#pragma unroll
    for (int q = 0; q < NB; ++q) {
      const int i = i0 + q * nt;
      if (i >= Tr * mr) continue;
      const int m = i % mr, jj = i / mr;
      // w[p] = inputs (2p, 2p+1) of the item, p < 8
      uint32_t w[8] = {xl[q].x, xl[q].y, xl[q].z, xl[q].w, xh[q].x, xh[q].y, xh[q].z, xh[q].w};
      if constexpr (WF == WF_BF16) {
        if (gm) {
          const uint32_t gw[8] = {gl[q].x, gl[q].y, gl[q].z, gl[q].w,
                                  gh[q].x, gh[q].y, gh[q].z, gh[q].w};
          const uint64_t r2 = pack_f32x2(rinv[m], rinv[m]);
#pragma unroll
          for (int p = 0; p < 8; ++p) {
            const uint32_t t1 = f32x2_to_bf16x2(fmul2(bf16x2_to_f32x2(w[p]), r2));
            w[p] = f32x2_to_bf16x2(fmul2(bf16x2_to_f32x2(gw[p]), bf16x2_to_f32x2(t1)));
          }
        }
        if (h_out) {
          uint4* h = reinterpret_cast<uint4*>(h_out + (size_t)m * K + 16 * (kt0 + jj));
          h[0] = make_uint4(w[0], w[1], w[2], w[3]);
          h[1] = make_uint4(w[4], w[5], w[6], w[7]);
        }
        uint4* dst = reinterpret_cast<uint4*>(xs + ((size_t)jj * mr + m) * 4);
        dst[0] = make_uint4(w[0], w[4], w[1], w[5]);
        dst[1] = make_uint4(w[2], w[6], w[3], w[7]);
      } else {
        if (gm) {
          const uint32_t gw[8] = {gl[q].x, gl[q].y, gl[q].z, gl[q].w,
                                  gh[q].x, gh[q].y, gh[q].z, gh[q].w};
          const uint64_t r2 = pack_f32x2(rinv[m], rinv[m]);
#pragma unroll
          for (int p = 0; p < 8; ++p) {
            const uint32_t t1 = f32x2_to_bf16x2(fmul2(bf16x2_to_f32x2(w[p]), r2));
            w[p] = f32x2_to_bf16x2(fmul2(bf16x2_to_f32x2(gw[p]), bf16x2_to_f32x2(t1)));
          }
        }
        if (h_out) {
          uint4* h = reinterpret_cast<uint4*>(h_out + (size_t)m * K + 16 * (kt0 + jj));
          h[0] = make_uint4(w[0], w[1], w[2], w[3]);
          h[1] = make_uint4(w[4], w[5], w[6], w[7]);
        }
        if (first) {
          // |bf16| bits as fp32 bits order like the magnitudes
          uint32_t mx = 0u;
#pragma unroll
          for (int p = 0; p < 8; ++p)
            mx = max(mx, max((w[p] << 16) & 0x7FFFFFFFu, w[p] & 0x7FFF0000u));
          if (mx >= 0x47000000u) {  // 2^15
            atomicMax(big + m, mx);
            big[16] = 1u;
          }
        }
        const uint64_t s2 = first ? pack_f32x2(1.0f, 1.0f)
                                  : pack_f32x2(1.0f / rpow[m], 1.0f / rpow[m]);  // powers of two
        uint32_t f[8];
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          const float2 v = unpack_f32x2(fmul2(bf16x2_to_f32x2(w[p]), s2));
          f[p] = pack_f16x2(v.x, v.y);
        }
        // f[p] = inputs (2p, 2p+1): entry t = {pair t, pair t + 4}
        uint4* dst = reinterpret_cast<uint4*>(xs + ((size_t)jj * mr + m) * 4);
        dst[0] = make_uint4(f[0], f[4], f[1], f[5]);
        dst[1] = make_uint4(f[2], f[6], f[3], f[7]);
      }
    }
  };
  load_x(tid);
  if (have_ss) {
    // the row statistics from the previous kernel's partials, loaded while
    // this thread's first activations are in flight: one partial per thread
    // and row, a shuffle tree per warp, the warps in order
    const int n = a.ssq_n;
    if (mr <= 4 && n <= nt) {
      float v[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) v[m] = (m < mr && tid < n) ? a.ssq_in[m * n + tid] : 0.0f;
#pragma unroll
      for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v[m] += __shfl_xor_sync(0xffffffffu, v[m], o);
      if (lane == 0)
#pragma unroll
        for (int m = 0; m < 4; ++m)
          if (m < mr) sq[warp * 16 + m] = v[m];
      named_bar_sync(1, nt);
      if (tid < mr) {
        float t = 0.0f;
        for (int w = 0; w < nwarps; ++w) t += sq[w * 16 + tid];
        set_rinv(tid, t);
      }
    } else {
      rows_reduce<false>(a.ssq_in, n, mr, warp, nwarps, lane, set_rinv);
    }
    named_bar_sync(1, nt);
  }
  store_batch(tid, true);
  for (int i0 = tid + NB * nt; i0 < Tr * mr; i0 += NB * nt) {
    load_gamma(i0);
    load_x(i0);
    store_batch(i0, true);
  }
  named_bar_sync(1, nt);
  if (WF == WF_I8ROW && big[16]) {  // some row reaches 2^15: its exponent, then again
    if (tid < mr) {
      const float mxf = __uint_as_float(big[tid]);
      int e = 0;  // largest magnitude below 2^15 after scaling by 2^-e
      if (mxf >= 32768.0f) e = ilogbf(mxf) - 14;
      rpow[tid] = ldexpf(1.0f, e);
    }
    named_bar_sync(1, nt);
    for (int i0 = tid; i0 < Tr * mr; i0 += NB * nt) {
      load_gamma(i0);
      load_x(i0);
      store_batch(i0, false);
    }
    named_bar_sync(1, nt);
  }
}

// ------------------------------------------------------------ top-k draw --
// Order-preserving bits of a float (larger float, larger unsigned).
__device__ __forceinline__ uint32_t f32_order(float f) {
  const uint32_t b = __float_as_uint(f == 0.0f ? 0.0f : f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// One key's top-k draw over the guided logits g = smp.gbuf[p][0, N), by one
// CTA (nt threads): radix select (8 bits per pass, most significant first)
// of the k-th largest value T; the kept set is every index with g > T plus
// the lowest-indexed ties at T that fill k; then Gumbel-argmax over the kept
// set (the lowest index on equal z) and the code written for the key's rows.
static __device__ __noinline__ void topk_draw(const GemvArgs& a, int p, int k, bool cfg, int tid, int nt,
                          unsigned long long* best) {
  __shared__ unsigned hist[256];
  __shared__ unsigned sel[2];        // prefix of T, ties still to take
  __shared__ unsigned eq_before[kTThreads + 1];
  const int N = a.N;
  const float* g = a.smp.gbuf + (size_t)p * N;
  if (tid == 0) {
    sel[0] = 0u;
    sel[1] = (unsigned)k;
    best[0] = 0ull;
  }
  uint32_t mask = 0u;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = tid; b < 256; b += nt) hist[b] = 0u;
    __syncthreads();
    const uint32_t prefix = sel[0];
    for (int i = tid; i < N; i += nt) {
      const uint32_t v = f32_order(__ldcg(g + i));
      if ((v & mask) == prefix) atomicAdd(&hist[(v >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid == 0) {
      unsigned need = sel[1], cum = 0u;
      for (int b = 255; b >= 0; --b) {
        if (cum + hist[b] >= need) {
          sel[0] = prefix | ((uint32_t)b << shift);
          sel[1] = need - cum;  // taken from inside bin b
          break;
        }
        cum += hist[b];
      }
    }
    mask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t T = sel[0];
  const unsigned ties = sel[1];  // the lowest-indexed `ties` values equal to T are kept
  // ties before each thread's contiguous chunk of indices
  const int chunk = (N + nt - 1) / nt;
  const int c0 = min(N, tid * chunk), c1 = min(N, c0 + chunk);
  unsigned eq = 0u;
  for (int i = c0; i < c1; ++i) eq += f32_order(__ldcg(g + i)) == T;
  eq_before[tid + 1] = eq;
  __syncthreads();
  if (tid == 0) {
    eq_before[0] = 0u;
    for (int t = 1; t <= nt; ++t) eq_before[t] += eq_before[t - 1];
  }
  __syncthreads();
  const unsigned long long key = cfg ? (unsigned long long)(a.row0 / 2 + p)
                                     : (unsigned long long)(a.row0 + p);
  unsigned rank = eq_before[tid];
  for (int i = c0; i < c1; ++i) {
    const float gi = __ldcg(g + i);
    const uint32_t v = f32_order(gi);
    bool keep = v > T;
    if (v == T) keep = rank++ < ties;
    if (!keep) continue;
    const float gn = gumbel_noise(a.fp->seed, a.fp->frame, key, smp_index(a.smp, i));
    const float z = __fadd_rn(__fdiv_rn(gi, a.fp->temperature), gn);
    atomicMax(&best[0], argmax_key(z, i));
  }
  __syncthreads();
  if (tid == 0) {
    const int bi = key_idx(best[0]);
    const int nm = cfg ? 2 : 1;
    for (int q = 0; q < nm; ++q) {
      const int r = a.row0 + (cfg ? 2 * p + q : p);
      a.smp.codes[(size_t)r * a.smp.code_stride] = bi;
      if (a.smp.prev)
        a.smp.prev[r] = a.smp.forced ? a.smp.forced[(size_t)r * a.smp.forced_stride] : bi;
    }
  }
  __syncthreads();
}

// ------------------------------------------------------- static kernel ----
// HI: more than 8 batch rows (a second MMA per tile for rows 8..15).
template <int WF, int EPI, bool HI>
__global__ void __launch_bounds__(kTThreads, 1) gemv_tile_kernel(const GemvArgs a) {
  static_assert(WF == WF_BF16 || WF == WF_I8ROW, "tiled formats: bf16, int8 row scale");
  constexpr int ESZ = WF == WF_BF16 ? 2 : 1;
  constexpr int LB = 8 * ESZ;  // bytes of one lane's A fragment
  constexpr int TB = 256 * ESZ;
  constexpr int NT = kTW * 32;
  namespace cg = cooperative_groups;

  const int C = a.tc;
  const int mr = a.mr;
  const int rank = (int)(blockIdx.x % (unsigned)C), cl = (int)(blockIdx.x / (unsigned)C);
  const int ncl = (int)gridDim.x / C;
  const TilePlan P = tile_plan(a.N, a.K, ESZ, C, ncl, a.tsb, a.tsb * a.tns);
  const int u0 = (int)((long long)P.U * cl / ncl), u1 = (int)((long long)P.U * (cl + 1) / ncl);
  const int nu = u1 - u0;
  const int nst = nu * P.ppr;
  const int ns = P.slots;
  const int kt0 = rank * P.Tr;  // first k-tile of this CTA's slice
  const int WU = mr * kUnitRows;  // sums per unit

  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)ns * P.stage);
  uint64_t* empty = full + kTMaxSlots;
  uint8_t* misc = reinterpret_cast<uint8_t*>(empty + kTMaxSlots);
  float* rinv = reinterpret_cast<float*>(misc);  // [16] RMSNorm 1/rms
  float* rpow = rinv + 16;                       // [16] int8: 2^e undoing the x scale
  unsigned long long* best = reinterpret_cast<unsigned long long*>(misc + 640);  // [16]
  int* flag = reinterpret_cast<int*>(misc + 768);
  uint2* zpad = reinterpret_cast<uint2*>(misc + 800);  // zero B fragment of absent rows
  uint2* xs = reinterpret_cast<uint2*>(misc + kTMiscBytes);               // [Tr][mr][4]
  float* part = reinterpret_cast<float*>(xs + (size_t)P.Tr * mr * 4);      // [2][kTW][WU]
  float* cpart = part + (size_t)2 * kTW * WU;                              // [nu_max][WU]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < ns; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kTW);
    }
    fence_barrier_init();
    *zpad = make_uint2(0u, 0u);
  }
  if (EPI == EPI_SAMPLE && tid < 16) best[tid] = 0ull;
  __syncthreads();
  pdl_launch_dependents();

  if (warp == kTW) {
    // ---------------------------------------------------------- producer --
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      const uint8_t* wb = static_cast<const uint8_t*>(a.w);
      for (int s = 0; s < nst; ++s) {
        const int slot = s % ns;
        if (s >= ns && !mbar_wait(&empty[slot], ((s / ns) - 1) & 1, a.err)) break;
        const int u = u0 + s / P.ppr, p = s % P.ppr;
        const int t0 = p * P.pt, t1 = min(P.Tr, t0 + P.pt);
        const uint32_t bytes = (uint32_t)((t1 - t0) * TB);
        mbar_arrive_expect_tx(&full[slot], bytes);
        bulk_g2s(ring + (size_t)slot * P.stage, wb + ((size_t)u * P.T + kt0 + t0) * TB, bytes,
                 &full[slot], pol);
      }
    }
  } else {
    // --------------------------------------------------------- consumers --
    __nv_bfloat16* h_out =
        (EPI == EPI_SAMPLE && a.smp.h_out && cl == 0) ? a.smp.h_out + (size_t)a.row0 * a.K : nullptr;
    if (a.gamma)
      stage_activations<WF, 4, true>(a, mr, kt0, P.Tr, rinv, rpow, reinterpret_cast<float*>(xs),
                                     xs, h_out, tid, NT);
    else
      stage_activations<WF, kStageItems<WF>, false>(a, mr, kt0, P.Tr, rinv, rpow, reinterpret_cast<float*>(xs),
                                      xs, h_out, tid, NT);

    const int g = lane >> 2, t = lane & 3;
    // this lane's B-fragment streams: batch rows g and g + 8, or the zero pad
    const uint2* xl = g < mr ? xs + g * 4 + t : zpad;
    const uint2* xh = g + 8 < mr ? xs + (g + 8) * 4 + t : zpad;
    const int xsl = g < mr ? mr * 4 : 0, xsh = g + 8 < mr ? mr * 4 : 0;
    float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
    float hcc0[4] = {0.f, 0.f, 0.f, 0.f}, hcc1[4] = {0.f, 0.f, 0.f, 0.f};

    for (int s = 0; s < nst; ++s) {
      const int slot = s % ns;
      const int ul = s / P.ppr, p = s % P.ppr;
      const int t0 = p * P.pt, nt = min(P.Tr, t0 + P.pt) - t0;
      // On a timeout the error word is set and the stage is consumed as is, so
      // that every thread still reaches the same barriers.
      mbar_wait(&full[slot], (s / ns) & 1, a.err);
      // this warp's tiles of the stage: warp, warp + kTW, ...
      const uint8_t* wp = ring + (size_t)slot * P.stage + (size_t)warp * TB + lane * LB;
      const uint2* pl = xl + (size_t)(t0 + warp) * xsl;
      const uint2* ph = xh + (size_t)(t0 + warp) * xsh;
      int n = nt > warp ? (nt - warp + kTW - 1) / kTW : 0;
      for (; n >= 2; n -= 2) {
        const uint4 w0 = load_afrag<WF>(wp), w1 = load_afrag<WF>(wp + kTW * TB);
        mma_w<WF>(acc0, w0, *pl);
        mma_w<WF>(acc1, w1, pl[kTW * xsl]);
        if constexpr (HI) {
          mma_w<WF>(hcc0, w0, *ph);
          mma_w<WF>(hcc1, w1, ph[kTW * xsh]);
        }
        wp += 2 * kTW * TB;
        pl += 2 * kTW * xsl;
        ph += 2 * kTW * xsh;
      }
      if (n) {
        const uint4 w0 = load_afrag<WF>(wp);
        mma_w<WF>(acc0, w0, *pl);
        if constexpr (HI) mma_w<WF>(hcc0, w0, *ph);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
      if (p == P.ppr - 1) {
        // the unit is complete: per-warp partials, then the sum over warps
        float* pb = part + ((size_t)(ul & 1) * kTW + warp) * WU;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc0[q] += acc1[q];
          hcc0[q] += hcc1[q];
        }
        put_cfrag(pb, acc0, lane, 0, mr);
        if constexpr (HI) put_cfrag(pb, hcc0, lane, 8, mr);
#pragma unroll
        for (int q = 0; q < 4; ++q) acc0[q] = acc1[q] = hcc0[q] = hcc1[q] = 0.f;
        named_bar_sync(1, NT);
        // in warp order; buffer (ul & 1) is written again two units on, after
        // the next unit's barrier
        const float* pu = part + (size_t)(ul & 1) * kTW * WU;
        for (int r = tid; r < WU; r += NT) {
          float y = 0.0f;
#pragma unroll
          for (int w = 0; w < kTW; ++w) y += pu[(size_t)w * WU + r];
          // int8: this CTA's own power-of-two activation scale (a cluster's
          // CTAs stage different K ranges and may scale them differently);
          // exact in fp32
          if constexpr (WF == WF_I8ROW) y *= rpow[r / kUnitRows];
          cpart[(size_t)ul * WU + r] = y;
        }
      }
    }
  }

  // ------------------------------------------------------------ epilogue --
  // every thread (producer warp included) takes the same barriers
  cg::cluster_group cluster = cg::this_cluster();
  if (C > 1) cluster.sync();
  else __syncthreads();

  // unit sum of (local unit ul, element r = m * 16 + row), over the
  // cluster's ranks in rank order
  auto usum = [&](int ul, int r) -> float {
    if (C == 1) return cpart[(size_t)ul * WU + r];
    float y = 0.0f;
    for (int q = 0; q < C; ++q) {
      const float* rp = cluster.map_shared_rank(cpart, q);
      y += rp[(size_t)ul * WU + r];
    }
    return y;
  };
  // this CTA finalises local units ul = rank, rank + C, ...
  const int nown = nu > rank ? (nu - rank + C - 1) / C : 0;
  if constexpr (EPI == EPI_STORE || EPI == EPI_RESID) {
    // a unit's 16 rows of one batch row are 16 consecutive items, held by a
    // half-warp (kTThreads is a multiple of 16): it sums their squares for
    // the next norm's partials
    static_assert(kTThreads % 16 == 0, "half-warp per (unit, row)");
    for (int e = tid; e < nown * WU; e += kTThreads) {
      const int ul = rank + (e / WU) * C, r = e % WU, m = r / kUnitRows;
      const int n = (u0 + ul) * kUnitRows + r % kUnitRows;
      float o2 = 0.0f;
      if (n < a.N) {
        float y = usum(ul, r);
        if constexpr (WF == WF_I8ROW) y = y * __ldg(a.scales + n);  // rpow is in the unit sums
        __nv_bfloat16* o = a.out + (size_t)m * a.ldo + n;
        __nv_bfloat16 ob;
        if constexpr (EPI == EPI_STORE) ob = __float2bfloat16_rn(y);
        else ob = __float2bfloat16_rn(__bfloat162float(*o) + round_bf16(y));
        *o = ob;
        const float of = __bfloat162float(ob);
        o2 = of * of;
      }
      if (EPI == EPI_RESID && a.ssq_out) {
        const unsigned hm = 0xFFFFu << (tid & 16);
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) o2 += __shfl_xor_sync(hm, o2, off);
        if ((tid & 15) == 0) a.ssq_out[(size_t)m * P.U + u0 + ul] = o2;
      }
    }
  } else if constexpr (EPI == EPI_SWIGLU) {
    constexpr int HP = kUnitRows / 2;  // (gate, up) row pairs per unit
    for (int e = tid; e < nown * mr * HP; e += kTThreads) {
      const int ul = rank + (e / (mr * HP)) * C, r = e % (mr * HP), m = r / HP, jj = r % HP;
      const int n = (u0 + ul) * kUnitRows + 2 * jj;  // gate row n, up row n + 1
      if (n >= a.N) continue;
      float yg = usum(ul, m * kUnitRows + 2 * jj), yu = usum(ul, m * kUnitRows + 2 * jj + 1);
      if constexpr (WF == WF_I8ROW) {
        yg = yg * __ldg(a.scales + n);  // rpow is in the unit sums
        yu = yu * __ldg(a.scales + n + 1);
      }
      const float gb = round_bf16(yg), ub = round_bf16(yu);
      const float act = round_bf16(round_bf16(silu_f(gb)) * ub);
      a.out[(size_t)m * a.ldo + n / 2] = __float2bfloat16_rn(act);
    }
  } else {  // EPI_SAMPLE: all of the CTA's outputs in parallel, then argmax
    const bool cfg = a.fp->cfg_on != 0;
    const int np = cfg ? mr / 2 : mr;
    // top-k: the guided logits go to smp.gbuf and the last CTA selects and
    // draws (k < N; the host passes 0 for "keep all")
    const int topk = a.smp.gbuf ? a.fp->top_k : 0;
    for (int e = tid; e < nown * kUnitRows * np; e += kTThreads) {
      const int ul = rank + (e / (kUnitRows * np)) * C, r = e % (kUnitRows * np);
      const int p = r / kUnitRows, nn = r % kUnitRows;
      const int n = (u0 + ul) * kUnitRows + nn;
      if (n >= a.N) continue;
      const int m0 = cfg ? 2 * p : p;
      float y0 = usum(ul, m0 * kUnitRows + nn);
      float y1 = cfg ? usum(ul, (m0 + 1) * kUnitRows + nn) : 0.0f;
      if constexpr (WF == WF_I8ROW) {
        const float sc = __ldg(a.scales + n);
        y0 = y0 * sc;  // rpow is in the unit sums
        if (cfg) y1 = y1 * sc;
      }
      if (a.smp.logits) {
        a.smp.logits[(size_t)(a.row0 + m0) * a.smp.logits_ld + n] = y0;
        if (cfg) a.smp.logits[(size_t)(a.row0 + m0 + 1) * a.smp.logits_ld + n] = y1;
      }
      float gl = y0;
      if (cfg) gl = __fadd_rn(y1, __fmul_rn(a.fp->cfg_scale, __fsub_rn(y0, y1)));
      if (topk > 0) {
        a.smp.gbuf[(size_t)p * a.N + n] = gl;
        continue;
      }
      const unsigned long long key = cfg ? (unsigned long long)(a.row0 / 2 + p)
                                         : (unsigned long long)(a.row0 + p);
      const float gn = gumbel_noise(a.fp->seed, a.fp->frame, key, smp_index(a.smp, n));
      const float z = __fadd_rn(__fdiv_rn(gl, a.fp->temperature), gn);
      atomicMax(&best[p], argmax_key(z, n));
    }
    __syncthreads();
    if (tid < np) {
      const unsigned long long b = best[tid];
      a.smp.part_z[blockIdx.x * kMaxRows + tid] = b ? key_z(b) : -INFINITY;
      a.smp.part_i[blockIdx.x * kMaxRows + tid] = b ? key_idx(b) : 0x7fffffff;
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      const unsigned old = atomicAdd(a.smp.counter, 1u);
      *flag = old == gridDim.x - 1;
    }
    __syncthreads();
    if (*flag && topk > 0) {  // the last CTA: top-k selection and draw per key
      __threadfence();
      for (int p = 0; p < np; ++p)
        topk_draw(a, p, topk, cfg, tid, kTThreads, best);
      if (tid == 0) *a.smp.counter = 0u;
    } else if (*flag) {  // the last CTA: argmax over the CTAs' winners
      __threadfence();
      // all threads at once (one CTA's winner each), the 64-bit key's max in
      // shared memory: the largest z, the lowest index on equal z
      if (tid < kMaxRows) best[tid] = 0ull;
      __syncthreads();
      for (int p = 0; p < np; ++p) {
        unsigned long long kb = 0ull;
        for (int bb = tid; bb < (int)gridDim.x; bb += kTThreads) {
          const int i = __ldcg(a.smp.part_i + bb * kMaxRows + p);
          if (i == 0x7fffffff) continue;  // a CTA without outputs
          const unsigned long long k = argmax_key(__ldcg(a.smp.part_z + bb * kMaxRows + p), i);
          kb = k > kb ? k : kb;
        }
        if (kb) atomicMax(&best[p], kb);
      }
      __syncthreads();
      if (tid < np) {
        const int bi = best[tid] ? key_idx(best[tid]) : 0x7fffffff;
        const int nm = cfg ? 2 : 1;
        for (int q = 0; q < nm; ++q) {
          const int r = a.row0 + (cfg ? 2 * tid + q : tid);
          a.smp.codes[(size_t)r * a.smp.code_stride] = bi;
          if (a.smp.prev)
            a.smp.prev[r] = a.smp.forced ? a.smp.forced[(size_t)r * a.smp.forced_stride] : bi;
        }
      }
      if (tid == 0) *a.smp.counter = 0u;
    }
  }
  // keep this CTA's unit sums alive until every rank has read them
  if (C > 1) cluster.sync();
}

}  // namespace m3
