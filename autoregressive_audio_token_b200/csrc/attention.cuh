// attention.cuh -- split-K flash-decode GQA attention over the paged KV cache,
// with the new token's q/k RMSNorm, RoPE and KV append fused in.
//
// Per row r, KV head g and split s (grid = splits x Hkv x rows, 4 warps;
// clusters of `splits` CTAs along x):
//   * before waiting for the QKV projection (programmatic dependent launch)
//     the CTA starts bulk copies of its first cached K/V tiles: positions
//     < pos were written by earlier frames and do not depend on it;
//   * it normalises and rotates q (and k) of the new token: per-head RMSNorm
//     with its own gain, then half-rotation RoPE with angle
//     pos * theta^(-2i/d) in fp64 ("MiniMax-Music3 ... DiffSynth-Studio",
//     "各子模型的结构要点": rope_theta 1e6; "MiniMax Music 3 on Metal",
//     "Precision": fp32 norms, rope, softmax and attention sums);
//   * split 0 appends k, v at position pos; the split holding pos takes the
//     new token from registers, so no CTA reads a slot written in this launch;
//   * each warp takes every 4th 32-position tile of the split and runs the
//     whole GQA group on it with warp-level tensor-core MMA (m16n8k16, fp32
//     accumulation): S = Q K^T for the group's heads (rows of A), online
//     softmax in fp32, O += P V with P split into two 16-bit halves
//     (P = P_hi + P_lo, "bf16 halves" as "MiniMax Music 3 on Metal" does for
//     its fp32 GEMMs) so the sums keep fp32 accuracy.  K/V pages are stored
//     chunk-swizzled (kv_elem_offset), so linear bulk copies land
//     conflict-free for ldmatrix;
//   * the warps' states merge in shared memory; the splits of one (r, g)
//     form a thread-block cluster, and its rank 0 merges their (max, sum,
//     unnormalised o) through distributed shared memory by log-sum-exp and
//     writes o in bf16 -- no global round trips, no atomics.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"
#include "gemv.cuh"

namespace m3 {

namespace cg = cooperative_groups;

constexpr int kAttnMaxSplits = 8;  // splits of one (row, KV head) = one portable cluster

constexpr int kAttnWarps = 4;
constexpr int kAttnTile = 32;
constexpr int kAttnBuf = kAttnWarps;  // one tile buffer per warp

struct AttnArgs {
  const __nv_bfloat16* qkv;   // [rows][ldqkv]: q (Hq*D) | k (Hkv*D) | v (Hkv*D)
  int ldqkv;
  const __nv_bfloat16* q_norm;  // [D]
  const __nv_bfloat16* k_norm;  // [D]
  float eps;
  const double* inv_freq;     // [D/2] theta^(-2i/D)
  const float2* rope;         // nullable: this frame's (cos, sin) [rows][D/2]
  int rope_ld;                // row stride of `rope` in entries (0: one position for all rows)
  const unsigned long long* pages;  // [rows][n_layers][max_pages] page base addresses
  int layer, n_layers, max_pages, page_size;
  int Hq, Hkv;
  __nv_bfloat16* out;         // [rows][Hq*D]
  const FrameParams* fp;
  int fixed_pos;              // >= 0: row r is at fixed_pos + r * pos_stride
  int pos_stride;             // 0: one position for all rows (depth decoder); 1: a prompt chunk
  int* err;
  // 0: decode (the new token's K/V are appended and attended from registers);
  // 1: append only (prefill: every row's K/V of its position, then exit);
  // 2: attend from the cache only, own position included (prefill, after 1)
  int mode;
};

template <int D>
__host__ __device__ constexpr size_t attn_smem_bytes() {
  return (size_t)kAttnBuf * 2 * kAttnTile * D * 2                  // K, V tiles
         + sizeof(float) * (kAttnWarps * D + 2 * D)                 // q, k, v of the new token
         + sizeof(float) * kAttnWarps * kAttnWarps * (D + 2)        // per-warp (m, l, o)
         + sizeof(float) * kAttnWarps                               // new-token scores
         + sizeof(uint64_t) * kAttnBuf + 64;
}

template <int KVF16>
__device__ __forceinline__ float kv_to_f32(uint16_t b) {
  if constexpr (KVF16) return __half2float(__ushort_as_half(b));
  return __uint_as_float(((uint32_t)b) << 16);
}

template <int KVF16>
__device__ __forceinline__ uint16_t f32_to_kv(float v) {
  if constexpr (KVF16) return __half_as_ushort(__float2half_rn(v));
  return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// Two fp32 -> packed 16-bit pair (low half = first), in the cache's type.
template <int KVF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if constexpr (KVF16) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  } else {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  }
}

template <int KVF16>
__device__ __forceinline__ float2 unpack2(uint32_t w) {
  if constexpr (KVF16) {
    __half2 h = *reinterpret_cast<__half2*>(&w);
    return __half22float2(h);
  } else {
    __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&w);
    return __bfloat1622float2(h);
  }
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D (16x8 fp32) += A (16x16) * B (16x8), A/B bf16 or f16 (same type).
template <int KVF16>
__device__ __forceinline__ void mma16816(float* d, uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  if constexpr (KVF16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
}

template <int D, int KVF16>
__global__ void __launch_bounds__(kAttnWarps * 32) attn_decode_kernel(const AttnArgs a) {
  constexpr int VPL = D / 32;           // dims per lane in the scalar parts (4 or 2)
  constexpr int NT = D / 8;             // n-tiles of O (8 dims each)
  constexpr int KS = D / 16;            // k-steps of Q K^T (16 dims each)
  constexpr int TILE_ELEMS = kAttnTile * D;
  constexpr int ROWB = D * 2;           // bytes per position row
  extern __shared__ __align__(1024) uint8_t smem[];
  uint16_t* kt = reinterpret_cast<uint16_t*>(smem);         // [BUF][TILE][D] (swizzled)
  uint16_t* vt = kt + kAttnBuf * TILE_ELEMS;                  // [BUF][TILE][D] (swizzled)
  float* q_s = reinterpret_cast<float*>(vt + kAttnBuf * TILE_ELEMS);  // [4][D]
  float* k_s = q_s + kAttnWarps * D;                          // [D]
  float* v_s = k_s + D;                                       // [D]
  float* w_s = v_s + D;                                       // [warp][head][D+2]
  float* sn_s = w_s + kAttnWarps * kAttnWarps * (D + 2);      // [head] new-token score
  uint64_t* bars = reinterpret_cast<uint64_t*>(sn_s + kAttnWarps);

  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int r = blockIdx.z, g = blockIdx.y, sidx = blockIdx.x, S = gridDim.x;
  const int grp = a.Hq / a.Hkv;
  const int pos = a.fixed_pos >= 0 ? a.fixed_pos + r * a.pos_stride : a.fp->pos[r];
  const int n = pos + 1;
  int chunk = (n + S - 1) / S;
  chunk = (chunk + kAttnTile - 1) / kAttnTile * kAttnTile;
  const int j0 = sidx * chunk;
  const int j1 = min(n, j0 + chunk);
  const int mode = a.mode;
  const int jc1 = mode == 2 ? j1 : min(j1, pos);  // cached positions [j0, jc1)
  const bool has_new = mode == 0 && (j0 <= pos) && (pos < j1);
  const int ntiles = (mode != 1 && jc1 > j0) ? (jc1 - j0 + kAttnTile - 1) / kAttnTile : 0;
  const unsigned long long* pt = a.pages + ((size_t)r * a.n_layers + a.layer) * a.max_pages;

  auto issue_tile = [&](int t) {
    const int js = j0 + t * kAttnTile;
    const int nv = min(kAttnTile, jc1 - js);
    const int page = js / a.page_size, off = js % a.page_size;
    const uint16_t* base = reinterpret_cast<const uint16_t*>(pt[page]);
    const uint32_t bytes = (uint32_t)(nv * ROWB);
    const int b = t % kAttnBuf;
    mbar_arrive_expect_tx(&bars[b], 2 * bytes);
    bulk_g2s_nohint(kt + b * TILE_ELEMS, base + ((size_t)g * a.page_size + off) * D, bytes,
                    &bars[b]);
    bulk_g2s_nohint(vt + b * TILE_ELEMS, base + ((size_t)(a.Hkv + g) * a.page_size + off) * D,
                    bytes, &bars[b]);
  };

  if (tid == 0) {
    for (int b = 0; b < kAttnBuf; ++b) mbar_init(&bars[b], 1);
    fence_barrier_init();
    for (int t = 0; t < min(kAttnBuf, ntiles); ++t) issue_tile(t);
  }
  __syncthreads();
  pdl_launch_dependents();

  // Everything the new token's norm + RoPE needs except q, k, v themselves
  // is static this frame: gains, and the rotation angles from the position.
  const float scale = 1.0f / sqrtf((float)D);
  const bool is_q = w < grp, is_k = (w == kAttnWarps - 1);
  float gq[VPL], gk[VPL], rc[VPL / 2], rs[VPL / 2];
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    gq[i] = is_q ? __bfloat162float(a.q_norm[lane + 32 * i]) : 0.0f;
    gk[i] = is_k ? __bfloat162float(a.k_norm[lane + 32 * i]) : 0.0f;
  }
  if (is_q || is_k) {
#pragma unroll
    for (int i = 0; i < VPL / 2; ++i) {
      if (a.rope) {
        const float2 cs = a.rope[(size_t)r * a.rope_ld + lane + 32 * i];
        rc[i] = cs.x;
        rs[i] = cs.y;
      } else {
        const double ang = (double)pos * a.inv_freq[lane + 32 * i];
        rc[i] = (float)cos(ang);
        rs[i] = (float)sin(ang);
      }
    }
  }
  pdl_wait();  // q, k, v of the new token come from the QKV projection

  // ---- new token: q/k RMSNorm + RoPE (lane l holds dims l + 32i) --------
  // every load of the new token is issued before any of them is used
  const __nv_bfloat16* row_qkv = a.qkv + (size_t)r * a.ldqkv;
  const __nv_bfloat16* qraw = row_qkv + (size_t)(g * grp + w) * D;
  const __nv_bfloat16* kraw = row_qkv + (size_t)a.Hq * D + (size_t)g * D;
  const __nv_bfloat16* vraw = row_qkv + (size_t)(a.Hq + a.Hkv) * D + (size_t)g * D;
  float qin[VPL], kin[VPL], vin[VPL];  // a warp may hold a query head and the key
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    qin[i] = is_q ? __bfloat162float(qraw[lane + 32 * i]) : 0.0f;
    kin[i] = is_k ? __bfloat162float(kraw[lane + 32 * i]) : 0.0f;
    vin[i] = is_k ? __bfloat162float(vraw[lane + 32 * i]) : 0.0f;
  }
  auto norm_rope = [&](float* v, const float* gamma, float* dst) {
    float ss = 0.0f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) ss = fmaf(v[i], v[i], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = 1.0f / sqrtf(ss / (float)D + a.eps);
#pragma unroll
    for (int i = 0; i < VPL; ++i) v[i] = round_bf16(gamma[i] * round_bf16(v[i] * inv));
    // pairs (i, i + D/2): dims lane + 32i with i < VPL/2 pair with i + VPL/2
#pragma unroll
    for (int i = 0; i < VPL / 2; ++i) {
      const float x0 = v[i], x1 = v[i + VPL / 2];
      v[i] = __fsub_rn(__fmul_rn(x0, rc[i]), __fmul_rn(x1, rs[i]));
      v[i + VPL / 2] = __fadd_rn(__fmul_rn(x1, rc[i]), __fmul_rn(x0, rs[i]));
    }
#pragma unroll
    for (int i = 0; i < VPL; ++i) dst[lane + 32 * i] = round_bf16(v[i]);
  };

  if (is_q) norm_rope(qin, gq, q_s + w * D);
  if (is_k) {
    // the key (and value) of the new token, as they will be stored
    norm_rope(kin, gk, k_s);
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int dim = lane + 32 * i;
      const uint16_t kb = f32_to_kv<KVF16>(k_s[dim]);
      const uint16_t vb = f32_to_kv<KVF16>(vin[i]);
      k_s[dim] = kv_to_f32<KVF16>(kb);
      v_s[dim] = kv_to_f32<KVF16>(vb);
      if (sidx == 0 && mode != 2) {
        const int page = pos / a.page_size, off = pos % a.page_size;
        uint16_t* base = reinterpret_cast<uint16_t*>(pt[page]);
        base[kv_elem_offset(g, a.page_size, off, D, dim)] = kb;
        base[kv_elem_offset(a.Hkv + g, a.page_size, off, D, dim)] = vb;
      }
    }
  }
  __syncthreads();
  // append only: the K/V are stored (no tile was issued, no cluster barrier
  // is taken by any CTA of this launch)
  if (mode == 1) return;
  if (w < grp) {  // score of the new token for head w
    float p = 0.0f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) p = fmaf(q_s[w * D + lane + 32 * i], k_s[lane + 32 * i], p);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
    if (lane == 0) sn_s[w] = p * scale;
  }

  // ---- cached positions: each warp runs every 4th tile on tensor cores ----
  // A fragments of Q (rows = the group's heads; rows >= grp and 8..15 zero).
  const int gid = lane >> 2, tig = lane & 3;
  const bool row_ok = gid < grp;
  uint32_t qa[KS][2];
#pragma unroll
  for (int kk = 0; kk < KS; ++kk) {
    const float* qh = q_s + gid * D + 16 * kk + 2 * tig;
    qa[kk][0] = row_ok ? pack2<KVF16>(qh[0], qh[1]) : 0u;
    qa[kk][1] = row_ok ? pack2<KVF16>(qh[8], qh[9]) : 0u;
  }
  float o_acc[NT][4];
#pragma unroll
  for (int j = 0; j < NT; ++j) o_acc[j][0] = o_acc[j][1] = o_acc[j][2] = o_acc[j][3] = 0.0f;
  float m_run = -INFINITY, l_run = 0.0f;  // of head gid (replicated in the quad)

  for (int t = w; t < ntiles; t += kAttnWarps) {
    const int b = t % kAttnBuf;
    mbar_wait(&bars[b], (t / kAttnBuf) & 1, a.err);
    const int nv = min(kAttnTile, jc1 - (j0 + t * kAttnTile));
    if (nv < kAttnTile) {
      // rows past the end of a partial tile hold stale (or never written)
      // shared memory; zero them so that p = 0 never multiplies a NaN pattern
      uint4* kz = reinterpret_cast<uint4*>(kt + b * TILE_ELEMS);
      uint4* vz = reinterpret_cast<uint4*>(vt + b * TILE_ELEMS);
      for (int c = nv * (D / 8) + lane; c < kAttnTile * (D / 8); c += 32) {
        kz[c] = make_uint4(0, 0, 0, 0);
        vz[c] = make_uint4(0, 0, 0, 0);
      }
      __syncwarp();
    }
    const uint32_t kb = smem_u32(kt + b * TILE_ELEMS);
    const uint32_t vb = smem_u32(vt + b * TILE_ELEMS);
    // S = Q K^T: 4 n-tiles of 8 positions
    float sc[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      sc[j][0] = sc[j][1] = sc[j][2] = sc[j][3] = 0.0f;
      const int prow = 8 * j + (lane & 7);
#pragma unroll
      for (int kk = 0; kk < KS; kk += 2) {
        const int chunk = 2 * kk + (lane >> 3);
        const uint32_t addr = kb + prow * ROWB + ((chunk ^ (prow & 7)) << 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(addr, b0, b1, b2, b3);
        mma16816<KVF16>(sc[j], qa[kk][0], 0u, qa[kk][1], 0u, b0, b1);
        mma16816<KVF16>(sc[j], qa[kk + 1][0], 0u, qa[kk + 1][1], 0u, b2, b3);
      }
    }
    // online softmax of row gid over this tile's positions 8j + 2 tig + {0,1}
    float mt = -INFINITY;
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int p = 8 * j + 2 * tig + e;
        const float s = p < nv ? sc[j][e] * scale : -INFINITY;
        sc[j][e] = s;
        mt = fmaxf(mt, s);
      }
    mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
    mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
    const float m_new = fmaxf(m_run, mt);
    const float corr = expf(m_run - m_new);  // 0 when m_run = -inf
    float ls = 0.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float p = expf(sc[j][e] - m_new);  // 0 for masked positions
        sc[j][e] = p;
        ls += p;
      }
    ls += __shfl_xor_sync(0xffffffffu, ls, 1);
    ls += __shfl_xor_sync(0xffffffffu, ls, 2);
    l_run = l_run * corr + ls;
    m_run = m_new;
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      o_acc[j][0] *= corr;
      o_acc[j][1] *= corr;
    }
    // O += P V, P = P_hi + P_lo (16-bit halves), two k-steps of 16 positions
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
      const float p0 = sc[2 * kk][0], p1 = sc[2 * kk][1];
      const float p2 = sc[2 * kk + 1][0], p3 = sc[2 * kk + 1][1];
      const uint32_t h0 = pack2<KVF16>(p0, p1), h2 = pack2<KVF16>(p2, p3);
      const float2 f0 = unpack2<KVF16>(h0), f2 = unpack2<KVF16>(h2);
      const uint32_t l0 = pack2<KVF16>(p0 - f0.x, p1 - f0.y);
      const uint32_t l2 = pack2<KVF16>(p2 - f2.x, p3 - f2.y);
      const int prow = 16 * kk + (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
      for (int j = 0; j < NT; j += 2) {
        const int chunk = j + (lane >> 4);
        const uint32_t addr = vb + prow * ROWB + ((chunk ^ (prow & 7)) << 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(addr, b0, b1, b2, b3);
        mma16816<KVF16>(o_acc[j], h0, 0u, h2, 0u, b0, b1);
        mma16816<KVF16>(o_acc[j], l0, 0u, l2, 0u, b0, b1);
        mma16816<KVF16>(o_acc[j + 1], h0, 0u, h2, 0u, b2, b3);
        mma16816<KVF16>(o_acc[j + 1], l0, 0u, l2, 0u, b2, b3);
      }
    }
    __syncwarp();
    if (lane == 0 && t + kAttnBuf < ntiles) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // reads before the refill
      issue_tile(t + kAttnBuf);
    }
  }

  // ---- merge the warps' states (and the new token) in shared memory ------
  {
    float* ws = w_s + (size_t)w * kAttnWarps * (D + 2);
    if (row_ok) {
      float* wh = ws + gid * (D + 2);
      if (tig == 0) {
        wh[0] = m_run;
        wh[1] = l_run;
      }
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        wh[2 + 8 * j + 2 * tig] = o_acc[j][0];
        wh[2 + 8 * j + 2 * tig + 1] = o_acc[j][1];
      }
    }
  }
  __syncthreads();
  // ---- this split's (max, sum, unnormalised o) per head, in shared memory --
  // (the tile buffers are free now: every warp has consumed its tiles)
  const int stride = D + 2;
  float* cp_s = reinterpret_cast<float*>(kt);  // [grp][D + 2]
  if (w < grp) {
    float M = has_new ? sn_s[w] : -INFINITY;
#pragma unroll
    for (int ww = 0; ww < kAttnWarps; ++ww) M = fmaxf(M, w_s[(ww * kAttnWarps + w) * (D + 2)]);
    float L = 0.0f, o[VPL];
#pragma unroll
    for (int e = 0; e < VPL; ++e) o[e] = 0.0f;
#pragma unroll
    for (int ww = 0; ww < kAttnWarps; ++ww) {
      const float* wh = w_s + (ww * kAttnWarps + w) * (D + 2);
      const float f = wh[0] == -INFINITY ? 0.0f : expf(wh[0] - M);
      L = fmaf(wh[1], f, L);
#pragma unroll
      for (int e = 0; e < VPL; ++e) o[e] = fmaf(wh[2 + VPL * lane + e], f, o[e]);
    }
    if (has_new) {
      const float f = expf(sn_s[w] - M);
      L += f;
#pragma unroll
      for (int e = 0; e < VPL; ++e) o[e] = fmaf(f, v_s[VPL * lane + e], o[e]);
    }
    float* cw = cp_s + w * stride;
    if (lane == 0) {
      cw[0] = M;
      cw[1] = L;
    }
#pragma unroll
    for (int e = 0; e < VPL; ++e) cw[2 + VPL * lane + e] = o[e];
  }

  // ---- the splits of (r, g) form one cluster and merge through distributed
  // shared memory (log-sum-exp): rank s finishes its slice of the group's
  // (head, dim) outputs, reading every rank's partial in parallel ----------
  cg::cluster_group cluster = cg::this_cluster();
  cluster.sync();
  {
    const int items = grp * D;
    const int per = (items + S - 1) / S;
    const int it_end = min(items, (sidx + 1) * per);
    for (int it = sidx * per + tid; it < it_end; it += blockDim.x) {
      const int hl = it / D, d = it % D;
      float ms[kAttnMaxSplits], ls[kAttnMaxSplits], os[kAttnMaxSplits];
#pragma unroll
      for (int s2 = 0; s2 < kAttnMaxSplits; ++s2) {
        if (s2 < S) {
          const float* rem = cluster.map_shared_rank(cp_s, s2) + hl * stride;
          ms[s2] = rem[0];
          ls[s2] = rem[1];
          os[s2] = rem[2 + d];
        }
      }
      float M = -INFINITY;
#pragma unroll
      for (int s2 = 0; s2 < kAttnMaxSplits; ++s2)
        if (s2 < S) M = fmaxf(M, ms[s2]);
      float L = 0.0f, o = 0.0f;
#pragma unroll
      for (int s2 = 0; s2 < kAttnMaxSplits; ++s2) {
        if (s2 < S) {
          const float f = ms[s2] == -INFINITY ? 0.0f : expf(ms[s2] - M);
          L = fmaf(ls[s2], f, L);
          o = fmaf(os[s2], f, o);
        }
      }
      a.out[(size_t)r * a.Hq * D + (size_t)(g * grp + hl) * D + d] = __float2bfloat16_rn(o / L);
    }
  }
  cluster.sync();  // no CTA leaves while another still reads its shared memory
}

}  // namespace m3
