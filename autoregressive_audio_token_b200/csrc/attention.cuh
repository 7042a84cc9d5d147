// attention.cuh -- split-K flash-decode GQA attention over the paged KV cache,
// with the new token's q/k RMSNorm, RoPE and KV append fused in.
//
// Per row r, KV head g and split s (grid = splits x Hkv x rows; 4 warps, one
// per query head of the GQA group):
//   * before waiting for the QKV projection (programmatic dependent launch),
//     the CTA starts bulk copies of its first cached K/V tiles (positions
//     < pos were written by earlier frames, so they do not depend on it);
//   * it then normalises and rotates q (and k) of the new token: per-head
//     RMSNorm with its own gain, half-rotation RoPE with angle
//     pos * theta^(-2i/d) in fp64 ("MiniMax-Music3 ... DiffSynth-Studio",
//     "各子模型的结构要点": rope_theta 1e6; "MiniMax Music 3 on Metal",
//     "Precision": fp32 norms, rope, softmax and attention sums);
//   * split 0 appends k, v at position pos; the split holding pos takes the
//     new token from registers, so no CTA reads a slot written in this launch;
//   * scores s_j = q.k_j / sqrt(d) use a transposed butterfly so that lane j
//     ends with position j; online softmax in fp32; o += p_j v_j;
//   * each split writes (max, sum, unnormalised o); the last CTA of (r, g)
//     to finish (an atomic ticket, no waiting) merges the splits by their
//     log-sum-exp and writes o in bf16.
#pragma once

#include "common.cuh"
#include "gemv.cuh"

namespace m3 {

constexpr int kAttnWarps = 4;
constexpr int kAttnTile = 32;
constexpr int kAttnBuf = 4;

struct AttnArgs {
  const __nv_bfloat16* qkv;   // [rows][ldqkv]: q (Hq*D) | k (Hkv*D) | v (Hkv*D)
  int ldqkv;
  const __nv_bfloat16* q_norm;  // [D]
  const __nv_bfloat16* k_norm;  // [D]
  float eps;
  const double* inv_freq;     // [D/2] theta^(-2i/D)
  const unsigned long long* pages;  // [rows][n_layers][max_pages] page base addresses
  int layer, n_layers, max_pages, page_size;
  int Hq, Hkv;
  float* part;                // [rows][Hq][splits][D+2]
  unsigned int* counters;     // [rows][Hkv], zero at rest
  __nv_bfloat16* out;         // [rows][Hq*D]
  const FrameParams* fp;
  int fixed_pos;              // >= 0: every row is at this position (depth decoder)
  int* err;
};

template <int D>
__host__ __device__ constexpr size_t attn_smem_bytes() {
  return (size_t)kAttnBuf * 2 * kAttnTile * D * 2 + sizeof(float) * (kAttnWarps * D + 2 * D) +
         sizeof(uint64_t) * kAttnBuf + 64;
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

// One step of a reduce-scatter over the warp: lanes exchange the half of
// their values that the partner keeps, so after the step with HALF = 1 lane l
// holds in v[0] the sum over all lanes of their v[l].
template <int HALF>
__device__ __forceinline__ void butterfly_step(float* v, int lane) {
  const bool up = (lane & HALF) != 0;
#pragma unroll
  for (int i = 0; i < HALF; ++i) {
    const float send = up ? v[i] : v[i + HALF];
    const float keep = up ? v[i + HALF] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, HALF);
  }
}

template <int D, int KVF16>
__global__ void __launch_bounds__(kAttnWarps * 32) attn_decode_kernel(const AttnArgs a) {
  constexpr int VPL = D / 32;  // dims per lane (4 or 2)
  constexpr int TILE_ELEMS = kAttnTile * D;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint16_t* kt = reinterpret_cast<uint16_t*>(smem);         // [BUF][TILE][D]
  uint16_t* vt = kt + kAttnBuf * TILE_ELEMS;                  // [BUF][TILE][D]
  float* q_s = reinterpret_cast<float*>(vt + kAttnBuf * TILE_ELEMS);  // [4][D]
  float* k_s = q_s + kAttnWarps * D;                          // [D]
  float* v_s = k_s + D;                                       // [D]
  uint64_t* bars = reinterpret_cast<uint64_t*>(v_s + D);
  __shared__ int s_last;

  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int r = blockIdx.z, g = blockIdx.y, sidx = blockIdx.x, S = gridDim.x;
  const int grp = a.Hq / a.Hkv;
  const int pos = a.fixed_pos >= 0 ? a.fixed_pos : a.fp->pos[r];
  const int n = pos + 1;
  int chunk = (n + S - 1) / S;
  chunk = (chunk + kAttnTile - 1) / kAttnTile * kAttnTile;
  const int j0 = sidx * chunk;
  const int j1 = min(n, j0 + chunk);
  const int jc1 = min(j1, pos);  // cached positions [j0, jc1)
  const bool has_new = (j0 <= pos) && (pos < j1);
  const int ntiles = jc1 > j0 ? (jc1 - j0 + kAttnTile - 1) / kAttnTile : 0;
  const unsigned long long* pt = a.pages + ((size_t)r * a.n_layers + a.layer) * a.max_pages;

  auto issue_tile = [&](int t) {
    const int js = j0 + t * kAttnTile;
    const int nv = min(kAttnTile, jc1 - js);
    const int page = js / a.page_size, off = js % a.page_size;
    const uint16_t* base = reinterpret_cast<const uint16_t*>(pt[page]);
    const uint32_t bytes = (uint32_t)(nv * D * 2);
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
  pdl_wait();  // q, k, v of the new token come from the QKV projection

  // ---- new token: q/k RMSNorm + RoPE (lane l holds dims l + 32i) --------
  const float scale = 1.0f / sqrtf((float)D);
  auto norm_rope = [&](const __nv_bfloat16* src, const __nv_bfloat16* gamma, float* dst) {
    float v[VPL];
    float ss = 0.0f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      v[i] = __bfloat162float(src[lane + 32 * i]);
      ss = fmaf(v[i], v[i], ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = 1.0f / sqrtf(ss / (float)D + a.eps);
#pragma unroll
    for (int i = 0; i < VPL; ++i)
      v[i] = round_bf16(__bfloat162float(gamma[lane + 32 * i]) * round_bf16(v[i] * inv));
    // pairs (i, i + D/2): dims lane + 32i with i < VPL/2 pair with i + VPL/2
#pragma unroll
    for (int i = 0; i < VPL / 2; ++i) {
      const int dim = lane + 32 * i;
      const double ang = (double)pos * a.inv_freq[dim];
      const float c = (float)cos(ang), s = (float)sin(ang);
      const float x0 = v[i], x1 = v[i + VPL / 2];
      v[i] = __fsub_rn(__fmul_rn(x0, c), __fmul_rn(x1, s));
      v[i + VPL / 2] = __fadd_rn(__fmul_rn(x1, c), __fmul_rn(x0, s));
    }
#pragma unroll
    for (int i = 0; i < VPL; ++i) dst[lane + 32 * i] = round_bf16(v[i]);
  };

  const __nv_bfloat16* row_qkv = a.qkv + (size_t)r * a.ldqkv;
  if (w < grp) norm_rope(row_qkv + (size_t)(g * grp + w) * D, a.q_norm, q_s + w * D);
  if (w == kAttnWarps - 1) {
    // the key (and value) of the new token, as they will be stored
    const __nv_bfloat16* kraw = row_qkv + (size_t)a.Hq * D + (size_t)g * D;
    const __nv_bfloat16* vraw = row_qkv + (size_t)(a.Hq + a.Hkv) * D + (size_t)g * D;
    norm_rope(kraw, a.k_norm, k_s);
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int dim = lane + 32 * i;
      const uint16_t kb = f32_to_kv<KVF16>(k_s[dim]);
      const uint16_t vb = f32_to_kv<KVF16>(__bfloat162float(vraw[dim]));
      k_s[dim] = kv_to_f32<KVF16>(kb);
      v_s[dim] = kv_to_f32<KVF16>(vb);
      if (sidx == 0) {
        const int page = pos / a.page_size, off = pos % a.page_size;
        uint16_t* base = reinterpret_cast<uint16_t*>(pt[page]);
        base[((size_t)g * a.page_size + off) * D + dim] = kb;
        base[((size_t)(a.Hkv + g) * a.page_size + off) * D + dim] = vb;
      }
    }
  }
  __syncthreads();

  // ---- cached positions: online softmax over tiles ----------------------
  float m_run = -INFINITY, l_run = 0.0f;
  float acc[VPL];
#pragma unroll
  for (int e = 0; e < VPL; ++e) acc[e] = 0.0f;
  float qv[VPL];
  if (w < grp) {
#pragma unroll
    for (int e = 0; e < VPL; ++e) qv[e] = q_s[w * D + VPL * lane + e];
  }

  for (int t = 0; t < ntiles; ++t) {
    const int b = t % kAttnBuf;
    mbar_wait(&bars[b], (t / kAttnBuf) & 1, a.err);
    const int nv = min(kAttnTile, jc1 - (j0 + t * kAttnTile));
    if (w < grp) {
      const uint16_t* K = kt + b * TILE_ELEMS;
      const uint16_t* V = vt + b * TILE_ELEMS;
      float sc[kAttnTile];
#pragma unroll
      for (int j = 0; j < kAttnTile; ++j) {
        float p = 0.0f;
        if (j < nv) {
          if constexpr (VPL == 4) {
            const uint2 kv = *reinterpret_cast<const uint2*>(K + j * D + 4 * lane);
            p = qv[0] * kv_to_f32<KVF16>(kv.x & 0xFFFF);
            p = fmaf(qv[1], kv_to_f32<KVF16>(kv.x >> 16), p);
            p = fmaf(qv[2], kv_to_f32<KVF16>(kv.y & 0xFFFF), p);
            p = fmaf(qv[3], kv_to_f32<KVF16>(kv.y >> 16), p);
          } else {
            const uint32_t kv = *reinterpret_cast<const uint32_t*>(K + j * D + 2 * lane);
            p = qv[0] * kv_to_f32<KVF16>(kv & 0xFFFF);
            p = fmaf(qv[1], kv_to_f32<KVF16>(kv >> 16), p);
          }
        }
        sc[j] = p;
      }
      // transposed butterfly: lane j ends with the full dot product of position j
      butterfly_step<16>(sc, lane);
      butterfly_step<8>(sc, lane);
      butterfly_step<4>(sc, lane);
      butterfly_step<2>(sc, lane);
      butterfly_step<1>(sc, lane);
      const float s = lane < nv ? sc[0] * scale : -INFINITY;
      float mt = s;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
      const float m_new = fmaxf(m_run, mt);
      const float p = lane < nv ? expf(s - m_new) : 0.0f;
      float ps = p;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
      const float corr = expf(m_run - m_new);  // 0 when m_run = -inf
      l_run = l_run * corr + ps;
#pragma unroll
      for (int e = 0; e < VPL; ++e) acc[e] *= corr;
      m_run = m_new;
      for (int j = 0; j < nv; ++j) {
        const float pj = __shfl_sync(0xffffffffu, p, j);
        if constexpr (VPL == 4) {
          const uint2 vv = *reinterpret_cast<const uint2*>(V + j * D + 4 * lane);
          acc[0] = fmaf(pj, kv_to_f32<KVF16>(vv.x & 0xFFFF), acc[0]);
          acc[1] = fmaf(pj, kv_to_f32<KVF16>(vv.x >> 16), acc[1]);
          acc[2] = fmaf(pj, kv_to_f32<KVF16>(vv.y & 0xFFFF), acc[2]);
          acc[3] = fmaf(pj, kv_to_f32<KVF16>(vv.y >> 16), acc[3]);
        } else {
          const uint32_t vv = *reinterpret_cast<const uint32_t*>(V + j * D + 2 * lane);
          acc[0] = fmaf(pj, kv_to_f32<KVF16>(vv & 0xFFFF), acc[0]);
          acc[1] = fmaf(pj, kv_to_f32<KVF16>(vv >> 16), acc[1]);
        }
      }
    }
    __syncthreads();  // buffer b is free
    if (tid == 0 && t + kAttnBuf < ntiles) issue_tile(t + kAttnBuf);
  }

  // ---- the new token -----------------------------------------------------
  if (has_new && w < grp) {
    float p = 0.0f;
#pragma unroll
    for (int e = 0; e < VPL; ++e) p = fmaf(qv[e], k_s[VPL * lane + e], p);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
    const float s = p * scale;
    const float m_new = fmaxf(m_run, s);
    const float pe = expf(s - m_new), corr = expf(m_run - m_new);
    l_run = l_run * corr + pe;
#pragma unroll
    for (int e = 0; e < VPL; ++e) acc[e] = fmaf(pe, v_s[VPL * lane + e], acc[e] * corr);
    m_run = m_new;
  }

  // ---- partial result, then the last CTA of (r, g) merges ----------------
  const int stride = D + 2;
  if (w < grp) {
    const int h = g * grp + w;
    float* pp = a.part + (((size_t)r * a.Hq + h) * S + sidx) * stride;
    if (lane == 0) {
      pp[0] = m_run;
      pp[1] = l_run;
    }
#pragma unroll
    for (int e = 0; e < VPL; ++e) pp[2 + VPL * lane + e] = acc[e];
    __threadfence();
  }
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const unsigned old = atomicAdd(a.counters + (size_t)r * a.Hkv + g, 1u);
    s_last = (old == (unsigned)(S - 1));
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (w < grp) {
    const int h = g * grp + w;
    const float* pp = a.part + ((size_t)r * a.Hq + h) * S * stride;
    // lanes hold the splits' (max, sum): S <= 64, two per lane at most
    const float m0 = lane < S ? __ldcg(pp + lane * stride) : -INFINITY;
    const float m1 = lane + 32 < S ? __ldcg(pp + (lane + 32) * stride) : -INFINITY;
    const float l0 = lane < S ? __ldcg(pp + lane * stride + 1) : 0.0f;
    const float l1 = lane + 32 < S ? __ldcg(pp + (lane + 32) * stride + 1) : 0.0f;
    float M = fmaxf(m0, m1);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float f0 = m0 == -INFINITY ? 0.0f : expf(m0 - M);
    const float f1 = m1 == -INFINITY ? 0.0f : expf(m1 - M);
    float L = l0 * f0 + l1 * f1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    float o[VPL];
#pragma unroll
    for (int e = 0; e < VPL; ++e) o[e] = 0.0f;
#pragma unroll 8
    for (int s2 = 0; s2 < S; ++s2) {
      const float f = __shfl_sync(0xffffffffu, s2 < 32 ? f0 : f1, s2 & 31);
      const float* src = pp + s2 * stride + 2 + VPL * lane;
#pragma unroll
      for (int e = 0; e < VPL; ++e) o[e] = fmaf(__ldcg(src + e), f, o[e]);
    }
    __nv_bfloat16* dst = a.out + (size_t)r * a.Hq * D + (size_t)h * D + VPL * lane;
#pragma unroll
    for (int e = 0; e < VPL; ++e) dst[e] = __float2bfloat16_rn(o[e] / L);
  }
  if (tid == 0) a.counters[(size_t)r * a.Hkv + g] = 0u;
}

}  // namespace m3
