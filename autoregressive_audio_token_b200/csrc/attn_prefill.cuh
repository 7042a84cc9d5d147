// attn_prefill.cuh -- causal attention of a prompt chunk over the row's paged
// KV cache, tiled (flash-attention style) on warp-level tensor-core MMA.
//
// The prefill is the token-by-token decode run in chunks (DiffSynth-Studio
// article, "第一阶段"): token t of the chunk sits at position p0 + t and
// attends to positions 0 .. p0 + t of its row, its own K/V included (they are
// appended before this kernel runs).  Run as the decode attention once per
// token, every token re-reads the chunk's K/V from L2; here the 4 query heads
// of one KV head share every K/V tile:
//   * a CTA of 4 warps takes (16 query rows per warp) x (one KV head): a row
//     is (token, query head of the group), tokens consecutive, so a warp holds
//     16 / group tokens; it normalises and rotates its q rows itself (per-head
//     RMSNorm with its gain, half-rotation RoPE at the token's position, bf16
//     like the decode path) into shared memory, then A fragments;
//   * K/V tiles of 32 positions come by bulk copies (the cache's chunk
//     swizzle lands them conflict-free for ldmatrix) into a 3-deep ring,
//     up to the CTA's last position; S = Q K^T (m16n8k16, fp32), the causal
//     mask per row, online softmax in fp32, O += P V with P in two 16-bit
//     halves (P = P_hi + P_lo) as in the decode kernel, so the sums keep fp32
//     accuracy; o / l in bf16.
// Every mbarrier wait is bounded.
#pragma once

#include "attention.cuh"

namespace m3 {

constexpr int kApWarps = 4;
constexpr int kApKT = 32;    // positions per K/V tile
constexpr int kApBuf = 3;    // K/V tiles in flight

template <int D>
__host__ __device__ constexpr size_t attn_prefill_smem() {
  return (size_t)kApWarps * 16 * D * 2          // q rows
         + (size_t)kApBuf * 2 * kApKT * D * 2  // K, V tiles
         + kApBuf * sizeof(uint64_t);
}

// Query rows a CTA covers: 16 per warp.
__host__ __device__ constexpr int attn_prefill_rows() { return kApWarps * 16; }

template <int D, int KVF16>
__global__ void __launch_bounds__(kApWarps * 32)
    attn_prefill_kernel(const AttnArgs a, int T) {
  constexpr int ROWB = D * 2;        // bytes per position (or q) row
  constexpr int KS = D / 16;         // k-steps of Q K^T
  constexpr int NTO = D / 8;         // n-tiles of O
  constexpr int VPL = D / 32;        // dims per lane in the q preparation
  constexpr int TILE_ELEMS = kApKT * D;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint16_t* qs = reinterpret_cast<uint16_t*>(smem);                   // [4 warps][16][D]
  uint16_t* kt = qs + kApWarps * 16 * D;                               // [BUF][KT][D]
  uint16_t* vt = kt + kApBuf * TILE_ELEMS;                             // [BUF][KT][D]
  uint64_t* bars = reinterpret_cast<uint64_t*>(vt + kApBuf * TILE_ELEMS);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grp = a.Hq / a.Hkv, tpw = 16 / grp;   // tokens per warp
  const int g = blockIdx.y;
  // heavy tiles (late tokens, long contexts) first
  const int tile = (int)gridDim.x - 1 - (int)blockIdx.x;
  const int t0 = tile * kApWarps * tpw;           // first token of the CTA
  const int tw0 = t0 + warp * tpw;                // first token of the warp
  const int t_last = min(T, t0 + kApWarps * tpw) - 1;
  const int p0 = a.fixed_pos;
  const int n_pos = p0 + t_last + 1;              // positions the CTA reads
  const int ntiles = (n_pos + kApKT - 1) / kApKT;
  const unsigned long long* pt = a.pages + (size_t)a.layer * a.max_pages;  // the row's pages

  auto issue_tile = [&](int t) {
    const int js = t * kApKT;
    const int nv = min(kApKT, n_pos - js);
    const int page = js / a.page_size, off = js % a.page_size;
    const uint16_t* base = reinterpret_cast<const uint16_t*>(pt[page]);
    const uint32_t bytes = (uint32_t)(nv * ROWB);
    const int b = t % kApBuf;
    mbar_arrive_expect_tx(&bars[b], 2 * bytes);
    bulk_g2s_nohint(kt + b * TILE_ELEMS, base + ((size_t)g * a.page_size + off) * D, bytes, &bars[b]);
    bulk_g2s_nohint(vt + b * TILE_ELEMS, base + ((size_t)(a.Hkv + g) * a.page_size + off) * D,
                    bytes, &bars[b]);
  };
  if (tid == 0) {
    for (int b = 0; b < kApBuf; ++b) mbar_init(&bars[b], 1);
    fence_barrier_init();
    for (int t = 0; t < min(kApBuf, ntiles); ++t) issue_tile(t);
  }

  // ---- this warp's q rows: RMSNorm (gain q_norm), RoPE at the token's
  // position, bf16 (then the cache's type for the MMA) ------------------------
  const float scale = 1.0f / sqrtf((float)D);
  uint16_t* qw = qs + (size_t)warp * 16 * D;
  for (int r = 0; r < 16; ++r) {
    const int t = tw0 + r / grp, h = g * grp + r % grp;
    float v[VPL];
    if (t < T) {
      const __nv_bfloat16* src = a.qkv + (size_t)t * a.ldqkv + (size_t)h * D;
#pragma unroll
      for (int i = 0; i < VPL; ++i) v[i] = __bfloat162float(__ldcg(src + lane + 32 * i));
      float ss = 0.0f;
#pragma unroll
      for (int i = 0; i < VPL; ++i) ss = fmaf(v[i], v[i], ss);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float inv = 1.0f / sqrtf(ss / (float)D + a.eps);
#pragma unroll
      for (int i = 0; i < VPL; ++i)
        v[i] = round_bf16(__bfloat162float(a.q_norm[lane + 32 * i]) * round_bf16(v[i] * inv));
#pragma unroll
      for (int i = 0; i < VPL / 2; ++i) {
        const float2 cs = a.rope[(size_t)t * a.rope_ld + lane + 32 * i];
        const float x0 = v[i], x1 = v[i + VPL / 2];
        v[i] = __fsub_rn(__fmul_rn(x0, cs.x), __fmul_rn(x1, cs.y));
        v[i + VPL / 2] = __fadd_rn(__fmul_rn(x1, cs.x), __fmul_rn(x0, cs.y));
      }
#pragma unroll
      for (int i = 0; i < VPL; ++i) v[i] = round_bf16(v[i]);
    } else {
#pragma unroll
      for (int i = 0; i < VPL; ++i) v[i] = 0.0f;
    }
    // row r of the warp's q tile, in the swizzle the K tiles use
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int d = lane + 32 * i;
      qw[r * D + ((((d >> 3) ^ (r & 7))) << 3) + (d & 7)] = f32_to_kv<KVF16>(v[i]);
    }
  }
  __syncwarp();
  uint32_t qa[KS][4];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    const int r = lane & 15, ch = ks * 2 + (lane >> 4);
    ldsm_x4(smem_u32(qw) + r * ROWB + ((ch ^ (r & 7)) << 4), qa[ks][0], qa[ks][1], qa[ks][2],
            qa[ks][3]);
  }
  __syncthreads();  // the ring's barriers are initialised

  // rows gid and gid + 8 of the warp: their positions (causal limits)
  const int gid = lane >> 2, tig = lane & 3;
  const int pos_a = p0 + tw0 + gid / grp, pos_b = p0 + tw0 + (gid + 8) / grp;
  float o[NTO][4];
#pragma unroll
  for (int j = 0; j < NTO; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.0f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.0f, 0.0f};
  const int warp_last = p0 + min(T - 1, tw0 + tpw - 1);  // the warp's last position

  for (int t = 0; t < ntiles; ++t) {
    const int b = t % kApBuf;
    mbar_wait(&bars[b], (t / kApBuf) & 1, a.err);
    const int js = t * kApKT;
    const int nv = min(kApKT, n_pos - js);
    if (nv < kApKT) {
      // rows past the end of the last tile hold stale (or never written)
      // shared memory: zero them, so that p = 0 never multiplies a NaN pattern
      uint4* kz = reinterpret_cast<uint4*>(kt + b * TILE_ELEMS);
      uint4* vz = reinterpret_cast<uint4*>(vt + b * TILE_ELEMS);
      for (int c = nv * (D / 8) + tid; c < kApKT * (D / 8); c += kApWarps * 32) {
        kz[c] = make_uint4(0u, 0u, 0u, 0u);
        vz[c] = make_uint4(0u, 0u, 0u, 0u);
      }
      __syncthreads();
    }
    if (js <= warp_last) {
      const uint32_t kb = smem_u32(kt + b * TILE_ELEMS), vb = smem_u32(vt + b * TILE_ELEMS);
      // S = Q K^T: 4 n-tiles of 8 positions
      float s[4][4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.0f;
        const int prow = 8 * j + (lane & 7);
#pragma unroll
        for (int kk = 0; kk < KS; kk += 2) {
          const int ch = 2 * kk + (lane >> 3);
          uint32_t b0, b1, b2, b3;
          ldsm_x4(kb + prow * ROWB + ((ch ^ (prow & 7)) << 4), b0, b1, b2, b3);
          mma16816<KVF16>(s[j], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b0, b1);
          mma16816<KVF16>(s[j], qa[kk + 1][0], qa[kk + 1][1], qa[kk + 1][2], qa[kk + 1][3], b2, b3);
        }
      }
      // causal mask per row (positions past the row's own, or past the tile)
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int p = js + 8 * j + 2 * tig + (e & 1);
          const bool ok = (p - js) < nv && p <= ((e >> 1) ? pos_b : pos_a);
          s[j][e] = ok ? s[j][e] * scale : -INFINITY;
          mx[e >> 1] = fmaxf(mx[e >> 1], s[j][e]);
        }
      float corr[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
        const float mn = fmaxf(m_run[h], mx[h]);
        corr[h] = mn == -INFINITY ? 1.0f : expf(m_run[h] - mn);  // 0 when m_run = -inf
        m_run[h] = mn;
      }
      float ls[2] = {0.0f, 0.0f};
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float mm = m_run[e >> 1];
          const float pe = (s[j][e] == -INFINITY) ? 0.0f : expf(s[j][e] - mm);
          s[j][e] = pe;
          ls[e >> 1] += pe;
        }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        ls[h] += __shfl_xor_sync(0xffffffffu, ls[h], 1);
        ls[h] += __shfl_xor_sync(0xffffffffu, ls[h], 2);
        l_run[h] = l_run[h] * corr[h] + ls[h];
      }
#pragma unroll
      for (int j = 0; j < NTO; ++j) {
        o[j][0] *= corr[0];
        o[j][1] *= corr[0];
        o[j][2] *= corr[1];
        o[j][3] *= corr[1];
      }
      // O += P V over two k-steps of 16 positions, P = P_hi + P_lo
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        const uint32_t h0 = pack2<KVF16>(s[2 * kk][0], s[2 * kk][1]);
        const uint32_t h1 = pack2<KVF16>(s[2 * kk][2], s[2 * kk][3]);
        const uint32_t h2 = pack2<KVF16>(s[2 * kk + 1][0], s[2 * kk + 1][1]);
        const uint32_t h3 = pack2<KVF16>(s[2 * kk + 1][2], s[2 * kk + 1][3]);
        const float2 f0 = unpack2<KVF16>(h0), f1 = unpack2<KVF16>(h1);
        const float2 f2 = unpack2<KVF16>(h2), f3 = unpack2<KVF16>(h3);
        const uint32_t l0 = pack2<KVF16>(s[2 * kk][0] - f0.x, s[2 * kk][1] - f0.y);
        const uint32_t l1 = pack2<KVF16>(s[2 * kk][2] - f1.x, s[2 * kk][3] - f1.y);
        const uint32_t l2 = pack2<KVF16>(s[2 * kk + 1][0] - f2.x, s[2 * kk + 1][1] - f2.y);
        const uint32_t l3 = pack2<KVF16>(s[2 * kk + 1][2] - f3.x, s[2 * kk + 1][3] - f3.y);
        const int prow = 16 * kk + (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
        for (int j = 0; j < NTO; j += 2) {
          const int ch = j + (lane >> 4);
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(vb + prow * ROWB + ((ch ^ (prow & 7)) << 4), b0, b1, b2, b3);
          mma16816<KVF16>(o[j], h0, h1, h2, h3, b0, b1);
          mma16816<KVF16>(o[j], l0, l1, l2, l3, b0, b1);
          mma16816<KVF16>(o[j + 1], h0, h1, h2, h3, b2, b3);
          mma16816<KVF16>(o[j + 1], l0, l1, l2, l3, b2, b3);
        }
      }
    }
    __syncthreads();  // every warp is done with buffer b
    if (tid == 0 && t + kApBuf < ntiles) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // reads before the refill
      issue_tile(t + kApBuf);
    }
  }

  // o / l in bf16: rows gid and gid + 8 of the warp's 16
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int r = gid + 8 * h;
    const int t = tw0 + r / grp, hd = g * grp + r % grp;
    if (t >= T) continue;
    __nv_bfloat16* orow = a.out + (size_t)t * a.Hq * D + (size_t)hd * D;
#pragma unroll
    for (int j = 0; j < NTO; ++j) {
      const int d = j * 8 + 2 * tig;
      *reinterpret_cast<__nv_bfloat162*>(orow + d) =
          __floats2bfloat162_rn(o[j][2 * h] / l_run[h], o[j][2 * h + 1] / l_run[h]);
    }
  }
}

// The chunk's K/V into the row's cache before attn_prefill_kernel reads them:
// one warp per (token, KV head), the decode path's arithmetic (per-head
// RMSNorm with the k gain, RoPE at the token's position, bf16, then the
// cache's type; v converted as is).
template <int D, int KVF16>
__global__ void __launch_bounds__(256) kv_append_kernel(const AttnArgs a, int T) {
  constexpr int VPL = D / 32;
  const int lane = threadIdx.x & 31;
  const int item = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (item >= T * a.Hkv) return;
  const int t = item / a.Hkv, g = item % a.Hkv;
  const int pos = a.fixed_pos + t;
  const __nv_bfloat16* row = a.qkv + (size_t)t * a.ldqkv;
  const __nv_bfloat16* kraw = row + (size_t)a.Hq * D + (size_t)g * D;
  const __nv_bfloat16* vraw = row + (size_t)(a.Hq + a.Hkv) * D + (size_t)g * D;
  float k[VPL], v[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    k[i] = __bfloat162float(__ldcg(kraw + lane + 32 * i));
    v[i] = __bfloat162float(__ldcg(vraw + lane + 32 * i));
  }
  float ss = 0.0f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) ss = fmaf(k[i], k[i], ss);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = 1.0f / sqrtf(ss / (float)D + a.eps);
#pragma unroll
  for (int i = 0; i < VPL; ++i)
    k[i] = round_bf16(__bfloat162float(a.k_norm[lane + 32 * i]) * round_bf16(k[i] * inv));
#pragma unroll
  for (int i = 0; i < VPL / 2; ++i) {
    const float2 cs = a.rope[(size_t)t * a.rope_ld + lane + 32 * i];
    const float x0 = k[i], x1 = k[i + VPL / 2];
    k[i] = __fsub_rn(__fmul_rn(x0, cs.x), __fmul_rn(x1, cs.y));
    k[i + VPL / 2] = __fadd_rn(__fmul_rn(x1, cs.x), __fmul_rn(x0, cs.y));
  }
  const unsigned long long* pt = a.pages + (size_t)a.layer * a.max_pages;  // the row's pages
  uint16_t* base = reinterpret_cast<uint16_t*>(pt[pos / a.page_size]);
  const int off = pos % a.page_size;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int dim = lane + 32 * i;
    base[kv_elem_offset(g, a.page_size, off, D, dim)] = f32_to_kv<KVF16>(round_bf16(k[i]));
    base[kv_elem_offset(a.Hkv + g, a.page_size, off, D, dim)] = f32_to_kv<KVF16>(v[i]);
  }
}

}  // namespace m3
