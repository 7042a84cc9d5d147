// depth.cu -- the RVQ depth decoder as one persistent kernel (depth.cuh).
//
// One CTA per SM runs the decoder's whole chain of steps: the input
// projection, then for each of the NC + 1 frame-local positions and each
// layer the fused QKV projection, the attention, the O projection (+ the
// residual), gate/up (+ SwiGLU) and down (+ the residual), and after every
// position j >= 1 the codebook head j with the guided Gumbel-argmax draw
// (DiffSynth-Studio article, "第二阶段"; the draw of "MiniMax Music 3 modular
// pipeline", finding 3).
//
// What keeps a step short:
//   * no grid barrier: every value another CTA reads is written as a tagged
//     32-bit word (bf16 value, 16-bit tag = 1 + the writing step's number;
//     the buffers are cleared to tag 0 before each launch) and the reader
//     polls exactly the words it needs until they carry the expected tag --
//     a step waits only for its own inputs, one L2 round trip after they
//     land. It is sound because every reader of a buffer is upstream of the
//     buffer's next writer (the next write needs data the reader produces);
//   * each CTA owns a fixed slice of 16-row tiles of every projection and
//     copies the slice of the NEXT projection into shared memory (bulk
//     copies, mbarrier transaction counts) while the current one runs;
//   * the slice's dot products run on the tensor cores (m16n8k16 bf16 MMA,
//     the int8 weights widened exactly to bf16, fp32 sums, one group-128
//     scale per 8 MMAs), K split over the warps, partial sums reduced in a
//     fixed order (deterministic);
//   * RMSNorms are recomputed by every CTA from the staged rows, each CTA
//     keeps its own slice of the residual stream in shared memory, and with
//     few (row, head) pairs the attention itself runs inside the O
//     projection's step, two pairs per warp.
// The roundings are those of the per-launch kernels and of the oracle: bf16
// activations between steps, fp32 norms, RoPE, softmax and sums.
#include <climits>
#include <cuda_runtime.h>

#include "common.cuh"
#include "depth.cuh"
#include "noise.cuh"

namespace m3 {

namespace {

// Polls of one tagged word before a wait gives up (each poll is one L2
// round trip, well under a microsecond): seconds, far beyond any healthy
// wait.
constexpr long long kDepthSpinLimit = 1ll << 21;

// ------------------------------------------------------------ tagged words --
__device__ __forceinline__ uint4 ld_words4(const uint32_t* p) {
  uint4 v;
  asm volatile("ld.volatile.global.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p)
               : "memory");
  return v;
}

__device__ __forceinline__ unsigned long long ld_u64v(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.volatile.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_words4(uint32_t* p, uint4 v) {
  asm volatile("st.volatile.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}

__device__ __forceinline__ void st_u64v(unsigned long long* p, unsigned long long v) {
  asm volatile("st.volatile.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ uint32_t bf16_bits(float v) {
  const __nv_bfloat16 b = __float2bfloat16_rn(v);
  return (uint32_t)*reinterpret_cast<const uint16_t*>(&b);
}

// four values (already bf16) as tagged words
__device__ __forceinline__ uint4 tag4(float v0, float v1, float v2, float v3, uint32_t tag) {
  const uint32_t t = tag << 16;
  return make_uint4(t | bf16_bits(v0), t | bf16_bits(v1), t | bf16_bits(v2), t | bf16_bits(v3));
}

__device__ __forceinline__ bool tags_are(const uint4& w, uint32_t tag) {
  return ((w.x >> 16) == tag) & ((w.y >> 16) == tag) & ((w.z >> 16) == tag) & ((w.w >> 16) == tag);
}

__device__ __forceinline__ float word_value(uint32_t w) { return __uint_as_float(w << 16); }

// Poll until the four words at p carry `tag`, from a first load w (bounded:
// past the limit an error word is set; once any wait has given up, the
// others give up at once).
__device__ __forceinline__ void wait_words4(const uint32_t* p, uint32_t tag, uint4& w, int* err) {
  for (long long spin = 0; !tags_are(w, tag); ++spin) {
    if ((spin & 255) == 255) {
      if (spin >= kDepthSpinLimit) {
        record_error(err, kErrTimeout);
        return;
      }
      if (*reinterpret_cast<volatile int*>(err) != 0) return;
    }
    w = ld_words4(p);
  }
}

// Tag of step ph: 1 + ph (never 0, the value of every word when the launch
// starts; a launch has at most 1 + 32 * 8 * 5 + 31 steps).
struct Sched {
  int L, S, merge;
  __device__ __forceinline__ uint32_t tag(int ph) const { return 1u + (uint32_t)ph; }
  // step ids: 0 the input projection; per position j, per layer l: QKV,
  // [attention,] O, gate/up, down; for j >= 1 then the head of codebook j
  __device__ __forceinline__ int pos0(int j) const { return 1 + j * L * S + (j > 0 ? j - 1 : 0); }
  __device__ __forceinline__ int qkv(int j, int l) const { return pos0(j) + l * S; }
  __device__ __forceinline__ int attn(int j, int l) const { return pos0(j) + l * S + 1; }
  __device__ __forceinline__ int o(int j, int l) const { return pos0(j) + l * S + S - 3; }
  __device__ __forceinline__ int gu(int j, int l) const { return pos0(j) + l * S + S - 2; }
  __device__ __forceinline__ int down(int j, int l) const { return pos0(j) + l * S + S - 1; }
  __device__ __forceinline__ int head(int j) const { return pos0(j) + L * S; }
  // the step that writes the keys and values of position p
  __device__ __forceinline__ int kv(int p, int l) const { return merge ? o(p, l) : attn(p, l); }
};

// Tiles [t0, t0 + nt) of a projection with N outputs (N / 16 tiles): the
// first T % grid CTAs hold one tile more.
__device__ __forceinline__ void cta_tiles(int N, int& t0, int& nt) {
  const int T = N >> 4, G = gridDim.x, b = blockIdx.x;
  const int q = T / G, r = T % G;
  nt = q + (b < r ? 1 : 0);
  t0 = b * q + min(b, r);
}

// One projection of the chain and the static vectors copied with its slice.
struct Proj {
  DepthMat W;
  int N, K;
  const void* side[3];
  uint32_t side_bytes[3];
};

// Projections in the order the kernel runs them: 0 the input projection;
// then per position j the layers' QKV (+ the attention norm's gain), O (+ the
// q/k norm gains and the RoPE row of position j), gate/up (+ the MLP norm's
// gain), down, and for j >= 1 the head of codebook j (+ the final norm's gain).
__device__ __forceinline__ int proj_count(const DepthArgs& a) {
  return 1 + (a.NC + 1) * 4 * a.n_layers + a.NC;
}

__device__ __forceinline__ Proj proj_at(const DepthArgs& a, int gi) {
  Proj p{};
  const int QN = a.nh * a.hd;
  if (gi == 0) {
    p.W = a.proj;
    p.N = a.Dh;
    p.K = a.Hin;
    return p;
  }
  int r = gi - 1;
  for (int j = 0; j <= a.NC; ++j) {
    const int per = 4 * a.n_layers + (j >= 1 ? 1 : 0);
    if (r < per) {
      if (r < 4 * a.n_layers) {
        const int l = r >> 2;
        switch (r & 3) {
          case 0:
            p.W = a.L[l].qkv; p.N = 3 * QN; p.K = a.Dh;
            p.side[0] = a.L[l].attn_norm; p.side_bytes[0] = 2u * a.Dh;
            break;
          case 1:
            p.W = a.L[l].o; p.N = a.Dh; p.K = QN;
            p.side[0] = a.L[l].q_norm; p.side_bytes[0] = 2u * a.hd;
            p.side[1] = a.L[l].k_norm; p.side_bytes[1] = 2u * a.hd;
            p.side[2] = a.rope + (size_t)j * (a.hd / 2); p.side_bytes[2] = 4u * a.hd;
            break;
          case 2:
            p.W = a.L[l].gu; p.N = 2 * a.F; p.K = a.Dh;
            p.side[0] = a.L[l].mlp_norm; p.side_bytes[0] = 2u * a.Dh;
            break;
          default:
            p.W = a.L[l].d; p.N = a.Dh; p.K = a.F;
            break;
        }
      } else {
        p.W = a.heads[j - 1];
        p.N = a.V;
        p.K = a.Dh;
        p.side[0] = a.final_norm;
        p.side_bytes[0] = 2u * a.Dh;
      }
      return p;
    }
    r -= per;
  }
  return p;
}

// Shared-memory slot of projection gi's slice: even projections from the
// bottom of the weight region, odd ones from the top, so two consecutive
// slices never overlap.
__device__ __forceinline__ uint8_t* slot_base(const DepthArgs& a, uint8_t* wb, int gi, int nt,
                                              int K) {
  return wb + ((gi & 1) ? a.wb_bytes - depth_slice_bytes(nt, K, a.side_bytes) : 0);
}

// The slot's static vectors start after the rows and the scales.
__device__ __forceinline__ const uint8_t* slot_side(const uint8_t* slot, int nt, int K) {
  return slot + (size_t)16 * nt * (K + 64) + (size_t)16 * nt * (K / 128) * 4;
}

// Warp 0: bulk copies of this CTA's slice of projection gi (rows padded to
// K + 64 bytes, the scales, the static vectors), completing on wbar[gi & 1].
__device__ __forceinline__ void issue_slice(const DepthArgs& a, uint8_t* wb, uint64_t* wbar,
                                            int gi) {
  if (gi >= proj_count(a)) return;
  const Proj p = proj_at(a, gi);
  int t0, nt;
  cta_tiles(p.N, t0, nt);
  if (nt == 0) return;
  const int lane = threadIdx.x & 31;
  uint8_t* dst = slot_base(a, wb, gi, nt, p.K);
  const int nrow = 16 * nt, ng = p.K >> 7;
  const uint32_t wbytes = (uint32_t)nrow * (uint32_t)p.K, sbytes = (uint32_t)(nrow * ng * 4);
  const uint32_t vbytes = p.side_bytes[0] + p.side_bytes[1] + p.side_bytes[2];
  uint64_t* bar = &wbar[gi & 1];
  if (lane == 0) mbar_arrive_expect_tx(bar, wbytes + sbytes + vbytes);
  __syncwarp();
  const int8_t* src = p.W.q + (size_t)t0 * 16 * p.K;
  for (int r = lane; r < nrow; r += 32)
    bulk_g2s_nohint(dst + (size_t)r * (p.K + 64), src + (size_t)r * p.K, (uint32_t)p.K, bar);
  if (lane == 0) {
    uint8_t* sd = dst + (size_t)nrow * (p.K + 64);
    bulk_g2s_nohint(sd, p.W.s + (size_t)t0 * 16 * ng, sbytes, bar);
    sd += sbytes;
    for (int i = 0; i < 3; ++i)
      if (p.side_bytes[i]) {
        bulk_g2s_nohint(sd, p.side[i], p.side_bytes[i], bar);
        sd += p.side_bytes[i];
      }
  }
}

// RMSNorm in place over staged rows whose sums of squares are in sred
// (per 64 inputs, in order): bf16(gamma * bf16(v / rms)), gamma in shared
// memory.
__device__ __forceinline__ void norm_rows(__nv_bfloat16* xs, int rp, int K,
                                          const __nv_bfloat16* gamma, float eps,
                                          const float* sred, float* rinv) {
  const int k8 = K >> 3, xk = K + 8, per = K >> 6;
  if (threadIdx.x < rp) {
    float s = 0.0f;
    for (int q = 0; q < per; ++q) s += sred[threadIdx.x * per + q];
    rinv[threadIdx.x] = 1.0f / sqrtf(s / (float)K + eps);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < rp * k8; i += kDepthThreads) {
    const int m = i / k8, c = i - m * k8;
    uint4* p = reinterpret_cast<uint4*>(xs + (size_t)m * xk + 8 * c);
    const uint4 v = *p;
    const uint4 gv = *reinterpret_cast<const uint4*>(gamma + 8 * c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w}, g[4] = {gv.x, gv.y, gv.z, gv.w};
    const float r = rinv[m];
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float lo, hi, glo, ghi;
      bf16x2_to_f32(w[q], lo, hi);
      bf16x2_to_f32(g[q], glo, ghi);
      const __nv_bfloat162 b =
          __floats2bfloat162_rn(glo * round_bf16(lo * r), ghi * round_bf16(hi * r));
      o[q] = *reinterpret_cast<const uint32_t*>(&b);
    }
    *p = make_uint4(o[0], o[1], o[2], o[3]);
  }
  __syncthreads();
}

// Sum of squares of four values over 16 lanes (a half-warp: 64 inputs of
// one row when 64 | K), stored by the half's first lane.
__device__ __forceinline__ void half_ss(float f0, float f1, float f2, float f3, bool ok, int i,
                                        float* sred) {
  float s = fmaf(f0, f0, 0.0f);
  s = fmaf(f1, f1, s);
  s = fmaf(f2, f2, s);
  s = fmaf(f3, f3, s);
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (ok && (threadIdx.x & 15) == 0) sred[i >> 4] = s;
}

// Rows 0..rp-1 of a step's input into xs [rp][K + 8] (bf16), from tagged
// words [rp][ld] each waited for until it carries `tag`; RMSNormed with a
// gain (shared memory) when gamma is non-null.
__device__ __forceinline__ void stage_tagged(const uint32_t* base, int ld, int rp, int K,
                                             uint32_t tag, const __nv_bfloat16* gamma, float eps,
                                             __nv_bfloat16* xs, float* sred, float* rinv,
                                             int* err) {
  const int k4 = K >> 2, xk = K + 8, total = rp * k4;
  for (int b0 = threadIdx.x & ~31; b0 < total; b0 += kDepthThreads) {
    const int i = b0 + (threadIdx.x & 31);
    const bool ok = i < total;
    const int m = ok ? i / k4 : 0, c = i - m * k4;
    uint4 w = make_uint4(0u, 0u, 0u, 0u);
    if (ok) {
      const uint32_t* p = base + (size_t)m * ld + 4 * c;
      w = ld_words4(p);
      wait_words4(p, tag, w, err);
      *reinterpret_cast<uint2*>(xs + (size_t)m * xk + 4 * c) =
          make_uint2((w.x & 0xFFFFu) | (w.y << 16), (w.z & 0xFFFFu) | (w.w << 16));
    }
    if (gamma)
      half_ss(word_value(w.x), word_value(w.y), word_value(w.z), word_value(w.w), ok, i, sred);
  }
  __syncthreads();
  if (gamma) norm_rows(xs, rp, K, gamma, eps, sred, rinv);
}

// The same from plain bf16 rows (src[m], null for a zero row) that no step
// of this launch writes (the frame's hidden state, embedding tables).
__device__ __forceinline__ void stage_plain(const __nv_bfloat16* const* src, int rp, int K,
                                            const __nv_bfloat16* gamma, float eps,
                                            __nv_bfloat16* xs, float* sred, float* rinv) {
  const int k4 = K >> 2, xk = K + 8, total = rp * k4;
  for (int b0 = threadIdx.x & ~31; b0 < total; b0 += kDepthThreads) {
    const int i = b0 + (threadIdx.x & 31);
    const bool ok = i < total;
    const int m = ok ? i / k4 : 0, c = i - m * k4;
    uint2 v = make_uint2(0u, 0u);
    if (ok) {
      if (src[m]) v = *reinterpret_cast<const uint2*>(src[m] + 4 * c);
      *reinterpret_cast<uint2*>(xs + (size_t)m * xk + 4 * c) = v;
    }
    if (gamma)
      half_ss(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u),
              __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xFFFF0000u), ok, i, sred);
  }
  __syncthreads();
  if (gamma) norm_rows(xs, rp, K, gamma, eps, sred, rinv);
}

__device__ __forceinline__ void mma_bf16_16816(float* c, const uint32_t* a, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Four int8 -> two exact bf16 pairs (bytes 0, 1) and (2, 3).
__device__ __forceinline__ void s8x4_to_bf16x2(uint32_t w, uint32_t& p01, uint32_t& p23) {
  uint64_t f01, f23;
  s8x4_to_f32x2(w, f01, f23);
  p01 = f32x2_to_bf16x2(f01);
  p23 = f32x2_to_bf16x2(f23);
}

// ys[m][16 nt] = the CTA's nt tiles of the projection applied to the staged
// rows 0..rp-1 of xs [rp][K + 8].
//
// Warp w takes tile w % nt and the groups of 128 inputs g = w / nt (mod
// 16 / nt). Within a 64-input block, lane (gid, tig) loads inputs
// 16 tig .. 16 tig + 15 of weight rows gid and gid + 8 and of activation row
// gid; MMA step s of the block uses inputs 16 tig + 4 s .. + 3 as the
// fragment columns 2 tig, 2 tig + 1, 2 tig + 8, 2 tig + 9 -- one fixed
// permutation of the 16 inputs of the step for A and B alike, which the dot
// product does not see.
template <int NB>
__device__ __forceinline__ void tile_dots(const uint8_t* wq, int nt, int K,
                                          const __nv_bfloat16* xs, int rp, float* part,
                                          float* ys) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
  const int nsub = kDepthWarps / nt, t = warp % nt, sub = warp / nt;
  const int ng = K >> 7, xk = K + 8;
  const float* wsc = reinterpret_cast<const float*>(wq + (size_t)16 * nt * (K + 64));
  float tot[NB][4];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb)
#pragma unroll
    for (int c = 0; c < 4; ++c) tot[nb][c] = 0.0f;
  if (sub < nsub) {
    const uint8_t* wlo = wq + (size_t)(16 * t + gid) * (K + 64) + 16 * tig;
    const uint8_t* whi = wlo + (size_t)8 * (K + 64);
    const float* slo = wsc + (size_t)(16 * t + gid) * ng;
    const float* shi = slo + 8 * ng;
    for (int g = sub; g < ng; g += nsub) {
      float acc[NB][4];
#pragma unroll
      for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[nb][c] = 0.0f;
#pragma unroll
      for (int blk = 0; blk < 2; ++blk) {
        const int k0 = 128 * g + 64 * blk;
        const uint4 alo = *reinterpret_cast<const uint4*>(wlo + k0);
        const uint4 ahi = *reinterpret_cast<const uint4*>(whi + k0);
        uint4 b0[NB], b1[NB];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
          const int m = nb * 8 + gid;
          if (m < rp) {
            const __nv_bfloat16* xr = xs + (size_t)m * xk + k0 + 16 * tig;
            b0[nb] = *reinterpret_cast<const uint4*>(xr);
            b1[nb] = *reinterpret_cast<const uint4*>(xr + 8);
          } else {
            b0[nb] = make_uint4(0u, 0u, 0u, 0u);
            b1[nb] = b0[nb];
          }
        }
        const uint32_t al[4] = {alo.x, alo.y, alo.z, alo.w};
        const uint32_t ah[4] = {ahi.x, ahi.y, ahi.z, ahi.w};
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          uint32_t A[4];
          s8x4_to_bf16x2(al[s], A[0], A[2]);
          s8x4_to_bf16x2(ah[s], A[1], A[3]);
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) {
            const uint4& bv = s < 2 ? b0[nb] : b1[nb];
            const uint32_t B0 = (s & 1) ? bv.z : bv.x;
            const uint32_t B1 = (s & 1) ? bv.w : bv.y;
            mma_bf16_16816(acc[nb], A, B0, B1);
          }
        }
      }
      const float sl = slo[g], sh = shi[g];
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        tot[nb][0] = fmaf(sl, acc[nb][0], tot[nb][0]);
        tot[nb][1] = fmaf(sl, acc[nb][1], tot[nb][1]);
        tot[nb][2] = fmaf(sh, acc[nb][2], tot[nb][2]);
        tot[nb][3] = fmaf(sh, acc[nb][3], tot[nb][3]);
      }
    }
  }
#pragma unroll
  for (int nb = 0; nb < NB; ++nb)
    *reinterpret_cast<float4*>(part + ((size_t)(warp * NB + nb) * 32 + lane) * 4) =
        make_float4(tot[nb][0], tot[nb][1], tot[nb][2], tot[nb][3]);
  __syncthreads();
  // fixed-order sum over the warps of each tile; C fragment (gid, tig, c):
  // weight row gid (+ 8 for c >= 2), activation row 2 tig + (c & 1)
  const int n16 = 16 * nt;
  for (int i = threadIdx.x; i < nt * NB * 128; i += kDepthThreads) {
    const int t2 = i / (NB * 128), rem = i - t2 * NB * 128;
    const int nb = rem >> 7, l2 = (rem & 127) >> 2, c = rem & 3;
    const int m = nb * 8 + 2 * (l2 & 3) + (c & 1);
    if (m >= rp) continue;
    float y = 0.0f;
    for (int s2 = 0; s2 < nsub; ++s2)
      y += part[((size_t)((s2 * nt + t2) * NB + nb) * 32 + l2) * 4 + c];
    const int row = (l2 >> 2) + (c >= 2 ? 8 : 0);
    ys[(size_t)m * n16 + 16 * t2 + row] = y;
  }
  __syncthreads();
}

// Attention of (row m, head h) at position j of layer l by one half-warp
// (lane e of the half holds dims VP e .. VP e + VP - 1, VP = HD / 16): q/k
// RMSNorm (gains gq, gk) and RoPE at position j ((cos, sin) pairs `rope`)
// with the roundings of the decode attention kernel; the key and value of
// position j stored as tagged words when write_kv; softmax attention over
// positions 0..j, a chunk of positions at a time: their dot products reduced
// together, the weights exp(s - max) summed in position order (as the oracle
// does within a chunk; chunks merged by rescaling). The head's output: bf16
// at out_x[0..HD), or tagged words at out_w[0..HD).
template <int HD>
__device__ __forceinline__ void attend(const DepthArgs& a, const Sched& sc, int l, int j, int m,
                                       int h, const __nv_bfloat16* gq, const __nv_bfloat16* gk,
                                       const float2* rope, __nv_bfloat16* out_x, uint32_t* out_w,
                                       uint32_t out_tag, bool write_kv) {
  constexpr int VP = HD / 16, VQ = VP / 4;  // dims per lane, their 16-byte groups
  constexpr int CH = HD == 64 ? 4 : 2;      // earlier positions fetched together
  const int e = threadIdx.x & 15;
  const unsigned hm = 0xFFFFu << (threadIdx.x & 16);  // this half-warp
  const int QN = a.nh * HD;
  const uint32_t* qw = a.qkvw + (size_t)m * 3 * QN + (size_t)h * HD + VP * e;
  uint32_t* kvb =
      a.kvw + ((size_t)m * a.n_layers + l) * (size_t)(a.NC + 1) * 2 * QN + (size_t)h * HD + VP * e;
  const uint32_t tq = sc.tag(sc.qkv(j, l));
  uint4 wq[VQ], wk[VQ], wv[VQ], ck[CH][VQ], cv[CH][VQ];
  // every load first: q, k, v of position j and the first chunk of earlier
  // positions' keys and values, then their tags
#pragma unroll
  for (int u = 0; u < VQ; ++u) {
    wq[u] = ld_words4(qw + 4 * u);
    wk[u] = ld_words4(qw + QN + 4 * u);
    wv[u] = ld_words4(qw + 2 * QN + 4 * u);
  }
  auto fetch = [&](int p0) {
#pragma unroll
    for (int t = 0; t < CH; ++t)
#pragma unroll
      for (int u = 0; u < VQ; ++u)
        if (p0 + t < j) {
          ck[t][u] = ld_words4(kvb + (size_t)(p0 + t) * 2 * QN + 4 * u);
          cv[t][u] = ld_words4(kvb + (size_t)(p0 + t) * 2 * QN + QN + 4 * u);
        }
  };
  auto check = [&](int p0) {
#pragma unroll
    for (int t = 0; t < CH; ++t)
      if (p0 + t < j) {
        const uint32_t tp = sc.tag(sc.kv(p0 + t, l));
#pragma unroll
        for (int u = 0; u < VQ; ++u) {
          wait_words4(kvb + (size_t)(p0 + t) * 2 * QN + 4 * u, tp, ck[t][u], a.err);
          wait_words4(kvb + (size_t)(p0 + t) * 2 * QN + QN + 4 * u, tp, cv[t][u], a.err);
        }
      }
  };
  fetch(0);
#pragma unroll
  for (int u = 0; u < VQ; ++u) {
    wait_words4(qw + 4 * u, tq, wq[u], a.err);
    wait_words4(qw + QN + 4 * u, tq, wk[u], a.err);
    wait_words4(qw + 2 * QN + 4 * u, tq, wv[u], a.err);
  }
  float q[VP], k[VP], v[VP];
#pragma unroll
  for (int u = 0; u < VQ; ++u) {
    const uint32_t aq[4] = {wq[u].x, wq[u].y, wq[u].z, wq[u].w};
    const uint32_t ak[4] = {wk[u].x, wk[u].y, wk[u].z, wk[u].w};
    const uint32_t av[4] = {wv[u].x, wv[u].y, wv[u].z, wv[u].w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      q[4 * u + c] = word_value(aq[c]);
      k[4 * u + c] = word_value(ak[c]);
      v[4 * u + c] = word_value(av[c]);
    }
  }
  // lane e < 8 holds dims d < HD / 2, lane e + 8 their rotation partners d + HD / 2
  const bool lo = e < 8;
  float cs[VP], sn[VP];
#pragma unroll
  for (int u = 0; u < VP; ++u) {
    const float2 t = rope[VP * (e & 7) + u];
    cs[u] = t.x;
    sn[u] = t.y;
  }
  auto norm_rope = [&](float* t, const __nv_bfloat16* gamma) {
    float ss = 0.0f;
#pragma unroll
    for (int u = 0; u < VP; ++u) ss = fmaf(t[u], t[u], ss);
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) ss += __shfl_xor_sync(hm, ss, o);
    const float inv = 1.0f / sqrtf(ss / (float)HD + a.eps);
#pragma unroll
    for (int u = 0; u < VP; ++u)
      t[u] = round_bf16(__bfloat162float(gamma[VP * e + u]) * round_bf16(t[u] * inv));
#pragma unroll
    for (int u = 0; u < VP; ++u) {
      const float pt = __shfl_xor_sync(hm, t[u], 8);
      t[u] = lo ? __fsub_rn(__fmul_rn(t[u], cs[u]), __fmul_rn(pt, sn[u]))
                : __fadd_rn(__fmul_rn(t[u], cs[u]), __fmul_rn(pt, sn[u]));
    }
#pragma unroll
    for (int u = 0; u < VP; ++u) t[u] = round_bf16(t[u]);
  };
  norm_rope(q, gq);
  norm_rope(k, gk);
  const uint32_t tkv = sc.tag(sc.kv(j, l));
  if (write_kv) {
#pragma unroll
    for (int u = 0; u < VQ; ++u) {
      st_words4(kvb + (size_t)j * 2 * QN + 4 * u,
                tag4(k[4 * u], k[4 * u + 1], k[4 * u + 2], k[4 * u + 3], tkv));
      st_words4(kvb + (size_t)j * 2 * QN + QN + 4 * u,
                tag4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3], tkv));
    }
  }
  const float scale = 1.0f / sqrtf((float)HD);
  float mrun = -INFINITY, lrun = 0.0f, o[VP];
#pragma unroll
  for (int u = 0; u < VP; ++u) o[u] = 0.0f;
  for (int p0 = 0; p0 <= j; p0 += CH) {
    if (p0 > 0) fetch(p0);
    check(p0);
    float d[CH];
#pragma unroll
    for (int t = 0; t < CH; ++t) {
      const bool cur = p0 + t == j;
      float acc = 0.0f;
#pragma unroll
      for (int u = 0; u < VQ; ++u) {
        const uint32_t c4[4] = {ck[t][u].x, ck[t][u].y, ck[t][u].z, ck[t][u].w};
#pragma unroll
        for (int c = 0; c < 4; ++c)
          acc = fmaf(q[4 * u + c], cur ? k[4 * u + c] : word_value(c4[c]), acc);
      }
      d[t] = acc;
    }
#pragma unroll
    for (int off = 8; off > 0; off >>= 1)
#pragma unroll
      for (int t = 0; t < CH; ++t) d[t] += __shfl_xor_sync(hm, d[t], off);
    float cm = -INFINITY;
#pragma unroll
    for (int t = 0; t < CH; ++t)
      if (p0 + t <= j) cm = fmaxf(cm, d[t] * scale);
    const float mnew = fmaxf(mrun, cm);
    const float corr = expf(mrun - mnew);  // 0 for the first chunk
    lrun *= corr;
#pragma unroll
    for (int u = 0; u < VP; ++u) o[u] *= corr;
#pragma unroll
    for (int t = 0; t < CH; ++t) {
      const int p = p0 + t;
      if (p <= j) {
        const float w = expf(d[t] * scale - mnew);
        lrun += w;
#pragma unroll
        for (int u = 0; u < VQ; ++u) {
          const uint32_t c4[4] = {cv[t][u].x, cv[t][u].y, cv[t][u].z, cv[t][u].w};
#pragma unroll
          for (int c = 0; c < 4; ++c)
            o[4 * u + c] = fmaf(w, p == j ? v[4 * u + c] : word_value(c4[c]), o[4 * u + c]);
        }
      }
    }
    mrun = mnew;
  }
  if (out_x) {
#pragma unroll
    for (int u = 0; u < VP; u += 2) {
      const __nv_bfloat162 b = __floats2bfloat162_rn(o[u] / lrun, o[u + 1] / lrun);
      *reinterpret_cast<__nv_bfloat162*>(out_x + VP * e + u) = b;
    }
  } else {
#pragma unroll
    for (int u = 0; u < VQ; ++u)
      st_words4(out_w + VP * e + 4 * u,
                tag4(o[4 * u] / lrun, o[4 * u + 1] / lrun, o[4 * u + 2] / lrun,
                     o[4 * u + 3] / lrun, out_tag));
  }
}

// The draw of codebook jj (1-based) from the best keys (tag t) of the CTAs
// that hold head tiles (the first min(grid, V / 16)): warp p takes key p;
// pcode[r] becomes the code row r feeds forward; CTA 0 writes the outputs.
// A key: order-preserving bits of z (high 32), 0xFFFF - index (next 16: the
// lower index wins a tie), the tag (low 16). Only CTAs upstream of the next
// head step read the keys (those with QKV or O tiles), so no key is
// overwritten before every reader has it.
__device__ __forceinline__ void take_codes(const DepthArgs& a, int jj, uint32_t t, int* pcode) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool cfg = a.fp->cfg_on != 0;
  const int keys = cfg ? a.rows / 2 : a.rows;
  const int nhc = min((int)gridDim.x, a.V >> 4);
  if (warp < keys) {
    unsigned long long b = 0ull;
    for (int c = lane; c < nhc; c += 32) {
      const unsigned long long* p = a.part + (size_t)c * kMaxRows + warp;
      unsigned long long v = ld_u64v(p);
      for (long long spin = 0; (uint32_t)(v & 0xFFFFu) != t; ++spin) {
        if ((spin & 255) == 255) {
          if (spin >= kDepthSpinLimit) {
            record_error(a.err, kErrTimeout);
            break;
          }
          if (*reinterpret_cast<volatile int*>(a.err) != 0) break;
        }
        v = ld_u64v(p);
      }
      b = v > b ? v : b;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long y = __shfl_xor_sync(0xffffffffu, b, o);
      b = y > b ? y : b;
    }
    if (lane == 0) {
      const int code = (b >> 16) ? (int)(0xFFFFu - (uint32_t)((b >> 16) & 0xFFFFu)) : 0x7fffffff;
      for (int q = 0; q < (cfg ? 2 : 1); ++q) {
        const int r = cfg ? 2 * warp + q : warp;
        const int fed = a.forced ? a.forced[(size_t)r * a.NC + jj - 1] : code;
        pcode[r] = fed;
        if (blockIdx.x == 0) {
          a.codes[(size_t)r * a.NC + jj - 1] = code;
          a.prev[r] = fed;
        }
      }
    }
  }
  __syncthreads();
}

template <int NB, int HD>
__global__ void __launch_bounds__(kDepthThreads, 1) depth_kernel(const DepthArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* wb = smem;
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(smem + a.wb_bytes);
  float* part = reinterpret_cast<float*>(smem + a.wb_bytes + a.xs_bytes);
  float* ys = part + kDepthWarps * NB * 128;
  float* xown = ys + (size_t)a.max_tiles * 256;  // [rows][16 own tiles] this CTA's residual slice
  float* sred = xown + (size_t)a.own_tiles * 256;  // [rows * K / 64] norm partials
  __shared__ uint64_t wbar[2];
  __shared__ unsigned long long best[kMaxRows];
  __shared__ int pcode[kMaxRows];
  __shared__ float rinv[kMaxRows];
  __shared__ const __nv_bfloat16* src[kMaxRows];

  const int tid = threadIdx.x, warp = tid >> 5;
  const int rows = a.rows, Dh = a.Dh, QN = a.nh * HD, F = a.F;
  Sched sc;
  sc.L = a.n_layers;
  sc.S = a.merge_attn ? 4 : 5;
  sc.merge = a.merge_attn;
  if (tid == 0) {
    mbar_init(&wbar[0], 1);
    mbar_init(&wbar[1], 1);
    fence_barrier_init();
  }
  if (tid < rows) pcode[tid] = a.code0[tid];
  __syncthreads();
  unsigned wpar = 0u;  // phase parity of each weight slot's mbarrier
  auto wwait = [&](int gi) {
    const int s = gi & 1;
    mbar_wait(&wbar[s], (wpar >> s) & 1u, a.err);
    wpar ^= 1u << s;
  };
  if (warp == 0) {
    issue_slice(a, wb, wbar, 0);
    issue_slice(a, wb, wbar, 1);
  }
  // this CTA's tiles of the residual stream (those of the O and down
  // projections): x = bf16(xown + bf16(y)), kept here and published
  int ot0, ont;
  cta_tiles(Dh, ot0, ont);
  auto publish_x = [&](int nt, uint32_t tag, bool add) {
    const int n16 = 16 * nt, q4 = n16 / 4;
    for (int i = tid; i < rows * q4; i += kDepthThreads) {
      const int m = i / q4, c = 4 * (i - m * q4);
      float xv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float y = ys[(size_t)m * n16 + c + u];
        xv[u] = add ? round_bf16(xown[(size_t)m * n16 + c + u] + round_bf16(y)) : round_bf16(y);
        xown[(size_t)m * n16 + c + u] = xv[u];
      }
      st_words4(a.xw + (size_t)m * Dh + 16 * ot0 + c, tag4(xv[0], xv[1], xv[2], xv[3], tag));
    }
  };
  auto gamma_of = [&](const uint8_t* slot, int nt, int K) {
    return reinterpret_cast<const __nv_bfloat16*>(slot_side(slot, nt, K));
  };

  // ---- position 0's input: x = bf16(W_proj h)
  if (ont > 0) {
    const int rpmax = a.xs_bytes / ((a.Hin + 8) * 2);
    wwait(0);
    const uint32_t t0tag = sc.tag(0);
    for (int m0 = 0; m0 < rows; m0 += rpmax) {
      const int rp = min(rpmax, rows - m0);
      if (tid < rp) src[tid] = a.h_in + (size_t)(m0 + tid) * a.Hin;
      __syncthreads();
      stage_plain(src, rp, a.Hin, nullptr, a.eps, xs, sred, rinv);
      tile_dots<NB>(slot_base(a, wb, 0, ont, a.Hin), ont, a.Hin, xs, rp, part, ys);
      const int n16 = 16 * ont, q4 = n16 / 4;
      for (int i = tid; i < rp * q4; i += kDepthThreads) {
        const int m = i / q4, c = 4 * (i - m * q4);
        float xv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          xv[u] = round_bf16(ys[(size_t)m * n16 + c + u]);
          xown[(size_t)(m0 + m) * n16 + c + u] = xv[u];
        }
        st_words4(a.xw + (size_t)(m0 + m) * Dh + 16 * ot0 + c, tag4(xv[0], xv[1], xv[2], xv[3], t0tag));
      }
      __syncthreads();
    }
  }
  __syncthreads();
  int gi = 1;

  for (int j = 0; j <= a.NC; ++j) {
    for (int l = 0; l < a.n_layers; ++l) {
      // ---- qkv = W_qkv norm(x); at layer 0 of position j >= 1 the input is
      // E_{j-1}[code] (a zero vector for the end token's code at j = 1)
      if (warp == 0) issue_slice(a, wb, wbar, gi + 1);
      {
        const bool emb = l == 0 && j >= 1;
        int t0, nt;
        cta_tiles(3 * QN, t0, nt);
        if (emb && (nt > 0 || ont > 0)) {
          if (j >= 2) take_codes(a, j - 1, sc.tag(sc.head(j - 1)), pcode);
          if (tid < rows) {
            const int c = pcode[tid];
            const bool zero = (j == 1 && c == a.zero_code);
            const bool ok = c >= 0 && c < a.emb_rows[j - 1];
            if (!zero && !ok && blockIdx.x == 0) record_error(a.err, kErrBounds);
            src[tid] = (zero || !ok) ? nullptr : a.emb[j - 1] + (size_t)c * Dh;
          }
          __syncthreads();
          // this CTA's slice of the residual stream starts at the input
          const int n16 = 16 * ont;
          for (int i = tid; i < rows * n16; i += kDepthThreads) {
            const int m = i / n16, nl = i - m * n16;
            xown[(size_t)m * n16 + nl] =
                src[m] ? __bfloat162float(src[m][16 * ot0 + nl]) : 0.0f;
          }
        }
        if (nt > 0) {
          wwait(gi);
          const uint8_t* slot = slot_base(a, wb, gi, nt, Dh);
          if (emb) {
            stage_plain(src, rows, Dh, gamma_of(slot, nt, Dh), a.eps, xs, sred, rinv);
          } else {
            const int xph = l > 0 ? sc.down(j, l - 1) : (j == 0 ? 0 : sc.down(j - 1, a.n_layers - 1));
            stage_tagged(a.xw, Dh, rows, Dh, sc.tag(xph), gamma_of(slot, nt, Dh), a.eps, xs, sred,
                         rinv, a.err);
          }
          tile_dots<NB>(slot, nt, Dh, xs, rows, part, ys);
          const int n16 = 16 * nt, q4 = n16 / 4;
          const uint32_t tg = sc.tag(sc.qkv(j, l));
          for (int i = tid; i < rows * q4; i += kDepthThreads) {
            const int m = i / q4, c = 4 * (i - m * q4);
            const float* y = ys + (size_t)m * n16 + c;
            st_words4(a.qkvw + (size_t)m * 3 * QN + 16 * t0 + c, tag4(y[0], y[1], y[2], y[3], tg));
          }
        }
      }
      __syncthreads();
      ++gi;

      // ---- attention as its own step (many (row, head) pairs): two pairs per warp
      if (!a.merge_attn) {
        const int items = rows * a.nh;
        const uint32_t tg = sc.tag(sc.attn(j, l));
        for (int it = 2 * (blockIdx.x + (int)gridDim.x * warp) + ((tid >> 4) & 1); it - ((tid >> 4) & 1) < items;
             it += 2 * (int)gridDim.x * kDepthWarps) {
          if (it < items) {
            const int m = it / a.nh, h = it - m * a.nh;
            attend<HD>(a, sc, l, j, m, h, a.L[l].q_norm, a.L[l].k_norm,
                       a.rope + (size_t)j * (HD / 2), nullptr,
                       a.attw + (size_t)m * QN + (size_t)h * HD, tg, true);
          }
        }
        __syncthreads();
      }

      // ---- x += bf16(W_o att)
      if (warp == 0) issue_slice(a, wb, wbar, gi + 1);
      if (ont > 0) {
        wwait(gi);
        const uint8_t* slot = slot_base(a, wb, gi, ont, QN);
        if (a.merge_attn) {
          // every (row, head) here, two per warp; CTA 0 stores the keys and values
          const uint8_t* sd = slot_side(slot, ont, QN);
          const __nv_bfloat16* gq = reinterpret_cast<const __nv_bfloat16*>(sd);
          const __nv_bfloat16* gk = gq + HD;
          const float2* rope = reinterpret_cast<const float2*>(gk + HD);
          const int it = 2 * warp + ((tid >> 4) & 1);
          if (it < rows * a.nh) {
            const int m = it / a.nh, h = it - m * a.nh;
            attend<HD>(a, sc, l, j, m, h, gq, gk, rope, xs + (size_t)m * (QN + 8) + (size_t)h * HD,
                       nullptr, 0u, blockIdx.x == 0);
          }
          __syncthreads();
        } else {
          stage_tagged(a.attw, QN, rows, QN, sc.tag(sc.attn(j, l)), nullptr, a.eps, xs, sred, rinv,
                       a.err);
        }
        tile_dots<NB>(slot, ont, QN, xs, rows, part, ys);
        publish_x(ont, sc.tag(sc.o(j, l)), true);
      }
      __syncthreads();
      ++gi;

      // ---- act = SwiGLU(W_gu norm(x)): gate rows 2i, up rows 2i + 1
      if (warp == 0) issue_slice(a, wb, wbar, gi + 1);
      {
        int t0, nt;
        cta_tiles(2 * F, t0, nt);
        if (nt > 0) {
          wwait(gi);
          const uint8_t* slot = slot_base(a, wb, gi, nt, Dh);
          stage_tagged(a.xw, Dh, rows, Dh, sc.tag(sc.o(j, l)), gamma_of(slot, nt, Dh), a.eps, xs,
                       sred, rinv, a.err);
          tile_dots<NB>(slot, nt, Dh, xs, rows, part, ys);
          const int n16 = 16 * nt, q4 = 2 * nt;  // 8 nt outputs per row, 4 per word group
          const uint32_t tg = sc.tag(sc.gu(j, l));
          for (int i = tid; i < rows * q4; i += kDepthThreads) {
            const int m = i / q4, c = 4 * (i - m * q4);
            float av[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float gb = round_bf16(ys[(size_t)m * n16 + 2 * (c + u)]);
              const float ub = round_bf16(ys[(size_t)m * n16 + 2 * (c + u) + 1]);
              av[u] = round_bf16(silu_f(gb)) * ub;
            }
            st_words4(a.actw + (size_t)m * F + 8 * t0 + c, tag4(av[0], av[1], av[2], av[3], tg));
          }
        }
      }
      __syncthreads();
      ++gi;

      // ---- x += bf16(W_d act)
      if (warp == 0) issue_slice(a, wb, wbar, gi + 1);
      if (ont > 0) {
        wwait(gi);
        stage_tagged(a.actw, F, rows, F, sc.tag(sc.gu(j, l)), nullptr, a.eps, xs, sred, rinv,
                     a.err);
        tile_dots<NB>(slot_base(a, wb, gi, ont, F), ont, F, xs, rows, part, ys);
        publish_x(ont, sc.tag(sc.down(j, l)), true);
      }
      __syncthreads();
      ++gi;
    }
    if (j == 0) continue;

    // ---- codebook j: logits of head j on norm_f(x), guided, Gumbel-argmax
    if (warp == 0) issue_slice(a, wb, wbar, gi + 1);
    if (tid < kMaxRows) best[tid] = 0ull;
    __syncthreads();
    {
      int t0, nt;
      cta_tiles(a.V, t0, nt);
      if (nt > 0) {
        wwait(gi);
        const uint8_t* slot = slot_base(a, wb, gi, nt, Dh);
        stage_tagged(a.xw, Dh, rows, Dh, sc.tag(sc.down(j, a.n_layers - 1)),
                     gamma_of(slot, nt, Dh), a.eps, xs, sred, rinv, a.err);
        tile_dots<NB>(slot, nt, Dh, xs, rows, part, ys);
        const int n16 = 16 * nt;
        for (int i = tid; i < rows * n16; i += kDepthThreads) {
          const int m = i / n16, nl = i - m * n16;
          a.logits[((size_t)m * a.NC + (j - 1)) * a.V + 16 * t0 + nl] = ys[(size_t)m * n16 + nl];
        }
        const FrameParams* fp = a.fp;
        const bool cfg = fp->cfg_on != 0;
        const int keys = cfg ? rows / 2 : rows;
        const unsigned long long ib = (unsigned long long)j << 32;
        for (int i = tid; i < keys * n16; i += kDepthThreads) {
          const int p = i / n16, nl = i - p * n16, n = 16 * t0 + nl;
          const float y0 = ys[(size_t)(cfg ? 2 * p : p) * n16 + nl];
          float gl = y0;
          if (cfg) {
            const float y1 = ys[(size_t)(2 * p + 1) * n16 + nl];
            gl = __fadd_rn(y1, __fmul_rn(fp->cfg_scale, __fsub_rn(y0, y1)));
          }
          const float z = __fadd_rn(__fdiv_rn(gl, fp->temperature),
                                    gumbel_noise(fp->seed, fp->frame, (unsigned long long)p,
                                                 ib | (unsigned long long)n));
          const uint32_t zb = (uint32_t)(argmax_key(z, 0) >> 32);
          atomicMax(&best[p], ((unsigned long long)zb << 32) |
                                  ((unsigned long long)(0xFFFFu - (uint32_t)n) << 16));
        }
        __syncthreads();
        if (tid < kMaxRows)
          st_u64v(a.part + (size_t)blockIdx.x * kMaxRows + tid, best[tid] | sc.tag(sc.head(j)));
      }
    }
    __syncthreads();
    ++gi;
  }
  // the last codebook's draw: CTA 0 writes it
  if (blockIdx.x == 0) take_codes(a, a.NC, sc.tag(sc.head(a.NC)), pcode);
}

template <int NB>
const void* depth_kernel_for(int hd) {
  return hd == 64 ? (const void*)depth_kernel<NB, 64> : (const void*)depth_kernel<NB, 128>;
}

}  // namespace

cudaError_t depth_plan(DepthArgs* a, int grid, size_t* smem) {
  const cudaError_t bad = cudaErrorInvalidConfiguration;
  if (grid < 1 || a->rows < 1 || a->rows > kMaxRows) return bad;
  if (a->n_layers < 1 || a->n_layers > kDepthMaxLayers || a->NC < 1 ||
      a->NC > kDepthMaxCodebooks)
    return bad;
  if (a->hd != 64 && a->hd != 128) return bad;
  const int QN = a->nh * a->hd;
  if (a->nh < 1 || a->Dh % 128 || QN % 128 || a->F % 128 || a->Hin % 128 || a->V < 16 ||
      a->V % 16 || a->V > 65535)  // a draw's index travels in 16 bits
    return bad;
  if (a->rows * a->nh > grid * kDepthWarps) return bad;
  // static vectors of a step: a norm gain (Dh bf16), or the q/k gains and a
  // RoPE row (2 hd bf16 + hd / 2 float2)
  int side = 2 * a->Dh > 8 * a->hd ? 2 * a->Dh : 8 * a->hd;
  side = (side + 15) & ~15;
  const int N[6] = {a->Dh, 3 * QN, a->Dh, 2 * a->F, a->Dh, a->V};
  const int K[6] = {a->Hin, a->Dh, QN, a->Dh, a->F, a->Dh};
  int sb[6], mt = 0;
  for (int i = 0; i < 6; ++i) {
    const int T = N[i] / 16, nt = (T + grid - 1) / grid;
    if (nt > kDepthMaxTiles) return bad;
    sb[i] = depth_slice_bytes(nt, K[i], side);
    mt = nt > mt ? nt : mt;
  }
  // consecutive projections: proj-qkv, qkv-o, o-gu, gu-down, down-qkv,
  // down-head, head-qkv
  const int pairs[7][2] = {{0, 1}, {1, 2}, {2, 3}, {3, 4}, {4, 1}, {4, 5}, {5, 1}};
  int wb = 0;
  for (const auto& p : pairs) wb = sb[p[0]] + sb[p[1]] > wb ? sb[p[0]] + sb[p[1]] : wb;
  int kmax = a->Dh;
  if (QN > kmax) kmax = QN;
  if (a->F > kmax) kmax = a->F;
  int xs = a->rows * (kmax + 8) * 2;
  if (xs < (a->Hin + 8) * 2) xs = (a->Hin + 8) * 2;  // at least one row of the projection's input
  xs = (xs + 127) & ~127;
  const int NB = a->rows > 8 ? 2 : 1;
  const int own = ((a->Dh / 16) + grid - 1) / grid;
  const size_t total = (size_t)wb + xs + (size_t)kDepthWarps * NB * 128 * 4 +
                       (size_t)mt * 256 * 4 + (size_t)own * 256 * 4 +
                       (size_t)a->rows * (a->Dh / 64) * 4;
  int dev = 0, optin = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  if (total + 1024 > (size_t)optin) return bad;
  a->wb_bytes = wb;
  a->xs_bytes = xs;
  a->max_tiles = mt;
  a->side_bytes = side;
  a->own_tiles = own;
  a->merge_attn = a->rows * a->nh <= 2 * kDepthWarps ? 1 : 0;
  const void* kern = NB == 2 ? depth_kernel_for<2>(a->hd) : depth_kernel_for<1>(a->hd);
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)total);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kDepthThreads, total);
  if (e != cudaSuccess) return e;
  int nsm = 0;
  e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  if (per_sm < 1 || grid > per_sm * nsm) return bad;
  *smem = total;
  return cudaSuccess;
}

// The tagged buffers cleared to tag 0 (so that a word carries a step's tag
// only once that step of this launch has written it), then one cooperative
// launch (every CTA resident at once: a step waits for other CTAs' outputs).
cudaError_t launch_depth(const DepthArgs& a, int grid, size_t smem, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(a.words, 0, a.words_bytes, st);
  if (e == cudaSuccess)
    e = cudaMemsetAsync(a.part, 0, sizeof(unsigned long long) * grid * kMaxRows, st);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kDepthThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (a.rows > 8)
    return a.hd == 64 ? cudaLaunchKernelEx(&cfg, depth_kernel<2, 64>, a)
                      : cudaLaunchKernelEx(&cfg, depth_kernel<2, 128>, a);
  return a.hd == 64 ? cudaLaunchKernelEx(&cfg, depth_kernel<1, 64>, a)
                    : cudaLaunchKernelEx(&cfg, depth_kernel<1, 128>, a);
}

}  // namespace m3
