// depth.cu -- launcher of the persistent depth-decoder kernel (depth.cuh).
#include <cuda_runtime.h>

#include "common.cuh"
#include "depth.cuh"
#include "gemv_tile.cuh"
#include "launch.cuh"
#include "noise.cuh"

namespace m3 {

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Every CTA of the launch meets here (all threads call it).
__device__ __forceinline__ void depth_grid_sync(unsigned* bar, unsigned& gen, int* err) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(&bar[0], 1u) == gridDim.x - 1) {
      bar[0] = 0u;  // nobody arrives again before the generation moves
      __threadfence();
      atomicAdd(&bar[1], 1u);
    } else {
      long long spins = 0;
      while (ld_acquire_u32(&bar[1]) == gen) {
        if (*reinterpret_cast<volatile unsigned*>(&bar[2])) break;
        if (++spins > kDepthSpinLimit) {
          record_error(err, kErrTimeout);
          atomicExch(&bar[2], 1u);
          break;
        }
        __nanosleep(64);
      }
    }
    __threadfence();
  }
  ++gen;
  __syncthreads();
}

// Data that other CTAs of the launch wrote is read through L2 (__ldcg): L1
// is not coherent across SMs.  Every staging is one round of 16-byte loads.
// Copy of `rows` bf16 vectors of length n (n % 8 == 0; row m at
// src[m], or zeros for a null pointer) into shared memory [rows][n].
static __device__ __noinline__ void depth_stage_rows(const __nv_bfloat16* const* src, int rows, int n,
                                                 __nv_bfloat16* out) {
  const int n8 = n >> 3;
  for (int i = threadIdx.x; i < rows * n8; i += kDepthThreads) {
    const int m = i / n8, c = i % n8;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (src[m]) v = __ldcg(reinterpret_cast<const uint4*>(src[m]) + c);
    reinterpret_cast<uint4*>(out)[i] = v;
  }
  __syncthreads();
}

// Rows of a strided bf16 matrix into shared memory [rows][n].
static __device__ __noinline__ void depth_copy_rows(const __nv_bfloat16* src, int ld, int rows, int n,
                                                __nv_bfloat16* out) {
  const int n8 = n >> 3;
  for (int i = threadIdx.x; i < rows * n8; i += kDepthThreads) {
    const int m = i / n8, c = i % n8;
    reinterpret_cast<uint4*>(out)[i] =
        __ldcg(reinterpret_cast<const uint4*>(src + (size_t)m * ld) + c);
  }
  __syncthreads();
}

// RMSNorm in place over the staged rows [rows][n] of shared memory:
// out = bf16(gamma * bf16(v / rms)), rms over the row in fp32 (one warp per
// row, lanes strided, a shuffle tree).
static __device__ __noinline__ void depth_norm_staged(__nv_bfloat16* xs, int rows, int n,
                                                  const __nv_bfloat16* gamma, float eps,
                                                  float* rinv) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int m = warp; m < rows; m += kDepthWarps) {
    float s = 0.0f;
    for (int i = lane; i < n; i += 32) {
      const float f = __bfloat162float(xs[(size_t)m * n + i]);
      s = fmaf(f, f, s);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) rinv[m] = 1.0f / sqrtf(s / (float)n + eps);
  }
  __syncthreads();
  for (int i = tid; i < rows * n; i += kDepthThreads) {
    const int m = i / n, k = i % n;
    const float f = __bfloat162float(xs[i]);
    xs[i] = __float2bfloat16_rn(__bfloat162float(gamma[k]) * round_bf16(f * rinv[m]));
  }
  __syncthreads();
}

// y[m] = sum_g s[n][g] sum_{k in g} q[n][k] x[m][k] for one output row n, by
// one warp: lane l takes inputs 128 g + 4 l .. + 3 of every group; fp32.
// The row's weights are fetched 8 groups at a time (one round trip for
// K = 1024).
static __device__ __noinline__ void depth_dot(const DepthMat& W, int n, int K,
                                         const __nv_bfloat16* xs, int rows, float* y) {
  const int lane = threadIdx.x & 31;
  const int G = K >> 7;
  const uint32_t* wr = reinterpret_cast<const uint32_t*>(W.q + (size_t)n * K) + lane;
  const float* sr = W.s + (size_t)n * G;
  float acc[kMaxRows];
#pragma unroll
  for (int m = 0; m < kMaxRows; ++m) acc[m] = 0.0f;
  for (int g0 = 0; g0 < G; g0 += 8) {
    uint32_t w[8];
    float sc[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      w[u] = g0 + u < G ? __ldg(wr + (size_t)(g0 + u) * 32) : 0u;
      sc[u] = g0 + u < G ? __ldg(sr + g0 + u) : 0.0f;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (g0 + u >= G) break;
      const float q0 = (float)(int8_t)(w[u] & 0xFF), q1 = (float)(int8_t)((w[u] >> 8) & 0xFF);
      const float q2 = (float)(int8_t)((w[u] >> 16) & 0xFF), q3 = (float)(int8_t)(w[u] >> 24);
      const int k = 128 * (g0 + u) + 4 * lane;
#pragma unroll
      for (int m = 0; m < kMaxRows; ++m) {
        if (m >= rows) break;
        const uint2 xv = *reinterpret_cast<const uint2*>(xs + (size_t)m * K + k);
        const float x0 = __uint_as_float(xv.x << 16), x1 = __uint_as_float(xv.x & 0xFFFF0000u);
        const float x2 = __uint_as_float(xv.y << 16), x3 = __uint_as_float(xv.y & 0xFFFF0000u);
        float p = q0 * x0;
        p = fmaf(q1, x1, p);
        p = fmaf(q2, x2, p);
        p = fmaf(q3, x3, p);
        acc[m] = fmaf(sc[u], p, acc[m]);
      }
    }
  }
#pragma unroll
  for (int m = 0; m < kMaxRows; ++m) {
    if (m >= rows) break;
    float v = acc[m];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    y[m] = v;
  }
}

// The same for up to 4 output rows nr[0..count) and at most 4 activation
// rows, K <= 1024: every weight word of all of them is fetched before any is
// used, so the rows cost one round trip together.  y[r][m] for row nr[r].
static __device__ __noinline__ void depth_dot4(const DepthMat& W, const int* nr, int count, int K,
                                          const __nv_bfloat16* xs, int rows, float (*y)[4]) {
  const int lane = threadIdx.x & 31;
  const int G = K >> 7;
  uint32_t w[4][8];
  float sc[4][8];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int n = r < count ? nr[r] : nr[0];
    const uint32_t* wr = reinterpret_cast<const uint32_t*>(W.q + (size_t)n * K) + lane;
    const float* sr = W.s + (size_t)n * G;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const bool ok = r < count && u < G;
      w[r][u] = ok ? __ldg(wr + (size_t)u * 32) : 0u;
      sc[r][u] = ok ? __ldg(sr + u) : 0.0f;
    }
  }
  float acc[4][4];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int m = 0; m < 4; ++m) acc[r][m] = 0.0f;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    if (u >= G) break;
    const int k = 128 * u + 4 * lane;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      if (m >= rows) break;
      const uint2 xv = *reinterpret_cast<const uint2*>(xs + (size_t)m * K + k);
      const float x0 = __uint_as_float(xv.x << 16), x1 = __uint_as_float(xv.x & 0xFFFF0000u);
      const float x2 = __uint_as_float(xv.y << 16), x3 = __uint_as_float(xv.y & 0xFFFF0000u);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const uint32_t q = w[r][u];
        float p = (float)(int8_t)(q & 0xFF) * x0;
        p = fmaf((float)(int8_t)((q >> 8) & 0xFF), x1, p);
        p = fmaf((float)(int8_t)((q >> 16) & 0xFF), x2, p);
        p = fmaf((float)(int8_t)(q >> 24), x3, p);
        acc[r][m] = fmaf(sc[r][u], p, acc[r][m]);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      float v = acc[r][m];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      y[r][m] = v;
    }
}

// Shared memory of the RoPE table of positions 0..NC (16-byte multiple).
__host__ __device__ __forceinline__ size_t depth_rope_bytes(const DepthArgs& a) {
  return ((size_t)(a.NC + 1) * (a.hd / 2) * sizeof(float2) + 15) / 16 * 16;
}

// One (row m, head h) of the attention phase, by one warp: q/k RMSNorm and
// RoPE at position j (as the body's attention kernel rounds them), the K/V of
// position j stored, then attention over positions 0..j (online softmax).
static __device__ __noinline__ void depth_attention(const DepthArgs& a, const float2* rope, int l,
                                                int j, int m, int h) {
  const int lane = threadIdx.x & 31, hd = a.hd, vpl = hd >> 5;
  const int QN = a.nh * hd;
  const __nv_bfloat16* qr = a.qkv + (size_t)m * 3 * QN + (size_t)h * hd;
  const __nv_bfloat16* kr = qr + QN;
  const __nv_bfloat16* vr = kr + QN;
  float q[4], k[4], v[4], cs[2], sn[2];  // rope: [NC + 1][hd / 2] (cos, sin)
  for (int i = 0; i < vpl; ++i) {
    q[i] = __bfloat162float(__ldcg(qr + lane + 32 * i));
    k[i] = __bfloat162float(__ldcg(kr + lane + 32 * i));
    v[i] = __bfloat162float(__ldcg(vr + lane + 32 * i));
  }
  for (int i = 0; i < vpl / 2; ++i) {
    const float2 t = rope[(size_t)j * (hd / 2) + lane + 32 * i];
    cs[i] = t.x;
    sn[i] = t.y;
  }
  auto norm_rope = [&](float* t, const __nv_bfloat16* gamma) {
    float ss = 0.0f;
    for (int i = 0; i < vpl; ++i) ss = fmaf(t[i], t[i], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = 1.0f / sqrtf(ss / (float)hd + a.eps);
    for (int i = 0; i < vpl; ++i)
      t[i] = round_bf16(__bfloat162float(gamma[lane + 32 * i]) * round_bf16(t[i] * inv));
    for (int i = 0; i < vpl / 2; ++i) {  // pairs (d, d + hd / 2)
      const float x0 = t[i], x1 = t[i + vpl / 2];
      t[i] = __fsub_rn(__fmul_rn(x0, cs[i]), __fmul_rn(x1, sn[i]));
      t[i + vpl / 2] = __fadd_rn(__fmul_rn(x1, cs[i]), __fmul_rn(x0, sn[i]));
    }
    for (int i = 0; i < vpl; ++i) t[i] = round_bf16(t[i]);
  };
  norm_rope(q, a.L[l].q_norm);
  norm_rope(k, a.L[l].k_norm);
  // K/V of every position of this (row, layer): [pos][2][nh][hd]
  __nv_bfloat16* kvb = a.kv + ((size_t)m * a.n_layers + l) * (size_t)(a.NC + 1) * 2 * QN;
  for (int i = 0; i < vpl; ++i) {
    kvb[((size_t)j * 2 + 0) * QN + (size_t)h * hd + lane + 32 * i] = __float2bfloat16_rn(k[i]);
    kvb[((size_t)j * 2 + 1) * QN + (size_t)h * hd + lane + 32 * i] = __float2bfloat16_rn(v[i]);
  }
  const float scale = 1.0f / sqrtf((float)hd);
  float mrun = -INFINITY, lrun = 0.0f, o[4] = {0.f, 0.f, 0.f, 0.f};
  for (int p0 = 0; p0 <= j; p0 += 8) {  // positions p0 .. p0 + 7, fetched together
    __nv_bfloat16 kb[8][4], vb[8][4];
#pragma unroll
    for (int t = 0; t < 8; ++t)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int p = p0 + t;
        kb[t][i] = vb[t][i] = __float2bfloat16_rn(0.0f);
        if (p < j && i < vpl) {
          kb[t][i] = __ldcg(kvb + ((size_t)p * 2 + 0) * QN + (size_t)h * hd + lane + 32 * i);
          vb[t][i] = __ldcg(kvb + ((size_t)p * 2 + 1) * QN + (size_t)h * hd + lane + 32 * i);
        }
      }
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const int p = p0 + t;
      if (p > j) break;
      float kp[4], vp[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        kp[i] = p == j ? k[i] : __bfloat162float(kb[t][i]);
        vp[i] = p == j ? v[i] : __bfloat162float(vb[t][i]);
      }
      float d = 0.0f;
      for (int i = 0; i < vpl; ++i) d = fmaf(q[i], kp[i], d);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
      const float sc = d * scale;
      const float mnew = fmaxf(mrun, sc);
      const float corr = expf(mrun - mnew), w = expf(sc - mnew);
      lrun = lrun * corr + w;
      for (int i = 0; i < vpl; ++i) o[i] = o[i] * corr + w * vp[i];
      mrun = mnew;
    }
  }
  __nv_bfloat16* out = a.att + (size_t)m * QN + (size_t)h * hd;
  for (int i = 0; i < vpl; ++i) out[lane + 32 * i] = __float2bfloat16_rn(o[i] / lrun);
}

__global__ void __launch_bounds__(kDepthThreads, 1) depth_decode_kernel(const DepthArgs a) {
  extern __shared__ __align__(16) uint8_t depth_smem[];
  // the RoPE rotations of positions 0..NC, then the staged activations
  float2* rope = reinterpret_cast<float2*>(depth_smem);  // [NC + 1][hd / 2]
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(depth_smem + depth_rope_bytes(a));
  __shared__ float rinv[kMaxRows];
  __shared__ unsigned long long best[kMaxRows];
  __shared__ int pcode[kMaxRows];  // the code each row feeds forward
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rows = a.rows, Dh = a.Dh, QN = a.nh * a.hd, F = a.F;
  const bool cfg = a.fp->cfg_on != 0;
  const int keys = cfg ? rows / 2 : rows;
  const int gw = blockIdx.x * kDepthWarps + warp, nw = gridDim.x * kDepthWarps;
  unsigned gen = 0;
  if (tid == 0) gen = ld_acquire_u32(&a.bar[1]);
  if (tid < rows) pcode[tid] = __ldcg(a.code0 + tid);
  for (int i = tid; i < (a.NC + 1) * (a.hd / 2); i += kDepthThreads) {
    const double ang = (double)(i / (a.hd / 2)) * a.inv_freq[i % (a.hd / 2)];
    rope[i] = make_float2((float)cos(ang), (float)sin(ang));
  }
  float y[kMaxRows], yu[kMaxRows], y4[4][4];
  // rows of up to 4 weight rows per warp at once (K <= 1024, up to 4 rows)
  const bool fast = a.Dh <= 1024 && a.rows <= 4;
  const __nv_bfloat16* src[kMaxRows];

  // ---- the frame's hidden state, projected
  depth_copy_rows(a.h_in, a.Hin, rows, a.Hin, xs);
  for (int n = gw; n < Dh; n += nw) {
    depth_dot(a.proj, n, a.Hin, xs, rows, y);
    if (lane == 0)
      for (int m = 0; m < rows; ++m) a.x[(size_t)m * Dh + n] = __float2bfloat16_rn(y[m]);
  }
  depth_grid_sync(a.bar, gen, a.err);

  for (int j = 0; j <= a.NC; ++j) {
    for (int l = 0; l < a.n_layers; ++l) {
      const DepthLayerW& L = a.L[l];
      // ---- A: n1 = norm(x); qkv (x of position j >= 1, layer 0: E_{j-1}[code])
      for (int m = 0; m < rows; ++m) {
        src[m] = a.x + (size_t)m * Dh;
        if (j >= 1 && l == 0) {
          const int c = pcode[m];
          const bool zero = (j == 1 && c == a.zero_code);
          const bool ok = c >= 0 && c < a.emb_rows[j - 1];
          if (!zero && !ok && tid == 0 && blockIdx.x == 0) record_error(a.err, kErrBounds);
          src[m] = (zero || !ok) ? nullptr : a.emb[j - 1] + (size_t)c * Dh;
        }
      }
      if (j >= 1 && l == 0 && blockIdx.x == 0) {  // the residual stream starts at the embedding
        for (int i = tid; i < rows * Dh; i += kDepthThreads) {
          const __nv_bfloat16* e = src[i / Dh];
          a.x[i] = e ? e[i % Dh] : __float2bfloat16_rn(0.0f);
        }
      }
      depth_stage_rows(src, rows, Dh, xs);
      depth_norm_staged(xs, rows, Dh, L.attn_norm, a.eps, rinv);
      if (fast) {
        for (int n0 = gw; n0 < 3 * QN; n0 += 4 * nw) {
          int nr[4], cnt = 0;
          for (int r = 0; r < 4 && n0 + r * nw < 3 * QN; ++r) nr[cnt++] = n0 + r * nw;
          depth_dot4(L.qkv, nr, cnt, Dh, xs, rows, y4);
          if (lane == 0)
            for (int r = 0; r < cnt; ++r)
              for (int m = 0; m < rows; ++m)
                a.qkv[(size_t)m * 3 * QN + nr[r]] = __float2bfloat16_rn(y4[r][m]);
        }
      } else {
        for (int n = gw; n < 3 * QN; n += nw) {
          depth_dot(L.qkv, n, Dh, xs, rows, y);
          if (lane == 0)
            for (int m = 0; m < rows; ++m) a.qkv[(size_t)m * 3 * QN + n] = __float2bfloat16_rn(y[m]);
        }
      }
      depth_grid_sync(a.bar, gen, a.err);
      // ---- B: attention, one warp per (row, head)
      for (int it = gw; it < rows * a.nh; it += nw)
        depth_attention(a, rope, l, j, it / a.nh, it % a.nh);
      depth_grid_sync(a.bar, gen, a.err);
      // ---- C: x = bf16(x + bf16(W_o att))
      depth_copy_rows(a.att, QN, rows, QN, xs);
      if (fast && QN <= 1024) {
        for (int n0 = gw; n0 < Dh; n0 += 4 * nw) {
          int nr[4], cnt = 0;
          for (int r = 0; r < 4 && n0 + r * nw < Dh; ++r) nr[cnt++] = n0 + r * nw;
          depth_dot4(L.o, nr, cnt, QN, xs, rows, y4);
          if (lane == 0)
            for (int r = 0; r < cnt; ++r)
              for (int m = 0; m < rows; ++m) {
                __nv_bfloat16* o = a.x + (size_t)m * Dh + nr[r];
                *o = __float2bfloat16_rn(__bfloat162float(__ldcg(o)) + round_bf16(y4[r][m]));
              }
        }
      } else {
        for (int n = gw; n < Dh; n += nw) {
          depth_dot(L.o, n, QN, xs, rows, y);
          if (lane == 0)
            for (int m = 0; m < rows; ++m) {
              __nv_bfloat16* o = a.x + (size_t)m * Dh + n;
              *o = __float2bfloat16_rn(__bfloat162float(__ldcg(o)) + round_bf16(y[m]));
            }
        }
      }
      depth_grid_sync(a.bar, gen, a.err);
      // ---- D: n2 = norm(x); act = SwiGLU(gate, up)
      for (int m = 0; m < rows; ++m) src[m] = a.x + (size_t)m * Dh;
      depth_stage_rows(src, rows, Dh, xs);
      depth_norm_staged(xs, rows, Dh, L.mlp_norm, a.eps, rinv);
      if (fast) {
        for (int p0 = gw; p0 < F; p0 += 2 * nw) {  // two (gate, up) pairs per call
          int nr[4], cnt = 0;
          for (int r = 0; r < 2 && p0 + r * nw < F; ++r) {
            nr[cnt++] = 2 * (p0 + r * nw);
            nr[cnt++] = 2 * (p0 + r * nw) + 1;
          }
          depth_dot4(L.gu, nr, cnt, Dh, xs, rows, y4);
          if (lane == 0)
            for (int r = 0; r < cnt / 2; ++r)
              for (int m = 0; m < rows; ++m) {
                const float gb = round_bf16(y4[2 * r][m]), ub = round_bf16(y4[2 * r + 1][m]);
                a.act[(size_t)m * F + p0 + r * nw] =
                    __float2bfloat16_rn(round_bf16(silu_f(gb)) * ub);
              }
        }
      } else {
        for (int pr = gw; pr < F; pr += nw) {
          depth_dot(L.gu, 2 * pr, Dh, xs, rows, y);
          depth_dot(L.gu, 2 * pr + 1, Dh, xs, rows, yu);
          if (lane == 0)
            for (int m = 0; m < rows; ++m) {
              const float gb = round_bf16(y[m]), ub = round_bf16(yu[m]);
              a.act[(size_t)m * F + pr] = __float2bfloat16_rn(round_bf16(silu_f(gb)) * ub);
            }
        }
      }
      depth_grid_sync(a.bar, gen, a.err);
      // ---- E: x = bf16(x + bf16(W_d act))
      depth_copy_rows(a.act, F, rows, F, xs);
      for (int n = gw; n < Dh; n += nw) {
        depth_dot(L.d, n, F, xs, rows, y);
        if (lane == 0)
          for (int m = 0; m < rows; ++m) {
            __nv_bfloat16* o = a.x + (size_t)m * Dh + n;
            *o = __float2bfloat16_rn(__bfloat162float(__ldcg(o)) + round_bf16(y[m]));
          }
      }
      depth_grid_sync(a.bar, gen, a.err);
    }
    if (j == 0) continue;
    // ---- codebook j: logits of head j on norm_f(x), guided, Gumbel-argmax
    for (int m = 0; m < rows; ++m) src[m] = a.x + (size_t)m * Dh;
    depth_stage_rows(src, rows, Dh, xs);
    depth_norm_staged(xs, rows, Dh, a.final_norm, a.eps, rinv);
    if (tid < kMaxRows) best[tid] = 0ull;
    __syncthreads();
    const FrameParams* fp = a.fp;
    const unsigned long long ib = (unsigned long long)j << 32;
    for (int n = gw; n < a.V; n += nw) {
      depth_dot(a.heads[j - 1], n, Dh, xs, rows, y);
      if (lane < keys) {
        const int k = lane;
        float g = y[k];
        if (cfg) g = __fadd_rn(y[2 * k + 1], __fmul_rn(fp->cfg_scale, __fsub_rn(y[2 * k], y[2 * k + 1])));
        const float z = __fadd_rn(__fdiv_rn(g, fp->temperature),
                                  gumbel_noise(fp->seed, fp->frame, (unsigned long long)k, ib | (unsigned long long)n));
        atomicMax(&best[k], argmax_key(z, n));
      }
      if (a.logits && lane == 0)
        for (int m = 0; m < rows; ++m) a.logits[((size_t)m * a.NC + (j - 1)) * a.V + n] = y[m];
    }
    __syncthreads();
    if (tid < keys) a.part[(size_t)blockIdx.x * kMaxRows + tid] = best[tid];
    depth_grid_sync(a.bar, gen, a.err);
    if (tid < keys) {  // every CTA: the winners in CTA order
      unsigned long long b = 0ull;
      for (int c = 0; c < (int)gridDim.x; ++c) {
        const unsigned long long v = __ldcg(a.part + (size_t)c * kMaxRows + tid);
        b = v > b ? v : b;
      }
      const int code = key_idx(b);
      const int nm = cfg ? 2 : 1;
      for (int q = 0; q < nm; ++q) {
        const int r = cfg ? 2 * tid + q : tid;
        if (blockIdx.x == 0) a.codes[(size_t)r * a.NC + (j - 1)] = code;
        pcode[r] = a.forced ? __ldcg(a.forced + (size_t)r * a.NC + (j - 1)) : code;
      }
    }
    __syncthreads();
    // the winners' buffer is read by every CTA before the next position's
    // head phase writes it again: at least five barriers lie between
  }
}


size_t depth_smem_bytes(const DepthArgs& a) {
  int k = a.Hin;
  if (a.F > k) k = a.F;
  if (a.Dh > k) k = a.Dh;
  if (a.nh * a.hd > k) k = a.nh * a.hd;
  return depth_rope_bytes(a) + (size_t)a.rows * k * sizeof(__nv_bfloat16);
}

// One cooperative launch of at most `max_grid` CTAs (one per SM), all resident.
cudaError_t launch_depth(const DepthArgs& a, int max_grid, cudaStream_t st) {
  const size_t smem = depth_smem_bytes(a);
  cudaError_t e = cudaFuncSetAttribute(depth_decode_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, depth_decode_kernel, kDepthThreads,
                                                    smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(max_grid);
  cfg.blockDim = dim3(kDepthThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, depth_decode_kernel, a);
}

}  // namespace m3
