// dit_kernels.cuh -- the DiT's kernels around its GEMMs: input assembly,
// Fourier timestep embedding and its MLP, LayerNorm, bidirectional attention
// over the chunk, and the guided velocity with the Euler step.
//
// Sources (page title, section): "MiniMax-Music3 ... DiffSynth-Studio",
// "各子模型的结构要点" (input = noisy latent | condition, 2*128 + 2048
// channels; partial rotary and Fourier time embeddings) and "第三阶段"
// (guided velocity uncond + cfg_scale * (cond - uncond), the all-zero
// condition as the unconditional branch, the scheduler step); "MiniMax Music 3
// on Metal", "Precision is the reference's" (fp16 with fp32 sums) and its
// kernel list (LayerNorm, timestep MLP, guided velocity, Euler step,
// attention with fp16 probabilities for P V).
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "attention.cuh"  // ldmatrix / mma.sync helpers
#include "common.cuh"

namespace m3 {

// Per-step scalars, written by a kernel before the step's graph so that the
// graph reads them from a fixed address.
struct DitParams {
  float sigma, sigma_next, cfg_scale, t;  // t = 1000 sigma
};

__global__ void dit_set_params_kernel(DitParams* dst, DitParams v) {
  if (threadIdx.x == 0) *dst = v;
}

// hin[b][t] = [f16(x[t]) | ctx[t] | cond[t] (b = 0) or 0 (b = 1)], B = 2.
__global__ void dit_assemble_kernel(const float* __restrict__ x, const __half* __restrict__ ctx,
                                    const __half* __restrict__ cond, int T, int L, int C,
                                    __half* __restrict__ hin) {
  const int Cin = 2 * L + C;
  const int row = blockIdx.x;  // 0 .. 2T-1
  const int b = row / T, t = row % T;
  __half* out = hin + (size_t)row * Cin;
  for (int i = threadIdx.x; i < Cin; i += blockDim.x) {
    __half v;
    if (i < L) v = __float2half_rn(x[(size_t)t * L + i]);
    else if (i < 2 * L) v = ctx[(size_t)t * L + (i - L)];
    else v = b == 0 ? cond[(size_t)t * C + (i - 2 * L)] : __float2half_rn(0.0f);
    out[i] = v;
  }
}

// Fourier features of t = 1000 sigma: feat[k] = f16(cos(t f_k)),
// feat[half + k] = f16(sin(t f_k)), f_k = 10000^(-k/half), in fp64.
__global__ void dit_time_features_kernel(const DitParams* __restrict__ p, int temb,
                                         __half* __restrict__ feat) {
  const int half = temb / 2;
  const double t = (double)p->t;
  for (int k = threadIdx.x; k < half; k += blockDim.x) {
    const double f = exp(-log(10000.0) * (double)k / (double)half);
    const double a = t * f;
    feat[k] = __float2half_rn((float)cos(a));
    feat[half + k] = __float2half_rn((float)sin(a));
  }
}

// y[o] = f16(act(f16(sum_k W[o][k] x[k]))), one warp per output row, W [N][K]
// fp16 (K a multiple of 8), x [K] fp16; act = SiLU when silu != 0.
__global__ void dit_gemv_kernel(const __half* __restrict__ W, const __half* __restrict__ x, int N,
                                int K, int silu, __half* __restrict__ y) {
  const int warps = blockDim.x >> 5;
  const int o = blockIdx.x * warps + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (o >= N) return;
  const __half* w = W + (size_t)o * K;
  float acc = 0.0f;
  for (int k = lane * 8; k < K; k += 256) {
    const uint4 wv = *reinterpret_cast<const uint4*>(w + k);
    const uint4 xv = *reinterpret_cast<const uint4*>(x + k);
    const __half2* wh = reinterpret_cast<const __half2*>(&wv);
    const __half2* xh = reinterpret_cast<const __half2*>(&xv);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 a = __half22float2(wh[j]), b = __half22float2(xh[j]);
      acc = __fadd_rn(acc, __fmul_rn(a.x, b.x));
      acc = __fadd_rn(acc, __fmul_rn(a.y, b.y));
    }
  }
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
  if (lane == 0) {
    float v = __half2float(__float2half_rn(acc));
    if (silu) v = __fdiv_rn(v, __fadd_rn(1.0f, expf(-v)));
    y[o] = __float2half_rn(v);
  }
}

// LayerNorm of rows of W fp16 values (W a multiple of 256): one warp per row,
// mean and variance in fp32 from registers (two passes), out =
// f16(((x - mean) * r) * g + b), r = 1 / sqrt(var + eps).
template <int W>
__global__ void dit_layernorm_kernel(const __half* __restrict__ x, const __half* __restrict__ g,
                                     const __half* __restrict__ b, int rows, float eps,
                                     __half* __restrict__ out) {
  constexpr int PER = W / 32;  // values per lane
  constexpr int CH = PER / 8;  // 16-byte chunks per lane
  const int warps = blockDim.x >> 5;
  const int row = blockIdx.x * warps + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= rows) return;
  const __half* xr = x + (size_t)row * W;
  float v[PER];
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    const uint4 u = *reinterpret_cast<const uint4*>(xr + (c * 32 + lane) * 8);
    const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __half22float2(h[j]);
      v[c * 8 + 2 * j] = f.x;
      v[c * 8 + 2 * j + 1] = f.y;
    }
  }
  float s = 0.0f;
#pragma unroll
  for (int i = 0; i < PER; ++i) s += v[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float mean = s / (float)W;
  float q = 0.0f;
#pragma unroll
  for (int i = 0; i < PER; ++i) q = fmaf(v[i] - mean, v[i] - mean, q);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
  const float r = 1.0f / sqrtf(q / (float)W + eps);
  __half* orow = out + (size_t)row * W;
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    const int i0 = (c * 32 + lane) * 8;
    const uint4 gu = *reinterpret_cast<const uint4*>(g + i0);
    const uint4 bu = *reinterpret_cast<const uint4*>(b + i0);
    const __half2* gh = reinterpret_cast<const __half2*>(&gu);
    const __half2* bh = reinterpret_cast<const __half2*>(&bu);
    uint32_t res[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 gf = __half22float2(gh[j]), bf = __half22float2(bh[j]);
      const float y0 = __fadd_rn(__fmul_rn(__fmul_rn(v[c * 8 + 2 * j] - mean, r), gf.x), bf.x);
      const float y1 = __fadd_rn(__fmul_rn(__fmul_rn(v[c * 8 + 2 * j + 1] - mean, r), gf.y), bf.y);
      const __half2 h = __floats2half2_rn(y0, y1);
      res[j] = *reinterpret_cast<const uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(orow + i0) = make_uint4(res[0], res[1], res[2], res[3]);
  }
}

// Partial-RoPE table of the chunk's positions: cs[p][i] = (cos, sin) of
// p * theta^(-2i/rot), i < rot/2, in fp64, then fp32.
__global__ void dit_rope_table_kernel(int T, int rot, double theta, float2* __restrict__ cs) {
  const int h = rot / 2;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < T * h; e += gridDim.x * blockDim.x) {
    const int p = e / h, i = e % h;
    const double ang = (double)p * pow(theta, -2.0 * (double)i / (double)rot);
    cs[e] = make_float2((float)cos(ang), (float)sin(ang));
  }
}

// ------------------------------------------------------------- attention --
// Bidirectional attention of one (batch element, head) over its T tokens,
// heads of 64: a CTA of 4 warps takes 64 queries (16 per warp) and walks the
// keys in tiles of 64 with warp-level tensor-core MMA (m16n8k16, fp16 in,
// fp32 accumulation): S = Q K^T / 8, online softmax in fp32 (in log2 units,
// exp2), P rounded to fp16 for O += P V, O / l at the end.  K / V tiles double-buffered in
// shared memory by cp.async.
constexpr int kDaWarps = 4;
constexpr int kDaQ = 16 * kDaWarps;  // queries per CTA
constexpr int kDaKT = 64;            // keys per tile
constexpr int kDaD = 64;             // head dim
constexpr int kDaRowB = kDaD * 2;    // 128 bytes per token row
constexpr size_t kDaSmem = (size_t)(kDaQ + 4 * kDaKT) * kDaRowB;  // Q + 2 x (K, V)

// Byte offset of 16-byte chunk c of row r in a [rows][64] fp16 tile whose
// chunks are XOR-swizzled by (r & 7): conflict-free ldmatrix.
__device__ __forceinline__ uint32_t da_off(int r, int c) {
  return (uint32_t)(r * kDaRowB + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ void cp16(uint32_t dst, const void* src, bool ok) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(ok ? 16 : 0)
               : "memory");
}

__global__ void __launch_bounds__(kDaWarps * 32)
    dit_attention_kernel(const __half* __restrict__ qkv, int T, int W, __half* __restrict__ out) {
  extern __shared__ __align__(128) uint8_t dsm[];
  const uint32_t sQ = smem_u32(dsm);
  const uint32_t sK0 = sQ + kDaQ * kDaRowB;  // [2][K tile | V tile]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q0 = blockIdx.x * kDaQ, hd = blockIdx.y, b = blockIdx.z;
  const size_t ld = (size_t)3 * W;
  const __half* base = qkv + (size_t)b * T * ld;
  const int nkt = (T + kDaKT - 1) / kDaKT;

  auto load_kv = [&](int kt, int buf) {
    const uint32_t sk = sK0 + (uint32_t)buf * 2 * kDaKT * kDaRowB, sv = sk + kDaKT * kDaRowB;
    for (int e = tid; e < kDaKT * 8; e += kDaWarps * 32) {
      const int r = e >> 3, c = e & 7, j = kt * kDaKT + r;
      const bool ok = j < T;
      const __half* row = base + (size_t)(ok ? j : 0) * ld;
      cp16(sk + da_off(r, c), row + W + hd * kDaD + c * 8, ok);
      cp16(sv + da_off(r, c), row + 2 * W + hd * kDaD + c * 8, ok);
    }
  };
  for (int e = tid; e < kDaQ * 8; e += kDaWarps * 32) {
    const int r = e >> 3, c = e & 7, t = q0 + r;
    const bool ok = t < T;
    cp16(sQ + da_off(r, c), base + (size_t)(ok ? t : 0) * ld + hd * kDaD + c * 8, ok);
  }
  load_kv(0, 0);
  asm volatile("cp.async.commit_group;" ::: "memory");

  // Q fragments of this warp's 16 rows: 4 k-steps of 16 dims
  uint32_t qa[4][4];
  float o[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.0f, 0.0f};
  // scores in log2 units: exp(s - m) = exp2(s log2e - m log2e), one MUFU op
  const float scale = 0.125f * 1.4426950408889634f;  // 1 / sqrt(64) * log2(e)

  for (int kt = 0; kt < nkt; ++kt) {
    if (kt + 1 < nkt) load_kv(kt + 1, (kt + 1) & 1);
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 1;" ::: "memory");
    __syncthreads();
    if (kt == 0) {
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const int r = warp * 16 + (lane & 15), c = ks * 2 + (lane >> 4);
        ldsm_x4(sQ + da_off(r, c), qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3]);
      }
    }
    const uint32_t sk = sK0 + (uint32_t)(kt & 1) * 2 * kDaKT * kDaRowB, sv = sk + kDaKT * kDaRowB;
    // S = Q K^T for 64 keys: 8 n-tiles of 8 keys
    float s[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.0f;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {  // two n-tiles (16 keys) per ldmatrix.x4
        uint32_t b0, b1, b2, b3;
        const int r = np * 16 + (lane & 7) + ((lane >> 4) << 3), c = ks * 2 + ((lane >> 3) & 1);
        ldsm_x4(sk + da_off(r, c), b0, b1, b2, b3);
        mma16816<1>(s[2 * np], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b0, b1);
        mma16816<1>(s[2 * np + 1], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b2, b3);
      }
    }
    // scale, mask keys beyond T, online softmax (rows lane/4 and lane/4 + 8)
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = kt * kDaKT + nt * 8 + (lane & 3) * 2 + (e & 1);
        s[nt][e] = key < T ? s[nt][e] * scale : -INFINITY;
        mx[e >> 1] = fmaxf(mx[e >> 1], s[nt][e]);
      }
    float alpha[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
      const float mn = fmaxf(m_run[h], mx[h]);
      alpha[h] = exp2f(m_run[h] - mn);  // 0 at the first tile (m_run = -inf)
      m_run[h] = mn;
    }
    float ls[2] = {0.0f, 0.0f};
    uint32_t pa[4][4];  // P as the A operand of P V: 4 k-steps of 16 keys
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const float e0 = exp2f(s[nt][0] - m_run[0]), e1 = exp2f(s[nt][1] - m_run[0]);
      const float e2 = exp2f(s[nt][2] - m_run[1]), e3 = exp2f(s[nt][3] - m_run[1]);
      ls[0] += e0 + e1;
      ls[1] += e2 + e3;
      const __half2 h01 = __floats2half2_rn(e0, e1), h23 = __floats2half2_rn(e2, e3);
      pa[nt >> 1][(nt & 1) * 2 + 0] = *reinterpret_cast<const uint32_t*>(&h01);
      pa[nt >> 1][(nt & 1) * 2 + 1] = *reinterpret_cast<const uint32_t*>(&h23);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      ls[h] += __shfl_xor_sync(0xffffffffu, ls[h], 1);
      ls[h] += __shfl_xor_sync(0xffffffffu, ls[h], 2);
      l_run[h] = l_run[h] * alpha[h] + ls[h];
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      o[i][0] *= alpha[0];
      o[i][1] *= alpha[0];
      o[i][2] *= alpha[1];
      o[i][3] *= alpha[1];
    }
    // O += P V: V tile [key][dim] via ldmatrix.trans as the B operand
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
      for (int dp = 0; dp < 4; ++dp) {  // two dim n-tiles (16 dims) per ldmatrix.x4
        uint32_t b0, b1, b2, b3;
        const int r = ks * 16 + (lane & 15), c = dp * 2 + (lane >> 4);
        ldsm_x4_t(sv + da_off(r, c), b0, b1, b2, b3);
        mma16816<1>(o[2 * dp], pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3], b0, b1);
        mma16816<1>(o[2 * dp + 1], pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3], b2, b3);
      }
    }
    __syncthreads();  // the buffer of this tile is refilled two tiles later
  }
  // o / l -> f16, rows lane/4 and lane/4 + 8 of the warp's 16
  const int r0 = q0 + warp * 16 + (lane >> 2);
  const float inv[2] = {1.0f / l_run[0], 1.0f / l_run[1]};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int t = r0 + h * 8;
    if (t >= T) continue;
    __half* orow = out + ((size_t)b * T + t) * W + hd * kDaD;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const int d = nt * 8 + (lane & 3) * 2;
      *reinterpret_cast<__half2*>(orow + d) =
          __floats2half2_rn(__fdiv_rn(o[nt][2 * h], l_run[h]), __fdiv_rn(o[nt][2 * h + 1], l_run[h]));
    }
  }
  (void)inv;
}

// vg = vu + c (vc - vu) (fp32 from the fp16 predictions); x += (sigma_next - sigma) vg.
__global__ void dit_guide_step_kernel(const DitParams* __restrict__ p, const __half* __restrict__ v,
                                      int n, float* __restrict__ x, float* __restrict__ vg_out) {
  const float dt = p->sigma_next - p->sigma, c = p->cfg_scale;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const float vc = __half2float(v[i]), vu = __half2float(v[n + i]);
    const float g = __fadd_rn(vu, __fmul_rn(c, __fsub_rn(vc, vu)));
    if (vg_out) vg_out[i] = g;
    x[i] = __fadd_rn(x[i], __fmul_rn(dt, g));
  }
}

}  // namespace m3
