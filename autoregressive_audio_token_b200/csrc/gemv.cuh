// gemv.cuh -- weight-streaming GEMV for the decode step (1..4 activation rows).
//
// The decode step reads every weight once per frame ("MiniMax Music 3
// modular pipeline", finding 4: the AR stage is memory-bandwidth bound), so
// each projection is a GEMV whose speed is the HBM stream of W:
//   * one CTA per SM, each owning a contiguous block of output rows;
//   * a producer warp streams that block through a 3-stage ring of 32 KB
//     shared-memory stages with non-multicast bulk copies (TMA engine,
//     mbarrier transaction counts, L2 evict-first), starting before the
//     previous kernel has finished (programmatic dependent launch: weights
//     do not depend on it);
//   * 8 consumer warps own fixed K positions, keep the (normalised)
//     activation in registers, and FMA 16 weights per row per thread; a
//     butterfly shuffle + one named barrier per stage reduces over K;
//   * the consumer of a norm computes RMSNorm itself (no separate pass):
//     "MiniMax Music 3 on Metal", section "Next steps", suggests folding the
//     RMS norms into the GEMVs that read them;
//   * epilogues: store bf16 (QKV), residual add (O, down), SwiGLU on
//     interleaved gate/up rows, or the fused lm_head sampler (fp32 logits,
//     CFG over row pairs, Gumbel noise, block argmax, last-CTA reduction).
// Weight formats: bf16, int8 + fp32 scale per row, int8 + fp32 scale per
// group of 128 inputs ("MiniMax Music 3 on Metal", section "Precision").
#pragma once

#include "common.cuh"
#include "noise.cuh"

namespace m3 {

enum : int { EPI_STORE = 0, EPI_RESID = 1, EPI_SWIGLU = 2, EPI_SAMPLE = 3 };
enum : int { WF_BF16 = 0, WF_I8ROW = 1, WF_I8G128 = 2 };

constexpr int kConsumers = 512;                  // 16 compute warps
constexpr int kEpiWarp = kConsumers / 32;        // warp 8: epilogue
constexpr int kGemvThreads = kConsumers + 64;    // + epilogue warp + producer warp
constexpr int kPartBufs = 4;                     // partial-sum buffers in flight
#ifndef M3_STAGE_BYTES
#define M3_STAGE_BYTES 65536
#endif
#ifndef M3_STAGES
#define M3_STAGES 3
#endif
#ifndef M3_PREFETCH_AHEAD
#define M3_PREFETCH_AHEAD 0
#endif
constexpr int kStageBytes = M3_STAGE_BYTES;
constexpr int kStages = M3_STAGES;
constexpr int kMaxRows = 16;
constexpr int kPrefetchAhead = M3_PREFETCH_AHEAD;  // stages prefetched into L2 beyond the ring

// Per-frame scalars, written once per frame by set_frame_params before the
// frame's first kernel.
struct FrameParams {
  int rows;
  int cfg_on;
  float cfg_scale;
  float temperature;
  unsigned long long seed;
  unsigned long long frame;
  int pos[kMaxRows];
  int top_k;  // the lm_head draw keeps the top_k guided logits; 0 keeps all
};

struct SampleArgs {
  float* logits;              // [rows][logits_ld] fp32 at column n; nullable
  int logits_ld;
  int* codes;                 // code of batch row r at codes[r * code_stride]
  int code_stride;
  int* prev;                  // nullable: fed-forward code per row [rows]
  const int* forced;          // nullable: forced[r * forced_stride] replaces prev
  int forced_stride;
  unsigned long long index_base;  // noise index of output row n is index_base + n
  float* part_z;              // [grid][kMaxRows] scratch
  int* part_i;                // [grid][kMaxRows] scratch
  unsigned int* counter;      // zero at rest; the last CTA resets it
  __nv_bfloat16* h_out;       // nullable: normalised input [rows][K] (CTA 0 writes)
  float* gbuf;                // nullable: [keys][N] guided logits for the top-k draw
  int end_row1;               // 1 + the output row that is the end token (0: none)
  unsigned long long end_index;  // that row's noise index (its vocab row)
};

// Noise index of output row n of a draw: the code block's vocab rows
// index_base + n, and the end token's own vocab row for the end candidate.
__device__ __forceinline__ unsigned long long smp_index(const SampleArgs& s, int n) {
  return n == s.end_row1 - 1 ? s.end_index : s.index_base + (unsigned long long)n;
}

// Order-preserving key for the sampler's argmax: larger z first, then the
// smaller index (-0.0 counts as +0.0, as in a float comparison).
__device__ __forceinline__ unsigned long long argmax_key(float z, int idx) {
  uint32_t b = __float_as_uint(z == 0.0f ? 0.0f : z);
  b = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  return ((unsigned long long)b << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)idx);
}

__device__ __forceinline__ float key_z(unsigned long long key) {
  uint32_t b = (uint32_t)(key >> 32);
  b = (b & 0x80000000u) ? (b & 0x7FFFFFFFu) : ~b;
  return __uint_as_float(b);
}

__device__ __forceinline__ int key_idx(unsigned long long key) {
  return (int)(0xFFFFFFFFu - (uint32_t)(key & 0xFFFFFFFFull));
}

struct GemvArgs {
  const void* w;              // [N][K] row-major, bf16 or int8
  const float* scales;        // int8: [N] or [N][K/128]
  int N, K;
  int row0;                   // first batch row of this launch
  int mr;                     // batch rows of this launch (<= MR)
  const __nv_bfloat16* x;     // [rows][ldx] input activations (row0-relative rows)
  int ldx;
  const __nv_bfloat16* gamma; // RMSNorm gain over K, nullable = no norm
  float eps;
  __nv_bfloat16* out;         // STORE/RESID: [rows][ldo] at column n; SWIGLU: column n/2
  int ldo;
  const FrameParams* fp;
  SampleArgs smp;
  int* err;
  // tiled kernels (gemv_tile.cuh, gemv_dyn.cuh) only: CTAs per cluster,
  // stage bytes, stages; the dynamic kernel's {claim, done} counter pair
  int tc, tsb, tns;
  int lazy_claim;  // dynamic GEMV: claim ahead only once the consumers run
  unsigned* ctr;
  // RMSNorm partials: a residual-add launch writes sum(x_new^2) per (row m,
  // 16-row unit u) at ssq_out[m * units + u]; a normalising launch reads
  // ssq_n such partials per row from ssq_in (either may be null)
  float* ssq_out;
  const float* ssq_in;
  int ssq_n;
};

template <int TPR, int ESZ>
struct GemvShape {
  static constexpr int EPT = 16 / ESZ;                // K elements per thread: one 16-B chunk
  static constexpr int KC = TPR * EPT;                // K elements per segment
  static constexpr int G = kConsumers / TPR;          // rows in flight per pass
  static constexpr int R = kStageBytes / (KC * ESZ);  // rows (segments) per stage
  static constexpr int P = R / G;                     // passes per stage
  static constexpr int W = TPR < 32 ? TPR : 32;       // shuffle width
  static constexpr int SLOTS = kConsumers / W;        // partial sums per row
  static_assert(R % G == 0 && R % 2 == 0, "stage geometry");
};

// Dynamic shared memory of one CTA (the host sizes it with the same formula).
template <int MR, int TPR, int ESZ>
__host__ __device__ constexpr size_t gemv_smem_bytes(int rows_cta_max) {
  using S = GemvShape<TPR, ESZ>;
  return (size_t)kStages * kStageBytes + 2 * kStages * sizeof(uint64_t) +
         sizeof(float) * (kPartBufs * S::SLOTS * S::P * MR + (kConsumers / 32 + 1) * MR +
                          (size_t)rows_cta_max * MR) +
         (sizeof(float) + sizeof(int)) * S::R * MR + 64;
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + expf(-g)); }

// Reduce V values (one per row-in-stage x batch row) over the 32 lanes of a
// warp as a reduce-scatter: after the call lane l holds in v[0] the warp
// total of value index l >> (5 - log2 V).  V - 1 + (5 - log2 V) shuffles
// instead of 5 V.
template <int V>
__device__ __forceinline__ void warp_reduce_scatter(float* v, int lane) {
  static_assert(V >= 1 && V <= 32 && (V & (V - 1)) == 0, "V must be a power of two <= 32");
  int n = V;
#pragma unroll
  for (int half = 16; half >= 1; half >>= 1) {
    if (n > 1) {
      const bool up = (lane & half) != 0;
      const int h = n / 2;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        if (i < h) {
          const float send = up ? v[i] : v[i + h];
          const float keep = up ? v[i + h] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, half);
        }
      }
      n = h;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], half);
    }
  }
}

template <int MR, int WF, int EPI, int TPR>
__global__ void __launch_bounds__(kGemvThreads, 1) gemv_kernel(const GemvArgs a) {
  constexpr int ESZ = WF == WF_BF16 ? 2 : 1;
  using S = GemvShape<TPR, ESZ>;
  constexpr int KC = S::KC, G = S::G, R = S::R, P = S::P, W = S::W, SLOTS = S::SLOTS;
  constexpr int EPT = S::EPT;
  constexpr int UNIT = EPI == EPI_SWIGLU ? 2 : 1;
  constexpr int V = P * MR;  // partial sums per thread per stage
  constexpr int LV = V == 1 ? 0 : V == 2 ? 1 : V == 4 ? 2 : V == 8 ? 3 : V == 16 ? 4 : 5;
  constexpr bool kScatter = (W == 32) && (V <= 32);
  // named barriers: 1 norm (compute warps); 2.. partial buffer full; 2+kPartBufs.. empty
  constexpr int kBarNorm = 1, kBarFull = 2, kBarEmpty = 2 + kPartBufs;
  constexpr int kPartThreads = kConsumers + 32;  // compute warps + epilogue warp

  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  float* part = reinterpret_cast<float*>(empty + kStages);  // [kPartBufs][SLOTS][V]
  float* nrm = part + kPartBufs * SLOTS * V;                 // [8][MR] + [MR]
  float* accr = nrm + (kConsumers / 32 + 1) * MR;              // [rows_cta][MR]

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int K = a.K;
  const int nkc = (K + KC - 1) / KC;
  const int U = a.N / UNIT;
  const int u0 = (int)((long long)U * blockIdx.x / gridDim.x);
  const int u1 = (int)((long long)U * (blockIdx.x + 1) / gridDim.x);
  const int r_begin = u0 * UNIT, r_end = u1 * UNIT;
  const int nrows = r_end - r_begin;
  const int spk = (nrows + R - 1) / R;
  const int nstages = spk * nkc;
  float* sbz = accr + (size_t)spk * R * MR;            // sampler: best z per role
  int* sbi = reinterpret_cast<int*>(sbz + R * MR);      // sampler: its index

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumers / 32);
    }
    fence_barrier_init();
  }
  if constexpr (EPI == EPI_SAMPLE) {
    for (int c = tid; c < R * MR; c += blockDim.x) {
      sbz[c] = -INFINITY;
      sbi[c] = 0x7fffffff;
    }
  }
  __syncthreads();
  pdl_launch_dependents();

  // ------------------------------------------------------------ producer --
  if (warp == kEpiWarp + 1) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      const uint8_t* wb = static_cast<const uint8_t*>(a.w);
      auto seg = [&](int s, int& rs, int& re, int& kc, uint32_t& segb) {
        kc = s / spk;
        const int sr = s % spk;
        rs = r_begin + sr * R;
        re = min(rs + R, r_end);
        segb = (uint32_t)(min(KC, K - kc * KC) * ESZ);
      };
      auto prefetch = [&](int s) {
        int rs, re, kc;
        uint32_t segb;
        seg(s, rs, re, kc, segb);
        for (int r = rs; r < re; ++r)
          bulk_prefetch_l2(wb + ((size_t)r * K + (size_t)kc * KC) * ESZ, segb);
      };
      constexpr int PFD = kStages + kPrefetchAhead;
      if (kPrefetchAhead > 0)
        for (int s = kStages; s < min(PFD, nstages); ++s) prefetch(s);
      for (int s = 0; s < nstages; ++s) {
        const int slot = s % kStages;
        if (s >= kStages && !mbar_wait(&empty[slot], ((s / kStages) - 1) & 1, a.err)) break;
        int rs, re, kc;
        uint32_t segb;
        seg(s, rs, re, kc, segb);
        mbar_arrive_expect_tx(&full[slot], segb * (uint32_t)(re - rs));
        uint8_t* dst = ring + slot * kStageBytes;
        for (int r = rs; r < re; ++r)
          bulk_g2s(dst + (size_t)(r - rs) * KC * ESZ,
                   wb + ((size_t)r * K + (size_t)kc * KC) * ESZ, segb, &full[slot], pol);
        if (kPrefetchAhead > 0 && s + PFD < nstages) prefetch(s + PFD);
      }
    }
    return;
  }

  // ------------------------------------------------------------ epilogue --
  // Sums the partials of each stage and applies the epilogue; the compute
  // warps never wait on its global-memory round trips (kPartBufs stages of
  // slack).
  if (warp == kEpiWarp) {
    pdl_wait();  // residual / outputs are shared with the previous kernel
    const int mr = a.mr;
    const int np = (EPI == EPI_SAMPLE) ? (a.fp->cfg_on ? mr / 2 : mr) : 0;
    int s = 0;
    for (int kc = 0; kc < nkc; ++kc) {
      const bool last_kc = (kc == nkc - 1);
      for (int sr = 0; sr < spk; ++sr, ++s) {
        const int b = s % kPartBufs;
        named_bar_sync(kBarFull + b, kPartThreads);
        const float* pb = part + b * SLOTS * V;
        const int rs = r_begin + sr * R;
        const int nr = min(R, r_end - rs);
        auto row_sum = [&](int rl, int m) -> float {
          const int gg = rl % G, pp = rl / G;
          constexpr int SPG = TPR / W;  // slots per row group
          float y = 0.0f;
#pragma unroll
          for (int q = 0; q < SPG; ++q) y += pb[(gg * SPG + q) * V + pp * MR + m];
          return y;
        };
        if constexpr (EPI == EPI_STORE || EPI == EPI_RESID) {
          for (int c = lane; c < R * MR; c += 32) {
            const int rl = c / MR, m = c % MR;
            if (rl >= nr || m >= mr) continue;
            float y = row_sum(rl, m);
            if (nkc > 1) {
              float* ar = accr + (size_t)(sr * R + rl) * MR + m;
              if (kc > 0) y += *ar;
              if (!last_kc) {
                *ar = y;
                continue;
              }
            }
            const int n = rs + rl;
            if constexpr (WF == WF_I8ROW) y *= __ldg(a.scales + n);
            __nv_bfloat16* o = a.out + (size_t)m * a.ldo + n;
            if constexpr (EPI == EPI_STORE) {
              *o = __float2bfloat16_rn(y);
            } else {
              *o = __float2bfloat16_rn(__bfloat162float(*o) + round_bf16(y));
            }
          }
        } else if constexpr (EPI == EPI_SWIGLU) {
          for (int c = lane; c < (R / 2) * MR; c += 32) {
            const int j = c / MR, m = c % MR;
            if (2 * j >= nr || m >= mr) continue;
            float yg = row_sum(2 * j, m), yu = row_sum(2 * j + 1, m);
            if (nkc > 1) {
              float* ag = accr + (size_t)(sr * R + 2 * j) * MR + m;
              float* au = accr + (size_t)(sr * R + 2 * j + 1) * MR + m;
              if (kc > 0) {
                yg += *ag;
                yu += *au;
              }
              if (!last_kc) {
                *ag = yg;
                *au = yu;
                continue;
              }
            }
            const int n = rs + 2 * j;
            if constexpr (WF == WF_I8ROW) {
              yg *= __ldg(a.scales + n);
              yu *= __ldg(a.scales + n + 1);
            }
            const float gb = round_bf16(yg), ub = round_bf16(yu);
            const float act = round_bf16(round_bf16(silu_f(gb)) * ub);
            a.out[(size_t)m * a.ldo + n / 2] = __float2bfloat16_rn(act);
          }
        } else {  // EPI_SAMPLE (K fits one segment): roles (row-in-stage, key)
          const bool cfg = a.fp->cfg_on != 0;
          for (int c = lane; c < R * MR; c += 32) {
            const int rl = c / MR, p = c % MR;
            if (rl >= nr || p >= np) continue;
            const int n = rs + rl;
            const int m0 = cfg ? 2 * p : p;
            float y0 = row_sum(rl, m0);
            float y1 = cfg ? row_sum(rl, m0 + 1) : 0.0f;
            if constexpr (WF == WF_I8ROW) {
              const float sc = __ldg(a.scales + n);
              y0 *= sc;
              y1 *= sc;
            }
            if (a.smp.logits) {
              a.smp.logits[(size_t)(a.row0 + m0) * a.smp.logits_ld + n] = y0;
              if (cfg) a.smp.logits[(size_t)(a.row0 + m0 + 1) * a.smp.logits_ld + n] = y1;
            }
            float gl = y0;
            if (cfg) gl = __fadd_rn(y1, __fmul_rn(a.fp->cfg_scale, __fsub_rn(y0, y1)));
            const unsigned long long key = cfg ? (unsigned long long)(a.row0 / 2 + p)
                                               : (unsigned long long)(a.row0 + p);
            const float gn = gumbel_noise(a.fp->seed, a.fp->frame, key, smp_index(a.smp, n));
            const float z = __fadd_rn(__fdiv_rn(gl, a.fp->temperature), gn);
            if (z > sbz[c] || (z == sbz[c] && n < sbi[c])) {
              sbz[c] = z;
              sbi[c] = n;
            }
          }
        }
        if (s + kPartBufs < nstages) named_bar_arrive(kBarEmpty + b, kPartThreads);
      }
    }
    if constexpr (EPI == EPI_SAMPLE) {
      // CTA-level argmax per key, then the last CTA reduces over CTAs.
      __syncwarp();
      int last = 0;
      if (lane < np) {
        float bz = -INFINITY;
        int bi = 0x7fffffff;
        for (int rl = 0; rl < R; ++rl) {
          const float z = sbz[rl * MR + lane];
          const int i = sbi[rl * MR + lane];
          if (z > bz || (z == bz && i < bi)) {
            bz = z;
            bi = i;
          }
        }
        a.smp.part_z[blockIdx.x * kMaxRows + lane] = bz;
        a.smp.part_i[blockIdx.x * kMaxRows + lane] = bi;
        __threadfence();
      }
      __syncwarp();
      if (lane == 0) {
        __threadfence();
        const unsigned old = atomicAdd(a.smp.counter, 1u);
        last = (old == gridDim.x - 1);
      }
      last = __shfl_sync(0xffffffffu, last, 0);
      if (!last) return;
      __threadfence();
      // per key, the warp's lanes take every 32nd CTA's winner; the 64-bit
      // key's max (largest z, lowest index on equal z) by a shuffle tree
      const bool cfg = a.fp->cfg_on != 0;
      for (int p = 0; p < np; ++p) {
        unsigned long long kb = 0ull;
        for (int bb = lane; bb < (int)gridDim.x; bb += 32) {
          const int i = __ldcg(a.smp.part_i + bb * kMaxRows + p);
          if (i == 0x7fffffff) continue;  // a CTA without outputs
          const unsigned long long k = argmax_key(__ldcg(a.smp.part_z + bb * kMaxRows + p), i);
          kb = k > kb ? k : kb;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const unsigned long long y = __shfl_xor_sync(0xffffffffu, kb, o);
          kb = y > kb ? y : kb;
        }
        if (lane == 0) {
          const int bi = kb ? key_idx(kb) : 0x7fffffff;
          const int nm = cfg ? 2 : 1;
          for (int q = 0; q < nm; ++q) {
            const int r = a.row0 + (cfg ? 2 * p + q : p);
            a.smp.codes[(size_t)r * a.smp.code_stride] = bi;
            if (a.smp.prev)
              a.smp.prev[r] = a.smp.forced ? a.smp.forced[(size_t)r * a.smp.forced_stride] : bi;
          }
        }
      }
      if (lane == 0) *a.smp.counter = 0u;
    }
    return;
  }

  // ------------------------------------------------------- compute warps --
  const int g = tid / TPR, t = tid % TPR;
  const int mr = a.mr;
  const __nv_bfloat16* __restrict__ x = a.x;

  pdl_wait();  // the activations come from the previous kernel

  float inv[MR];
#pragma unroll
  for (int m = 0; m < MR; ++m) inv[m] = 1.0f;
  if (a.gamma) {
    float ss[MR];
#pragma unroll
    for (int m = 0; m < MR; ++m) ss[m] = 0.0f;
    for (int k = tid; k < K; k += kConsumers) {
#pragma unroll
      for (int m = 0; m < MR; ++m)
        if (m < mr) {
          const float v = __bfloat162float(x[(size_t)m * a.ldx + k]);
          ss[m] = fmaf(v, v, ss[m]);
        }
    }
#pragma unroll
    for (int m = 0; m < MR; ++m) {
      float v = ss[m];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) nrm[warp * MR + m] = v;
    }
    named_bar_sync(kBarNorm, kConsumers);
#pragma unroll
    for (int m = 0; m < MR; ++m) {
      float tot = 0.0f;
#pragma unroll
      for (int w = 0; w < kConsumers / 32; ++w) tot += nrm[w * MR + m];
      inv[m] = 1.0f / sqrtf(tot / (float)K + a.eps);
    }
  }

  // x in registers: this thread's EPT K positions of the current segment
  // (one 16-byte weight chunk per row), as packed fp32 pairs (even, odd).
  uint64_t xr2[MR][EPT / 2];
  auto load_x = [&](int kc) {
    const bool write_h = (EPI == EPI_SAMPLE) && a.smp.h_out && blockIdx.x == 0 && g == 0;
#pragma unroll
    for (int e2 = 0; e2 < EPT / 2; ++e2) {
      float vv[MR][2];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int k = kc * KC + EPT * t + 2 * e2 + q;
        const bool ok = k < K;
        const float gm = (a.gamma && ok) ? __bfloat162float(a.gamma[k]) : 1.0f;
#pragma unroll
        for (int m = 0; m < MR; ++m) {
          float v = (ok && m < mr) ? __bfloat162float(x[(size_t)m * a.ldx + k]) : 0.0f;
          if (a.gamma) v = round_bf16(gm * round_bf16(v * inv[m]));
          vv[m][q] = v;
          if (write_h && ok && m < mr)
            a.smp.h_out[(size_t)(a.row0 + m) * K + k] = __float2bfloat16_rn(v);
        }
      }
#pragma unroll
      for (int m = 0; m < MR; ++m) xr2[m][e2] = pack_f32x2(vv[m][0], vv[m][1]);
    }
  };

  int s = 0;
  for (int kc = 0; kc < nkc; ++kc) {
    load_x(kc);
    const int kel = min(KC, K - kc * KC);
    for (int sr = 0; sr < spk; ++sr, ++s) {
      const int slot = s % kStages;
      // On a timeout the error word is set and the stage is consumed as is, so
      // that every thread still reaches the same barriers.
      mbar_wait(&full[slot], (s / kStages) & 1, a.err);
      const int rs = r_begin + sr * R;
      const int nr = min(R, r_end - rs);
      const uint8_t* st = ring + slot * kStageBytes;
      // per (row-in-pass, batch row) partial sums; each row's chunk is summed
      // in packed (even, odd) pairs and folded into one float
      float acc[V];
#pragma unroll
      for (int i = 0; i < V; ++i) acc[i] = 0.0f;
      const bool in_k = EPT * t < kel;
#pragma unroll
      for (int p = 0; p < P; ++p) {
        const int rl = p * G + g;
        if (rl < nr && in_k) {
          const uint4 wv = *reinterpret_cast<const uint4*>(st + (size_t)rl * KC * ESZ + 16 * t);
          const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
          uint64_t pm2[MR];
#pragma unroll
          for (int m = 0; m < MR; ++m) pm2[m] = 0ull;
          if constexpr (ESZ == 2) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              // (bf16 lo, bf16 hi) -> exact fp32 pair
              const uint64_t wp = pack_u32x2(ww[j] << 16, ww[j] & 0xFFFF0000u);
#pragma unroll
              for (int m = 0; m < MR; ++m) ffma2(pm2[m], wp, xr2[m][j]);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint64_t f01, f23;
              s8x4_to_f32x2(ww[j], f01, f23);
#pragma unroll
              for (int m = 0; m < MR; ++m) {
                ffma2(pm2[m], f01, xr2[m][2 * j]);
                ffma2(pm2[m], f23, xr2[m][2 * j + 1]);
              }
            }
          }
          float sc = 1.0f;
          if constexpr (WF == WF_I8G128) {
            const int n = rs + rl;
            const int kabs = kc * KC + 16 * t;
            sc = __ldg(a.scales + (size_t)n * (K / 128) + kabs / 128);
          }
#pragma unroll
          for (int m = 0; m < MR; ++m) {
            const float2 f = unpack_f32x2(pm2[m]);
            if constexpr (WF == WF_I8G128) acc[p * MR + m] = fmaf(sc, f.x + f.y, acc[p * MR + m]);
            else acc[p * MR + m] += f.x + f.y;
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);

      // reduce over the TPR threads of each row: shuffles, then partial slots
      const int b = s % kPartBufs;
      float* pb = part + b * SLOTS * V;
      if constexpr (kScatter) {
        warp_reduce_scatter<V>(acc, lane);
      } else {
#pragma unroll
        for (int i = 0; i < V; ++i) {
          float v = acc[i];
#pragma unroll
          for (int o = W / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o, W);
          acc[i] = v;
        }
      }
      if (s >= kPartBufs) named_bar_sync(kBarEmpty + b, kPartThreads);
      if constexpr (kScatter) {
        if ((lane & ((32 >> LV) - 1)) == 0) pb[warp * V + (lane >> (5 - LV))] = acc[0];
      } else {
        if ((tid % W) == 0) {
#pragma unroll
          for (int i = 0; i < V; ++i) pb[(tid / W) * V + i] = acc[i];
        }
      }
      named_bar_arrive(kBarFull + b, kPartThreads);
    }
  }
}

}  // namespace m3
