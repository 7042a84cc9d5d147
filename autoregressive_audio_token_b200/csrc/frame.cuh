// frame.cuh -- the whole decode frame of the 8B body as ONE persistent kernel.
//
// One CTA per SM, co-resident by cooperative launch.  The frame is a fixed
// sequence of phases: per layer QKV (RMSNorm + GEMV), ATT (q/k norm, RoPE,
// KV append, split-K attention), O (GEMV + residual), GU (RMSNorm + gate/up
// GEMV + SwiGLU), D (GEMV + residual); then LM (final norm + sliced lm_head +
// CFG + Gumbel-argmax).  Every phase reads what the previous one wrote, so
// phases are separated by grid barriers (an arrival counter per phase,
// bounded spins).  What the separate-kernel path pays at every kernel
// boundary -- launch, pipeline fill, tail -- disappears: the producer warp
// streams the CTA's weight rows and KV tiles for all phases back to back
// through the shared-memory ring (none of them depends on the frame's
// activations), so HBM keeps streaming while the compute warps wait at a
// barrier.  The weight and KV streams are the same bytes the separate GEMV
// and attention kernels read ("MiniMax Music 3 modular pipeline": the AR
// stage is memory-bandwidth bound, weights read once per frame).
//
// Warps: 0-7 compute (GEMV FMA / attention MMA), 8 epilogue (GEMV outputs,
// sampler), 9 producer (bulk copies).  GEMV phases use the layout of
// gemv.cuh with 256 threads per row (K >= 4096); the attention phase uses the
// MMA tiles of attention.cuh, one 32-position tile per ring stage.
#pragma once

#include "attention.cuh"
#include "gemv.cuh"

namespace m3 {

enum : int { PH_QKV = 0, PH_ATT = 1, PH_O = 2, PH_GU = 3, PH_D = 4, PH_LM = 5 };

struct FramePhase {
  int kind;
  int layer;
  const void* w;               // GEMV weights [N][K]
  const float* scales;         // int8 row scales
  int N, K;
  const __nv_bfloat16* x;      // GEMV input [rows][ldx]
  int ldx;
  const __nv_bfloat16* gamma;  // RMSNorm gain (nullable)
  __nv_bfloat16* out;          // GEMV output base
  int ldo;
  const __nv_bfloat16* q_norm; // ATT
  const __nv_bfloat16* k_norm;
};

struct FrameArgs {
  const FramePhase* ph;        // [nph] in device memory
  int nph;
  int mr;                      // batch rows (<= MR)
  float eps;
  const FrameParams* fp;
  // attention
  const __nv_bfloat16* qkv;
  int ldqkv;
  const double* inv_freq;
  const unsigned long long* pages;
  int n_layers, max_pages, page_size, Hq, Hkv, splits;
  float* apart;                // [rows][Hq][splits][D+2]
  unsigned int* acnt;          // [rows][Hkv] tickets, zero at rest
  __nv_bfloat16* att_out;      // [rows][Hq*D]
  SampleArgs smp;              // LM phase
  unsigned int* bar;           // [nph] arrivals, zeroed before the launch
  int* err;
};

// The frame kernel keeps its own warp layout: 8 compute warps owning 16 K
// positions each per 4096-wide segment (bf16: two 16-byte chunks), 1
// epilogue warp, 1 producer warp.
constexpr int kFC = 256;
constexpr int kFEpi = kFC / 32;
constexpr int kFrameThreads = kFC + 64;

template <int ESZ>
struct FrameShape {
  static constexpr int KC = 4096;                      // K elements per segment
  static constexpr int R = kStageBytes / (KC * ESZ);   // rows per stage
  static constexpr int P = R;                          // one row group
  static constexpr int SLOTS = kFC / 32;               // partial sums per row
};

// attention scratch of the frame kernel (head_dim 128): q, k, v of the new
// token, per-warp (m, l, o), new-token scores
constexpr int kFrameAttFloats = kAttnWarps * 128 + 2 * 128 + kAttnWarps * kAttnWarps * 130 +
                                kAttnWarps;

// Shared memory of the frame kernel: ring, ring barriers, partial-sum ring,
// norm scratch, attention scratch, then the K-chunk accumulators and the
// sampler's per-role bests.
template <int MR, int WF>
__host__ __device__ constexpr size_t frame_smem_bytes(int rows_cta_max) {
  using S = FrameShape<WF == WF_BF16 ? 2 : 1>;
  return (size_t)kStages * kStageBytes + 2 * kStages * sizeof(uint64_t) +
         sizeof(float) * ((size_t)kPartBufs * S::SLOTS * S::P * MR + 9 * MR + kFrameAttFloats +
                          (size_t)rows_cta_max * MR) +
         (sizeof(float) + sizeof(int)) * S::R * MR + 64;
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

template <int MR, int WF, int KVF16>
__global__ void __launch_bounds__(kFrameThreads, 1) frame_kernel(const FrameArgs a) {
  constexpr int D = 128, TPR = 256;
  constexpr int ESZ = WF == WF_BF16 ? 2 : 1;
  using S = FrameShape<ESZ>;
  constexpr int KC = S::KC, R = S::R, P = S::P, SLOTS = S::SLOTS;
  constexpr int V = P * MR;
  constexpr int LV = V == 1 ? 0 : V == 2 ? 1 : V == 4 ? 2 : V == 8 ? 3 : V == 16 ? 4 : 5;
  constexpr bool kScatter = V <= 32;
  constexpr int kBarCompute = 1, kBarFull = 2, kBarEmpty = 2 + kPartBufs;
  constexpr int kPartThreads = kFC + 32;
  constexpr int VPL = D / 32, NT = D / 8, KS = D / 16;
  constexpr int TILE_BYTES = kAttnTile * D * 2;
  static_assert(2 * TILE_BYTES <= kStageBytes, "a K/V tile pair fits one ring stage");

  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  float* part = reinterpret_cast<float*>(empty + kStages);  // [kPartBufs][SLOTS][V]
  float* nrm = part + kPartBufs * SLOTS * V;                 // [8][MR] + [MR]
  float* att = nrm + 9 * MR;                                  // kFrameAttFloats
  float* accr = att + kFrameAttFloats;                        // [rows_cta_max][MR] + bests
  __shared__ int s_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x;
  const int mr = a.mr;

  // per-phase geometry of this CTA's GEMV rows
  auto rows_of = [&](const FramePhase& ph, int& r_begin, int& r_end) {
    const int unit = ph.kind == PH_GU ? 2 : 1;
    const int U = ph.N / unit;
    r_begin = (int)((long long)U * blockIdx.x / G) * unit;
    r_end = (int)((long long)U * (blockIdx.x + 1) / G) * unit;
  };
  const int n_items = mr * a.Hkv * a.splits;
  auto item_range = [&](int item, int& r, int& g, int& sidx, int& pos, int& j0, int& jc1,
                        bool& has_new, int& ntiles) {
    r = item / (a.Hkv * a.splits);
    g = (item / a.splits) % a.Hkv;
    sidx = item % a.splits;
    pos = a.fp->pos[r];
    const int n = pos + 1;
    int chunk = (n + a.splits - 1) / a.splits;
    chunk = (chunk + kAttnTile - 1) / kAttnTile * kAttnTile;
    j0 = sidx * chunk;
    const int j1 = min(n, j0 + chunk);
    jc1 = min(j1, pos);
    has_new = (j0 <= pos) && (pos < j1);
    ntiles = jc1 > j0 ? (jc1 - j0 + kAttnTile - 1) / kAttnTile : 0;
  };
  auto page_table = [&](int r, int layer) {
    return a.pages + ((size_t)r * a.n_layers + layer) * a.max_pages;
  };

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kFC / 32);
    }
    fence_barrier_init();
  }
  __syncthreads();

  // =============================================================== producer
  if (warp == kFEpi + 1) {
    if (lane != 0) return;
    const uint64_t pol = policy_evict_first();
    int s = 0;
    auto next_slot = [&](int& slot) -> bool {
      slot = s % kStages;
      if (s >= kStages && !mbar_wait(&empty[slot], ((s / kStages) - 1) & 1, a.err)) return false;
      return true;
    };
    for (int p = 0; p < a.nph; ++p) {
      const FramePhase& ph = a.ph[p];
      if (ph.kind == PH_ATT) {
        for (int item = blockIdx.x; item < n_items; item += G) {
          int r, g, sidx, pos, j0, jc1, ntiles;
          bool has_new;
          item_range(item, r, g, sidx, pos, j0, jc1, has_new, ntiles);
          const unsigned long long* pt = page_table(r, ph.layer);
          for (int t = 0; t < ntiles; ++t, ++s) {
            int slot;
            if (!next_slot(slot)) return;
            const int js = j0 + t * kAttnTile;
            const int nv = min(kAttnTile, jc1 - js);
            const int page = js / a.page_size, off = js % a.page_size;
            const uint16_t* base = reinterpret_cast<const uint16_t*>(pt[page]);
            const uint32_t bytes = (uint32_t)(nv * D * 2);
            mbar_arrive_expect_tx(&full[slot], 2 * bytes);
            uint8_t* dst = ring + slot * kStageBytes;
            bulk_g2s_nohint(dst, base + ((size_t)g * a.page_size + off) * D, bytes, &full[slot]);
            bulk_g2s_nohint(dst + TILE_BYTES, base + ((size_t)(a.Hkv + g) * a.page_size + off) * D,
                            bytes, &full[slot]);
          }
        }
      } else {
        int r_begin, r_end;
        rows_of(ph, r_begin, r_end);
        const int nrows = r_end - r_begin;
        const int spk = (nrows + R - 1) / R;
        const int nkc = (ph.K + KC - 1) / KC;
        const uint8_t* wb = static_cast<const uint8_t*>(ph.w);
        for (int kc = 0; kc < nkc; ++kc)
          for (int sr = 0; sr < spk; ++sr, ++s) {
            int slot;
            if (!next_slot(slot)) return;
            const int rs = r_begin + sr * R, re = min(rs + R, r_end);
            const uint32_t segb = (uint32_t)(min(KC, ph.K - kc * KC) * ESZ);
            mbar_arrive_expect_tx(&full[slot], segb * (uint32_t)(re - rs));
            uint8_t* dst = ring + slot * kStageBytes;
            for (int rr = rs; rr < re; ++rr)
              bulk_g2s(dst + (size_t)(rr - rs) * KC * ESZ,
                       wb + ((size_t)rr * ph.K + (size_t)kc * KC) * ESZ, segb, &full[slot], pol);
          }
      }
    }
    return;
  }

  // =============================================================== epilogue
  if (warp == kFEpi) {
    // total partial stages of this CTA (the compute warps wait on EMPTY only
    // for stages that have a successor kPartBufs later)
    int total_sp = 0;
    for (int p = 0; p < a.nph; ++p) {
      const FramePhase& ph = a.ph[p];
      if (ph.kind == PH_ATT) continue;
      int r_begin, r_end;
      rows_of(ph, r_begin, r_end);
      total_sp += ((r_end - r_begin + R - 1) / R) * ((ph.K + KC - 1) / KC);
    }
    float* sbz = accr;  // sampler bests reuse the accumulator area's tail (set below)
    int sp = 0;
    for (int p = 0; p < a.nph; ++p) {
      const FramePhase& ph = a.ph[p];
      if (ph.kind == PH_ATT) continue;
      int r_begin, r_end;
      rows_of(ph, r_begin, r_end);
      const int nrows = r_end - r_begin;
      const int spk = (nrows + R - 1) / R;
      const int nkc = (ph.K + KC - 1) / KC;
      const int epi = ph.kind == PH_QKV ? EPI_STORE
                      : (ph.kind == PH_GU ? EPI_SWIGLU : (ph.kind == PH_LM ? EPI_SAMPLE : EPI_RESID));
      sbz = accr + (size_t)spk * R * MR;
      int* sbi = reinterpret_cast<int*>(sbz + R * MR);
      const int np = a.fp->cfg_on ? mr / 2 : mr;
      if (epi == EPI_SAMPLE) {
        for (int c = lane; c < R * MR; c += 32) {
          sbz[c] = -INFINITY;
          sbi[c] = 0x7fffffff;
        }
        __syncwarp();
      }
      for (int kc = 0; kc < nkc; ++kc) {
        const bool last_kc = (kc == nkc - 1);
        for (int sr = 0; sr < spk; ++sr, ++sp) {
          const int b = sp % kPartBufs;
          named_bar_sync(kBarFull + b, kPartThreads);
          const float* pb = part + b * SLOTS * V;
          const int rs = r_begin + sr * R;
          const int nr = min(R, r_end - rs);
          auto row_sum = [&](int rl, int m) -> float {
            float y = 0.0f;
#pragma unroll
            for (int q = 0; q < SLOTS; ++q) y += pb[q * V + rl * MR + m];
            return y;
          };
          if (epi == EPI_STORE || epi == EPI_RESID) {
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
              if constexpr (WF == WF_I8ROW) y *= __ldg(ph.scales + n);
              __nv_bfloat16* o = ph.out + (size_t)m * ph.ldo + n;
              if (epi == EPI_STORE) *o = __float2bfloat16_rn(y);
              else *o = __float2bfloat16_rn(__bfloat162float(*o) + round_bf16(y));
            }
          } else if (epi == EPI_SWIGLU) {
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
                yg *= __ldg(ph.scales + n);
                yu *= __ldg(ph.scales + n + 1);
              }
              const float gb = round_bf16(yg), ub = round_bf16(yu);
              const float act = round_bf16(round_bf16(silu_f(gb)) * ub);
              ph.out[(size_t)m * ph.ldo + n / 2] = __float2bfloat16_rn(act);
            }
          } else {  // EPI_SAMPLE
            const bool cfg = a.fp->cfg_on != 0;
            for (int c = lane; c < R * MR; c += 32) {
              const int rl = c / MR, pk = c % MR;
              if (rl >= nr || pk >= np) continue;
              const int n = rs + rl;
              const int m0 = cfg ? 2 * pk : pk;
              float y0 = row_sum(rl, m0);
              float y1 = cfg ? row_sum(rl, m0 + 1) : 0.0f;
              if constexpr (WF == WF_I8ROW) {
                const float sc = __ldg(ph.scales + n);
                y0 *= sc;
                y1 *= sc;
              }
              if (a.smp.logits) {
                a.smp.logits[(size_t)m0 * a.smp.logits_ld + n] = y0;
                if (cfg) a.smp.logits[(size_t)(m0 + 1) * a.smp.logits_ld + n] = y1;
              }
              float gl = y0;
              if (cfg) gl = __fadd_rn(y1, __fmul_rn(a.fp->cfg_scale, __fsub_rn(y0, y1)));
              const float gn = gumbel_noise(a.fp->seed, a.fp->frame, (unsigned long long)pk,
                                            a.smp.index_base + (unsigned long long)n);
              const float z = __fadd_rn(__fdiv_rn(gl, a.fp->temperature), gn);
              if (z > sbz[c] || (z == sbz[c] && n < sbi[c])) {
                sbz[c] = z;
                sbi[c] = n;
              }
            }
          }
          if (sp + kPartBufs < total_sp) named_bar_arrive(kBarEmpty + b, kPartThreads);
        }
      }
      __syncwarp();
      if (epi == EPI_SAMPLE) {
        // CTA argmax per key, then the last CTA reduces over CTAs
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
          last = atomicAdd(a.smp.counter, 1u) == (unsigned)(G - 1);
        }
        last = __shfl_sync(0xffffffffu, last, 0);
        if (last) {
          __threadfence();
          if (lane < np) {
            float bz = -INFINITY;
            int bi = 0x7fffffff;
            for (int bb = 0; bb < G; ++bb) {
              const float z = __ldcg(a.smp.part_z + bb * kMaxRows + lane);
              const int i = __ldcg(a.smp.part_i + bb * kMaxRows + lane);
              if (z > bz || (z == bz && i < bi)) {
                bz = z;
                bi = i;
              }
            }
            const bool cfg = a.fp->cfg_on != 0;
            for (int q = 0; q < (cfg ? 2 : 1); ++q) a.smp.codes[cfg ? 2 * lane + q : lane] = bi;
          }
          if (lane == 0) *a.smp.counter = 0u;
        }
      } else if (lane == 0) {
        __threadfence();  // this CTA's outputs of phase p, then its arrival
        atomicAdd(a.bar + p, 1u);
      }
    }
    return;
  }

  // ========================================================== compute warps
  const int t = tid;  // 256 threads per row (one row group)
  int s = 0, sp = 0;

  auto grid_wait = [&](int p) {  // all CTAs have finished phase p
    if (tid == 0) {
      long long it = 0;
      while (ld_acquire_u32(a.bar + p) < (unsigned)G) {
        __nanosleep(32);
        if (++it > kSpinLimit) {
          record_error(a.err, kErrTimeout);
          break;
        }
        if ((it & 1023) == 0 && *reinterpret_cast<volatile int*>(a.err) != 0) break;
      }
    }
    named_bar_sync(kBarCompute, kFC);
  };

  for (int p = 0; p < a.nph; ++p) {
    const FramePhase& ph = a.ph[p];
    if (p > 0) grid_wait(p - 1);

    if (ph.kind == PH_ATT) {
      float* q_s = att;
      float* k_s = q_s + kAttnWarps * D;
      float* v_s = k_s + D;
      float* w_s = v_s + D;
      float* sn_s = w_s + kAttnWarps * kAttnWarps * (D + 2);
      const int grp = a.Hq / a.Hkv;
      const float scale = 1.0f / sqrtf((float)D);
      const int gid = lane >> 2, tig = lane & 3;
      for (int item = blockIdx.x; item < n_items; item += G) {
        int r, g, sidx, pos, j0, jc1, ntiles;
        bool has_new;
        item_range(item, r, g, sidx, pos, j0, jc1, has_new, ntiles);
        const unsigned long long* pt = page_table(r, ph.layer);
        const bool is_q = warp < grp, is_k = (warp == kAttnWarps - 1);
        // ---- new token: norm + RoPE (lane holds dims lane + 32 i) --------
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
#pragma unroll
          for (int i = 0; i < VPL / 2; ++i) {
            const double ang = (double)pos * a.inv_freq[lane + 32 * i];
            const float c = (float)cos(ang), sn = (float)sin(ang);
            const float x0 = v[i], x1 = v[i + VPL / 2];
            v[i] = __fsub_rn(__fmul_rn(x0, c), __fmul_rn(x1, sn));
            v[i + VPL / 2] = __fadd_rn(__fmul_rn(x1, c), __fmul_rn(x0, sn));
          }
#pragma unroll
          for (int i = 0; i < VPL; ++i) dst[lane + 32 * i] = round_bf16(v[i]);
        };
        const __nv_bfloat16* row_qkv = a.qkv + (size_t)r * a.ldqkv;
        if (is_q) norm_rope(row_qkv + (size_t)(g * grp + warp) * D, ph.q_norm, q_s + warp * D);
        if (is_k) {
          const __nv_bfloat16* kraw = row_qkv + (size_t)a.Hq * D + (size_t)g * D;
          const __nv_bfloat16* vraw = row_qkv + (size_t)(a.Hq + a.Hkv) * D + (size_t)g * D;
          norm_rope(kraw, ph.k_norm, k_s);
#pragma unroll
          for (int i = 0; i < VPL; ++i) {
            const int dim = lane + 32 * i;
            const uint16_t kb = f32_to_kv<KVF16>(k_s[dim]);
            const uint16_t vb = f32_to_kv<KVF16>(__bfloat162float(vraw[dim]));
            k_s[dim] = kv_to_f32<KVF16>(kb);
            v_s[dim] = kv_to_f32<KVF16>(vb);
            if (sidx == 0) {
              const int page = pos / a.page_size, off = pos % a.page_size;
              uint16_t* pb2 = reinterpret_cast<uint16_t*>(pt[page]);
              pb2[kv_elem_offset(g, a.page_size, off, D, dim)] = kb;
              pb2[kv_elem_offset(a.Hkv + g, a.page_size, off, D, dim)] = vb;
            }
          }
        }
        named_bar_sync(kBarCompute, kFC);
        if (is_q) {
          float pq = 0.0f;
#pragma unroll
          for (int i = 0; i < VPL; ++i) pq = fmaf(q_s[warp * D + lane + 32 * i], k_s[lane + 32 * i], pq);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) pq += __shfl_xor_sync(0xffffffffu, pq, o);
          if (lane == 0) sn_s[warp] = pq * scale;
        }
        // ---- cached tiles: warp (t % 4) computes tile t; all warps pass the ring
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
        float m_run = -INFINITY, l_run = 0.0f;
        for (int tt = 0; tt < ntiles; ++tt, ++s) {
          const int slot = s % kStages;
          mbar_wait(&full[slot], (s / kStages) & 1, a.err);
          if (warp == (tt % kAttnWarps)) {
            const int nv = min(kAttnTile, jc1 - (j0 + tt * kAttnTile));
            if (nv < kAttnTile) {
              // rows past the tile's end hold weight bytes of an earlier stage:
              // zero them so that p = 0 multiplies zeros, not stray NaN patterns
              uint4* kz = reinterpret_cast<uint4*>(ring + slot * kStageBytes);
              uint4* vz = reinterpret_cast<uint4*>(ring + slot * kStageBytes + TILE_BYTES);
              for (int c = nv * (D / 8) + lane; c < kAttnTile * (D / 8); c += 32) {
                kz[c] = make_uint4(0, 0, 0, 0);
                vz[c] = make_uint4(0, 0, 0, 0);
              }
              __syncwarp();
            }
            const uint32_t kb = smem_u32(ring + slot * kStageBytes);
            const uint32_t vb = kb + TILE_BYTES;
            float sc[4][4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              sc[j][0] = sc[j][1] = sc[j][2] = sc[j][3] = 0.0f;
              const int prow = 8 * j + (lane & 7);
#pragma unroll
              for (int kk = 0; kk < KS; kk += 2) {
                const int chunk = 2 * kk + (lane >> 3);
                uint32_t b0, b1, b2, b3;
                ldsm_x4(kb + prow * (D * 2) + ((chunk ^ (prow & 7)) << 4), b0, b1, b2, b3);
                mma16816<KVF16>(sc[j], qa[kk][0], 0u, qa[kk][1], 0u, b0, b1);
                mma16816<KVF16>(sc[j], qa[kk + 1][0], 0u, qa[kk + 1][1], 0u, b2, b3);
              }
            }
            float mt = -INFINITY;
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int pp = 8 * j + 2 * tig + e;
                const float sv = pp < nv ? sc[j][e] * scale : -INFINITY;
                sc[j][e] = sv;
                mt = fmaxf(mt, sv);
              }
            mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
            mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
            const float m_new = fmaxf(m_run, mt);
            const float corr = expf(m_run - m_new);
            float ls = 0.0f;
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const float pv = expf(sc[j][e] - m_new);
                sc[j][e] = pv;
                ls += pv;
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
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(vb + prow * (D * 2) + ((chunk ^ (prow & 7)) << 4), b0, b1, b2, b3);
                mma16816<KVF16>(o_acc[j], h0, 0u, h2, 0u, b0, b1);
                mma16816<KVF16>(o_acc[j], l0, 0u, l2, 0u, b0, b1);
                mma16816<KVF16>(o_acc[j + 1], h0, 0u, h2, 0u, b2, b3);
                mma16816<KVF16>(o_acc[j + 1], l0, 0u, l2, 0u, b2, b3);
              }
            }
          }
          __syncwarp();
          if (lane == 0) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // before the refill
            mbar_arrive(&empty[slot]);
          }
        }
        // ---- merge the 4 warps (+ the new token), then this split's partial
        if (warp < kAttnWarps && row_ok) {
          float* wh = w_s + ((size_t)warp * kAttnWarps + gid) * (D + 2);
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
        named_bar_sync(kBarCompute, kFC);
        const int stride = D + 2;
        if (is_q) {
          const int h = g * grp + warp;
          float M = has_new ? sn_s[warp] : -INFINITY;
          for (int ww = 0; ww < kAttnWarps; ++ww) {
            const bool any = ww < ntiles;
            if (any) M = fmaxf(M, w_s[(ww * kAttnWarps + warp) * (D + 2)]);
          }
          float L = 0.0f, o[VPL];
#pragma unroll
          for (int e = 0; e < VPL; ++e) o[e] = 0.0f;
          for (int ww = 0; ww < kAttnWarps && ww < ntiles; ++ww) {
            const float* wh = w_s + (ww * kAttnWarps + warp) * (D + 2);
            const float f = wh[0] == -INFINITY ? 0.0f : expf(wh[0] - M);
            L = fmaf(wh[1], f, L);
#pragma unroll
            for (int e = 0; e < VPL; ++e) o[e] = fmaf(wh[2 + VPL * lane + e], f, o[e]);
          }
          if (has_new) {
            const float f = expf(sn_s[warp] - M);
            L += f;
#pragma unroll
            for (int e = 0; e < VPL; ++e) o[e] = fmaf(f, v_s[VPL * lane + e], o[e]);
          }
          float* pp = a.apart + (((size_t)r * a.Hq + h) * a.splits + sidx) * stride;
          if (lane == 0) {
            pp[0] = M;
            pp[1] = L;
          }
#pragma unroll
          for (int e = 0; e < VPL; ++e) pp[2 + VPL * lane + e] = o[e];
          __threadfence();
        }
        named_bar_sync(kBarCompute, kFC);
        if (tid == 0) {
          __threadfence();
          const unsigned old = atomicAdd(a.acnt + (size_t)r * a.Hkv + g, 1u);
          s_flag = (old == (unsigned)(a.splits - 1));
        }
        named_bar_sync(kBarCompute, kFC);
        if (s_flag) {
          __threadfence();
          if (is_q) {
            const int h = g * grp + warp;
            const float* pp = a.apart + ((size_t)r * a.Hq + h) * a.splits * stride;
            float M = -INFINITY;
            for (int s2 = 0; s2 < a.splits; ++s2) M = fmaxf(M, __ldcg(pp + s2 * stride));
            float L = 0.0f, o[VPL];
#pragma unroll
            for (int e = 0; e < VPL; ++e) o[e] = 0.0f;
            for (int s2 = 0; s2 < a.splits; ++s2) {
              const float ms = __ldcg(pp + s2 * stride);
              const float f = ms == -INFINITY ? 0.0f : expf(ms - M);
              L = fmaf(__ldcg(pp + s2 * stride + 1), f, L);
#pragma unroll
              for (int e = 0; e < VPL; ++e)
                o[e] = fmaf(__ldcg(pp + s2 * stride + 2 + VPL * lane + e), f, o[e]);
            }
            __nv_bfloat16* dst = a.att_out + (size_t)r * a.Hq * D + (size_t)h * D + VPL * lane;
#pragma unroll
            for (int e = 0; e < VPL; ++e) dst[e] = __float2bfloat16_rn(o[e] / L);
          }
          if (tid == 0) a.acnt[(size_t)r * a.Hkv + g] = 0u;
        }
        named_bar_sync(kBarCompute, kFC);  // before the next item reuses q_s ...
      }
      if (tid == 0) {
        __threadfence();
        atomicAdd(a.bar + p, 1u);
      }
      continue;
    }

    // ---------------------------------------------------------- GEMV phase
    int r_begin, r_end;
    rows_of(ph, r_begin, r_end);
    const int nrows = r_end - r_begin;
    const int spk = (nrows + R - 1) / R;
    const int K = ph.K;
    const int nkc = (K + KC - 1) / KC;
    const __nv_bfloat16* __restrict__ x = ph.x;

    float inv[MR];
#pragma unroll
    for (int m = 0; m < MR; ++m) inv[m] = 1.0f;
    if (ph.gamma) {
      float ss[MR];
#pragma unroll
      for (int m = 0; m < MR; ++m) ss[m] = 0.0f;
      for (int k = tid; k < K; k += kFC) {
#pragma unroll
        for (int m = 0; m < MR; ++m)
          if (m < mr) {
            const float v = __bfloat162float(x[(size_t)m * ph.ldx + k]);
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
      named_bar_sync(kBarCompute, kFC);
#pragma unroll
      for (int m = 0; m < MR; ++m) {
        float tot = 0.0f;
#pragma unroll
        for (int w = 0; w < kFC / 32; ++w) tot += nrm[w * MR + m];
        inv[m] = 1.0f / sqrtf(tot / (float)K + a.eps);
      }
      named_bar_sync(kBarCompute, kFC);  // nrm is reused by the next norm
    }
    const bool write_h = ph.kind == PH_LM && a.smp.h_out && blockIdx.x == 0;

    uint64_t xr2[MR][8];
    for (int kc = 0; kc < nkc; ++kc) {
      // load this thread's 16 inputs of the chunk (normalised when gamma)
#pragma unroll
      for (int e2 = 0; e2 < 8; ++e2) {
        float vv[MR][2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int e = 2 * e2 + q;
          const int k = ESZ == 2 ? kc * KC + (e < 8 ? 8 * t + e : 8 * (t + TPR) + (e - 8))
                                 : kc * KC + 16 * t + e;
          const bool ok = k < K;
          const float gm = (ph.gamma && ok) ? __bfloat162float(ph.gamma[k]) : 1.0f;
#pragma unroll
          for (int m = 0; m < MR; ++m) {
            float v = (ok && m < mr) ? __bfloat162float(x[(size_t)m * ph.ldx + k]) : 0.0f;
            if (ph.gamma) v = round_bf16(gm * round_bf16(v * inv[m]));
            vv[m][q] = v;
            if (write_h && ok && m < mr) a.smp.h_out[(size_t)m * K + k] = __float2bfloat16_rn(v);
          }
        }
#pragma unroll
        for (int m = 0; m < MR; ++m) xr2[m][e2] = pack_f32x2(vv[m][0], vv[m][1]);
      }
      const int kel = min(KC, K - kc * KC);
      for (int sr = 0; sr < spk; ++sr, ++s, ++sp) {
        const int slot = s % kStages;
        mbar_wait(&full[slot], (s / kStages) & 1, a.err);
        const int rs = r_begin + sr * R;
        const int nr = min(R, r_end - rs);
        const uint8_t* st = ring + slot * kStageBytes;
        uint64_t acc2[V];
#pragma unroll
        for (int i = 0; i < V; ++i) acc2[i] = 0ull;
#pragma unroll
        for (int pp = 0; pp < P; ++pp) {
          const int rl = pp;
          if (rl < nr) {
            const uint8_t* sg = st + (size_t)rl * KC * ESZ;
            if constexpr (ESZ == 2) {
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int c = t + h * TPR;
                if (8 * c < kel) {
                  const uint4 wv = *reinterpret_cast<const uint4*>(sg + 16 * c);
                  const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
                  for (int j = 0; j < 4; ++j) {
                    const uint64_t wp = pack_u32x2(ww[j] << 16, ww[j] & 0xFFFF0000u);
#pragma unroll
                    for (int m = 0; m < MR; ++m) ffma2(acc2[pp * MR + m], wp, xr2[m][4 * h + j]);
                  }
                }
              }
            } else {
              if (16 * t < kel) {
                const uint4 wv = *reinterpret_cast<const uint4*>(sg + 16 * t);
                const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  uint64_t f01, f23;
                  s8x4_to_f32x2(ww[j], f01, f23);
#pragma unroll
                  for (int m = 0; m < MR; ++m) {
                    ffma2(acc2[pp * MR + m], f01, xr2[m][2 * j]);
                    ffma2(acc2[pp * MR + m], f23, xr2[m][2 * j + 1]);
                  }
                }
              }
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
        float acc[V];
#pragma unroll
        for (int i = 0; i < V; ++i) {
          const float2 f = unpack_f32x2(acc2[i]);
          acc[i] = f.x + f.y;
        }
        const int b = sp % kPartBufs;
        float* pb = part + b * SLOTS * V;
        if constexpr (kScatter) {
          warp_reduce_scatter<V>(acc, lane);
        } else {
#pragma unroll
          for (int i = 0; i < V; ++i) {
            float v = acc[i];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            acc[i] = v;
          }
        }
        if (sp >= kPartBufs) named_bar_sync(kBarEmpty + b, kPartThreads);
        if constexpr (kScatter) {
          if ((lane & ((32 >> LV) - 1)) == 0) pb[warp * V + (lane >> (5 - LV))] = acc[0];
        } else {
          if (lane == 0) {
#pragma unroll
            for (int i = 0; i < V; ++i) pb[warp * V + i] = acc[i];
          }
        }
        named_bar_arrive(kBarFull + b, kPartThreads);
      }
    }
  }
}

}  // namespace m3
