// gemv_dyn.cuh -- the tiled tensor-core GEMV with dynamic work distribution
// (the body's projections: store, residual add, SwiGLU; up to 8 rows).
//
// Same weight layout, MMA formulation and epilogues as gemv_tile.cuh, but
// every CTA holds the whole K and CTAs claim 16-row units from a per-launch
// counter in global memory instead of owning a fixed range.  Measured
// per-SM streaming rates differ by up to a third within one launch, so a
// static partition ends with its slowest SM; claiming units balances that to
// within one unit.
//   * producer warp: claims a unit one ahead of streaming it, copies its K
//     run in ring stages (non-multicast bulk copies, L2 evict-first) and tags
//     each stage with (unit, part); an end tag closes the stream; it then
//     counts its CTA out, and the last CTA out resets the counter pair for
//     the launch site's next use;
//   * 8 consumer warps: MMA the stage's tiles against the activations held
//     in shared memory in B-fragment order; per unit, each warp hands its
//     partial sums to the epilogue warp through a 4-deep mbarrier ring;
//   * epilogue warp: sums the warps' partials in warp order (deterministic)
//     and applies store / residual add / SwiGLU to the unit's 16 rows.
#pragma once

#include "gemv_tile.cuh"

namespace m3 {

constexpr int kDW = 8;                     // consumer warps
constexpr int kDEpi = kDW;                 // epilogue warp index
constexpr int kDThreads = (kDW + 2) * 32;  // + epilogue warp + producer warp
constexpr int kDPB = 4;                    // unit partial buffers in flight
constexpr int kDMaxRows = 8;               // batch rows (one B fragment)

// Stage geometry of the dynamic kernel: a unit's run of T tiles in ppr parts
// of pt tiles, `slots` stages in the ring (host and device agree).
struct DynPlan {
  int T, TB, ppr, pt, stage, slots;
};

__host__ __device__ __forceinline__ DynPlan dyn_plan(int K, int esz, int sb, int ring_bytes) {
  DynPlan d;
  d.T = K >> 4;
  d.TB = 256 * esz;
  d.ppr = (d.T * d.TB + sb - 1) / sb;
  d.pt = (d.T + d.ppr - 1) / d.ppr;
  d.stage = d.pt * d.TB;
  d.slots = ring_bytes / d.stage < kTMaxSlots ? ring_bytes / d.stage : kTMaxSlots;
  return d;
}

// Dynamic shared memory of one CTA: the ring, its barriers and tags, the
// partial-sum ring's barriers and unit tags, per-row scalars, the
// activations [T][mr][4] in B-fragment order, kDPB partial buffers.
__host__ __device__ __forceinline__ size_t dyn_smem_bytes(const DynPlan& d, int mr) {
  return (size_t)d.slots * d.stage + 2 * kTMaxSlots * sizeof(uint64_t) +
         kTMaxSlots * sizeof(int) + 2 * kDPB * sizeof(uint64_t) + kDPB * sizeof(int) +
         kTMiscBytes + (size_t)d.T * mr * 32 + (size_t)kDPB * kDW * mr * kUnitRows * sizeof(float);
}

template <int WF, int EPI>
__global__ void __maxnreg__(128) gemv_dyn_kernel(const GemvArgs a) {
  static_assert(WF == WF_BF16 || WF == WF_I8ROW, "tiled formats: bf16, int8 row scale");
  static_assert(EPI == EPI_STORE || EPI == EPI_RESID || EPI == EPI_SWIGLU, "no sampler here");
  constexpr int ESZ = WF == WF_BF16 ? 2 : 1;
  constexpr int LB = 8 * ESZ;
  constexpr int TB = 256 * ESZ;
  constexpr int NT = kDW * 32;

  const int mr = a.mr;
  const int U = (a.N + kUnitRows - 1) / kUnitRows;
  const DynPlan D = dyn_plan(a.K, ESZ, a.tsb, a.tsb * a.tns);
  const int T = D.T, ppr = D.ppr, pt = D.pt, ns = D.slots;
  const int WU = mr * kUnitRows;

  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)ns * D.stage);
  uint64_t* empty = full + kTMaxSlots;
  int* tag = reinterpret_cast<int*>(empty + kTMaxSlots);             // unit*ppr+part, -1 end
  uint64_t* pfull = reinterpret_cast<uint64_t*>(tag + kTMaxSlots);  // [kDPB]
  uint64_t* pempty = pfull + kDPB;                                   // [kDPB]
  int* punit = reinterpret_cast<int*>(pempty + kDPB);                // [kDPB] unit, -1 end
  uint8_t* misc = reinterpret_cast<uint8_t*>(punit + kDPB);
  float* rinv = reinterpret_cast<float*>(misc);  // [16]
  float* rpow = rinv + 16;                       // [16]
  uint2* zpad = reinterpret_cast<uint2*>(misc + 800);
  uint2* xs = reinterpret_cast<uint2*>(misc + kTMiscBytes);         // [T][mr][4]
  float* part = reinterpret_cast<float*>(xs + (size_t)T * mr * 4);   // [kDPB][kDW][WU]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  unsigned* claim = a.ctr;     // next unit to hand out
  unsigned* done = a.ctr + 1;  // CTAs that have stopped claiming
  if (tid == 0) {
    for (int s = 0; s < ns; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kDW);
    }
    for (int b = 0; b < kDPB; ++b) {
      mbar_init(&pfull[b], kDW);
      mbar_init(&pempty[b], 1);
    }
    fence_barrier_init();
    *zpad = make_uint2(0u, 0u);
  }
  __syncthreads();
  pdl_launch_dependents();

  if (warp == kDW + 1) {
    // ---------------------------------------------------------- producer --
    // Weights and the claim counter belong to this launch alone, so the
    // producer starts before the previous kernel has finished.
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      const uint8_t* wb = static_cast<const uint8_t*>(a.w);
      // Before the consumers run, a CTA claims only its first unit: claiming
      // ahead that early would let the CTAs that launch first take two units
      // each before the others start, which unbalances launches of about two
      // units per CTA.  Once a slot has come back (the consumers run), the
      // next unit is claimed as soon as the current one starts.
      int u = (int)atomicAdd(claim, 1u);  // the unit being loaded; -1: take the next
      int un = -1;                         // the next unit, once claimed
      int p = 0;                           // next part of u
      bool started = false;                // a slot has come back
      for (int s = 0;; ++s) {
        const int slot = s % ns;
        if (s >= ns) {
          if (!mbar_wait(&empty[slot], ((s / ns) - 1) & 1, a.err)) break;
          started = true;
        }
        if (u < 0) {
          u = un >= 0 ? un : (int)atomicAdd(claim, 1u);
          un = -1;
          p = 0;
        }
        if ((started || !a.lazy_claim) && un < 0 && u < U) un = (int)atomicAdd(claim, 1u);
        if (u >= U) {  // the end tag takes a stage
          tag[slot] = -1;
          mbar_arrive(&full[slot]);
          break;
        }
        const int t0 = p * pt, t1 = min(T, t0 + pt);
        const uint32_t bytes = (uint32_t)((t1 - t0) * TB);
        tag[slot] = u * ppr + p;
        mbar_arrive_expect_tx(&full[slot], bytes);
        bulk_g2s(ring + (size_t)slot * D.stage, wb + ((size_t)u * T + t0) * TB, bytes,
                 &full[slot], pol);
        if (++p == ppr) u = -1;
      }
      // this CTA claims no more; the last CTA to stop resets the pair
      if (atomicAdd(done, 1u) == gridDim.x - 1) {
        *claim = 0u;
        *done = 0u;
      }
    }
  } else if (warp == kDEpi) {
    // ---------------------------------------------------------- epilogue --
    pdl_wait();  // outputs (and the residual) are shared with the previous kernel
    for (int i = 0;; ++i) {
      const int b = i % kDPB;
      if (!mbar_wait(&pfull[b], (i / kDPB) & 1, a.err)) break;
      const int u = punit[b];
      if (u < 0) break;
      const float* pb = part + (size_t)b * kDW * WU;
      if constexpr (EPI == EPI_SWIGLU) {
        constexpr int HP = kUnitRows / 2;  // (gate, up) row pairs per unit
        for (int e = lane; e < mr * HP; e += 32) {
          const int m = e / HP, jj = e % HP;
          const int n = u * kUnitRows + 2 * jj;  // gate row n, up row n + 1
          float yg = 0.0f, yu = 0.0f;
#pragma unroll
          for (int w = 0; w < kDW; ++w) {
            yg += pb[(size_t)w * WU + m * kUnitRows + 2 * jj];
            yu += pb[(size_t)w * WU + m * kUnitRows + 2 * jj + 1];
          }
          if (n >= a.N) continue;
          if constexpr (WF == WF_I8ROW) {
            yg = yg * rpow[m] * __ldg(a.scales + n);
            yu = yu * rpow[m] * __ldg(a.scales + n + 1);
          }
          const float gb = round_bf16(yg), ub = round_bf16(yu);
          const float act = round_bf16(round_bf16(silu_f(gb)) * ub);
          a.out[(size_t)m * a.ldo + n / 2] = __float2bfloat16_rn(act);
        }
      } else {
        // WU = 16 mr is a multiple of 16: each pass covers two rows, one per
        // half-warp, so the RMSNorm partial of (row, unit) is a 16-lane sum
        for (int e0 = 0; e0 < WU; e0 += 32) {
          const int e = e0 + lane;
          const int m = e / kUnitRows, n = u * kUnitRows + e % kUnitRows;
          float y = 0.0f, o2 = 0.0f;
          if (e < WU) {
#pragma unroll
            for (int w = 0; w < kDW; ++w) y += pb[(size_t)w * WU + e];
          }
          if (e < WU && n < a.N) {
            if constexpr (WF == WF_I8ROW) y = y * rpow[m] * __ldg(a.scales + n);
            __nv_bfloat16* o = a.out + (size_t)m * a.ldo + n;
            __nv_bfloat16 ob;
            if constexpr (EPI == EPI_STORE) ob = __float2bfloat16_rn(y);
            else ob = __float2bfloat16_rn(__bfloat162float(*o) + round_bf16(y));
            *o = ob;
            const float of = __bfloat162float(ob);
            o2 = of * of;
          }
          if (EPI == EPI_RESID && a.ssq_out) {
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) o2 += __shfl_xor_sync(0xffffffffu, o2, off);
            if ((lane & 15) == 0 && e < WU) a.ssq_out[(size_t)m * U + u] = o2;
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&pempty[b]);
    }
  } else {
    // --------------------------------------------------------- consumers --
    if (a.gamma)
      stage_activations<WF, 4, true>(a, mr, 0, T, rinv, rpow, reinterpret_cast<float*>(xs), xs,
                                     nullptr, tid, NT);
    else
      stage_activations<WF, kStageItems<WF>, false>(a, mr, 0, T, rinv, rpow, reinterpret_cast<float*>(xs), xs,
                                      nullptr, tid, NT);
    const int g = lane >> 2, t = lane & 3;
    const uint2* xl = g < mr ? xs + g * 4 + t : zpad;  // B fragment stream of batch row g
    const int xsl = g < mr ? mr * 4 : 0;
    float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
    int nunit = 0;
    for (int s = 0;; ++s) {
      const int slot = s % ns;
      const bool got = mbar_wait(&full[slot], (s / ns) & 1, a.err);
      const int tg = got ? tag[slot] : -1;
      const int b = nunit % kDPB;
      if (tg < 0) {
        // end of the stream: tell the epilogue warp
        if (nunit >= kDPB) mbar_wait(&pempty[b], ((nunit / kDPB) - 1) & 1, a.err);
        if (tid == 0) punit[b] = -1;
        __syncwarp();
        if (lane == 0) mbar_arrive(&pfull[b]);
        break;
      }
      const int u = tg / ppr, p = tg % ppr;
      const int t0 = p * pt, nt = min(T, t0 + pt) - t0;
      const uint8_t* wp = ring + (size_t)slot * D.stage + (size_t)warp * TB + lane * LB;
      const uint2* pl = xl + (size_t)(t0 + warp) * xsl;
      int n = nt > warp ? (nt - warp + kDW - 1) / kDW : 0;
      for (; n >= 2; n -= 2) {
        const uint4 w0 = load_afrag<WF>(wp), w1 = load_afrag<WF>(wp + kDW * TB);
        mma_w<WF>(acc0, w0, *pl);
        mma_w<WF>(acc1, w1, pl[kDW * xsl]);
        wp += 2 * kDW * TB;
        pl += 2 * kDW * xsl;
      }
      if (n) mma_w<WF>(acc0, load_afrag<WF>(wp), *pl);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
      if (p == ppr - 1) {
        // the unit is complete: this warp's partial sums to the epilogue warp
        if (nunit >= kDPB) mbar_wait(&pempty[b], ((nunit / kDPB) - 1) & 1, a.err);
#pragma unroll
        for (int q = 0; q < 4; ++q) acc0[q] += acc1[q];
        put_cfrag(part + ((size_t)b * kDW + warp) * WU, acc0, lane, 0, mr);
        if (tid == 0) punit[b] = u;
#pragma unroll
        for (int q = 0; q < 4; ++q) acc0[q] = acc1[q] = 0.f;
        __syncwarp();
        if (lane == 0) mbar_arrive(&pfull[b]);
        ++nunit;
      }
    }
  }
}

}  // namespace m3
