// misc.cuh -- the small kernels around the decode step: per-frame parameter
// block, GPU int8 quantiser, embedding lookup, KV prefill / readback.
#pragma once

#include "common.cuh"
#include "gemv.cuh"
#include "gemv_tile.cuh"
#include "noise.cuh"

namespace m3 {

// The frame's scalars go to a device block by a kernel launch (not a
// host-to-device copy), so they are ordered on the stream like any kernel
// and the captured graph reads them from a fixed address.
__global__ void set_frame_params_kernel(FrameParams* dst, FrameParams v) {
  if (threadIdx.x == 0) *dst = v;
}

// The frame's RoPE rotations, (cos, sin) of pos[r] * inv_freq[i] (fp64,
// then fp32), for rows r < rows and i < half: one table per frame instead
// of the trigonometry in every attention CTA of every layer.  The positions
// are read from the frame's parameter block on the device, so a captured
// loop of frames sees the positions the loop advanced.
__global__ void rope_table_kernel(const FrameParams* __restrict__ fp,
                                  const double* __restrict__ inv_freq, int half, float2* table) {
  const int r = blockIdx.x;
  const int pos = fp->pos[r];
  for (int i = threadIdx.x; i < half; i += blockDim.x) {
    const double ang = (double)pos * inv_freq[i];
    table[(size_t)r * half + i] = make_float2((float)cos(ang), (float)sin(ang));
  }
}

// (cos, sin) of p * inv_freq[i] (fp64, then fp32) for positions
// p = p0 .. p0 + npos - 1: the depth decoder's frame-local positions (once),
// a prompt chunk's positions.
__global__ void rope_positions_kernel(const double* __restrict__ inv_freq, int half, int p0,
                                      int npos, float2* table) {
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < npos * half; k += gridDim.x * blockDim.x) {
    const double ang = (double)(p0 + k / half) * inv_freq[k % half];
    table[k] = make_float2((float)cos(ang), (float)sin(ang));
  }
}

// int8 weight-only quantisation ("MiniMax Music 3 on Metal", section
// "Precision": one scale per row for the body and lm_head, per group of 128
// for the depth decoder, quantised on the GPU at load):
//   s = absmax / 127 (IEEE fp32 division), q = clamp(rint(w / s), -127, 127),
//   s == 0 -> q = 0.
// One CTA per (row, group) for groups >= 1024 elements; the output row r is
// written at q + r * q_ld and its scales at s + r * s_ld.
__global__ void quantize_rows_kernel(const __nv_bfloat16* __restrict__ w, int64_t cols,
                                     int64_t group, int8_t* q, int64_t q_ld, float* s,
                                     int64_t s_ld) {
  const int64_t row = blockIdx.y;
  const int64_t g = blockIdx.x;
  const __nv_bfloat16* src = w + row * cols + g * group;
  __shared__ float red[32];
  float amax = 0.0f;
  for (int64_t i = threadIdx.x; i < group; i += blockDim.x)
    amax = fmaxf(amax, fabsf(__bfloat162float(src[i])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  const float sc = __fdiv_rn(red[0], 127.0f);
  if (threadIdx.x == 0) s[row * s_ld + g] = sc;
  int8_t* dst = q + row * q_ld + g * group;
  for (int64_t i = threadIdx.x; i < group; i += blockDim.x) {
    int8_t v = 0;
    if (sc != 0.0f) {
      float r = rintf(__fdiv_rn(__bfloat162float(src[i]), sc));
      r = fminf(127.0f, fmaxf(-127.0f, r));
      v = (int8_t)r;
    }
    dst[i] = v;
  }
}

// Groups of 128: one warp per (row, group), 4 elements per lane.
__global__ void quantize_g128_kernel(const __nv_bfloat16* __restrict__ w, int64_t rows,
                                     int64_t cols, int8_t* q, int64_t q_ld, float* s,
                                     int64_t s_ld) {
  const int64_t ng = cols / 128;
  const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= rows * ng) return;
  const int64_t row = gw / ng, g = gw % ng;
  const __nv_bfloat16* src = w + row * cols + g * 128;
  float v[4];
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[i] = __bfloat162float(src[lane + 32 * i]);
    amax = fmaxf(amax, fabsf(v[i]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float sc = __fdiv_rn(amax, 127.0f);
  if (lane == 0) s[row * s_ld + g] = sc;
  int8_t* dst = q + row * q_ld + g * 128;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int8_t qq = 0;
    if (sc != 0.0f) {
      float r = rintf(__fdiv_rn(v[i], sc));
      r = fminf(127.0f, fmaxf(-127.0f, r));
      qq = (int8_t)r;
    }
    dst[lane + 32 * i] = qq;
  }
}

// Row-major [rows][K] weights (bf16 or int8) -> the tiled layout of
// gemv_tile.cuh, source row r going to matrix row dst_row0 + r * row_step;
// int8 is stored biased, byte = q + 128 (the GEMV's f16 conversion).
template <typename T>
__global__ void tile_rows_kernel(const T* __restrict__ src, int rows, int K, uint8_t* dst,
                                 int dst_row0, int row_step) {
  const int64_t total = (int64_t)rows * K;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int r = (int)(i / K), k = (int)(i % K);
    const int n = dst_row0 + r * row_step;
    T v = src[i];
    if constexpr (sizeof(T) == 1) v = (T)((uint8_t)v ^ 0x80u);  // int8 stored biased: q + 128
    *reinterpret_cast<T*>(dst + tile_byte_offset(n, k, K, (int)sizeof(T))) = v;
  }
}

// The inverse of tile_rows_kernel for bf16: a tiled [N][K] matrix back to
// row-major out[n][k] (rows N..pad of the tiling are not written).
__global__ void untile_rows_kernel(const uint8_t* __restrict__ src, int N, int K,
                                   __nv_bfloat16* __restrict__ out) {
  const int64_t total = (int64_t)N * K;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int n = (int)(i / K), k = (int)(i % K);
    out[i] = *reinterpret_cast<const __nv_bfloat16*>(src + tile_byte_offset(n, k, K, 2));
  }
}

// x_out[r] = table[offset + codes[r]] for r < rows; an out-of-range code
// records kErrBounds and yields a zero row.
// A code equal to zero_code (the end token's code, at the depth decoder's
// first lookup) gives a zero row without an error.
__global__ void embed_kernel(const int* __restrict__ codes, const __nv_bfloat16* __restrict__ table,
                             int n_table, int offset, int H, __nv_bfloat16* x_out, int* err,
                             int zero_code) {
  const int r = blockIdx.x;
  pdl_launch_dependents();
  pdl_wait();
  const int code = codes[r];
  const int idx = offset + code;
  const bool zero = code == zero_code;
  const bool ok = !zero && idx >= 0 && idx < n_table;
  if (!ok && !zero && threadIdx.x == 0) record_error(err, kErrBounds);
  for (int k = threadIdx.x * 8; k < H; k += blockDim.x * 8) {
    uint4 v = make_uint4(0, 0, 0, 0);
    if (ok) v = *reinterpret_cast<const uint4*>(table + (size_t)idx * H + k);
    *reinterpret_cast<uint4*>(x_out + (size_t)r * H + k) = v;
  }
}

// KV prefill: src bf16 [n_layers][n_pos][Hkv][D] -> pages (chunk-swizzled,
// see kv_elem_offset), converted to the cache type (bf16 copy or f16
// round-to-nearest-even).
__global__ void kv_set_kernel(const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                              const unsigned long long* __restrict__ pages, int n_layers,
                              int max_pages, int page_size, int n_pos, int Hkv, int D, int f16) {
  const int64_t total = (int64_t)n_layers * n_pos * Hkv * D;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int d = (int)(i % D);
    const int hh = (int)((i / D) % Hkv);
    const int p = (int)((i / ((int64_t)D * Hkv)) % n_pos);
    const int l = (int)(i / ((int64_t)D * Hkv * n_pos));
    uint16_t* base = reinterpret_cast<uint16_t*>(pages[(size_t)l * max_pages + p / page_size]);
    const int off = p % page_size;
    const float kf = __bfloat162float(k[i]), vf = __bfloat162float(v[i]);
    uint16_t kb, vb;
    if (f16) {
      kb = __half_as_ushort(__float2half_rn(kf));
      vb = __half_as_ushort(__float2half_rn(vf));
    } else {
      kb = __bfloat16_as_ushort(k[i]);
      vb = __bfloat16_as_ushort(v[i]);
    }
    base[kv_elem_offset(hh, page_size, off, D, d)] = kb;
    base[kv_elem_offset(Hkv + hh, page_size, off, D, d)] = vb;
  }
}

// KV readback: pages -> raw cache-type bits [n_layers][n_pos][Hkv][D].
__global__ void kv_get_kernel(uint16_t* k, uint16_t* v, const unsigned long long* __restrict__ pages,
                              int n_layers, int max_pages, int page_size, int n_pos, int Hkv,
                              int D) {
  const int64_t total = (int64_t)n_layers * n_pos * Hkv * D;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int d = (int)(i % D);
    const int hh = (int)((i / D) % Hkv);
    const int p = (int)((i / ((int64_t)D * Hkv)) % n_pos);
    const int l = (int)(i / ((int64_t)D * Hkv * n_pos));
    const uint16_t* base =
        reinterpret_cast<const uint16_t*>(pages[(size_t)l * max_pages + p / page_size]);
    const int off = p % page_size;
    k[i] = base[kv_elem_offset(hh, page_size, off, D, d)];
    v[i] = base[kv_elem_offset(Hkv + hh, page_size, off, D, d)];
  }
}

// One RMSNorm row per CTA (any blockDim multiple of 32, up to 1024):
// out = bf16(gamma * bf16(x / rms)), the sum of squares in fp32.  Rows of a
// multiple of 8 elements (16-byte aligned) go 16 bytes at a time (a thread's
// 8 consecutive elements, then the threads, then the warps, in that order).
__global__ void rmsnorm_rows_kernel(const __nv_bfloat16* __restrict__ x,
                                    const __nv_bfloat16* __restrict__ gamma, float eps, int n,
                                    __nv_bfloat16* out) {
  __shared__ float red[32];
  const __nv_bfloat16* xr = x + (size_t)blockIdx.x * n;
  __nv_bfloat16* orow = out + (size_t)blockIdx.x * n;
  const bool vec = n % 8 == 0 &&
                   ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(gamma) |
                     reinterpret_cast<uintptr_t>(out)) & 15) == 0;
  float s = 0.0f;
  if (vec) {
    for (int c = threadIdx.x; c < n / 8; c += blockDim.x) {
      const uint4 w = *reinterpret_cast<const uint4*>(xr + 8 * c);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float lo, hi;
        bf16x2_to_f32(ws[k], lo, hi);
        s = fmaf(lo, lo, s);
        s = fmaf(hi, hi, s);
      }
    }
  } else {
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      const float f = __bfloat162float(xr[i]);
      s = fmaf(f, f, s);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  float t = 0.0f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
  const float r = 1.0f / sqrtf(t / (float)n + eps);
  if (vec) {
    for (int c = threadIdx.x; c < n / 8; c += blockDim.x) {
      const uint4 w = *reinterpret_cast<const uint4*>(xr + 8 * c);
      const uint4 gv = *reinterpret_cast<const uint4*>(gamma + 8 * c);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w}, gs[4] = {gv.x, gv.y, gv.z, gv.w};
      uint32_t os[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float lo, hi, glo, ghi;
        bf16x2_to_f32(ws[k], lo, hi);
        bf16x2_to_f32(gs[k], glo, ghi);
        const __nv_bfloat162 o2 = __floats2bfloat162_rn(glo * round_bf16(lo * r), ghi * round_bf16(hi * r));
        os[k] = *reinterpret_cast<const uint32_t*>(&o2);
      }
      *reinterpret_cast<uint4*>(orow + 8 * c) = make_uint4(os[0], os[1], os[2], os[3]);
    }
  } else {
    for (int i = threadIdx.x; i < n; i += blockDim.x)
      orow[i] = __float2bfloat16_rn(__bfloat162float(gamma[i]) * round_bf16(__bfloat162float(xr[i]) * r));
  }
}

// ------------------------------------------------------ generation loop --
// Device state of a generation loop ("第二阶段" of the DiffSynth-Studio
// article: each frame's codes are embedded back as the next input until the
// end token; "MiniMax Music 3 on Metal": position, step and count advance
// on the GPU, the host reading the state every 16 frames).
struct LoopState {
  int step;               // frames run so far
  int keys;               // CFG pairs, or rows without CFG
  int active[kMaxRows];   // per key: still generating
  int count[kMaxRows];    // per key: frames generated before the end token
  int* codes_out;         // [max_frames][rows][1 + nc], filled with -1 beforehand
  __nv_bfloat16* h_hist;  // nullable: [max_frames][rows][H]
};

struct LoopArgs {
  FrameParams* fp;
  LoopState* ls;
  const int* codes;                 // [rows] this frame's semantic code
  const int* dcodes;                // [rows][nc] its residual codes
  const __nv_bfloat16* h;           // [rows][H] its final-normed hidden state
  const __nv_bfloat16* tok;         // [S][H] token embeddings of the code block
  const __nv_bfloat16* const* aud;  // nc audio-embedding tables [V][H]
  __nv_bfloat16* x;                 // [rows][H] the next frame's input
  int* err;
  int nc, V, H, S, has_end;
  float scale;                      // (1 + nc)^-0.5
};

__global__ void loop_init_kernel(LoopState* dst, LoopState v) {
  if (threadIdx.x == 0) *dst = v;
}

// One CTA per row.  For a row whose key still runs: record the frame (its
// codes, the residual ones -1 on the end frame, and its hidden state) at
// index step.  Then the next input: bf16(scale * (tok[c0] + aud[0][c1] + ...
// + aud[nc-1][c_nc])) with the sum in fp32 in that order, or zeros for a key
// that has stopped (now or before).
__global__ void loop_feedback_kernel(LoopArgs a) {
  __shared__ int cs[32];
  __shared__ int feed_s;
  const int r = blockIdx.x;
  const int rows = a.fp->rows;
  const int key = a.fp->cfg_on ? r / 2 : r;
  const LoopState* ls = a.ls;
  const int step = ls->step;
  const bool act = ls->active[key] != 0;
  const int c0 = a.codes[r];
  const bool ends = a.has_end && c0 == a.S;
  const int W = 1 + a.nc;
  if (threadIdx.x == 0) {
    cs[0] = c0;
    for (int j = 0; j < a.nc; ++j) cs[1 + j] = a.dcodes[r * a.nc + j];
    if (act) {
      int* out = ls->codes_out + ((size_t)step * rows + r) * W;
      out[0] = c0;
      for (int j = 0; j < a.nc; ++j) out[1 + j] = ends ? -1 : cs[1 + j];
    }
    bool feed = act && !ends;
    if (feed) {  // the codes fed forward must index the tables
      bool ok = c0 >= 0 && c0 < a.S;
      for (int j = 0; j < a.nc; ++j) ok = ok && cs[1 + j] >= 0 && cs[1 + j] < a.V;
      if (!ok) record_error(a.err, kErrBounds);
      feed = ok;
    }
    feed_s = feed;
  }
  if (act && ls->h_hist) {
    const uint4* src = reinterpret_cast<const uint4*>(a.h + (size_t)r * a.H);
    uint4* dst = reinterpret_cast<uint4*>(ls->h_hist + ((size_t)step * rows + r) * a.H);
    for (int k = threadIdx.x; k < a.H / 8; k += blockDim.x) dst[k] = src[k];
  }
  __syncthreads();
  const bool feed = feed_s != 0;
  for (int k = threadIdx.x * 8; k < a.H; k += blockDim.x * 8) {
    uint4 o = make_uint4(0u, 0u, 0u, 0u);
    if (feed) {
      float t[8];
      const uint4 e = *reinterpret_cast<const uint4*>(a.tok + (size_t)cs[0] * a.H + k);
      const uint32_t ew[4] = {e.x, e.y, e.z, e.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        t[2 * q] = __uint_as_float(ew[q] << 16);
        t[2 * q + 1] = __uint_as_float(ew[q] & 0xFFFF0000u);
      }
      for (int j = 0; j < a.nc; ++j) {
        const uint4 v = *reinterpret_cast<const uint4*>(a.aud[j] + (size_t)cs[1 + j] * a.H + k);
        const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          t[2 * q] = __fadd_rn(t[2 * q], __uint_as_float(vw[q] << 16));
          t[2 * q + 1] = __fadd_rn(t[2 * q + 1], __uint_as_float(vw[q] & 0xFFFF0000u));
        }
      }
      uint32_t ow[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(t[2 * q], a.scale)));
        const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(t[2 * q + 1], a.scale)));
        ow[q] = lo | (hi << 16);
      }
      o = make_uint4(ow[0], ow[1], ow[2], ow[3]);
    }
    *reinterpret_cast<uint4*>(a.x + (size_t)r * a.H + k) = o;
  }
}

// One warp: the stop rule and the counts per key, then the next frame's
// positions, noise frame and step.
__global__ void loop_advance_kernel(LoopArgs a) {
  FrameParams* fp = a.fp;
  LoopState* ls = a.ls;
  const int t = threadIdx.x;
  if (t < ls->keys && ls->active[t]) {
    const int r = fp->cfg_on ? 2 * t : t;
    if (a.has_end && a.codes[r] == a.S) ls->active[t] = 0;
    else ls->count[t] += 1;
  }
  if (t < fp->rows) fp->pos[t] += 1;
  __syncwarp();
  if (t == 0) {
    ls->step += 1;
    fp->frame += 1ull;
  }
}

// ------------------------------------------------------------ noise export --
// G(seed, frame, row, index0 + i) for i < n, by the same device function the
// samplers draw with (noise.cuh): the noise made visible for a bit-for-bit
// comparison with any other implementation of its definition.
__global__ void gumbel_fill_kernel(unsigned long long seed, unsigned long long frame,
                                   unsigned long long row, unsigned long long index0, long long n,
                                   float* __restrict__ out) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x)
    out[i] = gumbel_noise(seed, frame, row, index0 + (unsigned long long)i);
}

// ------------------------------------------------------- bounded-wait check --
// One mbarrier that nothing ever arrives on, waited for with at most `polls`
// try_wait polls: the wait gives up, records kErrTimeout and the kernel
// returns -- the path every bounded wait of the library takes when its
// producer never comes, exercised without hanging or faulting the GPU.
__global__ void stalled_wait_kernel(int* err, long long polls) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    bool done = false;
    for (long long i = 0; i < polls && !done; ++i) done = mbar_try_wait(&bar, 0);
    if (!done) record_error(err, kErrTimeout);
  }
}

}  // namespace m3
