// Memory-bound kernels of libfs4 (sm_100a): standalone NVFP4 quantise /
// dequantise, and the preamble of the Newton-Schulz step (Frobenius norm and
// max reduction, then normalise + clip + quantise to both NVFP4 views).
//
// "Full-Stack FP4" (arXiv 2607.04422): Section 2 "NVFP4 format" for the block
// encoding; Section 3.4 for clipping before the NVFP4 iteration and for the two
// views Q1x16(X) (Gram operand) and Q16x1(X) (update operand).
#include <algorithm>
#include <cfloat>
#include <mutex>
#include <cmath>

#include "fs4_device.cuh"
#include "fs4_internal.h"

namespace fs4 {

namespace {

constexpr int kEwThreads = 256;
constexpr int kT = 64;           // elementwise tile edge
constexpr float kBoundInflate = 1.0f + 1.0f / 256.0f;

__device__ __forceinline__ bool is_finite_bits(float v) {
  return (__float_as_uint(v) & 0x7F800000u) != 0x7F800000u;
}

// Index of the matrix that owns work unit u (prefix is ascending, prefix[0] == 0).
__device__ __forceinline__ int owner_of(const int32_t* prefix, int count, int32_t u) {
  int lo = 0, hi = count - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= u) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// Max over all threads of the block (blockDim.x == kEwThreads); result valid in thread 0.
__device__ __forceinline__ float block_max(float v, float* red) {
  v = warp_max(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  if (w == 0) {
    v = l < (kEwThreads / 32) ? red[l] : 0.0f;
    v = warp_max(v);
  }
  return v;
}

// Read-and-clear max of a float vector in global memory (values >= 0), block-wide;
// len is a multiple of 4 and vec 16-byte aligned.  Result valid in thread 0.
__device__ float drain_max(float* vec, int64_t len, float* red) {
  float m = 0.0f;
  float4* v4 = reinterpret_cast<float4*>(vec);
  const int32_t n4 = (int32_t)(len >> 2);
  for (int32_t i = threadIdx.x; i < n4; i += 2 * kEwThreads) {
    const bool two = i + kEwThreads < n4;
    const float4 a = __ldcg(v4 + i);
    const float4 b = two ? __ldcg(v4 + i + kEwThreads) : make_float4(0.f, 0.f, 0.f, 0.f);
    __stcg(v4 + i, make_float4(0.f, 0.f, 0.f, 0.f));
    if (two) __stcg(v4 + i + kEwThreads, make_float4(0.f, 0.f, 0.f, 0.f));
    m = fmaxf(m, fmaxf(fmaxf(fmaxf(a.x, a.y), fmaxf(a.z, a.w)), fmaxf(fmaxf(b.x, b.y), fmaxf(b.z, b.w))));
  }
  return block_max(m, red);
}

// Write 16 codes + 1 scale of the block starting at (row r, column c) of an
// NVFP4 matrix with Cp padded columns, TILED layout.
__device__ __forceinline__ void store_block_tiled(uint8_t* codes, uint8_t* scales, int64_t r,
                                                  int64_t c, int64_t Cp, const QBlock16& q) {
  const int64_t off = tiled_chunk_offset(r, c & ~int64_t(31), Cp) + ((c & 16) ? 8 : 0);
  *reinterpret_cast<uint2*>(codes + off) = make_uint2(q.w0, q.w1);
  scales[tiled_scale_offset(r, c >> 4, Cp)] = static_cast<uint8_t>(q.scale);
}

// ------------------------------------------------------------------ standalone quantise
// Pass 1: max |x| (hdr[1], as float bits) and a non-finite flag (hdr[0]) by atomics.
__device__ __forceinline__ void amax_pass(const float* __restrict__ x, int64_t rows, int64_t cols,
                                          int64_t ld, uint32_t* __restrict__ hdr) {
  __shared__ float red[kEwThreads / 32];
  float m = 0.0f;
  bool bad = false;
  const bool vec = ((reinterpret_cast<uintptr_t>(x) & 15) == 0) && ((ld & 3) == 0) && ((cols & 3) == 0);
  if (vec && ld == cols) {  // contiguous: one flat float4 stream, four loads in flight per thread
    const float4* x4 = reinterpret_cast<const float4*>(x);
    const int64_t n4 = rows * (cols >> 2);
    const int64_t stride = (int64_t)gridDim.x * kEwThreads;
    for (int64_t f = blockIdx.x * (int64_t)kEwThreads + threadIdx.x; f < n4; f += 4 * stride) {
      float4 v[4];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        v[k] = f + k * stride < n4 ? __ldg(x4 + f + k * stride) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        bad |= !(is_finite_bits(v[k].x) && is_finite_bits(v[k].y) && is_finite_bits(v[k].z) &&
                 is_finite_bits(v[k].w));
        m = fmaxf(m, fmaxf(fmaxf(fabsf(v[k].x), fabsf(v[k].y)), fmaxf(fabsf(v[k].z), fabsf(v[k].w))));
      }
    }
  } else {
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
      const float* row = x + r * ld;
      if (vec) {  // float4 loads: one request per thread covers 16 bytes
        const float4* row4 = reinterpret_cast<const float4*>(row);
        for (int64_t c = threadIdx.x; c < (cols >> 2); c += kEwThreads) {
          const float4 v = __ldg(row4 + c);
          bad |= !(is_finite_bits(v.x) && is_finite_bits(v.y) && is_finite_bits(v.z) &&
                   is_finite_bits(v.w));
          m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
        }
      } else {
        for (int64_t c = threadIdx.x; c < cols; c += kEwThreads) {
          const float v = __ldg(row + c);
          bad |= !is_finite_bits(v);
          m = fmaxf(m, fabsf(v));
        }
      }
    }
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(&hdr[0], kStatusNonFinite);
  m = block_max(m, red);
  if (threadIdx.x == 0) atomicMax(&hdr[1], __float_as_uint(m));
}

// Pass 2: quantise the R x C matrix Y (Y = x for the row axis, Y = x^T for the column
// axis) in 1x16 blocks along Y's rows.  Work unit = one 64 x 64 tile of Y's (padded)
// extent, staged through shared memory so both axes read x with coalesced loads.
// Persistent CTAs: the next unit's x tile is loaded into registers while the current
// one is quantised (interior tiles of 16-byte aligned inputs; edge tiles load on the
// guarded path).  Tiles are visited in x's row-major order, last tile first: the amax
// pass just streamed x top to bottom, so the tail of x is still resident in L2.
__device__ __forceinline__ void quantize_pass(
    const float* __restrict__ x, int64_t ld, int64_t R, int64_t C, int col_axis, int tiled,
    int sg_amax_mode, int64_t Rext, int64_t Cext, int64_t Cp, int64_t ntiles,
    uint8_t* __restrict__ codes, uint8_t* __restrict__ scales, float* __restrict__ s_g_out,
    const uint32_t* __restrict__ hdr) {
  __shared__ float tile[kT][kT + 1];
  const float amax = __uint_as_float(__ldcg(&hdr[1]));
  float s_g;
  if (sg_amax_mode) {
    s_g = amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f;
  } else {
    s_g = pow2_tensor_scale(amax);
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) *s_g_out = s_g;
  const float six_sg = __fmul_rn(6.0f, s_g);
  const float rcp_six = __frcp_rn(six_sg);

  const int t = threadIdx.x;
  const int64_t xtiles_c = (col_axis ? Rext : Cext) / kT;
  const int64_t xrows = col_axis ? C : R, xcols = col_axis ? R : C;       // x's extent
  const bool aligned = ((reinterpret_cast<uintptr_t>(x) & 15) == 0) && ((ld & 3) == 0);
  auto origin = [&](int64_t u, int64_t& xr0, int64_t& xc0) {   // tile origin in x
    const int64_t xt = ntiles - 1 - u;
    xr0 = (xt / xtiles_c) * kT;
    xc0 = (xt % xtiles_c) * kT;
  };
  // 16 threads per 256-byte line segment of x, four passes of 16 lines
  float4 pf[4];
  bool pf_fast = false;
  auto prefetch = [&](int64_t u) {
    pf_fast = false;
    if (u >= ntiles) return;
    int64_t xr0, xc0;
    origin(u, xr0, xc0);
    if (aligned && xr0 + kT <= xrows && xc0 + kT <= xcols) {
      pf_fast = true;
#pragma unroll
      for (int pass = 0; pass < 4; ++pass) {
        const int f = t + kEwThreads * pass;
        pf[pass] = __ldg(reinterpret_cast<const float4*>(x + (xr0 + (f >> 4)) * ld + xc0 + (f & 15) * 4));
      }
    }
  };
  prefetch(blockIdx.x);
  for (int64_t u = blockIdx.x; u < ntiles; u += gridDim.x) {
    float4 cur[4];
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) cur[pass] = pf[pass];
    const bool cur_fast = pf_fast;
    prefetch(u + gridDim.x);
    int64_t xr0, xc0;
    origin(u, xr0, xc0);
    const int64_t i0 = col_axis ? xc0 : xr0, j0 = col_axis ? xr0 : xc0;
    // Row axis: x line = row i of the quantised matrix Y; column axis: x line = column
    // of Y (Y = x^T), stored transposed.
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
      const int f = t + kEwThreads * pass;
      const int line = f >> 4, c4 = (f & 15) * 4;
      float v[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      if (cur_fast) {
        v[0] = cur[pass].x; v[1] = cur[pass].y; v[2] = cur[pass].z; v[3] = cur[pass].w;
      } else if (xr0 + line < xrows) {
        const float* src = x + (xr0 + line) * ld + xc0 + c4;
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (xc0 + c4 + e < xcols) v[e] = __ldg(src + e);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (!col_axis) tile[line][c4 + e] = v[e];
        else tile[c4 + e][line] = v[e];
      }
    }
    __syncthreads();
    const int r = t >> 2, cb = (t & 3) * 16;
    const int64_t i = i0 + r, j = j0 + cb;
    float v[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) v[e] = tile[r][cb + e];
    const QBlock16 q = sg_amax_mode ? quantize16<false>(v, s_g, six_sg, rcp_six)
                                    : quantize16<true>(v, s_g, six_sg, rcp_six);
    if (tiled) {
      store_block_tiled(codes, scales, i, j, Cp, q);
    } else if (i < R && j < C) {
      *reinterpret_cast<uint2*>(codes + i * (C / 2) + j / 2) = make_uint2(q.w0, q.w1);
      scales[i * (C / 16) + j / 16] = static_cast<uint8_t>(q.scale);
    }
    __syncthreads();   // the tile is restaged by the next unit
  }
}

// Arrive at a grid-wide barrier and wait (thread 0 of each CTA) until all `expected`
// CTAs have arrived; the fence makes this CTA's earlier atomics visible to every CTA
// that passes the barrier.  The wait is bounded: after kWaitLimitNs it records
// kStatusTimeout and returns false (the CTA then skips the rest of its work).  Only
// for cooperative launches, whose CTAs are all resident at once.
__device__ __forceinline__ bool grid_barrier(uint32_t* count, uint32_t expected, uint32_t* status) {
  __shared__ int passed;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(count, 1u);
    const uint64_t t0 = global_timer_ns();
    int ok = 0;
    for (;;) {
      uint32_t v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(count) : "memory");
      if (v >= expected) { ok = 1; break; }
      if (global_timer_ns() - t0 > kWaitLimitNs) { atomicOr(status, kStatusTimeout); break; }
      __nanosleep(64);
    }
    passed = ok;
  }
  __syncthreads();
  return passed != 0;
}

struct QuantArgs {
  const float* x;
  int64_t rows, cols, ld;             // x as given
  int64_t R, C, Rext, Cext, Cp, ntiles;
  int col_axis, tiled, sg_amax_mode;
  int stall;                          // test only: the barrier waits for one CTA too many
  uint8_t* codes;
  uint8_t* scales;
  float* s_g;
  uint32_t* hdr;                      // [0] status, [1] amax bits, [2] barrier count (zeroed)
};

// One matrix of a batched quantise (kernel parameter).
struct QMat {
  const float* x;
  int64_t rows, cols, ld;             // x as given
  int64_t R, C, Cp, xtiles_c;         // the quantised matrix Y (x or x^T), its padded width,
                                      // tiles per line of x
  int32_t col_axis, vec;              // 16x1 blocks; float4 loads possible
  uint8_t* codes;
  uint8_t* scales;
  float* s_g;
};
// Workspace words of a batched quantise: [0] status, [kQBatchCountWord] barrier count,
// [kQBatchAmaxWord + i] amax of matrix i (float bits); all zeroed by the launcher.
constexpr int kQBatchCountWord = 2;
constexpr int kQBatchAmaxWord = 64;

struct QBatchArgs {
  int32_t count;
  int32_t tiled, sg_amax_mode, stall;
  uint32_t* hdr;
  int32_t pre_amax[kMaxBatch + 1];    // prefix sums of the 16-row amax units
  int32_t pre_tiles[kMaxBatch + 1];   // prefix sums of the 64 x 64 tiles
  QMat mat[kMaxBatch];
};
static_assert(sizeof(QBatchArgs) <= 32000, "kernel parameter block too large");

// Standalone quantise in one cooperative launch: the amax pass over x, a grid-wide
// barrier, then the quantise pass.  The barrier takes the place of a second launch and
// its ramp, and the quantise pass (last tile first) finds the tail of x in L2.
__global__ void __launch_bounds__(kEwThreads) quantize_fused_kernel(const __grid_constant__ QuantArgs a) {
  amax_pass(a.x, a.rows, a.cols, a.ld, a.hdr);
  if (!grid_barrier(&a.hdr[2], gridDim.x + (a.stall ? 1u : 0u), &a.hdr[0])) return;
  quantize_pass(a.x, a.ld, a.R, a.C, a.col_axis, a.tiled, a.sg_amax_mode, a.Rext, a.Cext, a.Cp,
                a.ntiles, a.codes, a.scales, a.s_g, a.hdr);
}

// ------------------------------------------------------------------ batched quantise
// Many matrices in one cooperative launch: the amax pass over units of 16 rows (one
// atomic per unit on the matrix's amax), a grid-wide barrier, then the quantise pass
// over the 64 x 64 tiles of every matrix, each staged through shared memory as in the
// single-matrix quantise.  Work units of all matrices are numbered consecutively
// (prefix sums), so one launch keeps every SM busy whatever the mix of sizes.
__global__ void __launch_bounds__(kEwThreads) quantize_batched_kernel(const __grid_constant__ QBatchArgs a) {
  __shared__ float red[kEwThreads / 32];
  __shared__ float tile[kT][kT + 1];
  uint32_t* status = a.hdr;
  uint32_t* amaxv = a.hdr + kQBatchAmaxWord;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  // ---- pass 1: per-matrix max |x| and the non-finite flag
  bool bad = false;
  for (int32_t u = blockIdx.x; u < a.pre_amax[a.count]; u += gridDim.x) {
    const int mi = owner_of(a.pre_amax, a.count, u);
    const QMat& m = a.mat[mi];
    const int64_t r0 = (int64_t)(u - a.pre_amax[mi]) * 16;
    float mx = 0.0f;
    for (int64_t r = r0 + warp; r < r0 + 16 && r < m.rows; r += kEwThreads / 32) {
      const float* row = m.x + r * m.ld;
      if (m.vec) {
        const float4* row4 = reinterpret_cast<const float4*>(row);
        for (int64_t c = lane; c < (m.cols >> 2); c += 32) {
          const float4 v = __ldg(row4 + c);
          bad |= !(is_finite_bits(v.x) && is_finite_bits(v.y) && is_finite_bits(v.z) &&
                   is_finite_bits(v.w));
          mx = fmaxf(mx, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
        }
      } else {
        for (int64_t c = lane; c < m.cols; c += 32) {
          const float v = __ldg(row + c);
          bad |= !is_finite_bits(v);
          mx = fmaxf(mx, fabsf(v));
        }
      }
    }
    mx = block_max(mx, red);
    if (t == 0 && mx > 0.0f) atomicMax(&amaxv[mi], __float_as_uint(mx));
  }
  if (__syncthreads_or(bad) && t == 0) atomicOr(&status[0], kStatusNonFinite);
  if (!grid_barrier(&a.hdr[kQBatchCountWord], gridDim.x + (a.stall ? 1u : 0u), &status[0])) return;
  // ---- pass 2: the tiles of every matrix
  for (int32_t u = blockIdx.x; u < a.pre_tiles[a.count]; u += gridDim.x) {
    const int mi = owner_of(a.pre_tiles, a.count, u);
    const QMat& m = a.mat[mi];
    const int64_t lu = u - a.pre_tiles[mi];
    const float amax = __uint_as_float(__ldcg(&amaxv[mi]));
    const float s_g = a.sg_amax_mode ? (amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f)
                                     : pow2_tensor_scale(amax);
    if (lu == 0 && t == 0) *m.s_g = s_g;
    const float six_sg = __fmul_rn(6.0f, s_g);
    const float rcp_six = __frcp_rn(six_sg);
    // tile origin in x; Y = x (row axis) or x^T (column axis) is quantised along its rows
    const int64_t xr0 = (lu / m.xtiles_c) * kT, xc0 = (lu % m.xtiles_c) * kT;
    const int64_t xrows = m.col_axis ? m.C : m.R, xcols = m.col_axis ? m.R : m.C;
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
      const int f = t + kEwThreads * pass;
      const int line = f >> 4, c4 = (f & 15) * 4;
      float v[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      if (xr0 + line < xrows) {
        const float* src = m.x + (xr0 + line) * m.ld + xc0 + c4;
        if (m.vec && xc0 + c4 + 4 <= xcols) {
          const float4 q4 = __ldg(reinterpret_cast<const float4*>(src));
          v[0] = q4.x; v[1] = q4.y; v[2] = q4.z; v[3] = q4.w;
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (xc0 + c4 + e < xcols) v[e] = __ldg(src + e);
        }
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (!m.col_axis) tile[line][c4 + e] = v[e];
        else tile[c4 + e][line] = v[e];
      }
    }
    __syncthreads();
    const int64_t i0 = m.col_axis ? xc0 : xr0, j0 = m.col_axis ? xr0 : xc0;
    const int r = t >> 2, cb = (t & 3) * 16;
    const int64_t i = i0 + r, j = j0 + cb;
    float v[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) v[e] = tile[r][cb + e];
    const QBlock16 q = a.sg_amax_mode ? quantize16<false>(v, s_g, six_sg, rcp_six)
                                      : quantize16<true>(v, s_g, six_sg, rcp_six);
    if (a.tiled) {
      store_block_tiled(m.codes, m.scales, i, j, m.Cp, q);
    } else if (i < m.R && j < m.C) {
      *reinterpret_cast<uint2*>(m.codes + i * (m.C / 2) + j / 2) = make_uint2(q.w0, q.w1);
      m.scales[i * (m.C / 16) + j / 16] = static_cast<uint8_t>(q.scale);
    }
    __syncthreads();   // the tile is restaged by the next unit
  }
}

// y = fp32(fp32(code * scale) * s_g), one thread per group of 4 consecutive elements
// of a row, so a warp writes 512 contiguous bytes (float4 stores when y is 16-byte
// aligned with ld % 4 == 0).  The flat group index advances by a fixed (row, column)
// stride, so the loop needs no 64-bit division; each pass handles kDqUnroll groups
// whose code and scale loads are all issued before the first store.
constexpr int kDqUnroll = 4;

__global__ void __launch_bounds__(kEwThreads) dequantize_kernel(
    const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
    const float* __restrict__ s_g_ptr, int64_t R, int64_t C, int tiled, int64_t Cp,
    float* __restrict__ y, int64_t ld) {
  const float s_g = __ldg(s_g_ptr);
  const int64_t C4 = C / 4;
  if (R <= 0 || C4 <= 0) return;
  const bool vec = ((reinterpret_cast<uintptr_t>(y) & 15) == 0) && ((ld & 3) == 0);
  const int64_t g0 = blockIdx.x * (int64_t)kEwThreads + threadIdx.x;
  const int64_t step = (int64_t)gridDim.x * kEwThreads;
  const int64_t step_i = step / C4, step_c = step % C4;
  int64_t i = g0 / C4, c4 = g0 % C4;
  while (i < R) {
    int64_t gi[kDqUnroll], gc[kDqUnroll];
    uint32_t w[kDqUnroll], sb[kDqUnroll];
#pragma unroll
    for (int k = 0; k < kDqUnroll; ++k) {
      gi[k] = i;
      gc[k] = c4 * 4;
      if (i < R) {
        const int64_t c = gc[k];
        if (tiled) {
          w[k] = *reinterpret_cast<const uint16_t*>(
              codes + tiled_chunk_offset(i, c & ~int64_t(31), Cp) + ((c & 31) >> 1));
          sb[k] = scales[tiled_scale_offset(i, c >> 4, Cp)];
        } else {
          w[k] = *reinterpret_cast<const uint16_t*>(codes + i * (C / 2) + c / 2);
          sb[k] = scales[i * (C / 16) + c / 16];
        }
      }
      i += step_i;
      c4 += step_c;
      if (c4 >= C4) { c4 -= C4; ++i; }
    }
#pragma unroll
    for (int k = 0; k < kDqUnroll; ++k) {
      if (gi[k] >= R) break;
      const float s = e4m3_to_f32(sb[k]);
      const uint32_t hv[2] = {e2m1x2_to_f16x2(w[k] & 0xFFu), e2m1x2_to_f16x2((w[k] >> 8) & 0xFFu)};
      const float4 o = make_float4(__fmul_rn(__fmul_rn(half_lo(hv[0]), s), s_g),
                                   __fmul_rn(__fmul_rn(half_hi(hv[0]), s), s_g),
                                   __fmul_rn(__fmul_rn(half_lo(hv[1]), s), s_g),
                                   __fmul_rn(__fmul_rn(half_hi(hv[1]), s), s_g));
      float* dst = y + gi[k] * ld + gc[k];
      if (vec) {
        *reinterpret_cast<float4*>(dst) = o;
      } else {
        dst[0] = o.x; dst[1] = o.y; dst[2] = o.z; dst[3] = o.w;
      }
    }
  }
}

// ------------------------------------------------------------------ Newton-Schulz preamble
__device__ __forceinline__ NsState* state_of(const NsParams& p, const MatDesc& d) {
  return reinterpret_cast<NsState*>(p.ws + d.state_off);
}

// The 31-bit key of |g|: its float bits without the sign (non-negative floats order
// like their bit patterns).
__device__ __forceinline__ uint32_t abs_key(float v) { return __float_as_uint(v) & 0x7FFFFFFFu; }

// Block blk (16 elements from column 16 blk) of row r of a G given as an NVFP4 state
// (PLAIN 1x16 row blocks of G H16^r with n0 columns, as the first-moment step stores it),
// decoded by one thread: fp32(fp32(code * s) * s_g), then (H16^r)^-1 = H16 D / 4 (the
// butterfly and * 0.25 of rht16 without signs, then the signs of the state's mask).
__device__ __forceinline__ void nvfp4_src_block(const MatDesc& d, int64_t n0, int64_t r, int64_t blk,
                                                float (&v)[16]) {
  const int64_t b = r * (n0 / 16) + blk;
  const uint2 w = __ldg(reinterpret_cast<const uint2*>(d.qcodes) + b);
  const float sb = e4m3_to_f32(__ldg(d.qscales + b));
  const float sg = __ldg(d.qsg);
  e2m1_decode16(w.x, w.y, v);
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __fmul_rn(__fmul_rn(v[i], sb), sg);
  rht16(v, 0u);
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(__float_as_uint(v[i]) ^ (((d.qmask >> i) & 1u) << 31));
}

// Sum of G^2 (float64), max |G| and a non-finite flag per matrix; work unit =
// 16 rows of one matrix in the caller's orientation.  The last CTA to finish a
// matrix derives its normalisation and clip scalars and the tensor scale of X_0
// (Section 3.4: normalise, clip, quantise), so the preamble only reads them.
// kHist (quantile clip): also a histogram of the top 11 bits of every |g| key,
// accumulated per unit in shared memory and added to the matrix's histogram.
template <bool kHist, bool kNv>
__global__ void __launch_bounds__(kEwThreads) ns_reduce_kernel(const __grid_constant__ NsParams p) {
  __shared__ float redf[kEwThreads / 32];
  __shared__ double redd[kEwThreads / 32];
  __shared__ uint32_t hist[kHist ? kQBins1 : 1];
  const int32_t total = p.prefix[p.count];
  for (int32_t u = blockIdx.x; u < total; u += gridDim.x) {
    if constexpr (kHist) {
      for (int b = threadIdx.x; b < kQBins1; b += kEwThreads) hist[b] = 0u;
      __syncthreads();
    }
    const int mi = owner_of(p.prefix, p.count, u);
    const MatDesc& d = p.mat[mi];
    const int64_t rows0 = d.tall ? d.n : d.m, cols0 = d.tall ? d.m : d.n;
    const int64_t r0 = (u - p.prefix[mi]) * 16;
    const bool vec = ((reinterpret_cast<uintptr_t>(d.G) & 15) == 0) && ((d.ldg & 3) == 0);
    double s = 0.0;
    float mx = 0.0f;
    bool bad = false;
    for (int64_t r = r0; r < r0 + 16 && r < rows0; ++r) {
      const float* row = d.G + r * d.ldg;
      if constexpr (kNv) {   // NVFP4 source: one thread per 16-element block
        for (int64_t blk = threadIdx.x; blk < cols0 / 16; blk += kEwThreads) {
          float vv[16];
          nvfp4_src_block(d, cols0, r, blk, vv);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            bad |= !is_finite_bits(vv[e]);
            mx = fmaxf(mx, fabsf(vv[e]));
            s += (double)vv[e] * (double)vv[e];
            if constexpr (kHist) atomicAdd(&hist[abs_key(vv[e]) >> 20], 1u);
          }
        }
      } else if (vec) {
        for (int64_t c = 4 * threadIdx.x; c < cols0; c += 4 * kEwThreads) {
          const float4 v4 = __ldg(reinterpret_cast<const float4*>(row + c));
          const float vv[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            bad |= !is_finite_bits(vv[e]);
            mx = fmaxf(mx, fabsf(vv[e]));
            s += (double)vv[e] * (double)vv[e];
            if constexpr (kHist) atomicAdd(&hist[abs_key(vv[e]) >> 20], 1u);
          }
        }
      } else {
        for (int64_t c = threadIdx.x; c < cols0; c += kEwThreads) {
          const float v = __ldg(row + c);
          bad |= !is_finite_bits(v);
          mx = fmaxf(mx, fabsf(v));
          s += (double)v * (double)v;
          if constexpr (kHist) atomicAdd(&hist[abs_key(v) >> 20], 1u);
        }
      }
    }
    NsState* st = state_of(p, d);
    const bool any_bad = __syncthreads_or(bad);   // also orders the histogram updates
    if constexpr (kHist) {
      uint32_t* gh = reinterpret_cast<uint32_t*>(
          p.ws + mat_layout(d.mp, d.np, d.state_off, d.big_off).qhist);
      for (int b = threadIdx.x; b < kQBins1; b += kEwThreads)
        if (hist[b] != 0u) atomicAdd(&gh[b], hist[b]);
    }
    s = warp_sum(s);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    if (l == 0) redd[w] = s;
    mx = block_max(mx, redf);  // contains __syncthreads, orders the redd writes
    if (threadIdx.x == 0) {
      if (any_bad) {
        atomicOr(&st->nonfinite, 1u);
        atomicOr(p.status, kStatusNonFinite);
      }
      double tot = 0.0;
      for (int k = 0; k < kEwThreads / 32; ++k) tot += redd[k];
      atomicAdd(&st->sumsq, tot);
      atomicMax(&st->amaxG, __float_as_uint(mx));
      __threadfence();
      const uint32_t units = (uint32_t)(p.prefix[mi + 1] - p.prefix[mi]);
      if (atomicAdd(&st->done[4], 1u) == units - 1u) {
        __threadfence();
        const bool dead = __ldcg(&st->nonfinite) != 0u;
        const double norm = sqrt(__ldcg(&st->sumsq));
        const float inv = dead ? 0.0f : (float)(1.0 / (norm + 1e-7));
        float tau = FLT_MAX;   // the quantile clip sets it after the selection
        if (p.clip_k > 0.0f && !(p.opts & kOptQuantile))
          tau = (float)((double)p.clip_k * norm * (double)inv / sqrt((double)d.m * (double)d.n));
        const float amaxG = __uint_as_float(__ldcg(&st->amaxG));
        const float amax0 = dead ? 0.0f : fminf(__fmul_rn(amaxG, inv), tau);
        st->inv0 = inv;
        st->tau0 = tau;
        // with the Hadamard transform the quantised tensor is X_0 H: |X_0 H| <= 4 amax
        st->sg[kSgX + 0] = pow2_tensor_scale((p.opts & kOptRht) ? 4.0f * amax0 : amax0,
                                             (p.opts & kOpt46) != 0);
        st->amaxX[0] = __float_as_uint(amax0);
        st->done[4] = 0u;
      }
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------ quantile clip
// tau = the nearest-rank q-quantile of |X_0| = fp32(|G|_(k) * inv), |G|_(k) the k-th
// smallest |g| with k = ceil(fl64(q) * N) ("Full-Stack FP4" Section 3.4, "p99 outlier
// clipping"; fp32(. * inv) is monotone, so the order statistic of |X_0| is that of |G|
// scaled).  |G|_(k) is selected exactly on its 31-bit key, digit by digit: 11 bits from
// the reduction's histogram, then the keys of that bin are gathered and the last 11 + 9
// bits selected among them by one CTA per matrix.

// 1-based rank of the quantile (IEEE double, as the oracle computes it).
__device__ __forceinline__ uint64_t quantile_rank(float q, int64_t N) {
  double k = ceil((double)q * (double)N);
  if (k < 1.0) k = 1.0;
  if (k > (double)N) k = (double)N;
  return (uint64_t)k;
}

// Block-wide (kT threads): the bin b of `h` (nbins and kT powers of two) holding the
// element of rank k (1-based; sum(h) >= k), and the rank of that element within bin b.
// Result valid in every thread.
template <int kT>
__device__ void find_rank_bin(const uint32_t* h, int nbins, uint64_t k, int* bin_out,
                              uint64_t* rank_out) {
  __shared__ unsigned long long part[kT];
  __shared__ int s_bin;
  __shared__ unsigned long long s_rank;
  const int per = nbins >= kT ? nbins / kT : 1, t = threadIdx.x;
  const bool has = t * per < nbins;
  unsigned long long sum = 0;
  if (has)
    for (int i = 0; i < per; ++i) sum += h[t * per + i];
  part[t] = sum;
  if (t == 0) { s_bin = nbins - 1; s_rank = 1; }
  __syncthreads();
  // inclusive scan of the per-thread sums (Hillis-Steele over kT entries)
  for (int off = 1; off < kT; off <<= 1) {
    const unsigned long long v = t >= off ? part[t - off] : 0ull;
    __syncthreads();
    part[t] += v;
    __syncthreads();
  }
  const unsigned long long before = t > 0 ? part[t - 1] : 0ull;
  if (has && before < k && k <= part[t]) {
    unsigned long long acc = before;
    for (int i = 0; i < per; ++i) {
      const uint32_t c = h[t * per + i];
      if (k <= acc + c) { s_bin = t * per + i; s_rank = k - acc; break; }
      acc += c;
    }
  }
  __syncthreads();
  *bin_out = s_bin;
  *rank_out = s_rank;
  __syncthreads();
}

// One CTA per matrix: the first digit of the selected key and the rank within its bin.
__global__ void __launch_bounds__(kEwThreads) ns_quantile_select1_kernel(const __grid_constant__ NsParams p) {
  const MatDesc& d = p.mat[blockIdx.x];
  NsState* st = state_of(p, d);
  if (__ldcg(&st->nonfinite) != 0u) return;
  const uint32_t* gh = reinterpret_cast<const uint32_t*>(p.ws + mat_layout(d.mp, d.np, d.state_off, d.big_off).qhist);
  __shared__ uint32_t h[kQBins1];
  for (int b = threadIdx.x; b < kQBins1; b += kEwThreads) h[b] = __ldcg(&gh[b]);
  __syncthreads();
  int bin;
  uint64_t rank;
  find_rank_bin<kEwThreads>(h, kQBins1, quantile_rank(p.clip_k, (int64_t)d.m * d.n), &bin, &rank);
  if (threadIdx.x == 0) {
    st->q_bin1 = (uint32_t)bin;
    st->q_rank1 = rank;
  }
}

// Gather the keys of every |g| whose top 11 bits equal the selected first digit into the
// matrix's X buffer (unused until the preamble; it holds mp * np >= m * n words).  Work
// unit = 16 rows of one matrix, as in the reduction.  Hits are staged in a shared buffer
// (warp ballots, one shared atomic per warp and element step) and flushed with one global
// atomic per flush, so the matrix's counter sees a few atomics per unit, not one per warp.
constexpr int kGatherBuf = 8192;            // staged keys per CTA
constexpr int kGatherStep = 4 * 4 * kEwThreads;   // elements per column step (4 float4 per thread)
template <bool kNv>
__global__ void __launch_bounds__(kEwThreads) ns_quantile_gather_kernel(const __grid_constant__ NsParams p) {
  __shared__ uint32_t sbuf[kGatherBuf];
  __shared__ uint32_t s_n;
  __shared__ unsigned long long s_base;
  const int32_t total = p.prefix[p.count];
  const int lane = threadIdx.x & 31;
  for (int32_t u = blockIdx.x; u < total; u += gridDim.x) {
    const int mi = owner_of(p.prefix, p.count, u);
    const MatDesc& d = p.mat[mi];
    NsState* st = state_of(p, d);
    if (__ldcg(&st->nonfinite) != 0u) continue;   // uniform over the CTA
    const uint32_t bin = __ldcg(&st->q_bin1);
    uint32_t* cand = reinterpret_cast<uint32_t*>(p.ws + mat_layout(d.mp, d.np, d.state_off, d.big_off).X);
    const int64_t rows0 = d.tall ? d.n : d.m, cols0 = d.tall ? d.m : d.n;
    const int64_t r0 = (u - p.prefix[mi]) * 16;
    const bool vec = ((reinterpret_cast<uintptr_t>(d.G) & 15) == 0) && ((d.ldg & 3) == 0);
    if (threadIdx.x == 0) s_n = 0u;
    __syncthreads();
    auto append = [&](uint32_t key, bool valid) {   // warp-wide: every lane calls it
      const bool hit = valid && (key >> 20) == bin;
      const unsigned m = __ballot_sync(0xFFFFFFFFu, hit);
      if (m != 0u) {
        const int leader = __ffs(m) - 1;
        uint32_t pos = 0u;
        if (lane == leader) pos = atomicAdd(&s_n, (uint32_t)__popc(m));
        pos = __shfl_sync(0xFFFFFFFFu, pos, leader);
        if (hit) sbuf[pos + __popc(m & ((1u << lane) - 1u))] = key;
      }
    };
    // block-wide: move the staged keys to the matrix's candidate buffer
    auto flush = [&]() {
      __syncthreads();
      const uint32_t n = s_n;
      if (n != 0u) {
        if (threadIdx.x == 0) s_base = atomicAdd(&st->q_count, (unsigned long long)n);
        __syncthreads();
        const unsigned long long base = s_base;
        for (uint32_t i = threadIdx.x; i < n; i += kEwThreads) cand[base + i] = sbuf[i];
        __syncthreads();
        if (threadIdx.x == 0) s_n = 0u;
      }
      __syncthreads();
    };
    for (int64_t r = r0; r < r0 + 16 && r < rows0; ++r) {
      const float* row = d.G + r * d.ldg;
      // one column step adds at most kGatherStep keys: flush first when they might not fit
      for (int64_t c0 = 0; c0 < cols0; c0 += kGatherStep) {   // uniform over the CTA
        __syncthreads();
        const bool full = s_n > (uint32_t)(kGatherBuf - kGatherStep);
        __syncthreads();   // every thread has read s_n before any thread appends again
        if (full) flush();
        if constexpr (kNv) {   // NVFP4 source: one 16-element block per thread and step
          const int64_t blk = c0 / 16 + threadIdx.x;
          const bool valid = blk < cols0 / 16;
          float v[16];
          if (valid) {
            nvfp4_src_block(d, cols0, r, blk, v);
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] = 0.0f;
          }
#pragma unroll
          for (int e = 0; e < 16; ++e) append(abs_key(v[e]), valid);
        } else if (vec) {   // cols0 is a multiple of 16: a float4 is wholly inside or outside the row
          float4 v[4];
          bool valid[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int64_t c = c0 + 4 * (threadIdx.x + k * kEwThreads);
            valid[k] = c < cols0;
            v[k] = valid[k] ? __ldg(reinterpret_cast<const float4*>(row + c))
                            : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            append(abs_key(v[k].x), valid[k]);
            append(abs_key(v[k].y), valid[k]);
            append(abs_key(v[k].z), valid[k]);
            append(abs_key(v[k].w), valid[k]);
          }
        } else {
#pragma unroll 1
          for (int k = 0; k < 16; ++k) {
            const int64_t c = c0 + threadIdx.x + k * kEwThreads;
            const bool valid = c < cols0;
            append(valid ? abs_key(__ldg(row + c)) : 0u, valid);
          }
        }
      }
    }
    flush();
  }
}

// One CTA per matrix: the last two digits among the gathered keys, then tau, the clamp
// bound of X_0 and the tensor scale of X_0.
constexpr int kSelThreads = 1024;
__global__ void __launch_bounds__(kSelThreads) ns_quantile_select2_kernel(const __grid_constant__ NsParams p) {
  const MatDesc& d = p.mat[blockIdx.x];
  NsState* st = state_of(p, d);
  if (__ldcg(&st->nonfinite) != 0u) return;
  const uint32_t* cand = reinterpret_cast<const uint32_t*>(p.ws + mat_layout(d.mp, d.np, d.state_off, d.big_off).X);
  const uint64_t n = __ldcg(&st->q_count);
  const uint32_t b1 = __ldcg(&st->q_bin1);
  const uint64_t k1 = __ldcg(&st->q_rank1);
  __shared__ uint32_t h[kQBins2];
  for (int b = threadIdx.x; b < kQBins2; b += kSelThreads) h[b] = 0u;
  __syncthreads();
  for (uint64_t i = threadIdx.x; i < n; i += kSelThreads) atomicAdd(&h[(__ldcg(&cand[i]) >> 9) & (kQBins2 - 1)], 1u);
  __syncthreads();
  int b2;
  uint64_t k2;
  find_rank_bin<kSelThreads>(h, kQBins2, k1, &b2, &k2);
  for (int b = threadIdx.x; b < kQBins3; b += kSelThreads) h[b] = 0u;
  __syncthreads();
  for (uint64_t i = threadIdx.x; i < n; i += kSelThreads) {
    const uint32_t key = __ldcg(&cand[i]);
    if (((key >> 9) & (kQBins2 - 1)) == (uint32_t)b2) atomicAdd(&h[key & (kQBins3 - 1)], 1u);
  }
  __syncthreads();
  int b3;
  uint64_t k3;
  find_rank_bin<kSelThreads>(h, kQBins3, k2, &b3, &k3);
  if (threadIdx.x == 0) {
    const float gk = __uint_as_float((b1 << 20) | ((uint32_t)b2 << 9) | (uint32_t)b3);
    const float inv = __ldcg(&st->inv0);
    const float tau = __fmul_rn(gk, inv);
    const float amax0 = fminf(__fmul_rn(__uint_as_float(__ldcg(&st->amaxG)), inv), tau);
    st->tau0 = tau;
    st->amaxX[0] = __float_as_uint(amax0);
    st->sg[kSgX + 0] = pow2_tensor_scale((p.opts & kOptRht) ? 4.0f * amax0 : amax0,
                                         (p.opts & kOpt46) != 0);
  }
}

// Preamble tile in shared memory: 64 rows of 64 floats in 16-byte chunks, chunk c of row
// R stored at chunk c ^ pre_swz(R, c).  The XOR keeps every access of the kernel free of
// bank conflicts: a quarter-warp reading four chunks of each of two adjacent rows (row
// view, float4), a warp reading one column of four rows 16 apart (column view), and a
// quarter-warp writing eight consecutive chunks of one row (staging); the transposed
// staging of a tall matrix is 2-way.
__device__ __forceinline__ int pre_swz(int R, int c) {
  return (2 * (c >> 3)) ^ (R & 1) ^ ((R >> 2) & 1) ^ (2 * ((R >> 4) & 1)) ^ (4 * ((R >> 5) & 1));
}
__device__ __forceinline__ int pre_off(int R, int col) {   // float offset of (R, col)
  const int c = col >> 2;
  return R * kT + 4 * (c ^ pre_swz(R, c)) + (col & 3);
}

// clamp(fp32(x * inv), +-tau) of four values.
__device__ __forceinline__ float4 clip4(float4 x, float inv, float tau) {
  return make_float4(fminf(fmaxf(__fmul_rn(x.x, inv), -tau), tau), fminf(fmaxf(__fmul_rn(x.y, inv), -tau), tau),
                     fminf(fmaxf(__fmul_rn(x.z, inv), -tau), tau), fminf(fmaxf(__fmul_rn(x.w, inv), -tau), tau));
}

// Staging of a tile that the preamble's fast path does not take: an edge tile (rows_left
// rows and cols_left columns of G remain from the tile origin), a G that is not 16-byte
// aligned, or a matrix with a non-finite entry (dead: staged as zeros).  Kept out of line
// so that its per-element guards stay off the interior tiles' path.
__device__ __noinline__ void preamble_stage_guarded(float* tile, float* Xt, const float* gtile, int64_t ldg,
                                                    int32_t np, bool tall, bool dead, float inv, float tau,
                                                    int32_t rows_left, int32_t cols_left, int t) {
#pragma unroll
  for (int pass = 0; pass < 4; ++pass) {
    const int f = t + kEwThreads * pass;
    const int line = f >> 4, c4 = (f & 15) * 4;
    float v[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (!dead && line < rows_left) {
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (c4 + e < cols_left)
          v[e] = fminf(fmaxf(__fmul_rn(__ldg(gtile + (int64_t)line * ldg + c4 + e), inv), -tau), tau);
    }
    if (!tall) {
      const float4 v4 = make_float4(v[0], v[1], v[2], v[3]);
      *reinterpret_cast<float4*>(tile + pre_off(line, c4)) = v4;
      *reinterpret_cast<float4*>(Xt + line * np + c4) = v4;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) tile[pre_off(c4 + e, line)] = v[e];
    }
  }
}

// Normalise, clip and quantise: X0 = clamp(fp32(G * inv), +-tau) written as FP32
// and as both NVFP4 views, with row / column sums of the squared dequantised
// values.  Work unit = one 64 x 64 tile of the padded working extent; G and X
// are read and written as float4 with 16 threads per 64-float row segment.
// Each CTA takes one contiguous range of the unit sequence (matrix by matrix, the
// tiles of X in row-major order), so the next unit's position follows from the
// current one by an increment: the owning matrix is searched and the tile index
// divided once per CTA.
template <uint32_t kOpts>
__global__ void __launch_bounds__(kEwThreads, 4) ns_preamble_kernel(const __grid_constant__ NsParams p) {
  __shared__ __align__(16) float tile[kT * kT];
  __shared__ float scale_tab[256];
  const int t = threadIdx.x;
  if (t < 128) scale_tab_fill(scale_tab, t);   // read after the first barrier below

  const int32_t total = p.prefix[p.count];
  const int32_t per = total / (int32_t)gridDim.x, extra = total % (int32_t)gridDim.x;
  const int32_t bid = (int32_t)blockIdx.x;
  const int32_t first = bid * per + min(bid, extra);
  const int32_t n_units = per + (bid < extra ? 1 : 0);
  if (n_units <= 0) return;

  // position of the next unit to load: matrix, tile row and tile column of X
  int nmi = owner_of(p.prefix, p.count, first);
  int32_t ntn = p.mat[nmi].np / kT, ntm = p.mat[nmi].mp / kT, nti, ntj;
  {
    const int32_t lu = first - p.prefix[nmi];
    nti = lu / ntn;
    ntj = lu - nti * ntn;
  }

  // The next unit's G tile is loaded into registers while this unit is quantised
  // (interior tiles of 16-byte aligned inputs; edge tiles load on the guarded path).
  float4 pf[4];
  bool pf_fast = false;
  auto prefetch = [&](int mi, int32_t ti, int32_t tj) {
    pf_fast = false;
    const MatDesc& d = p.mat[mi];
    const int32_t i0 = ti * kT, j0 = tj * kT;
    const int32_t rows_g = d.tall ? d.n : d.m, cols_g = d.tall ? d.m : d.n;
    const int32_t gr0 = d.tall ? j0 : i0, gc0 = d.tall ? i0 : j0;
    const bool vec = ((reinterpret_cast<uintptr_t>(d.G) & 15) == 0) && ((d.ldg & 3) == 0);
    if (!(kOpts & kOptNvSrc) && vec && gr0 + kT <= rows_g && gc0 + kT <= cols_g) {
      pf_fast = true;
      const float* gtile = d.G + (int64_t)gr0 * d.ldg + gc0;
#pragma unroll
      for (int pass = 0; pass < 4; ++pass) {
        const int f = t + kEwThreads * pass;
        pf[pass] = __ldg(reinterpret_cast<const float4*>(gtile + (int64_t)(f >> 4) * d.ldg + (f & 15) * 4));
      }
    }
  };
  prefetch(nmi, nti, ntj);

  // scalars of the current matrix (derived once by the reduction kernel), reloaded only
  // when the unit belongs to another matrix than the previous one
  int cur_mi = -1;
  bool dead = false;
  float inv = 0.0f, tau = 0.0f, sg = 1.0f, six_sg = 6.0f, rcp_six = 1.0f, rcp_sg = 1.0f;

  for (int32_t it = 0; it < n_units; ++it) {
    float4 cur[4];
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) cur[pass] = pf[pass];
    const bool cur_fast = pf_fast;
    const int mi = nmi;
    const int32_t i0 = nti * kT, j0 = ntj * kT;
    if (it + 1 < n_units) {
      if (++ntj == ntn) {
        ntj = 0;
        if (++nti == ntm) {
          nti = 0;
          ++nmi;
          ntn = p.mat[nmi].np / kT;
          ntm = p.mat[nmi].mp / kT;
        }
      }
      prefetch(nmi, nti, ntj);
    }
    const MatDesc& d = p.mat[mi];
    const MatLayout L = mat_layout(d.mp, d.np, d.state_off, d.big_off, (kOpts & kOptBf16) != 0);
    if (mi != cur_mi) {
      const NsState* st = state_of(p, d);
      cur_mi = mi;
      dead = __ldcg(&st->nonfinite) != 0u;
      inv = __ldcg(&st->inv0);
      tau = __ldcg(&st->tau0);
      sg = __ldcg(&st->sg[kSgX + 0]);
      six_sg = __fmul_rn(6.0f, sg);
      rcp_six = __frcp_rn(six_sg);
      rcp_sg = __frcp_rn(sg);   // sg is a power of two
    }
    const ScaleTab stab{scale_tab, rcp_sg};
    // X0 of this tile (working orientation); a matrix with a non-finite entry is carried
    // as all zeros (its output is zero).  Non-tall: thread f holds X0 row f / 16, columns
    // 4 (f % 16) .. + 3, written to X straight from registers and staged as one float4.
    // Tall: it holds G row f / 16 = X0 column f / 16, staged transposed.
    const int32_t rows_g = d.tall ? d.n : d.m, cols_g = d.tall ? d.m : d.n;
    const int32_t gr0 = d.tall ? j0 : i0, gc0 = d.tall ? i0 : j0;   // tile origin in G
    const float* gtile = d.G + (int64_t)gr0 * d.ldg + gc0;
    float* Xt = reinterpret_cast<float*>(p.ws + L.X) + (int64_t)i0 * d.np + j0;
    if constexpr ((kOpts & kOptNvSrc) != 0) {
      // NVFP4 source: thread t decodes block t % 4 of G row t / 4 of the tile
      const int line = t >> 2, blk = t & 3;
      float v[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) v[e] = 0.0f;
      if (!dead && gr0 + line < rows_g && gc0 + 16 * blk < cols_g) {
        nvfp4_src_block(d, cols_g, gr0 + line, gc0 / 16 + blk, v);
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] = fminf(fmaxf(__fmul_rn(v[e], inv), -tau), tau);
      }
      if (!d.tall) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float4 v4 = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
          *reinterpret_cast<float4*>(tile + pre_off(line, 16 * blk + 4 * k)) = v4;
          *reinterpret_cast<float4*>(Xt + line * d.np + 16 * blk + 4 * k) = v4;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) tile[pre_off(16 * blk + e, line)] = v[e];
      }
    } else if (cur_fast && !dead) {
      // interior tile of a finite matrix, from the prefetched float4s (each case its own
      // uniform branch, so that the other cases' code is not predicated into this one)
      if (!d.tall) {
#pragma unroll
        for (int pass = 0; pass < 4; ++pass) {
          const int f = t + kEwThreads * pass;
          const int line = f >> 4, c4 = (f & 15) * 4;       // 64 lines of 64 floats
          const float4 v4 = clip4(cur[pass], inv, tau);
          *reinterpret_cast<float4*>(tile + pre_off(line, c4)) = v4;
          *reinterpret_cast<float4*>(Xt + line * d.np + c4) = v4;
        }
      } else {
#pragma unroll
        for (int pass = 0; pass < 4; ++pass) {
          const int f = t + kEwThreads * pass;
          const int line = f >> 4, c4 = (f & 15) * 4;
          const float4 v4 = clip4(cur[pass], inv, tau);
          tile[pre_off(c4, line)] = v4.x;
          tile[pre_off(c4 + 1, line)] = v4.y;
          tile[pre_off(c4 + 2, line)] = v4.z;
          tile[pre_off(c4 + 3, line)] = v4.w;
        }
      }
    } else {
      preamble_stage_guarded(tile, Xt, gtile, d.ldg, d.np, d.tall != 0, dead, inv, tau, rows_g - gr0,
                             cols_g - gc0, t);
    }
    __syncthreads();
    if (d.tall) {
#pragma unroll
      for (int pass = 0; pass < 4; ++pass) {
        const int f = t + kEwThreads * pass;
        const int r = f >> 4, c4 = (f & 15) * 4;
        *reinterpret_cast<float4*>(Xt + r * d.np + c4) = *reinterpret_cast<const float4*>(tile + pre_off(r, c4));
      }
    }
    // two views; thread t owns one 16-element block of line t/4 (four blocks per line)
#pragma unroll
    for (int view = 0; view < 2; ++view) {
      const int line = t >> 2, blk = t & 3;
      float v[16];
      if (view == 0) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float4 x4 = *reinterpret_cast<const float4*>(tile + pre_off(line, blk * 16 + 4 * k));
          v[4 * k] = x4.x; v[4 * k + 1] = x4.y; v[4 * k + 2] = x4.z; v[4 * k + 3] = x4.w;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] = tile[pre_off(blk * 16 + e, line)];
      }
      // row r0 + line of the view (view 0: row i0 + line of X, K from j0; view 1: row
      // j0 + line of X^T, K from i0)
      const int32_t r0 = view == 0 ? i0 : j0, k0 = view == 0 ? j0 : i0;
      const int32_t Cp = view == 0 ? d.np : d.mp;
      if constexpr ((kOpts & kOptBf16) != 0) {
        // the BF16 comparison step: both views are BF16 copies (round to nearest even) of
        // X0 (view 0) and of X0^T (view 1), two 16-byte chunks per block
        uint8_t* dst = p.ws + (view == 0 ? L.qX[0] : L.qXT[0]);
        uint32_t w[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) w[e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
        const int64_t R = r0 + line, K0 = k0 + blk * 16;
        *reinterpret_cast<uint4*>(dst + tiled_chunk_offset_bf16(R, K0, Cp)) = make_uint4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<uint4*>(dst + tiled_chunk_offset_bf16(R, K0 + 8, Cp)) = make_uint4(w[4], w[5], w[6], w[7]);
        continue;
      }
      // view 0 is the Gram operand of iteration 0, view 1 the update operand
      if constexpr ((kOpts & kOptRht) != 0) rht16(v, view == 0 ? p.rht[0] : p.rht[2]);
      const QBlock16 q = quantize16<true, true, true, (kOpts & kOpt46) != 0>(v, sg, six_sg, rcp_six, stab);
      // TILED destinations from the tile origin: r0 and k0 are multiples of 64, so the
      // row stays in one 128-row tile (at rr = r0 % 128 + line) and the block pair in one
      // 256-column tile (16-byte chunk (k0 % 256) / 32 + blk / 2, swizzled by rr % 8),
      // and the four scales of the line fill one word of one scale atom
      const int32_t rr = (r0 & 64) + line;
      uint8_t* codes = p.ws + (view == 0 ? L.qX[0] : L.qXT[0]) +
                       (int64_t)((r0 >> 7) * (Cp >> 8) + (k0 >> 8)) * kTileBytes + rr * 128;
      uint8_t* scales = p.ws + (view == 0 ? L.sX[0] : L.sXT[0]) +
                        (int64_t)((r0 >> 7) * (Cp >> 6) + (k0 >> 6)) * kAtomBytes + 16 * (rr & 31) +
                        4 * (rr >> 5);
      // pair blocks (0,1) and (2,3) into 16-byte chunks, the four scales into one word
      const uint32_t o0 = __shfl_xor_sync(0xFFFFFFFFu, q.w0, 1);
      const uint32_t o1 = __shfl_xor_sync(0xFFFFFFFFu, q.w1, 1);
      uint32_t sc = q.scale << (8 * blk);
      sc |= __shfl_xor_sync(0xFFFFFFFFu, sc, 1);
      sc |= __shfl_xor_sync(0xFFFFFFFFu, sc, 2);
      if ((blk & 1) == 0)
        *reinterpret_cast<uint4*>(codes + (((((k0 & 255) >> 5) + (blk >> 1)) ^ (line & 7)) << 4)) =
            make_uint4(q.w0, q.w1, o0, o1);
      if (blk == 0) *reinterpret_cast<uint32_t*>(scales) = sc;
      float ss = q.sumsq;
      ss += __shfl_xor_sync(0xFFFFFFFFu, ss, 1);
      ss += __shfl_xor_sync(0xFFFFFFFFu, ss, 2);
      if (blk == 0 && ss != 0.0f)
        atomicAdd(reinterpret_cast<float*>(p.ws + (view == 0 ? L.rowsumX : L.colsumX)) + r0 + line, ss);
    }
    __syncthreads();   // the tile is restaged by the next unit
  }
}

// After the preamble: each matrix's bounds for the first Gram product from the row and
// column sums of its quantised X_0 (one CTA per matrix; the sum vectors are cleared for
// the update phases).  A separate launch orders the preamble's sum atomics before
// these reads, so the preamble needs no fence or completion counter.
__global__ void __launch_bounds__(kEwThreads) ns_preamble_bounds_kernel(const __grid_constant__ NsParams p) {
  __shared__ float red[kEwThreads / 32];
  const int mi = blockIdx.x;
  const MatDesc& d = p.mat[mi];
  NsState* st = state_of(p, d);
  const MatLayout L = mat_layout(d.mp, d.np, d.state_off, d.big_off);
  const float ur = drain_max(reinterpret_cast<float*>(p.ws + L.rowsumX), d.mp, red);
  const float uc = drain_max(reinterpret_cast<float*>(p.ws + L.colsumX), d.np, red);
  if (threadIdx.x == 0) {
    st->u_rowX[0] = ur;
    st->u_colX[0] = uc;
    st->sg[kSgA + 0] = pow2_tensor_scale(ur * kBoundInflate * ((p.opts & kOptRht) ? 4.0f : 1.0f),
                                         (p.opts & kOpt46) != 0);
  }
}

int grid_for(int64_t units, int num_sms, int per_sm) {
  const int64_t cap = (int64_t)num_sms * per_sm;
  return (int)(units < cap ? (units > 0 ? units : 1) : cap);
}

// Grid of a persistent (grid-stride) kernel: as many CTAs as are resident at once,
// from the occupancy the compiled kernel actually reaches (a second wave would
// leave SMs half empty while it runs).  Cached per kernel address (kernels of one
// signature share a pointer type, so a per-type cache would mix them up).
template <typename Kernel>
int persistent_grid(Kernel kernel, int64_t units, int num_sms) {
  static std::mutex mu;
  static const void* keys[16];
  static int vals[16];
  static int used = 0;
  const void* key = reinterpret_cast<const void*>(kernel);
  int resident = 0;
  {
    std::lock_guard<std::mutex> lk(mu);
    for (int i = 0; i < used; ++i)
      if (keys[i] == key) resident = vals[i];
  }
  if (resident == 0) {
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, kEwThreads, 0) != cudaSuccess ||
        occ < 1)
      occ = 1;
    resident = occ;
    std::lock_guard<std::mutex> lk(mu);
    if (used < 16) { keys[used] = key; vals[used] = occ; ++used; }
  }
  return grid_for(units, num_sms, resident);
}

}  // namespace

cudaError_t launch_quantize(const float* x, int64_t rows, int64_t cols, int64_t ld, int axis,
                            uint8_t* codes, uint8_t* scales, float* s_g, uint32_t flags,
                            uint8_t* ws, cudaStream_t st, int num_sms) {
  cudaError_t e = cudaMemsetAsync(ws, 0, 12, st);
  if (e != cudaSuccess) return e;
  QuantArgs a;
  a.x = x; a.rows = rows; a.cols = cols; a.ld = ld;
  a.R = axis ? cols : rows;
  a.C = axis ? rows : cols;
  a.tiled = (flags & 2u) ? 1 : 0;
  a.Rext = a.tiled ? align_up(a.R, 128) : align_up(a.R, kT);
  a.Cp = align_up(a.C, 256);
  a.Cext = a.tiled ? a.Cp : align_up(a.C, kT);
  a.ntiles = (a.Rext / kT) * (a.Cext / kT);
  if (a.ntiles > 0x7FFFFFFF) return cudaErrorInvalidValue;
  a.col_axis = axis;
  a.sg_amax_mode = (flags & 1u) ? 1 : 0;
  a.stall = (flags & (1u << 30)) ? 1 : 0;   // FS4_TEST_STALL
  a.codes = codes; a.scales = scales; a.s_g = s_g;
  a.hdr = reinterpret_cast<uint32_t*>(ws);
  // as many CTAs as are resident at once (a cooperative launch refuses more), fewer
  // when neither pass has that much work (4 float4 per amax thread, one tile per unit)
  const int64_t amax_units = std::max<int64_t>(rows, (rows * cols + 4095) / 4096);
  const int grid = persistent_grid(quantize_fused_kernel, std::max<int64_t>(amax_units, a.ntiles), num_sms);
  void* args[] = {&a};
  return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(quantize_fused_kernel), dim3(grid),
                                     dim3(kEwThreads), args, 0, st);
}

size_t quantize_batched_workspace_bytes(int32_t count) {
  return (size_t)align_up(4 * (kQBatchAmaxWord + count), 256);
}

cudaError_t launch_quantize_batched(int32_t count, const QuantDesc* d, uint32_t flags, uint8_t* ws,
                                    cudaStream_t st, int num_sms) {
  static thread_local QBatchArgs a;   // 27 KB: too large for every caller's stack
  a.count = count;
  a.tiled = (flags & 2u) ? 1 : 0;
  a.sg_amax_mode = (flags & 1u) ? 1 : 0;
  a.stall = (flags & (1u << 30)) ? 1 : 0;   // FS4_TEST_STALL
  a.hdr = reinterpret_cast<uint32_t*>(ws);
  int64_t na = 0, nt = 0;
  a.pre_amax[0] = a.pre_tiles[0] = 0;
  for (int i = 0; i < count; ++i) {
    QMat& m = a.mat[i];
    m.x = d[i].x; m.rows = d[i].rows; m.cols = d[i].cols; m.ld = d[i].ld;
    m.col_axis = d[i].axis;
    m.R = m.col_axis ? m.cols : m.rows;
    m.C = m.col_axis ? m.rows : m.cols;
    const int64_t Rext = a.tiled ? align_up(m.R, 128) : align_up(m.R, kT);
    m.Cp = align_up(m.C, 256);
    const int64_t Cext = a.tiled ? m.Cp : align_up(m.C, kT);
    m.xtiles_c = (m.col_axis ? Rext : Cext) / kT;
    m.vec = ((reinterpret_cast<uintptr_t>(m.x) & 15) == 0 && (m.ld & 3) == 0 && (m.cols & 3) == 0) ? 1 : 0;
    m.codes = d[i].codes; m.scales = d[i].scales; m.s_g = d[i].s_g;
    na += (m.rows + 15) / 16;
    nt += (Rext / kT) * (Cext / kT);
    if (na > 0x7FFFFFFF || nt > 0x7FFFFFFF) return cudaErrorInvalidValue;
    a.pre_amax[i + 1] = (int32_t)na;
    a.pre_tiles[i + 1] = (int32_t)nt;
  }
  cudaError_t e = cudaMemsetAsync(ws, 0, quantize_batched_workspace_bytes(count), st);
  if (e != cudaSuccess) return e;
  // as many CTAs as are resident at once (a cooperative launch refuses more)
  const int grid = persistent_grid(quantize_batched_kernel, std::max<int64_t>(na, nt), num_sms);
  void* args[] = {&a};
  return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(quantize_batched_kernel), dim3(grid),
                                     dim3(kEwThreads), args, 0, st);
}

cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* scales, const float* s_g,
                              int64_t rows, int64_t cols, float* y, int64_t ld, uint32_t flags,
                              cudaStream_t st, int num_sms) {
  const int tiled = (flags & 2u) ? 1 : 0;
  const int64_t ngrp = rows * (cols / 4);
  dequantize_kernel<<<persistent_grid(dequantize_kernel, (ngrp + kEwThreads - 1) / kEwThreads, num_sms), kEwThreads, 0,
                      st>>>(codes, scales, s_g, rows, cols, tiled, align_up(cols, 256), y, ld);
  return cudaGetLastError();
}

cudaError_t launch_ns_reduce(const NsParams& p, cudaStream_t st, int num_sms) {
  const unsigned units = (unsigned)p.prefix[p.count];
  switch (p.opts & (kOptQuantile | kOptNvSrc)) {
    case kOptQuantile:
      ns_reduce_kernel<true, false><<<persistent_grid(ns_reduce_kernel<true, false>, units, num_sms), kEwThreads, 0, st>>>(p);
      break;
    case kOptNvSrc:
      ns_reduce_kernel<false, true><<<persistent_grid(ns_reduce_kernel<false, true>, units, num_sms), kEwThreads, 0, st>>>(p);
      break;
    case kOptQuantile | kOptNvSrc:
      ns_reduce_kernel<true, true><<<persistent_grid(ns_reduce_kernel<true, true>, units, num_sms), kEwThreads, 0, st>>>(p);
      break;
    default:
      ns_reduce_kernel<false, false><<<persistent_grid(ns_reduce_kernel<false, false>, units, num_sms), kEwThreads, 0, st>>>(p);
  }
  return cudaGetLastError();
}

// Quantile clip selection after the reduction (p.prefix holds the reduction's units).
cudaError_t launch_ns_quantile(const NsParams& p, cudaStream_t st, int num_sms) {
  ns_quantile_select1_kernel<<<p.count, kEwThreads, 0, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (p.opts & kOptNvSrc)
    ns_quantile_gather_kernel<true><<<persistent_grid(ns_quantile_gather_kernel<true>, p.prefix[p.count], num_sms),
                                      kEwThreads, 0, st>>>(p);
  else
    ns_quantile_gather_kernel<false><<<persistent_grid(ns_quantile_gather_kernel<false>, p.prefix[p.count], num_sms),
                                       kEwThreads, 0, st>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  ns_quantile_select2_kernel<<<p.count, kSelThreads, 0, st>>>(p);
  return cudaGetLastError();
}

template <uint32_t kOpts>
void preamble_launch(const NsParams& p, cudaStream_t st, int num_sms) {
  ns_preamble_kernel<kOpts><<<persistent_grid(ns_preamble_kernel<kOpts>, p.prefix[p.count], num_sms),
                              kEwThreads, 0, st>>>(p);
}

cudaError_t launch_ns_preamble(const NsParams& p, cudaStream_t st, int num_sms) {
  if (p.opts & kOptBf16) {
    // BF16 views carry no tensor scale: no bounds kernel follows
    preamble_launch<kOptBf16>(p, st, num_sms);
    return cudaGetLastError();
  }
  switch (p.opts & (kOptRht | kOpt46 | kOptNvSrc)) {
    case 0: preamble_launch<0>(p, st, num_sms); break;
    case kOpt46: preamble_launch<kOpt46>(p, st, num_sms); break;
    case kOptRht: preamble_launch<kOptRht>(p, st, num_sms); break;
    case kOptRht | kOpt46: preamble_launch<kOptRht | kOpt46>(p, st, num_sms); break;
    case kOptNvSrc: preamble_launch<kOptNvSrc>(p, st, num_sms); break;
    case kOptNvSrc | kOpt46: preamble_launch<kOptNvSrc | kOpt46>(p, st, num_sms); break;
    case kOptNvSrc | kOptRht: preamble_launch<kOptNvSrc | kOptRht>(p, st, num_sms); break;
    default: preamble_launch<kOptNvSrc | kOptRht | kOpt46>(p, st, num_sms); break;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  ns_preamble_bounds_kernel<<<p.count, kEwThreads, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace fs4
