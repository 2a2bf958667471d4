// Memory-bound kernels of libfs4 (sm_100a): standalone NVFP4 quantise /
// dequantise, and the preamble of the Newton-Schulz step (Frobenius norm and
// max reduction, then normalise + clip + quantise to both NVFP4 views).
//
// "Full-Stack FP4" (arXiv 2607.04422): Section 2 "NVFP4 format" for the block
// encoding; Section 3.4 for clipping before the NVFP4 iteration and for the two
// views Q1x16(X) (Gram operand) and Q16x1(X) (update operand).
#include <cfloat>
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
__device__ __forceinline__ int owner_of(const int32_t* prefix, int count, int64_t u) {
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

// Read-and-clear max of a float vector in global memory (values >= 0), block-wide.
__device__ float drain_max(float* vec, int64_t len, float* red) {
  float m = 0.0f;
  for (int64_t i = threadIdx.x; i < len; i += kEwThreads) {
    m = fmaxf(m, __ldcg(vec + i));
    __stcg(vec + i, 0.0f);
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
__global__ void __launch_bounds__(kEwThreads) amax_kernel(const float* __restrict__ x, int64_t rows,
                                                          int64_t cols, int64_t ld,
                                                          uint32_t* __restrict__ hdr) {
  __shared__ float red[kEwThreads / 32];
  float m = 0.0f;
  bool bad = false;
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const float* row = x + r * ld;
    for (int64_t c = threadIdx.x; c < cols; c += kEwThreads) {
      const float v = __ldg(row + c);
      bad |= !is_finite_bits(v);
      m = fmaxf(m, fabsf(v));
    }
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(&hdr[0], kStatusNonFinite);
  m = block_max(m, red);
  if (threadIdx.x == 0) atomicMax(&hdr[1], __float_as_uint(m));
}

// Quantise the R x C matrix Y (Y = x for the row axis, Y = x^T for the column
// axis) in 1x16 blocks along Y's rows.  One CTA per 64 x 64 tile of Y's
// (padded) extent; the tile is staged through shared memory so both axes read
// x with coalesced loads.
__global__ void __launch_bounds__(kEwThreads) quantize_kernel(
    const float* __restrict__ x, int64_t ld, int64_t R, int64_t C, int col_axis, int tiled,
    int sg_amax_mode, int64_t Rext, int64_t Cext, int64_t Cp, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ scales, float* __restrict__ s_g_out, const uint32_t* __restrict__ hdr) {
  __shared__ float tile[kT][kT + 1];
  const int64_t tiles_c = Cext / kT;
  const int64_t i0 = (blockIdx.x / tiles_c) * kT, j0 = (blockIdx.x % tiles_c) * kT;
  const float amax = __uint_as_float(__ldcg(&hdr[1]));
  float s_g;
  if (sg_amax_mode) {
    s_g = amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f;
  } else {
    s_g = pow2_tensor_scale(amax);
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) *s_g_out = s_g;
  const float six_sg = __fmul_rn(6.0f, s_g);

  const int t = threadIdx.x;
  // stage: thread t covers 16 consecutive elements of one line of x
  {
    const int line = t >> 2, part = (t & 3) * 16;
    if (!col_axis) {
      const int64_t i = i0 + line;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int64_t j = j0 + part + e;
        tile[line][part + e] = (i < R && j < C) ? __ldg(x + i * ld + j) : 0.0f;
      }
    } else {  // Y[i][j] = x[j][i]: read x row j0+line, columns i0+part..
      const int64_t jx = j0 + line;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int64_t ix = i0 + part + e;
        tile[part + e][line] = (jx < C && ix < R) ? __ldg(x + jx * ld + ix) : 0.0f;
      }
    }
  }
  __syncthreads();
  const int r = t >> 2, cb = (t & 3) * 16;
  const int64_t i = i0 + r, j = j0 + cb;
  float v[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) v[e] = tile[r][cb + e];
  const QBlock16 q = quantize16(v, s_g, six_sg);
  if (tiled) {
    store_block_tiled(codes, scales, i, j, Cp, q);
  } else if (i < R && j < C) {
    *reinterpret_cast<uint2*>(codes + i * (C / 2) + j / 2) = make_uint2(q.w0, q.w1);
    scales[i * (C / 16) + j / 16] = static_cast<uint8_t>(q.scale);
  }
}

// y = fp32(fp32(code * scale) * s_g), one thread per 16-element block.
__global__ void __launch_bounds__(kEwThreads) dequantize_kernel(
    const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
    const float* __restrict__ s_g_ptr, int64_t R, int64_t C, int tiled, int64_t Cp,
    float* __restrict__ y, int64_t ld) {
  const float s_g = __ldg(s_g_ptr);
  const int64_t nblk = R * (C / 16);
  for (int64_t b = blockIdx.x * (int64_t)kEwThreads + threadIdx.x; b < nblk;
       b += (int64_t)gridDim.x * kEwThreads) {
    const int64_t i = b / (C / 16), j = (b % (C / 16)) * 16;
    uint2 w;
    uint32_t sb;
    if (tiled) {
      w = *reinterpret_cast<const uint2*>(codes + tiled_chunk_offset(i, j & ~int64_t(31), Cp) +
                                          ((j & 16) ? 8 : 0));
      sb = scales[tiled_scale_offset(i, j >> 4, Cp)];
    } else {
      w = *reinterpret_cast<const uint2*>(codes + i * (C / 2) + j / 2);
      sb = scales[i * (C / 16) + j / 16];
    }
    const float s = e4m3_to_f32(sb);
    uint32_t words[2] = {w.x, w.y};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t hv[4];
      asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
          "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
          "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
          "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
          "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
          "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
          : "=r"(hv[0]), "=r"(hv[1]), "=r"(hv[2]), "=r"(hv[3])
          : "r"(words[h]));
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const int64_t c = j + h * 8 + p * 2;
        y[i * ld + c] = __fmul_rn(__fmul_rn(half_lo(hv[p]), s), s_g);
        y[i * ld + c + 1] = __fmul_rn(__fmul_rn(half_hi(hv[p]), s), s_g);
      }
    }
  }
}

// ------------------------------------------------------------------ Newton-Schulz preamble
__device__ __forceinline__ NsState* state_of(const NsParams& p, const MatDesc& d) {
  return reinterpret_cast<NsState*>(p.ws + d.state_off);
}

// Sum of G^2 (float64), max |G| and a non-finite flag per matrix; work unit =
// 16 rows of one matrix in the caller's orientation.
__global__ void __launch_bounds__(kEwThreads) ns_reduce_kernel(const __grid_constant__ NsParams p) {
  __shared__ float redf[kEwThreads / 32];
  __shared__ double redd[kEwThreads / 32];
  const int64_t total = p.prefix[p.count];
  for (int64_t u = blockIdx.x; u < total; u += gridDim.x) {
    const int mi = owner_of(p.prefix, p.count, u);
    const MatDesc& d = p.mat[mi];
    const int64_t rows0 = d.tall ? d.n : d.m, cols0 = d.tall ? d.m : d.n;
    const int64_t r0 = (u - p.prefix[mi]) * 16;
    double s = 0.0;
    float mx = 0.0f;
    bool bad = false;
    for (int64_t r = r0; r < r0 + 16 && r < rows0; ++r) {
      const float* row = d.G + r * d.ldg;
      for (int64_t c = threadIdx.x; c < cols0; c += kEwThreads) {
        const float v = __ldg(row + c);
        bad |= !is_finite_bits(v);
        mx = fmaxf(mx, fabsf(v));
        s += (double)v * (double)v;
      }
    }
    NsState* st = state_of(p, d);
    if (__syncthreads_or(bad) && threadIdx.x == 0) {
      atomicOr(&st->nonfinite, 1u);
      atomicOr(p.status, kStatusNonFinite);
    }
    s = warp_sum(s);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    if (l == 0) redd[w] = s;
    mx = block_max(mx, redf);  // contains __syncthreads, orders the redd writes
    if (threadIdx.x == 0) {
      double tot = 0.0;
      for (int k = 0; k < kEwThreads / 32; ++k) tot += redd[k];
      atomicAdd(&st->sumsq, tot);
      atomicMax(&st->amaxG, __float_as_uint(mx));
    }
    __syncthreads();
  }
}

// Normalise, clip and quantise: X0 = clamp(fp32(G * inv), +-tau) written as FP32
// and as both NVFP4 views, with row / column sums of the squared dequantised
// values.  Work unit = one 64 x 64 tile of the padded working extent.
__global__ void __launch_bounds__(kEwThreads) ns_preamble_kernel(const __grid_constant__ NsParams p) {
  __shared__ float tile[kT][kT + 1];
  __shared__ float red[kEwThreads / 32];
  __shared__ int s_last;
  const int64_t total = p.prefix[p.count];
  const int t = threadIdx.x;
  for (int64_t u = blockIdx.x; u < total; u += gridDim.x) {
    const int mi = owner_of(p.prefix, p.count, u);
    const MatDesc& d = p.mat[mi];
    NsState* st = state_of(p, d);
    const MatLayout L = mat_layout(d.mp, d.np, d.state_off, d.big_off);
    const int64_t tiles_n = d.np / kT;
    const int64_t lu = u - p.prefix[mi];
    const int64_t i0 = (lu / tiles_n) * kT, j0 = (lu % tiles_n) * kT;

    // scalars of this matrix (identical in every CTA)
    const bool dead = __ldcg(&st->nonfinite) != 0u;
    const double norm = sqrt(__ldcg(&st->sumsq));
    const float inv = dead ? 0.0f : (float)(1.0 / (norm + 1e-7));
    float tau = FLT_MAX;
    if (p.clip_k > 0.0f)
      tau = (float)((double)p.clip_k * norm * (double)inv / sqrt((double)d.m * (double)d.n));
    const float amaxG = __uint_as_float(__ldcg(&st->amaxG));
    const float amax0 = dead ? 0.0f : fminf(__fmul_rn(amaxG, inv), tau);
    const float sg = pow2_tensor_scale(amax0);
    const float six_sg = __fmul_rn(6.0f, sg);
    if (lu == 0 && t == 0) {
      st->sg[kSgX + 0] = sg;
      st->amaxX[0] = __float_as_uint(amax0);
    }

    // stage X0 tile (working orientation) in shared memory
    {
      const int line = t >> 2, part = (t & 3) * 16;
      if (!d.tall) {
        const int64_t i = i0 + line;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int64_t j = j0 + part + e;
          float v = 0.0f;
          if (!dead && i < d.m && j < d.n) v = fminf(fmaxf(__fmul_rn(__ldg(d.G + i * d.ldg + j), inv), -tau), tau);
          tile[line][part + e] = v;
        }
      } else {  // X[i][j] = G[j][i]
        const int64_t j = j0 + line;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int64_t i = i0 + part + e;
          float v = 0.0f;
          if (!dead && i < d.m && j < d.n) v = fminf(fmaxf(__fmul_rn(__ldg(d.G + j * d.ldg + i), inv), -tau), tau);
          tile[part + e][line] = v;
        }
      }
    }
    __syncthreads();
    // a matrix with a non-finite entry is carried as all zeros (its output is zero)
    float* X = reinterpret_cast<float*>(p.ws + L.X);
    {
      const int r = t >> 2, cb = (t & 3) * 16;
      const int64_t i = i0 + r, j = j0 + cb;
      float v[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) v[e] = tile[r][cb + e];
      float4* dst = reinterpret_cast<float4*>(X + i * d.np + j);
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) dst[q4] = make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
      // 1x16 view (Gram operand): rows of X
      const QBlock16 q = quantize16(v, sg, six_sg);
      store_block_tiled(p.ws + L.qX[0], p.ws + L.sX[0], i, j, d.np, q);
      float rs = q.sumsq;
      rs += __shfl_xor_sync(0xFFFFFFFFu, rs, 1);
      rs += __shfl_xor_sync(0xFFFFFFFFu, rs, 2);
      if ((t & 3) == 0 && rs != 0.0f) atomicAdd(reinterpret_cast<float*>(p.ws + L.rowsumX) + i, rs);
    }
    {
      // 16x1 view (update operand), stored as the 1x16 quantisation of X^T
      const int c = t >> 2, rb = (t & 3) * 16;
      const int64_t j = j0 + c, i = i0 + rb;
      float v[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) v[e] = tile[rb + e][c];
      const QBlock16 q = quantize16(v, sg, six_sg);
      store_block_tiled(p.ws + L.qXT[0], p.ws + L.sXT[0], j, i, d.mp, q);
      float cs = q.sumsq;
      cs += __shfl_xor_sync(0xFFFFFFFFu, cs, 1);
      cs += __shfl_xor_sync(0xFFFFFFFFu, cs, 2);
      if ((t & 3) == 0 && cs != 0.0f) atomicAdd(reinterpret_cast<float*>(p.ws + L.colsumX) + j, cs);
    }
    // the last CTA of this matrix turns the sums into the bounds the next phase needs;
    // every thread fences its own (fire-and-forget) sum atomics before the count
    __threadfence();
    __syncthreads();
    if (t == 0) {
      const uint32_t units = (uint32_t)(p.prefix[mi + 1] - p.prefix[mi]);
      s_last = (atomicAdd(&st->done[0], 1u) == units - 1u);
    }
    __syncthreads();
    if (s_last) {
      __threadfence();
      const float ur = drain_max(reinterpret_cast<float*>(p.ws + L.rowsumX), d.mp, red);
      const float uc = drain_max(reinterpret_cast<float*>(p.ws + L.colsumX), d.np, red);
      if (t == 0) {
        st->u_rowX[0] = ur;
        st->u_colX[0] = uc;
        st->sg[kSgA + 0] = pow2_tensor_scale(ur * kBoundInflate);
        st->done[0] = 0u;
      }
    }
    __syncthreads();
  }
}

int grid_for(int64_t units, int num_sms, int per_sm) {
  const int64_t cap = (int64_t)num_sms * per_sm;
  return (int)(units < cap ? (units > 0 ? units : 1) : cap);
}

}  // namespace

cudaError_t launch_quantize(const float* x, int64_t rows, int64_t cols, int64_t ld, int axis,
                            uint8_t* codes, uint8_t* scales, float* s_g, uint32_t flags,
                            uint8_t* ws, cudaStream_t st, int num_sms) {
  cudaError_t e = cudaMemsetAsync(ws, 0, 8, st);
  if (e != cudaSuccess) return e;
  uint32_t* hdr = reinterpret_cast<uint32_t*>(ws);
  amax_kernel<<<grid_for(rows, num_sms, 8), kEwThreads, 0, st>>>(x, rows, cols, ld, hdr);
  const int64_t R = axis ? cols : rows, C = axis ? rows : cols;
  const int tiled = (flags & 2u) ? 1 : 0;
  const int64_t Rext = tiled ? align_up(R, 128) : align_up(R, kT);
  const int64_t Cp = align_up(C, 256);
  const int64_t Cext = tiled ? Cp : align_up(C, kT);
  const int64_t ntiles = (Rext / kT) * (Cext / kT);
  if (ntiles > 0x7FFFFFFF) return cudaErrorInvalidValue;
  quantize_kernel<<<(unsigned)ntiles, kEwThreads, 0, st>>>(x, ld, R, C, axis, tiled,
                                                          (flags & 1u) ? 1 : 0, Rext, Cext, Cp,
                                                          codes, scales, s_g, hdr);
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* scales, const float* s_g,
                              int64_t rows, int64_t cols, float* y, int64_t ld, uint32_t flags,
                              cudaStream_t st, int num_sms) {
  const int tiled = (flags & 2u) ? 1 : 0;
  const int64_t nblk = rows * (cols / 16);
  dequantize_kernel<<<grid_for((nblk + kEwThreads - 1) / kEwThreads, num_sms, 8), kEwThreads, 0,
                      st>>>(codes, scales, s_g, rows, cols, tiled, align_up(cols, 256), y, ld);
  return cudaGetLastError();
}

cudaError_t launch_ns_reduce(const NsParams& p, cudaStream_t st, int num_sms) {
  ns_reduce_kernel<<<grid_for(p.prefix[p.count], num_sms, 8), kEwThreads, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_ns_preamble(const NsParams& p, cudaStream_t st, int num_sms) {
  ns_preamble_kernel<<<grid_for(p.prefix[p.count], num_sms, 8), kEwThreads, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace fs4
