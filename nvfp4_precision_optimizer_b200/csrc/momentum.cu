// NVFP4 storage of the first moment (momentum) of Q-Root (sm_100a).
//
// "Full-Stack FP4" (arXiv 2607.04422), Section 3.3 "Quantized-State AdamW": the first
// moment is stored after Hadamard mixing with stochastic rounding (SR) and adaptive 4/6
// quantisation; Section 3.4: Q-Root's first-order momentum follows that recipe.
//
// One step, per 16-element block of a row of the m x n momentum:
//   m_prev = deq(previous state) (H16^r_prev)^-1          (zero without a previous state)
//   m_t    = fp32(fp32(beta m_prev) + fp32(fp32(1 - beta) g))
//   y      = m_t H16^r                                      (FP32 butterfly)
//   state  = Q(y): tensor scale by the 1792 rule over max |y|, block scale by adaptive
//            4/6, element codes rounded stochastically with u from SplitMix64.
// Two passes: the first forms m_t (written out if asked) and max |y|; the second forms
// them again (the same operations, so the same values) and quantises.
#include <cstdint>

#include "fs4_device.cuh"
#include "fs4_internal.h"

namespace fs4 {
namespace {

constexpr int kMoThreads = 256;

__device__ __forceinline__ float mo_block_max(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  if (threadIdx.x < 32) {
    v = threadIdx.x < kMoThreads / 32 ? red[threadIdx.x] : 0.0f;
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  }
  return v;
}

// SplitMix64 (Steele, Lea and Flood, OOPSLA 2014) at counter value i of a generator
// started at `seed`; u = its top 24 bits times 2^-24 (exact in FP32).
__device__ __forceinline__ float splitmix_u24(uint64_t seed, uint64_t i) {
  uint64_t z = seed + (i + 1ull) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  z ^= z >> 31;
  return (float)(uint32_t)(z >> 40) * (1.0f / 16777216.0f);
}

// Stochastic E2M1 rounding of v >= 0: the magnitude code lo or lo + 1 around v, up when
// u < (v - lo) / (hi - lo) (exact: v - lo is exact and hi - lo a power of two); v >= 6
// saturates to code 7.
__device__ __forceinline__ uint32_t sr_e2m1_code(float v, float u) {
  const uint32_t idx = (v >= 0.5f) + (v >= 1.0f) + (v >= 1.5f) + (v >= 2.0f) + (v >= 3.0f) +
                       (v >= 4.0f) + (v >= 6.0f);
  if (idx >= 7u) return 7u;
  // grid value and 1 / gap of bin idx: {0,.5,1,1.5,2,3,4} and {2,2,2,2,1,1,0.5}
  const float lo = idx < 4u ? 0.5f * (float)idx : (idx == 4u ? 2.0f : (idx == 5u ? 3.0f : 4.0f));
  const float inv_gap = idx < 4u ? 2.0f : (idx < 6u ? 1.0f : 0.5f);
  const float frac = __fmul_rn(__fsub_rn(v, lo), inv_gap);
  return idx + (u < frac ? 1u : 0u);
}

// One 4/6 candidate of a block with SR codes: block scale RN_e4m3(scaled_amax), den =
// fp32(value * s_g), codes sign | SR(fp32(|y| / den)).
__device__ __forceinline__ void sr_candidate(const float* y, const float* u, float scaled_amax,
                                             float s_g, uint32_t& w0, uint32_t& w1,
                                             uint32_t& scale, float& den) {
  scale = f32_to_e4m3(scaled_amax);
  w0 = w1 = 0u;
  den = 0.0f;
  if (scale == 0u) return;
  den = __fmul_rn(e4m3_to_f32(scale), s_g);
  const float rcp = __frcp_rn(den);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float v = div_rn_fma(fabsf(y[i]), den, rcp);
    const uint32_t code = sr_e2m1_code(v, u[i]) | ((__float_as_uint(y[i]) >> 31) << 3);
    if (i < 8) w0 |= code << (4 * i);
    else w1 |= code << (4 * (i - 8));
  }
}

struct MoArgs {
  const float* g;
  int64_t rows, cols, ld;
  float beta;
  const uint8_t* prev_codes;   // null: no previous state
  const uint8_t* prev_scales;
  const float* prev_sg;
  uint32_t prev_mask, mask;
  uint8_t* codes;
  uint8_t* scales;
  float* s_g;
  uint64_t seed;
  float* m_out;                // may be null
  int64_t ld_out;
  uint32_t* hdr;               // [0] status, [1] max |y| bits, [2] previous s_g bits
};

// m_t and y = m_t H16^r of block (r, c) (16 elements from column c).
__device__ __forceinline__ void mo_block(const MoArgs& a, float prev_sg, int64_t r, int64_t c,
                                         float* m, float* y, bool& bad) {
  const float* gp = a.g + r * a.ld + c;
  float g[16];
  if (((reinterpret_cast<uintptr_t>(gp) & 15) == 0)) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(gp) + q);
      g[4 * q] = v.x; g[4 * q + 1] = v.y; g[4 * q + 2] = v.z; g[4 * q + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) g[i] = __ldg(gp + i);
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) bad |= (__float_as_uint(g[i]) & 0x7F800000u) == 0x7F800000u;
  float mp[16];
  if (a.prev_codes) {
    const int64_t blk = r * (a.cols / 16) + c / 16;
    // coherent loads: an in-place step overwrites this block later in the same kernel
    const uint2 w = __ldcg(reinterpret_cast<const uint2*>(a.prev_codes) + blk);
    const float sb = e4m3_to_f32(__ldcg(a.prev_scales + blk));
    e2m1_decode16(w.x, w.y, mp);
#pragma unroll
    for (int i = 0; i < 16; ++i) mp[i] = __fmul_rn(__fmul_rn(mp[i], sb), prev_sg);
    // (H16^r)^-1 = H16 D / 4: the butterfly and * 0.25 (rht16 without signs), then D
    rht16(mp, 0u);
#pragma unroll
    for (int i = 0; i < 16; ++i)
      mp[i] = __uint_as_float(__float_as_uint(mp[i]) ^ (((a.prev_mask >> i) & 1u) << 31));
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) mp[i] = 0.0f;
  }
  const float omb = __fsub_rn(1.0f, a.beta);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    m[i] = __fadd_rn(__fmul_rn(a.beta, mp[i]), __fmul_rn(omb, g[i]));
    y[i] = m[i];
  }
  rht16(y, a.mask);
}

__global__ void __launch_bounds__(kMoThreads, 4) momentum_pass1_kernel(const __grid_constant__ MoArgs a) {
  __shared__ float red[kMoThreads / 32];
  const float prev_sg = a.prev_codes ? __ldcg(a.prev_sg) : 0.0f;
  if (blockIdx.x == 0 && threadIdx.x == 0) a.hdr[2] = __float_as_uint(prev_sg);
  const int64_t nblk = a.rows * (a.cols / 16);
  float mx = 0.0f;
  bool bad = false;
  for (int64_t b = blockIdx.x * (int64_t)kMoThreads + threadIdx.x; b < nblk;
       b += (int64_t)gridDim.x * kMoThreads) {
    const int64_t r = b / (a.cols / 16), c = (b % (a.cols / 16)) * 16;
    float m[16], y[16];
    mo_block(a, prev_sg, r, c, m, y, bad);
    if (a.m_out) {
      float* op = a.m_out + r * a.ld_out + c;
      if ((reinterpret_cast<uintptr_t>(op) & 15) == 0) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
          reinterpret_cast<float4*>(op)[q] = make_float4(m[4 * q], m[4 * q + 1], m[4 * q + 2], m[4 * q + 3]);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) op[i] = m[i];
      }
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) mx = fmaxf(mx, fabsf(y[i]));
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(&a.hdr[0], kStatusNonFinite);
  mx = mo_block_max(mx, red);
  if (threadIdx.x == 0) atomicMax(&a.hdr[1], __float_as_uint(mx));
}

__global__ void __launch_bounds__(kMoThreads, 4) momentum_pass2_kernel(const __grid_constant__ MoArgs a) {
  const float prev_sg = __uint_as_float(__ldcg(&a.hdr[2]));
  const float s_g = pow2_tensor_scale(__uint_as_float(__ldcg(&a.hdr[1])), true);
  if (blockIdx.x == 0 && threadIdx.x == 0) *a.s_g = s_g;
  const float six_sg = __fmul_rn(6.0f, s_g);
  const float rcp_six = __frcp_rn(six_sg);
  const float quarter_rcp_sg = __fmul_rn(0.25f, __frcp_rn(s_g));   // 1 / (4 s_g), exact
  const int64_t nblk = a.rows * (a.cols / 16);
  for (int64_t b = blockIdx.x * (int64_t)kMoThreads + threadIdx.x; b < nblk;
       b += (int64_t)gridDim.x * kMoThreads) {
    const int64_t r = b / (a.cols / 16), c = (b % (a.cols / 16)) * 16;
    float m[16], y[16], u[16];
    bool bad = false;
    mo_block(a, prev_sg, r, c, m, y, bad);
    const uint64_t i0 = (uint64_t)r * (uint64_t)a.cols + (uint64_t)c;
#pragma unroll
    for (int i = 0; i < 16; ++i) u[i] = splitmix_u24(a.seed, i0 + i);
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(y[i]));
    uint32_t w6a, w6b, s6, w4a, w4b, s4;
    float d6, d4;
    sr_candidate(y, u, div_rn_fma(amax, six_sg, rcp_six), s_g, w6a, w6b, s6, d6);
    sr_candidate(y, u, __fmul_rn(amax, quarter_rcp_sg), s_g, w4a, w4b, s4, d4);
    const bool use4 = block_sq_error(y, w4a, w4b, d4) < block_sq_error(y, w6a, w6b, d6);
    reinterpret_cast<uint2*>(a.codes)[b] = use4 ? make_uint2(w4a, w4b) : make_uint2(w6a, w6b);
    a.scales[b] = static_cast<uint8_t>(use4 ? s4 : s6);
  }
}

int mo_grid(int64_t nblk, int num_sms) {
  const int64_t want = (nblk + kMoThreads - 1) / kMoThreads;
  const int64_t cap = (int64_t)num_sms * 8;
  return (int)(want < 1 ? 1 : (want < cap ? want : cap));
}

}  // namespace

cudaError_t launch_momentum(const float* g, int64_t rows, int64_t cols, int64_t ld, float beta,
                            const uint8_t* prev_codes, const uint8_t* prev_scales,
                            const float* prev_sg, uint32_t prev_mask, uint8_t* codes,
                            uint8_t* scales, float* s_g, uint32_t mask, uint64_t seed,
                            float* m_out, int64_t ld_out, uint8_t* ws, cudaStream_t st,
                            int num_sms) {
  cudaError_t e = cudaMemsetAsync(ws, 0, 12, st);
  if (e != cudaSuccess) return e;
  MoArgs a;
  a.g = g; a.rows = rows; a.cols = cols; a.ld = ld; a.beta = beta;
  a.prev_codes = prev_codes; a.prev_scales = prev_scales; a.prev_sg = prev_sg;
  a.prev_mask = prev_mask; a.mask = mask;
  a.codes = codes; a.scales = scales; a.s_g = s_g; a.seed = seed;
  a.m_out = m_out; a.ld_out = ld_out;
  a.hdr = reinterpret_cast<uint32_t*>(ws);
  const int grid = mo_grid(rows * (cols / 16), num_sms);
  momentum_pass1_kernel<<<grid, kMoThreads, 0, st>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  momentum_pass2_kernel<<<grid, kMoThreads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace fs4
