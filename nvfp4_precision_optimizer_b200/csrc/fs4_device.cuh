// Device-side building blocks of libfs4 (sm_100a): PTX wrappers for mbarriers,
// bulk copies and tcgen05, the TILED operand layout, and the 16-element NVFP4
// block quantiser used by every kernel that writes an NVFP4 view.
//
// NVFP4 block rule ("Full-Stack FP4", Section 2, paragraph "NVFP4 format",
// round-to-nearest per Section 3.4):
//   s      = RN_e4m3(fp32(amax_b / fp32(6 s_g)))      (saturating at 448)
//   code_i = sign_i | RN_e2m1(fp32(|x_i| / fp32(dec(s) s_g)))   (saturating at 6)
//   a block whose scale rounds to 0 gets all-zero codes.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace fs4 {

// ------------------------------------------------------------------ status word
// Device-detected conditions are OR-ed into a 32-bit status word in the workspace.
constexpr uint32_t kStatusNonFinite = 1u;
constexpr uint32_t kStatusTimeout = 2u;
// Bounded waits give up after this many nanoseconds of %globaltimer.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------------ TILED layout
// Operand layout of a row-blocked NVFP4 matrix with Rp rows (multiple of 128)
// and Cp columns (multiple of 256): 16 KB tiles of 128 rows x 256 elements in
// the 128-byte-swizzled K-major form the tensor core reads, and 512-byte scale
// atoms of 128 rows x 4 column blocks in the form tcgen05.cp copies to TMEM.
constexpr int kTileRows = 128;
constexpr int kTileK = 256;
constexpr int kTileBytes = kTileRows * kTileK / 2;  // 16384
constexpr int kAtomBytes = 512;

// Byte offset of the 16-byte chunk that holds columns [c, c+32) of row r (c % 32 == 0).
__host__ __device__ __forceinline__ int64_t tiled_chunk_offset(int64_t r, int64_t c, int64_t Cp) {
  const int64_t tile = (r >> 7) * (Cp >> 8) + (c >> 8);
  const int64_t rr = r & 127;
  const int64_t j = (c & 255) >> 5;
  return tile * kTileBytes + rr * 128 + ((j ^ (rr & 7)) << 4);
}

// The same TILED layout for BF16 operands (the BF16 comparison step): 16 KB tiles of
// 128 rows x 64 elements (128-byte rows, chunk j of row r at chunk position j ^ (r % 8)).
// Byte offset of the 16-byte chunk that holds columns [c, c+8) of row r (c % 8 == 0).
__host__ __device__ __forceinline__ int64_t tiled_chunk_offset_bf16(int64_t r, int64_t c, int64_t Cp) {
  const int64_t tile = (r >> 7) * (Cp >> 6) + (c >> 6);
  const int64_t rr = r & 127;
  const int64_t j = (c & 63) >> 3;
  return tile * kTileBytes + rr * 128 + ((j ^ (rr & 7)) << 4);
}

// Two FP32 values rounded to BF16 (round to nearest, ties to even), the first in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Byte offset of the scale of row r, column block kb = c / 16.
__host__ __device__ __forceinline__ int64_t tiled_scale_offset(int64_t r, int64_t kb, int64_t Cp) {
  const int64_t atom = (r >> 7) * (Cp >> 6) + (kb >> 2);
  return atom * kAtomBytes + 16 * (r & 31) + 4 * ((r & 127) >> 5) + (kb & 3);
}

// ------------------------------------------------------------------ conversions
__device__ __forceinline__ uint32_t f32_to_e4m3(float v) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
  return r & 0xFFu;
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t byte) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)byte));
  return __half2float(__ushort_as_half((uint16_t)(h2 & 0xFFFFu)));
}

// Eight FP32 values -> eight E2M1 codes packed low nibble first (RN, satfinite).
__device__ __forceinline__ uint32_t pack8_e2m1(float q0, float q1, float q2, float q3, float q4,
                                               float q5, float q6, float q7) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(q0), "f"(q1), "f"(q2), "f"(q3), "f"(q4), "f"(q5), "f"(q6), "f"(q7));
  return out;
}

// The two FP16 halves of a 32-bit register as FP32.
__device__ __forceinline__ float half_lo(uint32_t h2) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}
__device__ __forceinline__ float half_hi(uint32_t h2) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 >> 16)));
}

// 4 x the sum of the squared E2M1 values of the eight codes in `w`, in integer
// arithmetic: byte permutes look up (2 v)^2 in {0, 1, 4, 9, 16, 36, 64, 144} for
// each code magnitude (sign bits masked off) and dp4a adds the bytes.
__device__ __forceinline__ uint32_t sq4_e2m1_sum8(uint32_t w) {
  constexpr uint32_t kLutLo = 0x09040100u;   // codes 0..3: 0, 1, 4, 9
  constexpr uint32_t kLutHi = 0x90402410u;   // codes 4..7: 16, 36, 64, 144
  const uint32_t lo = __byte_perm(kLutLo, kLutHi, w & 0x7777u);
  const uint32_t hi = __byte_perm(kLutLo, kLutHi, (w >> 16) & 0x7777u);
  return __dp4a(lo, 0x01010101u, __dp4a(hi, 0x01010101u, 0u));
}

// ------------------------------------------------------------------ tensor scale
// Smallest power of two s_g with 2688 * s_g >= u, exponent clamped to [-116, 118];
// 1 for u == 0.  Exact: 2688 = 1.3125 * 2^11, so compare u's mantissa with 1.3125.
// for46 (adaptive 4/6 block scaling): the denominator is 1792 = 4 * 448 = 1.75 * 2^10,
// so that the M = 4 candidate's block scale cannot saturate either.
__host__ __device__ __forceinline__ float pow2_tensor_scale(float u, bool for46 = false) {
  if (!(u > 0.0f)) return 1.0f;
  uint32_t bits;
#ifdef __CUDA_ARCH__
  bits = __float_as_uint(u);
#else
  __builtin_memcpy(&bits, &u, 4);
#endif
  int e;
  if ((bits >> 23) == 0) {
    e = -126 - 11;  // subnormal u: far below the clamp
  } else {
    const int eu = (int)(bits >> 23) - 127;
    const uint32_t mant = bits & 0x7FFFFFu;
    if (for46) e = (mant <= 0x600000u) ? eu - 10 : eu - 9;
    else e = (mant <= 0x280000u) ? eu - 11 : eu - 10;
  }
  e = e < -116 ? -116 : (e > 118 ? 118 : e);
  uint32_t out = (uint32_t)(e + 127) << 23;
  float f;
#ifdef __CUDA_ARCH__
  f = __uint_as_float(out);
#else
  __builtin_memcpy(&f, &out, 4);
#endif
  return f;
}

// ------------------------------------------------------------------ block quantiser
// max(|a|, |b|, |c|) in one instruction (sm_100's three-input max with .abs); NaN
// operands are ignored as by fmaxf.
__device__ __forceinline__ float absmax3(float a, float b, float c) {
  float r;
  asm("max.abs.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
// max |x_i| of a 16-element block: a three-level tree of three-input maxima.
__device__ __forceinline__ float absmax16(const float* x) {
  const float m0 = absmax3(x[0], x[1], x[2]), m1 = absmax3(x[3], x[4], x[5]);
  const float m2 = absmax3(x[6], x[7], x[8]), m3 = absmax3(x[9], x[10], x[11]);
  const float m4 = absmax3(x[12], x[13], x[14]);
  return fmaxf(absmax3(m0, m1, m2), absmax3(m3, m4, x[15]));
}

struct QBlock16 {
  uint32_t w0, w1;   // 16 codes, element 0 in the low nibble of w0
  uint32_t scale;    // E4M3 byte
  float sumsq;       // sum of the squared dequantised values
  float amax;        // max |x| of the block
};

// Correctly rounded x / d from rcp = RN(1/d), by Markstein's FMA correction: the
// residual x - q0 d of q0 = RN(x rcp) is exact and q0 + residual * rcp rounds to
// RN(x / d).  Used where d has one of the eight 4-bit mantissas of an E4M3 value
// times a power of two (decoded block scales and 6 s_g for a power-of-two s_g),
// for which the identity is checked exhaustively, and |x / d| stays far from
// the FP32 underflow and overflow ranges.
__device__ __forceinline__ float div_rn_fma(float x, float d, float rcp) {
  const float q0 = x * rcp;
  return fmaf(fmaf(-q0, d, x), rcp, q0);
}

// Per-CTA table of the positive E4M3 block scales: tab[b] = {value of byte b,
// RN(1 / value)} for b = 1..126 (tab[0] and tab[127] unused).  With a
// power-of-two tensor scale s_g = 2^k the decoded scale is den = value * 2^k and
// RN(1 / den) = RN(1 / value) * 2^-k exactly, because the product stays a normal
// number for every block scale reachable from a tensor scale of the form chosen by
// pow2_tensor_scale (den <= 2^125.5, so 1 / den >= 2^-125.5).
// Decoded E4M3 block scales and their reciprocals, looked up by scale byte: tab[b] is
// the value of byte b and tab[128 + b] = RN(1 / value), 256 floats in shared memory.
// Two float arrays rather than one of float2: lanes with different bytes then share a
// bank only when the bytes differ by a multiple of 32 (scales 16x apart), where
// 8-byte entries collide already at bytes 16 apart (scales 4x apart).
struct ScaleTab {
  const float* tab;    // 256 floats in shared memory
  float rcp_sg;        // 1 / s_g, exact
};

// Fill entry b (0 <= b < 128) of a scale table.
__device__ __forceinline__ void scale_tab_fill(float* tab, uint32_t b) {
  float v = 0.0f, r = 0.0f;
  if (b != 0u && b < 127u) {
    v = e4m3_to_f32(b);
    r = __frcp_rn(v);
  }
  tab[b] = v;
  tab[128u + b] = r;
}

// ------------------------------------------------------------------ packed FP32 pairs
// sm_100 executes FP32 multiply and FMA on register pairs (f32x2); each lane of the
// pair is rounded exactly like the scalar instruction.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
// -RN(x / d) on a pair, by the same correction written for the negated quotient:
// nq0 = x * (-rcp) = -q0, r = x + d * nq0 = x - q0 d (exact), result nq0 - r * rcp.
// d2 = (d, d), nrcp = (-RN(1/d), -RN(1/d)).  A zero residual is +0, so the correction
// never changes a zero quotient, whose sign is the opposite of x's (-(+0) for x = +0
// and +0 for x = -0).
__device__ __forceinline__ uint64_t ndiv2_rn_fma(uint64_t x, uint64_t d2, uint64_t nrcp) {
  const uint64_t nq0 = f2_mul(x, nrcp);
  return f2_fma(f2_fma(nq0, d2, x), nrcp, nq0);
}

// Quantise 16 FP32 values with tensor scale s_g (six_sg = fp32(6 * s_g)).
// kPow2: s_g is a power of two and rcp_six = RN(1 / six_sg), so the block scale
// division may use the FMA-corrected form; otherwise IEEE division is used.
// With a table (kPow2 only) the decoded block scale and its reciprocal are looked up.
// ------------------------------------------------------------------ random Hadamard transform
// x <- x H16^r on one 16-element block, H16^r = D H16 / 4 ("Full-Stack FP4", Section 3.4):
// bit i of `mask` negates element i, then the in-place butterfly with strides 1, 2, 4, 8
// ((u, v) -> (u + v, u - v), FP32 round-to-nearest per addition), then the exact * 0.25.
__device__ __forceinline__ void rht16(float* x, uint32_t mask) {
#pragma unroll
  for (int i = 0; i < 16; ++i) x[i] = __uint_as_float(__float_as_uint(x[i]) ^ (((mask >> i) & 1u) << 31));
#pragma unroll
  for (int h = 1; h < 16; h *= 2) {
#pragma unroll
    for (int i = 0; i < 16; i += 2 * h) {
#pragma unroll
      for (int j = i; j < i + h; ++j) {
        const float u = x[j], v = x[j + h];
        x[j] = __fadd_rn(u, v);
        x[j + h] = __fsub_rn(u, v);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) x[i] = __fmul_rn(x[i], 0.25f);
}

// The two E2M1 values (signed) of one code byte as an f16x2: the low nibble in the low
// half.  The byte is handed to the conversion through its own 8-bit register, taken
// from a 32-bit value with cvt, so no vector unpacking of a packed word is involved.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
  uint32_t h;
  asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(h) : "r"(byte));
  return h;
}

// The 8 E2M1 values (signed) of one packed word as 4 f16x2: element 2i in the low
// half of h[i] (byte i of w, low nibble first).
__device__ __forceinline__ void e2m1_decode8(uint32_t w, uint32_t* h) {
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = e2m1x2_to_f16x2((w >> (8 * i)) & 0xFFu);
}

// The 16 E2M1 values (signed, as FP32) of a block's packed codes.
__device__ __forceinline__ void e2m1_decode16(uint32_t w0, uint32_t w1, float* v) {
  uint32_t h[8];
  e2m1_decode8(w0, h);
  e2m1_decode8(w1, h + 4);
#pragma unroll
  for (int b = 0; b < 8; ++b) {
    v[2 * b] = half_lo(h[b]);
    v[2 * b + 1] = half_hi(h[b]);
  }
}

// sum_i (x_i - code_i * den)^2 in FP32, one rounding per operation, in element order.
__device__ __forceinline__ float block_sq_error(const float* x, uint32_t w0, uint32_t w1, float den) {
  float v[16];
  e2m1_decode16(w0, w1, v);
  float err = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float d = __fsub_rn(x[i], __fmul_rn(v[i], den));
    err = __fadd_rn(err, __fmul_rn(d, d));
  }
  return err;
}

// kPacked: divide in f32x2 pairs (fewer instructions; the same roundings).
// k46: adaptive 4/6 block scaling (Section 3.4): the block is also quantised with
// its amax mapped to 4 (scale RN_e4m3(amax / (4 s_g)); 4 s_g is a power of two, so
// that division is exact) and keeps that candidate only when its squared error is
// strictly smaller.  Requires kPow2.
template <bool kPow2, bool kTab = false, bool kPacked = true, bool k46 = false>
__device__ __forceinline__ QBlock16 quantize16(const float* x, float s_g, float six_sg, float rcp_six,
                                               ScaleTab st = ScaleTab{nullptr, 0.0f}) {
  static_assert(kPow2 || !k46, "adaptive 4/6 needs a power-of-two tensor scale");
  static_assert(kPow2 || !kTab, "the scale table needs a power-of-two tensor scale");
  const float amax = absmax16(x);
  // one candidate: block scale byte from the scaled amax, codes, den = value(scale) * s_g
  auto candidate = [&](float scaled_amax, QBlock16& r, float& den) {
    r.amax = amax;
    r.scale = f32_to_e4m3(scaled_amax);
    if (r.scale == 0u) {
      r.w0 = r.w1 = 0u;
      r.sumsq = 0.0f;
      den = 0.0f;
      return;
    }
    float rcp = 0.0f;
    if constexpr (kTab) {
      den = __fmul_rn(st.tab[r.scale], s_g);
      rcp = st.tab[128u + r.scale] * st.rcp_sg;
    } else {
      den = __fmul_rn(e4m3_to_f32(r.scale), s_g);
      if (kPow2) rcp = __frcp_rn(den);
    }
    float q[16];
    if constexpr (kPow2) {
      // the FMA-corrected quotient in negated form (ndiv2_rn_fma): a zero quotient then
      // carries the opposite of x's sign, so flipping every code's sign bit afterwards
      // gives each element x's sign, -0 included (the plain form turns x = -0 into +0)
      if constexpr (kPacked) {
        const uint64_t d2 = f2_pack(den, den), nrcp2 = f2_pack(-rcp, -rcp);
#pragma unroll
        for (int i = 0; i < 16; i += 2)
          f2_unpack(ndiv2_rn_fma(f2_pack(x[i], x[i + 1]), d2, nrcp2), q[i], q[i + 1]);
      } else {
        const float nrcp = -rcp;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float nq0 = x[i] * nrcp;
          q[i] = fmaf(fmaf(nq0, den, x[i]), nrcp, nq0);
        }
      }
      r.w0 = pack8_e2m1(q[0], q[1], q[2], q[3], q[4], q[5], q[6], q[7]) ^ 0x88888888u;
      r.w1 = pack8_e2m1(q[8], q[9], q[10], q[11], q[12], q[13], q[14], q[15]) ^ 0x88888888u;
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) q[i] = __fdiv_rn(x[i], den);
      r.w0 = pack8_e2m1(q[0], q[1], q[2], q[3], q[4], q[5], q[6], q[7]);
      r.w1 = pack8_e2m1(q[8], q[9], q[10], q[11], q[12], q[13], q[14], q[15]);
    }
    const float s4 = static_cast<float>(sq4_e2m1_sum8(r.w0) + sq4_e2m1_sum8(r.w1));
    r.sumsq = 0.25f * s4 * den * den;
  };
  QBlock16 r6;
  float den6;
  candidate(kPow2 ? div_rn_fma(amax, six_sg, rcp_six) : __fdiv_rn(amax, six_sg), r6, den6);
  if constexpr (k46) {
    QBlock16 r4;
    float den4;
    // amax / (4 s_g): a division by a power of two, exact as a product
    candidate(__fmul_rn(amax, __fmul_rn(0.25f, kTab ? st.rcp_sg : __frcp_rn(s_g))), r4, den4);
    const float e6 = block_sq_error(x, r6.w0, r6.w1, den6);
    const float e4 = block_sq_error(x, r4.w0, r4.w1, den4);
    if (e4 < e6) return r4;
  }
  return r6;
}

// ------------------------------------------------------------------ shared memory / mbarriers
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

// Test for completion of the phase with `parity`; if it is not complete the thread
// may be suspended (it stops issuing) until it completes or about kSuspendNs pass
// (which also bounds how late a waiter notices an abort).
constexpr uint32_t kSuspendNs = 20000u;
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity), "r"(kSuspendNs)
      : "memory");
  return ok != 0u;
}

// Wait for the phase with `parity` of `bar` to complete.  Gives up after
// kWaitLimitNs (or within about kSuspendNs of *abort being set), records the
// timeout in the status word and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* status,
                                          volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    if (*abort) return false;
    if (mbar_try_wait(bar, parity)) return true;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      atomicOr(status, kStatusTimeout);
      *abort = 1;
      return false;
    }
  }
}

// 1-D bulk copy global -> shared (TMA engine), completion signalled on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// The same copy with the destination and the barrier given as shared-memory addresses.
__device__ __forceinline__ void bulk_g2s_addr(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// ------------------------------------------------------------------ tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_addr(slot)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor, K-major operand in 128-byte swizzled rows
// (8-row groups 1024 bytes apart).  The start address must lie in a tile whose
// base is 1024-byte aligned; advancing it by 32 bytes moves 64 FP4 along K.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);     // start address
  d |= (uint64_t)1 << 16;                        // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024 >> 4) << 32;              // stride byte offset: 8 rows x 128 bytes
  d |= (uint64_t)1 << 46;                        // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;                        // 128-byte swizzle
  return d;
}

// Descriptor of a plain 32-row x 16-byte block (one scale atom) for tcgen05.cp.
__device__ __forceinline__ uint64_t sdesc_sf_atom(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)(128 >> 4) << 32;               // 8-row core matrices 128 bytes apart
  d |= (uint64_t)1 << 46;
  return d;                                      // no swizzle
}

// Instruction descriptor: kind::mxf4nvf4, E2M1 x E2M1, UE4M3 scales, K-major A and B,
// FP32 accumulate, M x N.
__host__ __device__ constexpr uint32_t idesc_mxf4nvf4(int M, int N) {
  return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Instruction descriptor: kind::f16 with BF16 A and B, FP32 accumulate, K-major A and B, M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D (TMEM) (+)= A(smem) * B(smem)^T, BF16 operands, FP32 accumulator; K = 16.
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Copy one 512-byte scale atom from shared memory into 4 TMEM columns at
// `taddr`, replicated to all four 32-lane quarters.
__device__ __forceinline__ void tc_copy_sf(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

// D (TMEM) (+)= A(smem) * B(smem)^T with per-16 UE4M3 scales from TMEM; K = 64.
__device__ __forceinline__ void tc_mma_nvf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], "
      "[%6], p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Arrive on `bar` once every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_addr(bar))
      : "memory");
}

// Load 32 consecutive 32-bit TMEM columns of this warp's 32 lanes.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Issue a load of 32 consecutive TMEM columns of this warp's 32 lanes; the
// registers are valid only after tmem_wait_ld32.
__device__ __forceinline__ void tmem_ld32_async(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

// Wait for this thread's outstanding TMEM loads.  The 32 registers are passed
// through the statement so that no use of them can be scheduled before the wait;
// call it (or tmem_ld_order) once per register group filled by tmem_ld32_async.
__device__ __forceinline__ void tmem_wait_ld32(uint32_t* r) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
        "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
        "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]),
        "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]),
        "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
      :
      : "memory");
}

// Order a further register group after a preceding tmem_wait_ld32 (no instruction).
__device__ __forceinline__ void tmem_ld_order(uint32_t* r) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]),
                 "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                 "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                 "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}

// Per-warpgroup register budget changes (all 128 threads of the warpgroup execute them).
template <uint32_t N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// Named barrier among `count` threads (id 1..15; id 0 is __syncthreads).
__device__ __forceinline__ void named_bar(uint32_t id, uint32_t count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

}  // namespace fs4
