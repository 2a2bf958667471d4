// Block-scaled NVFP4 GEMMs on the 5th-generation tensor cores (sm_100a) with
// the fused epilogues of the direct NVFP4 Newton-Schulz iteration.
//
// "Full-Stack FP4" (arXiv 2607.04422), Section 3.4, one iteration:
//   G1  A   = qX qX^T                       epilogue: A (FP32), qA = Q1x16(A)
//   G2  P   = qA qA16x1,  B = b A + c P     epilogue: qB = Q1x16(B)
//   G3  X' = a X + qB qX16x1                epilogue: X' (FP32), Q1x16(X'), Q16x1(X')
// A and B are symmetric, so G1 and G2 compute only the 256 x 256 tiles on and
// above the diagonal; an off-diagonal tile also writes the transposed view,
// which is the mirrored tile's 1x16 quantisation (Q16x1(A) = Q1x16(A)^T).
//
// Kernel structure (one persistent CTA per SM, 384 threads = 3 warpgroups):
//   warp 0     producer: 1-D bulk copies (TMA engine) of pre-tiled operand tiles
//              and scale atoms into a 3-stage shared-memory ring
//   warp 1     allocates 512 TMEM columns; one thread copies the scale atoms to
//              TMEM (tcgen05.cp) and issues tcgen05.mma kind::mxf4nvf4
//              (M=128, N=256, K=64, UE4M3 per-16 scales), FP32 accumulator in TMEM
//   warp 2     tile counter: counts finished tiles per matrix and, in the CTA that
//              finishes a matrix, derives the next phase's tensor scale
//   warps 4-11 epilogue: tcgen05.ld of the 128 x 256 accumulator into registers
//              (the accumulator is handed back to the MMA warp at once, so the
//              next tile's MMAs overlap this epilogue), the fused element-wise
//              step, requantisation of the next operand, and the row/column sums
//              the next phase's tensor scales are bounded by
// setmaxnreg moves registers from warpgroup 0 (control, 40 per thread) to the
// two epilogue warpgroups (232 per thread).
// Every mbarrier wait is bounded (see mbar_wait); on a timeout the CTA stops
// issuing work, drains what it issued, frees TMEM and returns.
#include <cfloat>
#include <cmath>

#include "fs4_device.cuh"
#include "fs4_internal.h"

namespace fs4 {

namespace {

constexpr int BM = 128, BN = 256, BK = 256;
constexpr int kStages = 3;
// 12 warps: warpgroup 0 = producer (warp 0), MMA issuer (warp 1), two idle warps;
// warpgroups 1-2 = 8 epilogue warps.  Registers are rebalanced after launch:
// 384 threads x 168 = 40 x 128 (warpgroup 0) + 232 x 256 (epilogue warpgroups).
constexpr int kThreads = 384;
constexpr int kEpiThreads = 256;
constexpr int kEpiBase = 128;          // first epilogue thread
constexpr uint32_t kRegsLaunch = 168;
constexpr uint32_t kRegsCtl = 40;
constexpr uint32_t kRegsEpi = 232;
static_assert(kRegsCtl * 128 + kRegsEpi * 256 <= kRegsLaunch * kThreads, "register split over budget");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSfCol = 256;      // scale-factor columns follow the 256 accumulator columns
constexpr uint32_t kSfBufCols = 48;   // 16 (A: 4 k-steps x 4) + 32 (B: 4 k-steps x 8)
constexpr int A_BYTES = BM * BK / 2;
constexpr int B_BYTES = BN * BK / 2;
constexpr int SFA_BYTES = BM * BK / 16;
constexpr int SFB_BYTES = BN * BK / 16;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
constexpr int TRANS_FLOATS = 32 * 33;
constexpr int SMEM_BYTES = 1024 + kStages * STAGE_BYTES + 8 * TRANS_FLOATS * 4 + 256;
constexpr float kBoundInflate = 1.0f + 1.0f / 256.0f;
constexpr uint32_t kIdesc = idesc_mxf4nvf4(BM, BN);
static_assert(STAGE_BYTES % 1024 == 0, "stages must keep 1024-byte alignment");

struct Job {
  int mat;
  int64_t row0, col0;
  int mirror;        // off-diagonal symmetric tile
  int b_half;        // only the first 128 rows of the B tile exist
  int kt;            // number of 256-wide K tiles
  const uint8_t* a_codes; const uint8_t* a_sf;
  const uint8_t* b_codes; const uint8_t* b_sf;
  int64_t a_tile_row, b_tile_row;   // 128-row tile index of the A / B operand
  int64_t ktiles_total;             // K tiles per operand row band (Kp / 256)
};

__device__ __forceinline__ int owner_of(const int32_t* prefix, int count, int32_t u) {
  int lo = 0, hi = count - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= u) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Upper-triangle super tile s -> (P, Q), P <= Q, of a T x T grid, row-major.
__device__ __forceinline__ void upper_tile(int32_t s, int32_t T, int32_t& P, int32_t& Q) {
  P = 0;
  while (s >= T - P) { s -= T - P; ++P; }
  Q = P + s;
}

template <Epi E>
__device__ __forceinline__ Job make_job(int32_t u, const NsParams& p, const GemmPlainArgs& g) {
  Job j;
  j.mirror = 0;
  j.b_half = 0;
  if constexpr (E == Epi::Plain) {
    const int32_t nJ = (g.Np + BN - 1) / BN;
    const int32_t I = u / nJ;
    j.mat = 0;
    j.row0 = (int64_t)I * BM;
    j.col0 = (int64_t)(u - I * nJ) * BN;
    j.b_half = (j.col0 + 128 >= g.Np) ? 1 : 0;
    j.kt = g.Kp / BK;
    j.ktiles_total = g.Kp / BK;
    j.a_codes = g.a_codes; j.a_sf = g.a_scales;
    j.b_codes = g.b_codes; j.b_sf = g.b_scales;
  } else {
    const int mi = owner_of(p.prefix, p.count, u);
    const MatDesc& d = p.mat[mi];
    const MatLayout L = mat_layout(d.mp, d.np, d.state_off, d.big_off);
    const int32_t lu = u - p.prefix[mi];
    const int slot = p.iter & 1;
    j.mat = mi;
    if constexpr (E == Epi::GramX || E == Epi::GramA) {
      const int32_t T = d.mp / 256;
      int32_t P, Q;
      upper_tile(lu >> 1, T, P, Q);
      j.row0 = 256 * (int64_t)P + 128 * (lu & 1);
      j.col0 = 256 * (int64_t)Q;
      j.mirror = (P != Q) ? 1 : 0;
      if constexpr (E == Epi::GramX) {
        j.kt = d.np / BK;
        j.a_codes = j.b_codes = p.ws + (slot ? L.qX[1] : L.qX[0]);
        j.a_sf = j.b_sf = p.ws + (slot ? L.sX[1] : L.sX[0]);
      } else {
        j.kt = d.mp / BK;
        j.a_codes = j.b_codes = p.ws + L.qA;
        j.a_sf = j.b_sf = p.ws + L.sA;
      }
    } else {
      const int32_t nJ = d.np / BN;
      const int32_t I = lu / nJ;
      j.row0 = (int64_t)I * BM;
      j.col0 = (int64_t)(lu - I * nJ) * BN;
      j.kt = d.mp / BK;
      j.a_codes = p.ws + L.qB; j.a_sf = p.ws + L.sB;
      j.b_codes = p.ws + (slot ? L.qXT[1] : L.qXT[0]);
      j.b_sf = p.ws + (slot ? L.sXT[1] : L.sXT[0]);
    }
    j.ktiles_total = j.kt;
  }
  j.a_tile_row = j.row0 / 128;
  j.b_tile_row = j.col0 / 128;
  return j;
}

template <Epi E>
__device__ __forceinline__ int32_t total_units(const NsParams& p, const GemmPlainArgs& g) {
  if constexpr (E == Epi::Plain) {
    return (g.Mp / BM) * ((g.Np + BN - 1) / BN);
  } else {
    return p.prefix[p.count];
  }
}

struct ChunkSums {
  float sumsq;   // sum of squared dequantised values of the 32 elements
  float amax;    // max |x| of the 32 elements
};

// 1x16 quantisation of 32 consecutive values of row r starting at column c (c % 32 == 0),
// power-of-two tensor scale sg (six = 6 sg, rcp_six = RN(1 / six)).
__device__ __forceinline__ ChunkSums store_row_chunk(const float* v, int64_t r, int64_t c, int64_t Cp,
                                                     uint8_t* codes, uint8_t* scales, float sg,
                                                     float six, float rcp_six) {
  const QBlock16 q0 = quantize16<true>(v, sg, six, rcp_six);
  const QBlock16 q1 = quantize16<true>(v + 16, sg, six, rcp_six);
  *reinterpret_cast<uint4*>(codes + tiled_chunk_offset(r, c, Cp)) =
      make_uint4(q0.w0, q0.w1, q1.w0, q1.w1);
  *reinterpret_cast<uint16_t*>(scales + tiled_scale_offset(r, c >> 4, Cp)) =
      static_cast<uint16_t>(q0.scale | (q1.scale << 8));
  return {q0.sumsq + q1.sumsq, fmaxf(q0.amax, q1.amax)};
}

// Transpose this warp's 32 x 32 chunk through shared memory: on return w[t]
// holds the value of row t of the chunk in this lane's column.
__device__ __forceinline__ void warp_transpose(const float* v, float* w, float* tb, int lane) {
#pragma unroll
  for (int j = 0; j < 32; ++j) tb[lane * 33 + j] = v[j];
  __syncwarp();
#pragma unroll
  for (int t = 0; t < 32; ++t) w[t] = tb[t * 33 + lane];
  __syncwarp();
}

// Read-and-clear max of a float vector in global memory by one warp (values >= 0):
// float4 loads, four in flight per lane.
__device__ __forceinline__ float warp_drain_max4(float* vec, int64_t len, int lane) {
  float m = 0.0f;
  float4* v4 = reinterpret_cast<float4*>(vec);
  const int64_t n4 = len >> 2;     // len is a multiple of 256
  for (int64_t base = 0; base < n4; base += 128) {
    float4 a[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int64_t i = base + k * 32 + lane;
      a[k] = i < n4 ? __ldcg(v4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int64_t i = base + k * 32 + lane;
      if (i < n4) __stcg(v4 + i, make_float4(0.f, 0.f, 0.f, 0.f));
      m = fmaxf(m, fmaxf(fmaxf(a[k].x, a[k].y), fmaxf(a[k].z, a[k].w)));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  return m;
}

// Count one finished tile of matrix mi; in the CTA that completes the matrix's
// tiles of this launch, derive the next tensor scale from the row/column sums.
template <Epi E>
__device__ __forceinline__ void finalize_tile(const NsParams& p, int mi, int lane) {
  if constexpr (E != Epi::Plain) {
    const MatDesc& d = p.mat[mi];
    NsState* st = reinterpret_cast<NsState*>(p.ws + d.state_off);
    constexpr int kind = (E == Epi::GramX) ? 1 : (E == Epi::GramA ? 2 : 3);
    int last = 0;
    if (lane == 0) {
      const uint32_t units = (uint32_t)(p.prefix[mi + 1] - p.prefix[mi]);
      last = (atomicAdd(&st->done[kind], 1u) == units - 1u) ? 1 : 0;
    }
    last = __shfl_sync(0xFFFFFFFFu, last, 0);
    if (!last) return;
    __threadfence();
    const MatLayout L = mat_layout(d.mp, d.np, d.state_off, d.big_off);
    const int k = p.iter;
    if constexpr (E == Epi::GramX) {
      const float ua = warp_drain_max4(reinterpret_cast<float*>(p.ws + L.rowsumA), d.mp, lane);
      if (lane == 0) {
        st->u_rowA[k] = ua;
        const float ub = (fabsf(d.b) * __ldcg(&st->u_rowX[k]) + fabsf(d.c) * ua) * kBoundInflate;
        st->sg[kSgB + k] = pow2_tensor_scale(ub);
      }
    } else if constexpr (E == Epi::GramA) {
      const float ub = warp_drain_max4(reinterpret_cast<float*>(p.ws + L.rowsumB), d.mp, lane);
      if (lane == 0) {
        st->u_rowB[k] = ub;
        const float ax = __uint_as_float(__ldcg(&st->amaxX[k]));
        const float ux = (fabsf(d.a) * ax + sqrtf(ub * __ldcg(&st->u_colX[k]))) * kBoundInflate;
        st->sg[kSgX + k + 1] = pow2_tensor_scale(ux);
      }
    } else {
      const float ur = warp_drain_max4(reinterpret_cast<float*>(p.ws + L.rowsumX), d.mp, lane);
      const float uc = warp_drain_max4(reinterpret_cast<float*>(p.ws + L.colsumX), d.np, lane);
      if (lane == 0 && !p.last) {
        st->u_rowX[k + 1] = ur;
        st->u_colX[k + 1] = uc;
        st->sg[kSgA + k + 1] = pow2_tensor_scale(ur * kBoundInflate);
      }
    }
    if (lane == 0) st->done[kind] = 0u;
  }
}

template <Epi E>
__global__ void __launch_bounds__(kThreads, 1)
    nvfp4_gemm_kernel(const __grid_constant__ NsParams p, const __grid_constant__ GemmPlainArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  float* trans = reinterpret_cast<float*>(smem + kStages * STAGE_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * STAGE_BYTES + 8 * TRANS_FLOATS * 4);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* acc_full = bars + 2 * kStages;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* mma_done = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 3);
  uint32_t* arrivals = tmem_slot + 1;   // monotonic count of (epilogue warp, tile) completions
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);

  uint32_t* status = (E == Epi::Plain) ? g.status : p.status;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 8);
    mbar_init(mma_done, 1);
    *arrivals = 0u;
    *abort_flag = (__ldcg(status) & kStatusTimeout) ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int32_t total = total_units<E>(p, g);
  if (warp < 4) {
    regs_dec<kRegsCtl>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t it = 0;
      for (int32_t u = blockIdx.x; u < total && !*abort_flag; u += gridDim.x) {
        const Job j = make_job<E>(u, p, g);
        for (int kt = 0; kt < j.kt; ++kt, ++it) {
          const uint32_t s = it % kStages, use = it / kStages;
          if (!mbar_wait(&empty[s], (use & 1u) ^ 1u, status, abort_flag)) break;
          uint8_t* st = stage_base + s * STAGE_BYTES;
          const uint32_t bbytes = j.b_half ? (B_BYTES + SFB_BYTES) / 2 : (B_BYTES + SFB_BYTES);
          mbar_arrive_expect_tx(&full[s], A_BYTES + SFA_BYTES + bbytes);
          const int64_t at = j.a_tile_row * j.ktiles_total + kt;
          bulk_g2s(st, j.a_codes + at * kTileBytes, A_BYTES, &full[s]);
          bulk_g2s(st + A_BYTES + B_BYTES, j.a_sf + at * (4 * kAtomBytes), SFA_BYTES, &full[s]);
          for (int h = 0; h < (j.b_half ? 1 : 2); ++h) {
            const int64_t bt = (j.b_tile_row + h) * j.ktiles_total + kt;
            bulk_g2s(st + A_BYTES + h * kTileBytes, j.b_codes + bt * kTileBytes, kTileBytes, &full[s]);
            bulk_g2s(st + A_BYTES + B_BYTES + SFA_BYTES + h * (4 * kAtomBytes),
                     j.b_sf + bt * (4 * kAtomBytes), 4 * kAtomBytes, &full[s]);
          }
        }
      }
      // drain: every issued copy must land before the CTA may exit
      const uint32_t first = it > (uint32_t)kStages ? it - kStages : 0u;
      for (uint32_t k = first; k < it; ++k) {
        volatile int never = 0;
        mbar_wait(&full[k % kStages], (k / kStages) & 1u, status, &never);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, tl = 0;
      const uint32_t acc = tmem;   // lane 0, column 0
      for (int32_t u = blockIdx.x; u < total && !*abort_flag; u += gridDim.x, ++tl) {
        const Job j = make_job<E>(u, p, g);
        if (!mbar_wait(acc_empty, (tl & 1u) ^ 1u, status, abort_flag)) break;
        tc_fence_after();
        bool ok = true;
        for (int kt = 0; kt < j.kt; ++kt, ++it) {
          const uint32_t s = it % kStages, use = it / kStages;
          if (!mbar_wait(&full[s], use & 1u, status, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint8_t* st = stage_base + s * STAGE_BYTES;
          const uint32_t sa = smem_addr(st), sb = sa + A_BYTES;
          const uint32_t ssfa = sa + A_BYTES + B_BYTES, ssfb = ssfa + SFA_BYTES;
          const uint32_t sf = tmem + kSfCol + (it & 1u) * kSfBufCols;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            tc_copy_sf(sf + 4 * ks, sdesc_sf_atom(ssfa + ks * kAtomBytes));
            tc_copy_sf(sf + 16 + 8 * ks, sdesc_sf_atom(ssfb + ks * kAtomBytes));
            tc_copy_sf(sf + 16 + 8 * ks + 4, sdesc_sf_atom(ssfb + 4 * kAtomBytes + ks * kAtomBytes));
          }
          const uint64_t da = sdesc_sw128(sa), db = sdesc_sw128(sb);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            tc_mma_nvf4(acc, da + 2 * ks, db + 2 * ks, kIdesc, sf + 4 * ks, sf + 16 + 8 * ks,
                        (kt | ks) != 0 ? 1u : 0u);
          }
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(acc_full);
      }
      tc_commit(mma_done);
      volatile int never = 0;
      mbar_wait(mma_done, 0, status, &never);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ tile counter / finalizer
    // Trails the epilogue warps: once all eight have published tile tl's sums, count
    // the tile for its matrix; the CTA that finishes a matrix's last tile in this
    // launch turns the matrix's sums into the next tensor scale.  The epilogue warps
    // never wait for this warp.
    if constexpr (E != Epi::Plain) {
      uint32_t tl = 0;
      for (int32_t u = blockIdx.x; u < total; u += gridDim.x, ++tl) {
        const Job j = make_job<E>(u, p, g);
        const uint32_t target = 8u * (tl + 1u);
        bool seen = true;
        if (*reinterpret_cast<volatile uint32_t*>(arrivals) < target) {
          const uint64_t t0 = global_timer_ns();
          while (*reinterpret_cast<volatile uint32_t*>(arrivals) < target) {
            if (*abort_flag || global_timer_ns() - t0 > kWaitLimitNs) { seen = false; break; }
            __nanosleep(64);
          }
        }
        if (!seen) {
          if (lane == 0 && !*abort_flag) { atomicOr(status, kStatusTimeout); *abort_flag = 1; }
          break;
        }
        __threadfence();
        finalize_tile<E>(p, j.mat, lane);
      }
    }
  }
  } else {
    regs_inc<kRegsEpi>();
    // ------------------------------------------------------------ epilogue
    // Every epilogue warp walks the same tile list and never leaves it early (a
    // failed wait only skips that tile's work), so the block-wide barrier at the
    // end is reached by all threads.  Per tile, each warp fences its row/column
    // sum atomics and bumps the shared arrival counter that warp 2 trails.
    const int ew = warp - 4;          // 0..7
    const int quad = warp & 3;        // TMEM lanes 32*quad .. 32*quad+31
    const int ch = ew >> 2;           // column half of the 256-wide tile
    float* tb = trans + ew * TRANS_FLOATS;
    uint32_t tl = 0;
    for (int32_t u = blockIdx.x; u < total; u += gridDim.x, ++tl) {
      const Job j = make_job<E>(u, p, g);
      const bool ok = mbar_wait(acc_full, tl & 1u, status, abort_flag);
      const int64_t gr0 = j.row0 + 32 * quad;   // first row of this warp's band
      const int64_t gr = gr0 + lane;             // this lane's row

      // per-job constants
      float acc_scale, sg_out = 1.0f, six_out = 6.0f, rcp_six = 1.0f / 6.0f;
      float coef_a = 0.0f, coef_b = 0.0f, coef_c = 0.0f;
      const MatDesc* d = nullptr;
      NsState* st = nullptr;
      MatLayout L;
      const int k = p.iter;
      if constexpr (E == Epi::Plain) {
        acc_scale = __ldg(g.a_sg) * __ldg(g.b_sg);
      } else {
        d = &p.mat[j.mat];
        st = reinterpret_cast<NsState*>(p.ws + d->state_off);
        L = mat_layout(d->mp, d->np, d->state_off, d->big_off);
        coef_a = d->a; coef_b = d->b; coef_c = d->c;
        if constexpr (E == Epi::GramX) {
          const float sx = __ldcg(&st->sg[kSgX + k]);
          acc_scale = sx * sx;
          sg_out = __ldcg(&st->sg[kSgA + k]);
        } else if constexpr (E == Epi::GramA) {
          const float sa = __ldcg(&st->sg[kSgA + k]);
          acc_scale = sa * sa;
          sg_out = __ldcg(&st->sg[kSgB + k]);
        } else {
          acc_scale = __ldcg(&st->sg[kSgB + k]) * __ldcg(&st->sg[kSgX + k]);
          sg_out = p.last ? 1.0f : __ldcg(&st->sg[kSgX + k + 1]);
        }
        six_out = __fmul_rn(6.0f, sg_out);
        rcp_six = __frcp_rn(six_out);
      }

      float row_acc = 0.0f, amax = 0.0f;
      if (ok) {
        tc_fence_after();
        // drain this warp's 32 x 128 share of the accumulator into registers and hand
        // the accumulator back at once: the next tile's MMAs overlap this epilogue
        uint32_t accr[4][32];
        const uint32_t taddr = tmem + ((uint32_t)(32 * quad) << 16) + (uint32_t)(128 * ch);
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32_async(taddr + 32 * c, accr[c]);
        tmem_wait_ld32(accr[0]);
        tmem_ld_order(accr[1]);
        tmem_ld_order(accr[2]);
        tmem_ld_order(accr[3]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty);

#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int64_t gc = j.col0 + 128 * ch + 32 * c;
          float v[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(accr[c][e]) * acc_scale;

          // FP32 tiles are read and written after a per-warp transpose (lane = column,
          // w[t] = row gr0 + t): every warp access is then one contiguous 128-byte line.
          if constexpr (E == Epi::Plain) {
            float w[32];
            warp_transpose(v, w, tb, lane);
            const int64_t col = gc + lane;
            if (col < g.N) {
              float* dcol = g.d + gr0 * g.ldd + col;
#pragma unroll
              for (int t = 0; t < 32; ++t)
                if (gr0 + t < g.M) dcol[t * g.ldd] = w[t];
            }
          } else if constexpr (E == Epi::GramX) {
            row_acc += store_row_chunk(v, gr, gc, d->mp, p.ws + L.qA, p.ws + L.sA, sg_out, six_out, rcp_six).sumsq;
            float w[32];
            warp_transpose(v, w, tb, lane);
            float* Acol = reinterpret_cast<float*>(p.ws + L.A) + gr0 * d->mp + gc + lane;
#pragma unroll
            for (int t = 0; t < 32; ++t) Acol[t * d->mp] = w[t];
            if (j.mirror) {
              const float cs = store_row_chunk(w, gc + lane, gr0, d->mp, p.ws + L.qA, p.ws + L.sA,
                                               sg_out, six_out, rcp_six).sumsq;
              if (cs != 0.0f) atomicAdd(reinterpret_cast<float*>(p.ws + L.rowsumA) + gc + lane, cs);
            }
          } else if constexpr (E == Epi::GramA) {
            const float* Acol = reinterpret_cast<const float*>(p.ws + L.A) + gr0 * d->mp + gc + lane;
            float w[32], a_row[32];
#pragma unroll
            for (int t = 0; t < 32; ++t) w[t] = __ldcg(Acol + t * d->mp);
            warp_transpose(w, a_row, tb, lane);
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = fmaf(coef_b, a_row[e], coef_c * v[e]);
            row_acc += store_row_chunk(v, gr, gc, d->mp, p.ws + L.qB, p.ws + L.sB, sg_out, six_out, rcp_six).sumsq;
            if (j.mirror) {
              warp_transpose(v, w, tb, lane);
              const float cs = store_row_chunk(w, gc + lane, gr0, d->mp, p.ws + L.qB, p.ws + L.sB,
                                               sg_out, six_out, rcp_six).sumsq;
              if (cs != 0.0f) atomicAdd(reinterpret_cast<float*>(p.ws + L.rowsumB) + gc + lane, cs);
            }
          } else {  // Update
            float* Xcol = reinterpret_cast<float*>(p.ws + L.X) + gr0 * d->np + gc + lane;
            float w[32];
            warp_transpose(v, w, tb, lane);
#pragma unroll
            for (int t = 0; t < 32; ++t) w[t] = fmaf(coef_a, __ldcg(Xcol + t * d->np), w[t]);
            if (p.last) {
              if (!d->tall) {
                if (gc + lane < d->n) {
                  float* ocol = d->out + gr0 * d->ldo + gc + lane;
#pragma unroll
                  for (int t = 0; t < 32; ++t)
                    if (gr0 + t < d->m) ocol[t * d->ldo] = w[t];
                }
              } else {
                warp_transpose(w, v, tb, lane);
                if (gr < d->m) {
#pragma unroll
                  for (int e = 0; e < 32; ++e)
                    if (gc + e < d->n) d->out[(gc + e) * d->ldo + gr] = v[e];
                }
              }
            } else {
#pragma unroll
              for (int t = 0; t < 32; ++t) Xcol[t * d->np] = w[t];
              const int ns = (k + 1) & 1;
              const ChunkSums cs = store_row_chunk(w, gc + lane, gr0, d->mp,
                                                   p.ws + (ns ? L.qXT[1] : L.qXT[0]),
                                                   p.ws + (ns ? L.sXT[1] : L.sXT[0]), sg_out, six_out, rcp_six);
              amax = fmaxf(amax, cs.amax);
              if (cs.sumsq != 0.0f) atomicAdd(reinterpret_cast<float*>(p.ws + L.colsumX) + gc + lane, cs.sumsq);
              warp_transpose(w, v, tb, lane);
              row_acc += store_row_chunk(v, gr, gc, d->np, p.ws + (ns ? L.qX[1] : L.qX[0]),
                                         p.ws + (ns ? L.sX[1] : L.sX[0]), sg_out, six_out, rcp_six).sumsq;
            }
          }
        }
      }

      if constexpr (E != Epi::Plain) {
        float* rowsum = nullptr;
        if constexpr (E == Epi::GramX) rowsum = reinterpret_cast<float*>(p.ws + L.rowsumA);
        if constexpr (E == Epi::GramA) rowsum = reinterpret_cast<float*>(p.ws + L.rowsumB);
        if constexpr (E == Epi::Update) rowsum = reinterpret_cast<float*>(p.ws + L.rowsumX);
        if (row_acc != 0.0f) atomicAdd(rowsum + gr, row_acc);
        if constexpr (E == Epi::Update) {
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
          if (lane == 0 && !p.last && amax > 0.0f) atomicMax(&st->amaxX[k + 1], __float_as_uint(amax));
        }
        // publish this warp's sums for the counter warp (never waits)
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(arrivals, 1u);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <Epi E>
cudaError_t launch_impl(const NsParams* p, const GemmPlainArgs* g, int64_t units, cudaStream_t st,
                        int num_sms) {
  static unsigned long long attr_set = 0ull;   // one bit per device; a benign race
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(attr_set & (1ull << dev))) {
    e = cudaFuncSetAttribute(nvfp4_gemm_kernel<E>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set |= 1ull << dev;
  }
  // setmaxnreg.inc can only hand out what the block was launched with: refuse to
  // launch unless the compiled register count is exactly the split's budget
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, nvfp4_gemm_kernel<E>);
  if (e != cudaSuccess) return e;
  if ((uint32_t)fa.numRegs != kRegsLaunch) return cudaErrorInvalidConfiguration;
  const int grid = (int)(units < num_sms ? (units > 0 ? units : 1) : num_sms);
  static const NsParams zero_p{};
  static const GemmPlainArgs zero_g{};
  nvfp4_gemm_kernel<E><<<grid, kThreads, SMEM_BYTES, st>>>(p ? *p : zero_p, g ? *g : zero_g);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_plain(const GemmPlainArgs& a, cudaStream_t st, int num_sms) {
  const int64_t units = (int64_t)(a.Mp / BM) * ((a.Np + BN - 1) / BN);
  return launch_impl<Epi::Plain>(nullptr, &a, units, st, num_sms);
}

cudaError_t launch_gemm_ns(Epi epi, const NsParams& p, cudaStream_t st, int num_sms) {
  const int64_t units = p.prefix[p.count];
  switch (epi) {
    case Epi::GramX: return launch_impl<Epi::GramX>(&p, nullptr, units, st, num_sms);
    case Epi::GramA: return launch_impl<Epi::GramA>(&p, nullptr, units, st, num_sms);
    case Epi::Update: return launch_impl<Epi::Update>(&p, nullptr, units, st, num_sms);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace fs4
