// The standalone block-scaled NVFP4 GEMM D = deq(A) deq(B)^T (fs4_nvfp4_gemm) on
// the 5th-generation tensor cores (sm_100a).  The three products of the Newton-
// Schulz iteration, with their fused epilogues, are in gemm_ns.cu.
//
// "Full-Stack FP4" (arXiv 2607.04422), Section 2 "NVFP4 format": each operand is
// E2M1 values with an E4M3 scale per 16 elements along K and an FP32 tensor scale;
// the product of the dequantised operands is what every step of Section 3.4 takes.
//
// Kernel structure (one persistent CTA per SM, 384 threads = 3 warpgroups):
//   warp 0     producer: 1-D bulk copies (TMA engine) of pre-tiled operand tiles
//              and scale atoms into a 3-stage shared-memory ring
//   warp 1     allocates 512 TMEM columns; one thread copies the scale atoms to
//              TMEM (tcgen05.cp) and issues tcgen05.mma kind::mxf4nvf4
//              (M=128, N=256, K=64, UE4M3 per-16 scales), FP32 accumulator in TMEM
//   warps 4-11 epilogue: tcgen05.ld of the 128 x 256 accumulator into registers
//              (handed back to the MMA warp at once, so the next tile's MMAs
//              overlap this epilogue), scaling by s_a s_b and row-contiguous stores
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
// 12 warps: warpgroup 0 = producer (warp 0), MMA issuer (warp 1), two idle warps;
// warpgroups 1-2 = 8 epilogue warps.  Registers are rebalanced after launch:
// 384 threads x 168 = 40 x 128 (warpgroup 0) + 232 x 256 (epilogue warpgroups).
constexpr int kThreads = 384;
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
constexpr int kStages = 3;
constexpr int TRANS_FLOATS = 32 * 33;   // per-warp transpose buffer of the epilogue
constexpr int BAR_BYTES = 256;
constexpr int SMEM_BYTES = 1024 + kStages * STAGE_BYTES + 8 * TRANS_FLOATS * 4 + BAR_BYTES;
constexpr uint32_t kIdesc = idesc_mxf4nvf4(BM, BN);
static_assert(STAGE_BYTES % 1024 == 0, "stages must keep 1024-byte alignment");
static_assert(SMEM_BYTES <= 232448, "over the per-CTA shared-memory limit");
static_assert((2 * kStages + 3) * 8 + 12 <= BAR_BYTES, "barrier block too small");

// Work unit u: the 128 x 256 output tile (u / nJ, u % nJ); the last tile column may
// hold only 128 rows of B (b_half).
struct Job {
  int64_t row0, col0;
  int b_half;
};

__device__ __forceinline__ Job make_job(int32_t u, const GemmPlainArgs& g) {
  Job j;
  const int32_t nJ = (g.Np + BN - 1) / BN;
  const int32_t I = u / nJ;
  j.row0 = (int64_t)I * BM;
  j.col0 = (int64_t)(u - I * nJ) * BN;
  j.b_half = (j.col0 + 128 >= g.Np) ? 1 : 0;
  return j;
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

// Epilogue D = (sa sb) acc (one epilogue warp); tb is a 32 x 33 transpose buffer so
// that each store instruction writes one contiguous row segment.
__device__ __forceinline__ void epilogue_plain(const GemmPlainArgs& g, uint32_t tmem, uint64_t* acc_full,
                                               uint64_t* acc_empty, uint32_t* status,
                                               volatile int* abort_flag, float* tb, int quad,
                                               int ch, int lane, int32_t total) {
  uint32_t tl = 0;
  for (int32_t u = blockIdx.x; u < total; u += gridDim.x, ++tl) {
    const Job j = make_job(u, g);
    // one lane polls; the result is warp-uniform (the TMEM loads below are .sync.aligned)
    const bool ok = __shfl_sync(0xFFFFFFFFu,
                                lane == 0 ? (mbar_wait(acc_full, tl & 1u, status, abort_flag) ? 1 : 0) : 0,
                                0) != 0;
    __syncwarp();
    if (!ok) continue;
    const int64_t gr0 = j.row0 + 32 * quad;
    const float acc_scale = __ldg(g.a_sg) * __ldg(g.b_sg);
    tc_fence_after();
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
      float v[32], w[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(accr[c][e]) * acc_scale;
      warp_transpose(v, w, tb, lane);
      const int64_t col = j.col0 + 128 * ch + 32 * c + lane;
      if (col < g.N) {
        float* dcol = g.d + gr0 * g.ldd + col;
#pragma unroll
        for (int t = 0; t < 32; ++t)
          if (gr0 + t < g.M) dcol[t * g.ldd] = w[t];
      }
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1) nvfp4_gemm_kernel(const __grid_constant__ GemmPlainArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  float* epi_smem = reinterpret_cast<float*>(smem + kStages * STAGE_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * STAGE_BYTES + 8 * TRANS_FLOATS * 4);
  uint64_t* full = bars;                      // an operand stage landed
  uint64_t* empty = bars + kStages;           // the MMAs reading a stage finished
  uint64_t* acc_full = bars + 2 * kStages;
  uint64_t* acc_empty = acc_full + 1;         // the epilogue warps drained the accumulator
  uint64_t* mma_done = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);

  uint32_t* status = g.status;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t first = blockIdx.x, step = gridDim.x;
  const int32_t total = (g.Mp / BM) * ((g.Np + BN - 1) / BN);
  const int32_t kt_total = g.Kp / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 8);
    mbar_init(mma_done, 1);
    *abort_flag = (__ldcg(status) & kStatusTimeout) ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp < 4) {
    regs_dec<kRegsCtl>();
    if (warp == 0) {
      // ------------------------------------------------------------ producer
      if (lane == 0) {
        uint32_t it = 0;
        for (int32_t u = first; u < total && !*abort_flag; u += step) {
          const Job j = make_job(u, g);
          const int64_t a_row = j.row0 / 128, b_row = j.col0 / 128;
          for (int kt = 0; kt < kt_total; ++kt, ++it) {
            const uint32_t s = it % kStages, use = it / kStages;
            if (!mbar_wait(&empty[s], (use & 1u) ^ 1u, status, abort_flag)) break;
            uint8_t* st = stage_base + s * STAGE_BYTES;
            uint8_t* st_b = st + A_BYTES;
            uint8_t* st_sfa = st_b + B_BYTES;
            uint8_t* st_sfb = st_sfa + SFA_BYTES;
            const int64_t at = a_row * kt_total + kt;
            const uint32_t bbytes = j.b_half ? (B_BYTES + SFB_BYTES) / 2 : (B_BYTES + SFB_BYTES);
            mbar_arrive_expect_tx(&full[s], A_BYTES + SFA_BYTES + bbytes);
            bulk_g2s(st, g.a_codes + at * kTileBytes, A_BYTES, &full[s]);
            bulk_g2s(st_sfa, g.a_scales + at * (4 * kAtomBytes), SFA_BYTES, &full[s]);
            for (int h = 0; h < (j.b_half ? 1 : 2); ++h) {
              const int64_t bt = (b_row + h) * kt_total + kt;
              bulk_g2s(st_b + h * kTileBytes, g.b_codes + bt * kTileBytes, kTileBytes, &full[s]);
              bulk_g2s(st_sfb + h * (4 * kAtomBytes), g.b_scales + bt * (4 * kAtomBytes), 4 * kAtomBytes,
                       &full[s]);
            }
          }
        }
        // drain: every issued copy must land before the CTA may exit
        const uint32_t from = it > (uint32_t)kStages ? it - kStages : 0u;
        for (uint32_t k = from; k < it; ++k) {
          volatile int never = 0;
          mbar_wait(&full[k % kStages], (k / kStages) & 1u, status, &never);
        }
      }
    } else if (warp == 1) {
      if (lane == 0) {
        // ---------------------------------------------------------- MMA issuer
        uint32_t it = 0, tl = 0;
        const uint32_t acc = tmem;   // lane 0, column 0
        for (int32_t u = first; u < total && !*abort_flag; u += step, ++tl) {
          if (!mbar_wait(acc_empty, (tl & 1u) ^ 1u, status, abort_flag)) break;
          tc_fence_after();
          bool ok = true;
          for (int kt = 0; kt < kt_total; ++kt, ++it) {
            const uint32_t s = it % kStages, use = it / kStages;
            if (!mbar_wait(&full[s], use & 1u, status, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint8_t* st = stage_base + s * STAGE_BYTES;
            const uint32_t sa = smem_addr(st), sb = sa + A_BYTES;
            const uint32_t ssfa = sb + B_BYTES, ssfb = ssfa + SFA_BYTES;
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
    }
  } else {
    regs_inc<kRegsEpi>();
    // ------------------------------------------------------------ epilogue
    // Every epilogue warp walks the same tile list and never leaves it early (a
    // failed wait only skips that tile's work), so the block-wide barrier at the
    // end is reached by all threads.
    const int ew = warp - 4;          // 0..7
    const int quad = warp & 3;        // TMEM lanes 32*quad .. 32*quad+31
    const int ch = ew >> 2;           // column half of the 256-wide tile
    epilogue_plain(g, tmem, acc_full, acc_empty, status, abort_flag, epi_smem + ew * TRANS_FLOATS, quad,
                   ch, lane, total);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_gemm_plain(const GemmPlainArgs& a, cudaStream_t st, int num_sms) {
  static unsigned long long attr_set = 0ull;   // one bit per device; a benign race
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(attr_set & (1ull << dev))) {
    e = cudaFuncSetAttribute(nvfp4_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set |= 1ull << dev;
  }
  // setmaxnreg.inc can only hand out what the block was launched with: refuse to
  // launch unless the compiled register count is exactly the split's budget
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, nvfp4_gemm_kernel);
  if (e != cudaSuccess) return e;
  if ((uint32_t)fa.numRegs != kRegsLaunch) return cudaErrorInvalidConfiguration;
  const int64_t units = (int64_t)(a.Mp / BM) * ((a.Np + BN - 1) / BN);
  const int grid = (int)(units < num_sms ? (units > 0 ? units : 1) : num_sms);
  nvfp4_gemm_kernel<<<grid, kThreads, SMEM_BYTES, st>>>(a);
  return cudaGetLastError();
}

}  // namespace fs4
