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
//   warp 1     allocates 512 TMEM columns; one thread issues tcgen05.mma
//              kind::mxf4nvf4 (M=128, N=256, K=64, UE4M3 per-16 scales), FP32
//              accumulator in TMEM
//   warps 2-3  scale-factor copiers: one or two threads copy every stage's scale atoms
//              to TMEM (tcgen05.cp) into a ring of buffers (the update's MMA thread
//              copies its own)
//   (a one-CTA-per-matrix kernel after each launch turns the row/column sums
//    into the next phase's tensor scale)
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
#include <type_traits>

#include "fs4_device.cuh"
#include "fs4_internal.h"

namespace fs4 {

namespace {

constexpr int BM = 128, BN = 256, BK = 256;
// 12 warps: warpgroup 0 = producer (warp 0), MMA issuer (warp 1), scale copiers (2, 3);
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
constexpr int SFA_BYTES = BM * BK / 16;
constexpr int SFB_BYTES = BN * BK / 16;   // the scales of all BN rows of B, in either mode
constexpr int TRANS_FLOATS = 32 * 33;   // per-warp transpose buffer of the plain epilogue
// Each epilogue warp owns a 32 x 128 share of the 128 x 256 tile and walks it in
// chunks of 32 rows x 16 columns.  A chunk passes through a shared-memory stage
// where row r starts at float 16 (r + r / 16) and its four 16-byte quads sit at
// quad q ^ ((r / 2) % 4): one lane per row (the accumulator layout), one lane per
// (column, row half) (the 16x1 view) and four lanes per row (coalesced global
// traffic, rows r and r + 8 i) all hit 32 distinct banks.
constexpr int kChunkCols = 16;
constexpr int kChunks = 128 / kChunkCols;      // chunks per warp and tile
constexpr int kStageFloats = 33 * 16;           // one staged chunk (2112 bytes)
constexpr int kStageBufs = 3;                   // FP32 input runs two chunks ahead
constexpr int EPI_WARP_FLOATS = kStageBufs * kStageFloats;
static_assert(EPI_WARP_FLOATS >= TRANS_FLOATS, "the plain epilogue reuses the stage");
constexpr float kBoundInflate = 1.0f + 1.0f / 256.0f;

// Per-kernel configuration.  kBf16: the BF16 comparison step, whose operands are BF16
// tiles of the same 128-byte rows (64 elements of K per tile instead of 256) and carry
// no scale factors.
template <Epi E, bool kBf16 = false, bool kWide = false>
struct Cfg {
  static constexpr int kStages = 3;
  static constexpr int kTileK = kBf16 ? 64 : BK;              // K elements per stage
  static constexpr int B_BYTES = BN * 128;                    // 256 rows of 128 bytes
  static constexpr int SFA = kBf16 ? 0 : SFA_BYTES;
  static constexpr int SFB = kBf16 ? 0 : SFB_BYTES;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA + SFB;
  static constexpr int BAR_BYTES = 256;
  static constexpr int EPI_FLOATS = kStageBufs * kStageFloats;
  static constexpr int SMEM_BYTES =
      1024 + kStages * STAGE_BYTES + 8 * EPI_FLOATS * 4 + BAR_BYTES + 128 * 8;
  static constexpr uint32_t kIdesc = kBf16 ? idesc_bf16(BM, BN) : idesc_mxf4nvf4(BM, BN);
  // Scale-factor copies to TMEM (a ring of kSfBufs buffers).  A tcgen05.cp takes about 50
  // cycles to issue, so the twelve copies of a stage issued by the MMA thread take longer
  // than the stage's MMAs take to run: the first Gram product (and the plain GEMM), whose
  // time is set by the mainloop, leaves them to two copier threads (warps 2 and 3, six
  // atoms each).  Each waiting copier thread shares a scheduler with two epilogue warps,
  // and the products whose epilogue also streams an FP32 input measured best with fewer
  // on 3072-wide matrices: one copier thread for the second Gram product, the copies in
  // the MMA thread for the update.  With an inner dimension of 8192 (kWide) every product's
  // mainloop outlasts its epilogue, and all three take two copier threads.
  static constexpr int kSfCopiers =
      kBf16 ? 0 : (kWide ? 2 : (E == Epi::Update ? 0 : (E == Epi::GramA ? 1 : 2)));
  static constexpr bool kSfWarp = kSfCopiers > 0;
  static constexpr int kSfBufs = kSfWarp ? 4 : 2;
  static_assert(STAGE_BYTES % 1024 == 0, "stages must keep 1024-byte alignment");
  static_assert(SMEM_BYTES <= 232448, "over the per-CTA shared-memory limit");
  static_assert((3 * kStages + 4 + 2 * 4 + 1) * 8 + 12 <= BAR_BYTES, "barrier block too small");
  static_assert(kSfCol + kSfBufs * kSfBufCols <= kTmemCols, "scale-factor ring over the TMEM columns");
};

struct Job {
  int mat;
  int64_t row0, col0;
  int mirror;        // off-diagonal symmetric tile
  int b_half;        // only the first 128 rows of the B tile exist
  int kt;            // number of K tiles (256 NVFP4 or 64 BF16 elements each)
  const uint8_t* a_codes; const uint8_t* a_sf;
  const uint8_t* b_codes; const uint8_t* b_sf;
  int64_t a_tile_row, b_tile_row;   // 128-row tile index of the A / B operand
  int64_t ktiles_total;             // K tiles per operand row band
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

// Work unit u of kernel E: one 128 x 256 output tile.  The Newton-Schulz units of a
// matrix go through its 256 x 256 blocks in order, the two 128-row halves of a block
// one after the other (they share the block's B rows in L2).
template <Epi E, bool kBf16 = false>
__device__ __forceinline__ Job make_job(int32_t u, const NsParams& p, const GemmPlainArgs& g) {
  constexpr int TK = Cfg<E, kBf16>::kTileK;
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
    const MatLayout L = mat_layout(d.mp, d.np, d.state_off, d.big_off, kBf16);
    const int32_t lu = u - p.prefix[mi];
    const int slot = p.iter & 1;
    j.mat = mi;
    const int32_t tu = lu >> 1, half = lu & 1;   // 256 x 256 block, 128-row half
    if constexpr (E == Epi::GramX || E == Epi::GramA) {
      const int32_t T = d.mp / 256;
      int32_t P, Q;
      upper_tile(tu, T, P, Q);
      j.row0 = 256 * (int64_t)P + 128 * (int64_t)half;
      j.col0 = 256 * (int64_t)Q;
      j.mirror = (P != Q) ? 1 : 0;
      if constexpr (E == Epi::GramX) {
        j.kt = d.np / TK;
        j.a_codes = j.b_codes = p.ws + (slot ? L.qX[1] : L.qX[0]);
        j.a_sf = j.b_sf = p.ws + (slot ? L.sX[1] : L.sX[0]);
      } else {
        j.kt = d.mp / TK;
        j.a_codes = j.b_codes = p.ws + L.qA;
        j.a_sf = j.b_sf = p.ws + L.sA;
      }
    } else {
      const int32_t nJ = d.np / 256;
      const int32_t I = tu / nJ;
      j.row0 = 256 * (int64_t)I + 128 * (int64_t)half;
      j.col0 = (int64_t)(tu - I * nJ) * 256;
      j.kt = d.mp / TK;
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

// After a Newton-Schulz GEMM launch: turn each matrix's row / column sums into the
// bound that fixes the next tensor scale, and clear the sums for their next use (one
// CTA per matrix; the launch boundary orders the GEMM's sum atomics before the reads).
//   GramX:  u_rowA = max_i sum_j deq(qA)^2;  s_B from |b| u_rowX + |c| u_rowA
//   GramA:  u_rowB = max_i sum_j deq(qB)^2;  s_X' from |a| amax(X) + sqrt(u_rowB u_colX)
//   Update: u_rowX', u_colX' of the two views of X';  s_A' from u_rowX'
template <Epi E>
__global__ void __launch_bounds__(256) ns_bounds_kernel(const __grid_constant__ NsParams p) {
  __shared__ float red[8];
  const MatDesc& d = p.mat[blockIdx.x];
  NsState* st = reinterpret_cast<NsState*>(p.ws + d.state_off);
  const MatLayout L = mat_layout(d.mp, d.np, d.state_off, d.big_off);
  const int k = p.iter;
  // with the Hadamard transform the quantised tensor is T H: |T H| <= 4 max |T|
  const float rht4 = (p.opts & kOptRht) ? 4.0f : 1.0f;
  const bool for46 = (p.opts & kOpt46) != 0;   // tensor scales cover the M = 4 candidate
  auto drain = [&](int64_t off, int64_t len) -> float {
    float m = 0.0f;
    float4* v4 = reinterpret_cast<float4*>(p.ws + off);
    for (int64_t i = threadIdx.x; i < (len >> 2); i += 256) {
      const float4 a = __ldcg(v4 + i);
      __stcg(v4 + i, make_float4(0.f, 0.f, 0.f, 0.f));
      m = fmaxf(m, fmaxf(fmaxf(a.x, a.y), fmaxf(a.z, a.w)));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    float r = 0.0f;
#pragma unroll
    for (int w = 0; w < 8; ++w) r = fmaxf(r, red[w]);
    return r;
  };
  if constexpr (E == Epi::GramX) {
    const float ua = drain(L.rowsumA, d.mp);
    if (threadIdx.x == 0) {
      st->u_rowA[k] = ua;
      const float ub = (fabsf(d.b) * st->u_rowX[k] + fabsf(d.c) * ua) * kBoundInflate;
      st->sg[kSgB + k] = pow2_tensor_scale(ub * rht4, for46);
    }
  } else if constexpr (E == Epi::GramA) {
    const float ub = drain(L.rowsumB, d.mp);
    if (threadIdx.x == 0) {
      st->u_rowB[k] = ub;
      const float ax = __uint_as_float(st->amaxX[k]);
      const float ux = (fabsf(d.a) * ax + sqrtf(ub * st->u_colX[k])) * kBoundInflate;
      st->sg[kSgX + k + 1] = pow2_tensor_scale(ux * rht4, for46);
    }
  } else {
    const float ur = drain(L.rowsumX, d.mp);
    const float uc = drain(L.colsumX, d.np);
    if (threadIdx.x == 0 && !p.last) {
      st->u_rowX[k + 1] = ur;
      st->u_colX[k + 1] = uc;
      st->sg[kSgA + k + 1] = pow2_tensor_scale(ur * kBoundInflate * rht4, for46);
    }
  }
}

// ---------------------------------------------------------------- epilogue staging
__device__ __forceinline__ int stage_off(int r, int q) {
  return 16 * (r + (r >> 4)) + 4 * (q ^ ((r >> 1) & 3));
}

__device__ __forceinline__ void cp_async16(float* smem_dst, const float* gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(smem_dst)), "l"(gsrc)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Row r = lane of the stage <-> 16 registers.
__device__ __forceinline__ void stage_load_row(const float* buf, int lane, float* x) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float4 t = *reinterpret_cast<const float4*>(buf + stage_off(lane, q));
    x[4 * q] = t.x; x[4 * q + 1] = t.y; x[4 * q + 2] = t.z; x[4 * q + 3] = t.w;
  }
}
__device__ __forceinline__ void stage_store_row(float* buf, int lane, const float* x) {
#pragma unroll
  for (int q = 0; q < 4; ++q)
    *reinterpret_cast<float4*>(buf + stage_off(lane, q)) =
        make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
}
// Column cc, rows 16 hh .. 16 hh + 15 of the stage -> 16 registers.
__device__ __forceinline__ void stage_load_col(const float* buf, int cc, int hh, float* x) {
  // stage_off(16 hh + t, cc / 4) + cc % 4 = 272 hh + 16 t + 4 ((cc / 4) ^ ((t / 2) % 4)) + cc % 4
  const float* b = buf + 272 * hh + (cc & 3);
  const int q = cc >> 2;
#pragma unroll
  for (int t = 0; t < 16; ++t) x[t] = b[16 * t + 4 * (q ^ ((t >> 1) & 3))];
}

// FP32 rows of tile u for the four-lanes-per-row mapping: row row0 + 32 quad +
// (lane / 4) + 8 i, i = 0..3, starts at base + i * step (step = 8 rows, in floats),
// columns col0 + 128 ch + 4 (lane % 4) ...; the FP32 tile is A (GramX, GramA) or X (Update).
struct TileRows {
  float* base;
  uint32_t step;
};

template <Epi E>
__device__ __forceinline__ TileRows tile_rows(const NsParams& p, const GemmPlainArgs& g, int32_t u,
                                              int quad, int ch, int lane) {
  const Job j = make_job<E>(u, p, g);
  const MatDesc& d = p.mat[j.mat];
  const MatLayout L = mat_layout(d.mp, d.np, d.state_off, d.big_off);
  const int64_t pitch = (E == Epi::Update) ? d.np : d.mp;
  TileRows t;
  t.base = reinterpret_cast<float*>(p.ws + (E == Epi::Update ? L.X : L.A)) +
           (j.row0 + 32 * quad + (lane >> 2)) * pitch + j.col0 + 128 * ch + 4 * (lane & 3);
  t.step = (uint32_t)(8 * pitch);
  return t;
}

// Asynchronous copy of chunk c of the FP32 tile rows into a stage buffer.
__device__ __forceinline__ void stage_fetch(float* buf, TileRows t, int c, int lane) {
  const int rr = lane >> 2, qq = lane & 3;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    cp_async16(buf + stage_off(rr + 8 * i, qq), t.base + (size_t)i * t.step + kChunkCols * c);
}

// Coalesced store of the staged chunk c to the FP32 tile rows.
__device__ __forceinline__ void stage_flush(const float* buf, TileRows t, int c, int lane) {
  const int rr = lane >> 2, qq = lane & 3;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    *reinterpret_cast<float4*>(t.base + (size_t)i * t.step + kChunkCols * c) =
        *reinterpret_cast<const float4*>(buf + stage_off(rr + 8 * i, qq));
}

// Epilogue of the three Newton-Schulz GEMMs (one epilogue warp).
//   GramX   A = sX^2 acc            -> A (FP32), qA = Q1x16(A); mirrored tile: Q1x16 of A^T
//   GramA   B = b A + c sA^2 acc    -> qB = Q1x16(B);           mirrored tile: Q1x16 of B^T
//   Update  X' = a X + sB sX acc    -> X' (FP32), Q1x16(X'), Q16x1(X') (or the output, last)
template <Epi E, uint32_t kOpts>
__device__ __forceinline__ void epilogue_ns(const NsParams& p, const GemmPlainArgs& g,
                                            uint32_t tmem, uint64_t* acc_full,
                                            uint64_t* acc_empty,
                                            uint32_t* status, volatile int* abort_flag,
                                            float* wbuf, const float* scale_tab, int quad, int ch,
                                            int lane, int32_t total) {
  const int32_t first = blockIdx.x, step = gridDim.x;
  constexpr bool kIn = (E == Epi::GramA || E == Epi::Update);   // reads an FP32 tile
  constexpr bool kPackedQ = true;   // f32x2 quantiser (measured faster in all three kernels)
  constexpr bool kRht = (kOpts & kOptRht) != 0;    // Hadamard transform before quantising
  constexpr bool k46 = (kOpts & kOpt46) != 0;      // adaptive 4/6 block scaling
  constexpr bool kBf16 = (kOpts & kOptBf16) != 0;  // BF16 comparison step: BF16 views
  // H16^r masks of the tensors this epilogue quantises (Section 3.4): GramX -> qA (product
  // qA qA^T of iteration k), GramA -> qB (update product of iteration k), Update -> the
  // next iterate's Gram view and update view (iteration k + 1)
  const int kk = p.iter;
  const uint32_t mask_row = E == Epi::GramX ? p.rht[3 * kk + 1]
                           : E == Epi::GramA ? p.rht[3 * kk + 2]
                                             : (kk + 1 < kMaxIters ? p.rht[3 * (kk + 1)] : 0u);
  const uint32_t mask_col = E == Epi::Update ? (kk + 1 < kMaxIters ? p.rht[3 * (kk + 1) + 2] : 0u)
                                             : mask_row;
  const int k = p.iter;
  const int cc = lane & 15, hh = lane >> 4;
  TileRows fp{nullptr, 0u};   // FP32 tile rows of the current tile
  TileRows fn{nullptr, 0u};   // ... of the next tile (fetched ahead)
  if constexpr (kIn) {
    if (first < total) {
      fp = tile_rows<E>(p, g, first, quad, ch, lane);
      stage_fetch(wbuf, fp, 0, lane);
      cp_async_commit();
      stage_fetch(wbuf + kStageFloats, fp, 1, lane);
      cp_async_commit();
    }
  }
  int b = 0;   // stage buffer of the current chunk
  uint32_t tl = 0;
  for (int32_t u = first; u < total; u += step, ++tl) {
    const Job j = make_job<E>(u, p, g);
    const MatDesc& d = p.mat[j.mat];
    NsState* st = reinterpret_cast<NsState*>(p.ws + d.state_off);
    const MatLayout L = mat_layout(d.mp, d.np, d.state_off, d.big_off, kBf16);
    if constexpr (!kIn) fp = tile_rows<E>(p, g, u, quad, ch, lane);
    // One lane polls the barrier (32 lanes polling one mbarrier serialise on its bank);
    // the warp then synchronises, which with tcgen05.fence::after_thread_sync below
    // orders every lane's accumulator loads after the MMAs.  Warp-uniform by
    // construction: the chunk loop shuffles under this condition.
    const bool ok = __shfl_sync(0xFFFFFFFFu,
                                lane == 0 ? (mbar_wait(acc_full, tl & 1u, status, abort_flag) ? 1 : 0) : 0,
                                0) != 0;
    __syncwarp();
    const int64_t gr0 = j.row0 + 32 * quad;   // first row of this warp's band
    const int64_t gr = gr0 + lane;             // this lane's row
    const int64_t gc0 = j.col0 + 128 * ch;     // first column of this warp's half
    const bool last = (E == Epi::Update) && p.last;

    float acc_scale, sg_out;
    if constexpr (kBf16) {
      acc_scale = 1.0f;   // BF16 operands carry no tensor scales
      sg_out = 1.0f;
    } else if constexpr (E == Epi::GramX) {
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
    const float six_out = __fmul_rn(6.0f, sg_out);
    const float rcp_six = __frcp_rn(six_out);
    const ScaleTab stab{scale_tab, __frcp_rn(sg_out)};   // sg_out is a power of two

    // destinations of the two views and of their sums
    const int ns = (k + 1) & 1;
    uint8_t* row_codes = p.ws + (E == Epi::GramX ? L.qA : E == Epi::GramA ? L.qB : (ns ? L.qX[1] : L.qX[0]));
    uint8_t* row_scales = p.ws + (E == Epi::GramX ? L.sA : E == Epi::GramA ? L.sB : (ns ? L.sX[1] : L.sX[0]));
    const int64_t row_cp = (E == Epi::Update) ? d.np : d.mp;
    uint8_t* col_codes = (E == Epi::Update) ? p.ws + (ns ? L.qXT[1] : L.qXT[0]) : row_codes;
    uint8_t* col_scales = (E == Epi::Update) ? p.ws + (ns ? L.sXT[1] : L.sXT[0]) : row_scales;
    float* rowsum = reinterpret_cast<float*>(
        p.ws + (E == Epi::GramX ? L.rowsumA : E == Epi::GramA ? L.rowsumB : L.rowsumX));
    float* colsum = (E == Epi::Update) ? reinterpret_cast<float*>(p.ws + L.colsumX) : rowsum;
    const bool need_col = (E == Epi::Update) ? !last : (j.mirror != 0);
    // TILED-layout addresses of this warp's share: a per-tile base plus a per-chunk
    // constant (the share spans one 256-column tile of each view).  The update kernel,
    // which is tighter on registers, measured faster recomputing them per chunk.
    const int64_t rr = gr & 127;
    uint8_t* const rowc = row_codes + ((gr >> 7) * (row_cp >> 8) + (gc0 >> 8)) * kTileBytes + rr * 128;
    const uint32_t rjb = (uint32_t)((gc0 & 255) >> 5), rx = (uint32_t)(rr & 7);
    uint8_t* const rows = row_scales + ((gr >> 7) * (row_cp >> 6) + (gc0 >> 6)) * kAtomBytes +
                          16 * (gr & 31) + 4 * ((gr & 127) >> 5);
    uint8_t* const colc = col_codes + ((gc0 >> 7) * (d.mp >> 8) + (gr0 >> 8)) * kTileBytes + cc * 128 +
                          ((((gr0 & 255) >> 5) ^ (cc & 7)) << 4);
    uint8_t* const cols = col_scales + ((gc0 >> 7) * (d.mp >> 6) + (gr0 >> 6)) * kAtomBytes + 16 * cc +
                          ((gr0 >> 4) & 3);

    uint32_t accr[4][32];
    if (ok) {
      tc_fence_after();
      // drain this warp's 32 x 128 share of the accumulator into registers and hand
      // the accumulator back at once: the next tile's MMAs overlap this epilogue
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
    }

    float row_acc = 0.0f, amax = 0.0f;
    uint32_t prev_w0 = 0u, prev_w1 = 0u, scale_word = 0u;
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
      float* buf = wbuf + b * kStageFloats;
      if constexpr (kIn) {
        cp_async_wait<1>();   // this chunk's rows have landed (own copies) ...
        __syncwarp();         // ... and every lane's
      }
      if (ok) {
        const int64_t gcc = gc0 + kChunkCols * c;   // first column of the chunk
        float y[16];
        const uint64_t s2 = f2_pack(acc_scale, acc_scale);
        if constexpr (E == Epi::Update) {
          // (the update kernel measured faster with scalar arithmetic here)
          float xin[16];
          stage_load_row(buf, lane, xin);
#pragma unroll
          for (int e = 0; e < 16; ++e)
            y[e] = fmaf(d.a, xin[e], __uint_as_float(accr[c >> 1][16 * (c & 1) + e]) * acc_scale);
        } else if constexpr (kIn) {
          // GramA: b A + c (s acc)   (pairs of columns at a time)
          float xin[16];
          stage_load_row(buf, lane, xin);
          const uint64_t ca = f2_pack(d.b, d.b);
          const uint64_t cc2 = f2_pack(d.c, d.c);
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            uint64_t v = f2_mul(f2_pack(__uint_as_float(accr[c >> 1][16 * (c & 1) + e]),
                                        __uint_as_float(accr[c >> 1][16 * (c & 1) + e + 1])), s2);
            if constexpr (E == Epi::GramA) v = f2_mul(cc2, v);
            f2_unpack(f2_fma(ca, f2_pack(xin[e], xin[e + 1]), v), y[e], y[e + 1]);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 16; e += 2)
            f2_unpack(f2_mul(f2_pack(__uint_as_float(accr[c >> 1][16 * (c & 1) + e]),
                                     __uint_as_float(accr[c >> 1][16 * (c & 1) + e + 1])), s2),
                      y[e], y[e + 1]);
        }
        if (last) {
          // final iteration: write the output (transposed back for a tall input)
          if (d.tall) {
            if (gr < d.m) {
#pragma unroll
              for (int e = 0; e < 16; ++e)
                if (gcc + e < d.n) d.out[(gcc + e) * d.ldo + gr] = y[e];
            }
          } else {
            stage_store_row(buf, lane, y);
            __syncwarp();
            float xc[16];
            stage_load_col(buf, cc, hh, xc);
            const int64_t col = gcc + cc;
            if (col < d.n) {
#pragma unroll
              for (int t = 0; t < 16; ++t) {
                const int64_t row = gr0 + 16 * hh + t;
                if (row < d.m) d.out[row * d.ldo + col] = xc[t];
              }
            }
          }
        } else {
          // stage the chunk (FP32 store and/or the 16x1 view read it back); a debug
          // stop after the second product also stores B (FP32) over this tile of A,
          // whose chunk c was read already
          const bool dbg_b = (E == Epi::GramA) && p.dbg_b;
          if (E != Epi::GramA || need_col || dbg_b) {
            stage_store_row(buf, lane, y);
            __syncwarp();
          }
          if constexpr (E != Epi::GramA) stage_flush(buf, fp, c, lane);   // A or X' (FP32)
          else if (dbg_b) stage_flush(buf, fp, c, lane);
          if constexpr (kBf16) {
            // BF16 views (round to nearest even): the row's 16 values, and where needed
            // column gcc + cc, rows gr0 + 16 hh ..; two 16-byte chunks each
            uint32_t w[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) w[e] = pack_bf16x2(y[2 * e], y[2 * e + 1]);
            *reinterpret_cast<uint4*>(row_codes + tiled_chunk_offset_bf16(gr, gcc, row_cp)) =
                make_uint4(w[0], w[1], w[2], w[3]);
            *reinterpret_cast<uint4*>(row_codes + tiled_chunk_offset_bf16(gr, gcc + 8, row_cp)) =
                make_uint4(w[4], w[5], w[6], w[7]);
            if (need_col) {
              float xc[16];
              stage_load_col(buf, cc, hh, xc);
#pragma unroll
              for (int e = 0; e < 8; ++e) w[e] = pack_bf16x2(xc[2 * e], xc[2 * e + 1]);
              const int64_t rt = gcc + cc, k0 = gr0 + 16 * hh;
              *reinterpret_cast<uint4*>(col_codes + tiled_chunk_offset_bf16(rt, k0, d.mp)) =
                  make_uint4(w[0], w[1], w[2], w[3]);
              *reinterpret_cast<uint4*>(col_codes + tiled_chunk_offset_bf16(rt, k0 + 8, d.mp)) =
                  make_uint4(w[4], w[5], w[6], w[7]);
            }
          } else {
          // 1x16 view along this lane's row and, where needed, the 16x1 view of column
          // gcc + cc, rows gr0 + 16 hh ..: two independent quantiser chains side by side
          QBlock16 q, qc;
          float yamax = 0.0f;   // max |X'| of the untransformed block (update bound)
          if constexpr (kRht && E == Epi::Update) {
            yamax = absmax16(y);
          }
          if constexpr (kRht) rht16(y, mask_row);
          if (need_col) {
            float xc[16];
            stage_load_col(buf, cc, hh, xc);
            if constexpr (kRht) rht16(xc, mask_col);
            q = quantize16<true, true, kPackedQ, k46>(y, sg_out, six_out, rcp_six, stab);
            qc = quantize16<true, true, kPackedQ, k46>(xc, sg_out, six_out, rcp_six, stab);
          } else {
            q = quantize16<true, true, kPackedQ, k46>(y, sg_out, six_out, rcp_six, stab);
          }
          row_acc += q.sumsq;
          amax = fmaxf(amax, kRht ? yamax : q.amax);
          if (c & 1) {
            uint8_t* dst = (E == Epi::Update)
                               ? row_codes + tiled_chunk_offset(gr, gcc - 16, row_cp)
                               : rowc + (((rjb + (c >> 1)) ^ rx) << 4);
            *reinterpret_cast<uint4*>(dst) = make_uint4(prev_w0, prev_w1, q.w0, q.w1);
          } else {
            prev_w0 = q.w0;
            prev_w1 = q.w1;
          }
          scale_word |= q.scale << (8 * (c & 3));
          if ((c & 3) == 3) {
            uint8_t* dst = (E == Epi::Update)
                               ? row_scales + tiled_scale_offset(gr, (gcc - 48) >> 4, row_cp)
                               : rows + kAtomBytes * (c >> 2);
            *reinterpret_cast<uint32_t*>(dst) = scale_word;
            scale_word = 0u;
          }
          if (need_col) {
            // the two row halves of one column pair up into a 16-byte code chunk
            const uint32_t o0 = __shfl_xor_sync(0xFFFFFFFFu, qc.w0, 16);
            const uint32_t o1 = __shfl_xor_sync(0xFFFFFFFFu, qc.w1, 16);
            const uint32_t os = __shfl_xor_sync(0xFFFFFFFFu, qc.scale, 16);
            const float s2 = qc.sumsq + __shfl_xor_sync(0xFFFFFFFFu, qc.sumsq, 16);
            if (hh == 0) {
              const int64_t rt = gcc + cc;
              uint8_t* dc = (E == Epi::Update) ? col_codes + tiled_chunk_offset(rt, gr0, d.mp)
                                               : colc + 2048 * c;
              uint8_t* ds = (E == Epi::Update) ? col_scales + tiled_scale_offset(rt, gr0 >> 4, d.mp)
                                               : cols + 256 * (c & 1) + 4 * (c >> 1);
              *reinterpret_cast<uint4*>(dc) = make_uint4(qc.w0, qc.w1, o0, o1);
              *reinterpret_cast<uint16_t*>(ds) = static_cast<uint16_t>(qc.scale | (os << 8));
              if (s2 != 0.0f) atomicAdd(colsum + gcc + cc, s2);
            }
          }
          }
        }
      }
      __syncwarp();   // every lane is done with this stage buffer
      if constexpr (kIn) {
        // fetch chunk c + 2 (of this tile or the next) into the buffer chunk c - 1 used
        float* nb = wbuf + (b == 0 ? 2 : b - 1) * kStageFloats;
        const bool more = u + step < total;
        if (c + 2 < kChunks) {
          stage_fetch(nb, fp, c + 2, lane);
        } else if (more) {
          if (c + 2 == kChunks) fn = tile_rows<E>(p, g, u + step, quad, ch, lane);
          stage_fetch(nb, fn, c + 2 - kChunks, lane);
        }
        cp_async_commit();
      }
      b = (b == kStageBufs - 1) ? 0 : b + 1;
    }

    if (row_acc != 0.0f) atomicAdd(rowsum + gr, row_acc);
    if constexpr (E == Epi::Update) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
      if (lane == 0 && !p.last && amax > 0.0f) atomicMax(&st->amaxX[k + 1], __float_as_uint(amax));
    }
    if constexpr (kIn) fp = fn;
  }
  if constexpr (kIn) cp_async_wait<0>();
}

// Epilogue of the plain GEMM D = (sa sb) acc (one epilogue warp); tb is a 32 x 33
// transpose buffer so that each store instruction writes one contiguous row segment.
__device__ __forceinline__ void epilogue_plain(const NsParams& p, const GemmPlainArgs& g,
                                               uint32_t tmem, uint64_t* acc_full,
                                               uint64_t* acc_empty, uint32_t* status,
                                               volatile int* abort_flag, float* tb, int quad,
                                               int ch, int lane, int32_t total) {
  uint32_t tl = 0;
  for (int32_t u = blockIdx.x; u < total; u += gridDim.x, ++tl) {
    const Job j = make_job<Epi::Plain>(u, p, g);
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

template <Epi E, uint32_t kOpts>
__global__ void __launch_bounds__(kThreads, 1)
    nvfp4_gemm_kernel(const __grid_constant__ NsParams p, const __grid_constant__ GemmPlainArgs g) {
  constexpr bool kBf16 = (kOpts & kOptBf16) != 0;
  using C = Cfg<E, kBf16, (kOpts & kOptWideK) != 0>;
  constexpr int kStages = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  float* epi_smem = reinterpret_cast<float*>(smem + kStages * C::STAGE_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * C::STAGE_BYTES + 8 * EPI_WARP_FLOATS * 4);
  uint64_t* full = bars;                      // an operand stage landed
  uint64_t* empty = bars + kStages;           // the MMAs reading a stage finished
  uint64_t* acc_full = bars + 2 * kStages;
  uint64_t* acc_empty = acc_full + 1;         // the epilogue warps drained the accumulator
  uint64_t* mma_done = acc_full + 2;
  uint64_t* stall_bar = acc_full + 3;        // test only: never arrived on
  uint64_t* sf_full = acc_full + 4;           // [kSfBufs] scale copies into a TMEM buffer done
  uint64_t* sf_empty = sf_full + C::kSfBufs;  // [kSfBufs] the MMAs reading that buffer done
  uint64_t* sf_done = sf_empty + C::kSfBufs;  // the copier's last copies completed
  uint64_t* sf_land = sf_done + 1;            // [kStages] a stage's scale atoms landed (copier products)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sf_land + kStages);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);
  float* scale_tab = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + C::BAR_BYTES);
  if (threadIdx.x >= 128 && threadIdx.x < 256) scale_tab_fill(scale_tab, threadIdx.x - 128);

  uint32_t* status = (E == Epi::Plain) ? g.status : p.status;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t first = blockIdx.x, step = gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_land[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 8);
    mbar_init(mma_done, 1);
    mbar_init(stall_bar, 1);
    for (int b = 0; b < C::kSfBufs; ++b) {
      mbar_init(&sf_full[b], C::kSfCopiers > 0 ? C::kSfCopiers : 1);   // one arrival per copier thread
      mbar_init(&sf_empty[b], 1);
    }
    mbar_init(sf_done, C::kSfCopiers > 0 ? C::kSfCopiers : 1);
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
  // The control loops below each run on a single issuing thread, where every tcgen05 or
  // bulk-copy instruction costs tens of cycles to issue: they keep per-stage work to those
  // instructions, with the stage ring position, phases, descriptors and global addresses
  // advanced by constant steps.
  constexpr uint64_t kStageDesc = C::STAGE_BYTES >> 4;   // descriptor address units per stage
  const uint32_t s_base = smem_addr(stage_base);
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t it = 0, s = 0, ph = 0;   // stages issued; ring position and its phase
      for (int32_t u = first; u < total && !*abort_flag; u += step) {
        const Job j = make_job<E, kBf16>(u, p, g);
        // k-tile kt of a 128-row band sits kt tiles after the band's first; the second
        // half of the B tile is the next band
        const int64_t band = j.ktiles_total * kTileBytes, sband = j.ktiles_total * (4 * kAtomBytes);
        const uint8_t* pa = j.a_codes + j.a_tile_row * band;
        const uint8_t* pb = j.b_codes + j.b_tile_row * band;
        const uint8_t* psa = j.a_sf + j.a_tile_row * sband;
        const uint8_t* psb = j.b_sf + j.b_tile_row * sband;
        // with copier threads the scale atoms land on a barrier of their own (sf_land) and
        // are issued first, so the copies to TMEM start while the codes are still in flight
        const uint32_t tx_sf = C::SFA + (j.b_half ? C::SFB / 2 : C::SFB);
        const uint32_t tx_codes = A_BYTES + (j.b_half ? C::B_BYTES / 2 : C::B_BYTES);
        for (int kt = 0; kt < j.kt; ++kt, ++it) {
          if (!mbar_wait(&empty[s], ph ^ 1u, status, abort_flag)) break;
          const uint32_t st = s_base + s * C::STAGE_BYTES;
          uint64_t* fb = &full[s];
          if constexpr (!kBf16) {
            uint64_t* sb = C::kSfWarp ? &sf_land[s] : fb;
            if constexpr (C::kSfWarp) mbar_arrive_expect_tx(sb, tx_sf);
            bulk_g2s_addr(st + A_BYTES + C::B_BYTES, psa, SFA_BYTES, sb);
            bulk_g2s_addr(st + A_BYTES + C::B_BYTES + C::SFA, psb, 4 * kAtomBytes, sb);
            if (!j.b_half)
              bulk_g2s_addr(st + A_BYTES + C::B_BYTES + C::SFA + 4 * kAtomBytes, psb + sband, 4 * kAtomBytes, sb);
          }
          mbar_arrive_expect_tx(fb, C::kSfWarp ? tx_codes : tx_codes + (kBf16 ? 0u : tx_sf));
          bulk_g2s_addr(st, pa, A_BYTES, fb);
          bulk_g2s_addr(st + A_BYTES, pb, kTileBytes, fb);
          if (!j.b_half) bulk_g2s_addr(st + A_BYTES + kTileBytes, pb + band, kTileBytes, fb);
          pa += kTileBytes;
          pb += kTileBytes;
          psa += 4 * kAtomBytes;
          psb += 4 * kAtomBytes;
          if (++s == (uint32_t)kStages) { s = 0; ph ^= 1u; }
        }
      }
      // drain: every issued copy must land before the CTA may exit
      const uint32_t from = it > (uint32_t)kStages ? it - kStages : 0u;
      for (uint32_t k = from; k < it; ++k) {
        volatile int never = 0;
        mbar_wait(&full[k % kStages], (k / kStages) & 1u, status, &never);
        if constexpr (C::kSfWarp) mbar_wait(&sf_land[k % kStages], (k / kStages) & 1u, status, &never);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      uint32_t tl = 0, s = 0, ph = 0, b = 0, bph = 0;   // stage ring and scale-factor ring
      const uint32_t acc = tmem;   // lane 0, column 0
      const uint64_t da0 = sdesc_sw128(s_base), db0 = sdesc_sw128(s_base + A_BYTES);
      const uint64_t dsf0 = sdesc_sf_atom(s_base + A_BYTES + C::B_BYTES);
      if constexpr (E != Epi::Plain) {
        // test only: a wait that runs out (bounded), exercising the timeout path
        if (p.stall) mbar_wait(stall_bar, 0, status, abort_flag);
      }
      for (int32_t u = first; u < total && !*abort_flag; u += step, ++tl) {
        const Job j = make_job<E, kBf16>(u, p, g);
        if (!mbar_wait(acc_empty, (tl & 1u) ^ 1u, status, abort_flag)) break;
        tc_fence_after();
        bool ok = true;
        for (int kt = 0; kt < j.kt; ++kt) {
          if (!mbar_wait(&full[s], ph, status, abort_flag)) { ok = false; break; }
          const uint64_t da = da0 + s * kStageDesc, db = db0 + s * kStageDesc;
          if constexpr (kBf16) {
            tc_fence_after();
            // four K = 16 steps of BF16 per 128-byte row, no scale factors
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              tc_mma_bf16(acc, da + 2 * ks, db + 2 * ks, C::kIdesc, (kt | ks) != 0 ? 1u : 0u);
          } else {
            const uint32_t sf = tmem + kSfCol + b * kSfBufCols;
            if constexpr (C::kSfWarp) {
              // the copier threads filled scale-factor buffer b from this stage
              if (!mbar_wait(&sf_full[b], bph, status, abort_flag)) { ok = false; break; }
              tc_fence_after();
            } else {
              // this thread copies the stage's twelve scale atoms (A, k-steps 0-3; B rows
              // 0-127 and 128-255, k-steps 0-3; 512 bytes apart); the MMAs below queue
              // behind them
              tc_fence_after();
              const uint64_t d = dsf0 + s * kStageDesc;
#pragma unroll
              for (int a = 0; a < 12; ++a)
                tc_copy_sf(sf + (a < 4 ? 4 * a : (a < 8 ? 16 + 8 * (a - 4) : 20 + 8 * (a - 8))),
                           d + (uint64_t)(a * (kAtomBytes >> 4)));
            }
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              tc_mma_nvf4(acc, da + 2 * ks, db + 2 * ks, C::kIdesc, sf + 4 * ks, sf + 16 + 8 * ks,
                          (kt | ks) != 0 ? 1u : 0u);
            }
            if constexpr (C::kSfWarp) tc_commit(&sf_empty[b]);
            if (++b == (uint32_t)C::kSfBufs) { b = 0; bph ^= 1u; }
          }
          tc_commit(&empty[s]);
          if (++s == (uint32_t)kStages) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        tc_commit(acc_full);
      }
      tc_commit(mma_done);
      volatile int never = 0;
      mbar_wait(mma_done, 0, status, &never);
    }
  } else if (warp >= 2 && C::kSfWarp) {
    // ------------------------------------------------------------ scale-factor copiers
    // For each stage: once its scale atoms have landed (sf_land) and the MMAs of the stage
    // that last used the TMEM buffer have completed, copy the stage's twelve scale atoms
    // into the buffer: with two copiers lane 0 of warp 2 the first six (A, k-steps 0-3; B rows
    // 0-127, k-steps 0-1) and lane 0 of warp 3 the other six, with one copier lane 0 of
    // warp 2 all twelve; each copier thread commits once per stage (sf_full expects one
    // arrival per copier thread).  The MMAs that read the stage's shared memory wait for these copies
    // (sf_full), and the producer refills the stage only after those MMAs (empty), so
    // the copies never read a refilled stage.
    auto copier = [&](auto first_c) {
      constexpr int kA0 = decltype(first_c)::value;           // first atom of this thread
      constexpr int kNA = 12 / (C::kSfCopiers > 0 ? C::kSfCopiers : 1);   // atoms per copier thread
      uint32_t s = 0, ph = 0, b = 0, bph = 0;
      bool ok = true;
      const uint64_t dsf = sdesc_sf_atom(s_base + A_BYTES + C::B_BYTES);
      for (int32_t u = first; u < total && ok && !*abort_flag; u += step) {
        const Job j = make_job<E, kBf16>(u, p, g);
        for (int kt = 0; kt < j.kt; ++kt) {
          if (!mbar_wait(&sf_land[s], ph, status, abort_flag) ||
              !mbar_wait(&sf_empty[b], bph ^ 1u, status, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sf = tmem + kSfCol + b * kSfBufCols;
          const uint64_t d = dsf + s * kStageDesc;
#pragma unroll
          for (int q = 0; q < kNA; ++q) {
            // atom a: 0-3 A k-step a, 4-7 B rows 0-127 k-step a - 4, 8-11 B rows 128-255
            // k-step a - 8; atoms sit 512 bytes apart, A's then B's
            const int a = kA0 + q;
            const uint32_t col = a < 4 ? 4 * a : (a < 8 ? 16 + 8 * (a - 4) : 20 + 8 * (a - 8));
            tc_copy_sf(sf + col, d + (uint64_t)(a * (kAtomBytes >> 4)));
          }
          tc_commit(&sf_full[b]);
          if (++s == (uint32_t)kStages) { s = 0; ph ^= 1u; }
          if (++b == (uint32_t)C::kSfBufs) { b = 0; bph ^= 1u; }
        }
      }
      // every copy this thread issued completes before the TMEM is freed
      tc_commit(sf_done);
      volatile int never = 0;
      mbar_wait(sf_done, 0, status, &never);
    };
    if (lane == 0) {
      if (warp == 2) copier(std::integral_constant<int, 0>{});
      else if (C::kSfCopiers == 2) copier(std::integral_constant<int, 6>{});
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
    float* wbuf = epi_smem + ew * EPI_WARP_FLOATS;
    if constexpr (E == Epi::Plain)
      epilogue_plain(p, g, tmem, acc_full, acc_empty, status, abort_flag, wbuf, quad, ch, lane, total);
    else
      epilogue_ns<E, kOpts>(p, g, tmem, acc_full, acc_empty, status, abort_flag, wbuf, scale_tab,
                     quad, ch, lane, total);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <Epi E, uint32_t kOpts>
cudaError_t launch_impl(const NsParams* p, const GemmPlainArgs* g, int64_t units, cudaStream_t st,
                        int num_sms) {
  using C = Cfg<E, (kOpts & kOptBf16) != 0, (kOpts & kOptWideK) != 0>;
  static unsigned long long attr_set = 0ull;   // one bit per device; a benign race
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(attr_set & (1ull << dev))) {
    e = cudaFuncSetAttribute(nvfp4_gemm_kernel<E, kOpts>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set |= 1ull << dev;
  }
  // setmaxnreg.inc can only hand out what the block was launched with: refuse to
  // launch unless the compiled register count is exactly the split's budget
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, nvfp4_gemm_kernel<E, kOpts>);
  if (e != cudaSuccess) return e;
  if ((uint32_t)fa.numRegs != kRegsLaunch) return cudaErrorInvalidConfiguration;
  const int grid = (int)(units < num_sms ? (units > 0 ? units : 1) : num_sms);
  static const NsParams zero_p{};
  static const GemmPlainArgs zero_g{};
  nvfp4_gemm_kernel<E, kOpts><<<grid, kThreads, C::SMEM_BYTES, st>>>(p ? *p : zero_p, g ? *g : zero_g);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_plain(const GemmPlainArgs& a, cudaStream_t st, int num_sms) {
  const int64_t units = (int64_t)(a.Mp / BM) * ((a.Np + BN - 1) / BN);
  return launch_impl<Epi::Plain, 0>(nullptr, &a, units, st, num_sms);
}

namespace {

template <uint32_t kOpts>
cudaError_t launch_ns_opts(Epi epi, const NsParams& p, cudaStream_t st, int num_sms) {
  const int64_t units = p.prefix[p.count];
  cudaError_t e;
  switch (epi) {
    // (the BF16 step has no tensor scales, hence no bounds kernels)
    case Epi::GramX:
      if ((e = launch_impl<Epi::GramX, kOpts>(&p, nullptr, units, st, num_sms)) != cudaSuccess) return e;
      if (!(kOpts & kOptBf16)) ns_bounds_kernel<Epi::GramX><<<p.count, 256, 0, st>>>(p);
      break;
    case Epi::GramA:
      if ((e = launch_impl<Epi::GramA, kOpts>(&p, nullptr, units, st, num_sms)) != cudaSuccess) return e;
      if (!(kOpts & kOptBf16)) ns_bounds_kernel<Epi::GramA><<<p.count, 256, 0, st>>>(p);
      break;
    case Epi::Update:
      if ((e = launch_impl<Epi::Update, kOpts>(&p, nullptr, units, st, num_sms)) != cudaSuccess) return e;
      if (!p.last && !(kOpts & kOptBf16)) ns_bounds_kernel<Epi::Update><<<p.count, 256, 0, st>>>(p);
      break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_ns(Epi epi, const NsParams& p, cudaStream_t st, int num_sms) {
  if (p.opts & kOptBf16) return launch_ns_opts<kOptBf16>(epi, p, st, num_sms);
  switch (p.opts & (kOptRht | kOpt46 | kOptWideK)) {
    case 0: return launch_ns_opts<0>(epi, p, st, num_sms);
    case kOpt46: return launch_ns_opts<kOpt46>(epi, p, st, num_sms);
    case kOptRht: return launch_ns_opts<kOptRht>(epi, p, st, num_sms);
    case kOptRht | kOpt46: return launch_ns_opts<kOptRht | kOpt46>(epi, p, st, num_sms);
    case kOptWideK: return launch_ns_opts<kOptWideK>(epi, p, st, num_sms);
    case kOptWideK | kOpt46: return launch_ns_opts<kOptWideK | kOpt46>(epi, p, st, num_sms);
    case kOptWideK | kOptRht: return launch_ns_opts<kOptWideK | kOptRht>(epi, p, st, num_sms);
    default: return launch_ns_opts<kOptWideK | kOptRht | kOpt46>(epi, p, st, num_sms);
  }
}

}  // namespace fs4
