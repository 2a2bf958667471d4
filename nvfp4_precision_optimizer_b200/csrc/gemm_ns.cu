// The three block-scaled NVFP4 products of the direct NVFP4 Newton-Schulz
// iteration on CTA pairs (tcgen05 cta_group::2, sm_100a), with their fused
// epilogues.
//
// "Full-Stack FP4" (arXiv 2607.04422), Section 3.4, one iteration:
//   GramX   A  = qX qX^T                    epilogue: A (FP32), qA = Q1x16(A)
//   GramA   P  = qA qA16x1, B = b A + c P   epilogue: qB = Q1x16(B)
//   Update  X' = a X + qB qX16x1            epilogue: X' (FP32), Q1x16(X'), Q16x1(X')
// A and B are symmetric, so GramX and GramA compute only the 256 x 256 blocks on
// and above the diagonal; an off-diagonal block also writes its transposed view,
// which is the mirrored block's 1x16 quantisation (Q16x1(A) = Q1x16(A)^T).
//
// Work unit: a 256 x 128 output tile of one matrix, computed by a CTA pair (a
// cluster of 2).  Each CTA stages its own 128 rows of the A operand and 64 of the
// B operand's 128 rows; the pair's leader issues tcgen05.mma.cta_group::2
// kind::mxf4nvf4 (M = 256, N = 128, K = 64, UE4M3 scales per 16 elements), and
// each CTA accumulates its 128 x 128 share in its own TMEM.  The accumulator is
// double-buffered (2 x 128 columns), so the MMAs of tile t + 1 run while the
// epilogue reads tile t.
//
// One persistent CTA per SM, 640 threads:
//   warp 0      producer: 1-D bulk copies (TMA engine) of pre-tiled operand tiles
//               and scale atoms into a ring of shared-memory stages
//   warp 1      leader: allocates TMEM, copies scale atoms to TMEM (tcgen05.cp)
//               and issues the MMAs for both CTAs; peer: tells the leader each
//               time one of its stages has landed
//   warps 4-19  epilogue: each warp owns 32 rows (its TMEM lane quarter) x 32
//               columns of the CTA's 128 x 128 share, loads them from TMEM,
//               releases the accumulator buffer, then runs the fused step and
//               the requantisation in two chunks of 32 x 16
// setmaxnreg moves registers from the control warpgroup (32 per thread) to the
// four epilogue warpgroups (112 per thread).  No load uses cluster multicast.
// Every mbarrier wait is bounded (see mbar_wait); on a timeout a CTA stops
// issuing work, drains what it issued, frees TMEM and returns.
#include <cfloat>
#include <cmath>

#include "fs4_device.cuh"
#include "fs4_internal.h"

namespace fs4 {

namespace {

constexpr int BM = 128;          // rows per CTA (256 per pair)
constexpr int BN = 128;          // columns per tile
constexpr int BK = 256;          // K per stage
constexpr int kThreads = 640;    // 20 warps
constexpr int kEpiWarps = 16;
constexpr uint32_t kRegsLaunch = 96;
constexpr uint32_t kRegsCtl = 32;
constexpr uint32_t kRegsEpi = 112;
static_assert(kRegsCtl * 128 + kRegsEpi * 512 <= kRegsLaunch * kThreads, "register split over budget");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCols = 128;     // one accumulator buffer
constexpr uint32_t kSfCol = 256;       // scale factors follow the two accumulator buffers
constexpr uint32_t kSfBufCols = 32;    // 16 (A: 4 k-steps x 4) + 16 (B: 4 k-steps x 4)
constexpr int A_BYTES = BM * BK / 2;             // 16 KB: this CTA's 128 A rows
constexpr int B_BYTES = (BN / 2) * BK / 2;       //  8 KB: this CTA's 64 B rows
constexpr int SFA_BYTES = BM * BK / 16;          //  2 KB
constexpr int SFB_BYTES = BN * BK / 16;          //  2 KB: the scales of all 128 B rows
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
constexpr int kStages = 4;
static_assert(STAGE_BYTES % 1024 == 0, "stages must keep 1024-byte alignment");
// Each epilogue warp walks its 32 x 32 share in chunks of 32 rows x 16 columns.  A chunk
// passes through a shared-memory stage where row r starts at float 16 (r + r / 16) and
// its four 16-byte quads sit at quad q ^ ((r / 2) % 4): one lane per row (the
// accumulator layout), one lane per (column, row half) (the 16x1 view) and four lanes
// per row (coalesced global traffic, rows r and r + 8 i) all hit 32 distinct banks.
constexpr int kChunkCols = 16;
constexpr int kChunks = 32 / kChunkCols;        // chunks per warp and tile
constexpr int kStageFloats = 33 * 16;           // one staged chunk (2112 bytes)
constexpr int kStageBufs = 3;                   // FP32 input runs two chunks ahead
constexpr int EPI_WARP_FLOATS = kStageBufs * kStageFloats;
constexpr int BAR_BYTES = 256;
constexpr int SMEM_BYTES = 1024 + kStages * STAGE_BYTES + kEpiWarps * EPI_WARP_FLOATS * 4 + BAR_BYTES + 256 * 4;
static_assert(SMEM_BYTES <= 232448, "over the per-CTA shared-memory limit");
static_assert((3 * kStages + 6) * 8 + 12 <= BAR_BYTES, "barrier block too small");
constexpr uint32_t kIdesc = idesc_mxf4nvf4(2 * BM, BN);
constexpr float kBoundInflate = 1.0f + 1.0f / 256.0f;

struct Job {
  int mat;
  int64_t row0, col0;   // this CTA's first output row and the tile's first column
  int mirror;           // off-diagonal symmetric block
  int kt;               // number of 256-wide K tiles
  const uint8_t* a_codes; const uint8_t* a_sf;
  const uint8_t* b_codes; const uint8_t* b_sf;
};

__device__ __forceinline__ int owner_of(const int32_t* prefix, int count, int32_t u) {
  int lo = 0, hi = count - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= u) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Upper-triangle block s -> (P, Q), P <= Q, of a T x T grid, row-major.
__device__ __forceinline__ void upper_tile(int32_t s, int32_t T, int32_t& P, int32_t& Q) {
  P = 0;
  while (s >= T - P) { s -= T - P; ++P; }
  Q = P + s;
}

// Work unit u of kernel E for the CTA of rank `rank` in its pair.  A matrix's units go
// through its 256-row bands in order; inside a band, its 128-column tiles in order.
template <Epi E>
__device__ __forceinline__ Job make_job(int32_t u, const NsParams& p, uint32_t rank) {
  Job j;
  const int mi = owner_of(p.prefix, p.count, u);
  const MatDesc& d = p.mat[mi];
  const MatLayout L = mat_layout(d.mp, d.np, d.state_off, d.big_off);
  const int32_t lu = u - p.prefix[mi];
  const int slot = p.iter & 1;
  j.mat = mi;
  j.mirror = 0;
  if constexpr (E == Epi::GramX || E == Epi::GramA) {
    const int32_t T = d.mp / 256;
    int32_t P, Q;
    upper_tile(lu >> 1, T, P, Q);   // two 128-column tiles per 256 x 256 block
    j.row0 = 256 * (int64_t)P + 128 * (int64_t)rank;
    j.col0 = 256 * (int64_t)Q + 128 * (int64_t)(lu & 1);
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
    j.row0 = 256 * (int64_t)I + 128 * (int64_t)rank;
    j.col0 = (int64_t)(lu - I * nJ) * BN;
    j.kt = d.mp / BK;
    j.a_codes = p.ws + L.qB; j.a_sf = p.ws + L.sB;
    j.b_codes = p.ws + (slot ? L.qXT[1] : L.qXT[0]);
    j.b_sf = p.ws + (slot ? L.sXT[1] : L.sXT[0]);
  }
  return j;
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
// columns col0 + 32 slice + 4 (lane % 4) ...; the FP32 tile is A (GramX, GramA) or X
// (Update).
struct TileRows {
  float* base;
  uint32_t step;
};

template <Epi E>
__device__ __forceinline__ TileRows tile_rows(const NsParams& p, int32_t u, uint32_t rank, int quad,
                                              int slice, int lane) {
  const Job j = make_job<E>(u, p, rank);
  const MatDesc& d = p.mat[j.mat];
  const MatLayout L = mat_layout(d.mp, d.np, d.state_off, d.big_off);
  const int64_t pitch = (E == Epi::Update) ? d.np : d.mp;
  TileRows t;
  t.base = reinterpret_cast<float*>(p.ws + (E == Epi::Update ? L.X : L.A)) +
           (j.row0 + 32 * quad + (lane >> 2)) * pitch + j.col0 + 32 * slice + 4 * (lane & 3);
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

// Epilogue of the three Newton-Schulz products (one epilogue warp).
//   GramX   A = sX^2 acc            -> A (FP32), qA = Q1x16(A); mirrored tile: Q1x16 of A^T
//   GramA   B = b A + c sA^2 acc    -> qB = Q1x16(B);           mirrored tile: Q1x16 of B^T
//   Update  X' = a X + sB sX acc    -> X' (FP32), Q1x16(X'), Q16x1(X') (or the output, last)
template <Epi E, uint32_t kOpts>
__device__ __forceinline__ void epilogue_ns(const NsParams& p, uint32_t tmem, uint64_t* acc_full,
                                            uint64_t* acc_empty, uint32_t rank, uint32_t* status,
                                            volatile int* abort_flag, float* wbuf,
                                            const float* scale_tab, int quad, int slice, int lane,
                                            int32_t first, int32_t step, int32_t total) {
  constexpr bool kIn = (E == Epi::GramA || E == Epi::Update);   // reads an FP32 tile
  constexpr bool kRht = (kOpts & kOptRht) != 0;    // Hadamard transform before quantising
  constexpr bool k46 = (kOpts & kOpt46) != 0;      // adaptive 4/6 block scaling
  // H16^r masks of the tensors this epilogue quantises (Section 3.4): GramX -> qA (product
  // qA qA^T of iteration k), GramA -> qB (update product of iteration k), Update -> the
  // next iterate's Gram view and update view (iteration k + 1)
  const int k = p.iter;
  const uint32_t mask_row = E == Epi::GramX ? p.rht[3 * k + 1]
                           : E == Epi::GramA ? p.rht[3 * k + 2]
                                             : (k + 1 < kMaxIters ? p.rht[3 * (k + 1)] : 0u);
  const uint32_t mask_col = E == Epi::Update ? (k + 1 < kMaxIters ? p.rht[3 * (k + 1) + 2] : 0u)
                                             : mask_row;
  const int cc = lane & 15, hh = lane >> 4;
  TileRows fp{nullptr, 0u};   // FP32 tile rows of the current tile
  TileRows fn{nullptr, 0u};   // ... of the next tile (fetched ahead)
  if constexpr (kIn) {
    if (first < total) {
      fp = tile_rows<E>(p, first, rank, quad, slice, lane);
      stage_fetch(wbuf, fp, 0, lane);
      cp_async_commit();
      stage_fetch(wbuf + kStageFloats, fp, 1, lane);
      cp_async_commit();
    }
  }
  int b = 0;   // stage buffer of the current chunk
  uint32_t tl = 0;
  for (int32_t u = first; u < total; u += step, ++tl) {
    const Job j = make_job<E>(u, p, rank);
    const MatDesc& d = p.mat[j.mat];
    NsState* st = reinterpret_cast<NsState*>(p.ws + d.state_off);
    const MatLayout L = mat_layout(d.mp, d.np, d.state_off, d.big_off);
    if constexpr (!kIn) fp = tile_rows<E>(p, u, rank, quad, slice, lane);
    const uint32_t buf_i = tl & 1u;
    // One lane polls the barrier; the warp then synchronises, which with
    // tcgen05.fence::after_thread_sync below orders every lane's accumulator loads after
    // the MMAs.  Warp-uniform by construction: the chunk loop shuffles under it.
    const bool ok = __shfl_sync(0xFFFFFFFFu,
                                lane == 0 ? (mbar_wait(&acc_full[buf_i], (tl >> 1) & 1u, status, abort_flag) ? 1 : 0) : 0,
                                0) != 0;
    __syncwarp();
    const int64_t gr0 = j.row0 + 32 * quad;   // first row of this warp's band
    const int64_t gr = gr0 + lane;             // this lane's row
    const int64_t gc0 = j.col0 + 32 * slice;   // first column of this warp's share
    const bool last = (E == Epi::Update) && p.last;

    float acc_scale, sg_out;
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

    // this warp's 32 x 32 share of the accumulator, loaded at once; the buffer is
    // handed back before any element-wise work
    uint32_t accr[32];
    if (ok) {
      tc_fence_after();
      const uint32_t taddr = tmem + ((uint32_t)(32 * quad) << 16) + kAccCols * buf_i + (uint32_t)(32 * slice);
      tmem_ld32_async(taddr, accr);
      tmem_wait_ld32(accr);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0) mbar_arrive(&acc_empty[buf_i]);
        else mbar_arrive_cluster(&acc_empty[buf_i], 0);
      }
    }

    float row_acc = 0.0f, amax = 0.0f;
    uint32_t prev_w0 = 0u, prev_w1 = 0u, scale_word = 0u;
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
      float* sbuf = wbuf + b * kStageFloats;
      if constexpr (kIn) {
        cp_async_wait<1>();   // this chunk's rows have landed (own copies) ...
        __syncwarp();         // ... and every lane's
      }
      if (ok) {
        const int64_t gcc = gc0 + kChunkCols * c;   // first column of the chunk
        float y[16];
        const uint64_t s2 = f2_pack(acc_scale, acc_scale);
        if constexpr (E == Epi::Update) {
          float xin[16];
          stage_load_row(sbuf, lane, xin);
#pragma unroll
          for (int e = 0; e < 16; ++e)
            y[e] = fmaf(d.a, xin[e], __uint_as_float(accr[16 * c + e]) * acc_scale);
        } else if constexpr (kIn) {
          // GramA: b A + c (s acc)   (pairs of columns at a time)
          float xin[16];
          stage_load_row(sbuf, lane, xin);
          const uint64_t ca = f2_pack(d.b, d.b);
          const uint64_t cc2 = f2_pack(d.c, d.c);
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            uint64_t v = f2_mul(f2_pack(__uint_as_float(accr[16 * c + e]),
                                        __uint_as_float(accr[16 * c + e + 1])), s2);
            v = f2_mul(cc2, v);
            f2_unpack(f2_fma(ca, f2_pack(xin[e], xin[e + 1]), v), y[e], y[e + 1]);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 16; e += 2)
            f2_unpack(f2_mul(f2_pack(__uint_as_float(accr[16 * c + e]),
                                     __uint_as_float(accr[16 * c + e + 1])), s2),
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
            stage_store_row(sbuf, lane, y);
            __syncwarp();
            float xc[16];
            stage_load_col(sbuf, cc, hh, xc);
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
            stage_store_row(sbuf, lane, y);
            __syncwarp();
          }
          if constexpr (E != Epi::GramA) stage_flush(sbuf, fp, c, lane);   // A or X' (FP32)
          else if (dbg_b) stage_flush(sbuf, fp, c, lane);
          // 1x16 view along this lane's row and, where needed, the 16x1 view of column
          // gcc + cc, rows gr0 + 16 hh ..: two independent quantiser chains side by side
          QBlock16 q, qc;
          float yamax = 0.0f;   // max |X'| of the untransformed block (update bound)
          if constexpr (kRht && E == Epi::Update) yamax = absmax16(y);
          if constexpr (kRht) rht16(y, mask_row);
          if (need_col) {
            float xc[16];
            stage_load_col(sbuf, cc, hh, xc);
            if constexpr (kRht) rht16(xc, mask_col);
            q = quantize16<true, true, true, k46>(y, sg_out, six_out, rcp_six, stab);
            qc = quantize16<true, true, true, k46>(xc, sg_out, six_out, rcp_six, stab);
          } else {
            q = quantize16<true, true, true, k46>(y, sg_out, six_out, rcp_six, stab);
          }
          row_acc += q.sumsq;
          amax = fmaxf(amax, kRht ? yamax : q.amax);
          if (c == 1) {
            // the two chunks of the row form one 16-byte code chunk and two scale bytes
            *reinterpret_cast<uint4*>(row_codes + tiled_chunk_offset(gr, gc0, row_cp)) =
                make_uint4(prev_w0, prev_w1, q.w0, q.w1);
            *reinterpret_cast<uint16_t*>(row_scales + tiled_scale_offset(gr, gc0 >> 4, row_cp)) =
                static_cast<uint16_t>(scale_word | (q.scale << 8));
          } else {
            prev_w0 = q.w0;
            prev_w1 = q.w1;
            scale_word = q.scale;
          }
          if (need_col) {
            // the two row halves of one column pair up into a 16-byte code chunk
            const uint32_t o0 = __shfl_xor_sync(0xFFFFFFFFu, qc.w0, 16);
            const uint32_t o1 = __shfl_xor_sync(0xFFFFFFFFu, qc.w1, 16);
            const uint32_t os = __shfl_xor_sync(0xFFFFFFFFu, qc.scale, 16);
            const float s2c = qc.sumsq + __shfl_xor_sync(0xFFFFFFFFu, qc.sumsq, 16);
            if (hh == 0) {
              const int64_t rt = gcc + cc;
              *reinterpret_cast<uint4*>(col_codes + tiled_chunk_offset(rt, gr0, d.mp)) =
                  make_uint4(qc.w0, qc.w1, o0, o1);
              *reinterpret_cast<uint16_t*>(col_scales + tiled_scale_offset(rt, gr0 >> 4, d.mp)) =
                  static_cast<uint16_t>(qc.scale | (os << 8));
              if (s2c != 0.0f) atomicAdd(colsum + rt, s2c);
            }
          }
        }
      }
      __syncwarp();   // every lane is done with this stage buffer
      if constexpr (kIn) {
        // fetch chunk c + 2 (of the next tile) into the buffer chunk c - 1 used
        float* nb = wbuf + (b == 0 ? 2 : b - 1) * kStageFloats;
        if (u + step < total) {
          if (c == 0) fn = tile_rows<E>(p, u + step, rank, quad, slice, lane);
          stage_fetch(nb, fn, c, lane);
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

template <Epi E, uint32_t kOpts>
__global__ void __launch_bounds__(kThreads, 1)
    nvfp4_ns_pair_kernel(const __grid_constant__ NsParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  float* epi_smem = reinterpret_cast<float*>(smem + kStages * STAGE_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * STAGE_BYTES + kEpiWarps * EPI_WARP_FLOATS * 4);
  uint64_t* full = bars;                      // this CTA's operand stage landed
  uint64_t* empty = bars + kStages;           // the MMAs reading a stage finished
  uint64_t* peer_full = bars + 2 * kStages;   // (leader) the peer's stage landed
  uint64_t* acc_full = bars + 3 * kStages;    // [2] an accumulator buffer is complete
  uint64_t* acc_empty = acc_full + 2;         // [2] (leader) both CTAs drained a buffer
  uint64_t* mma_done = acc_full + 4;
  uint64_t* stall_bar = acc_full + 5;         // test only: never arrived on
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 6);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);
  float* scale_tab = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + BAR_BYTES);
  if (threadIdx.x >= 128 && threadIdx.x < 256) scale_tab_fill(scale_tab, threadIdx.x - 128);

  uint32_t* status = p.status;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int32_t first = (int32_t)(blockIdx.x >> 1), step = (int32_t)(gridDim.x >> 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&peer_full[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 2 * kEpiWarps);
    }
    mbar_init(mma_done, 1);
    mbar_init(stall_bar, 1);
    *abort_flag = (__ldcg(status) & kStatusTimeout) ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, kTmemCols);
  tc_fence_before();
  cluster_sync();   // the peer's barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int32_t total = p.prefix[p.count];
  if (warp < 4) {
    regs_dec<kRegsCtl>();
    if (warp == 0) {
      // ------------------------------------------------------------ producer
      if (lane == 0) {
        uint32_t it = 0;
        for (int32_t u = first; u < total && !*abort_flag; u += step) {
          const Job j = make_job<E>(u, p, rank);
          const int64_t a_row = j.row0 / 128, b_row = j.col0 / 128;
          for (int kt = 0; kt < j.kt; ++kt, ++it) {
            const uint32_t s = it % kStages, use = it / kStages;
            if (!mbar_wait(&empty[s], (use & 1u) ^ 1u, status, abort_flag)) break;
            uint8_t* st = stage_base + s * STAGE_BYTES;
            const int64_t at = a_row * j.kt + kt, bt = b_row * j.kt + kt;
            mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
            bulk_g2s(st, j.a_codes + at * kTileBytes, A_BYTES, &full[s]);
            bulk_g2s(st + A_BYTES, j.b_codes + bt * kTileBytes + rank * B_BYTES, B_BYTES, &full[s]);
            bulk_g2s(st + A_BYTES + B_BYTES, j.a_sf + at * (4 * kAtomBytes), SFA_BYTES, &full[s]);
            bulk_g2s(st + A_BYTES + B_BYTES + SFA_BYTES, j.b_sf + bt * (4 * kAtomBytes), SFB_BYTES,
                     &full[s]);
          }
        }
        // drain: every issued copy must land before the CTA may exit
        const uint32_t from = it > (uint32_t)kStages ? it - kStages : 0u;
        for (uint32_t k = from; k < it; ++k) {
          volatile int never = 0;
          mbar_wait(&full[k % kStages], (k / kStages) & 1u, status, &never);
        }
      }
    } else if (warp == 1 && rank != 0) {
      // ---------------------------------------------------------- relay (pair's peer)
      // Tell the leader's MMA thread each time one of this CTA's stages has landed.
      if (lane == 0) {
        uint32_t it = 0;
        bool ok = true;
        for (int32_t u = first; u < total && ok && !*abort_flag; u += step) {
          const Job j = make_job<E>(u, p, rank);
          for (int kt = 0; kt < j.kt; ++kt, ++it) {
            const uint32_t s = it % kStages, use = it / kStages;
            if (!mbar_wait(&full[s], use & 1u, status, abort_flag)) { ok = false; break; }
            mbar_arrive_cluster(&peer_full[s], 0);
          }
        }
      }
    } else if (warp == 1) {
      if (lane == 0) {
        // -------------------------------------------------------- MMA issuer (leader)
        // operands and accumulators of each CTA stay in that CTA; commits arrive on
        // the barriers of both
        uint32_t it = 0, tl = 0;
        if (p.stall) mbar_wait(stall_bar, 0, status, abort_flag);   // test only
        for (int32_t u = first; u < total && !*abort_flag; u += step, ++tl) {
          const Job j = make_job<E>(u, p, rank);
          const uint32_t buf_i = tl & 1u;
          if (!mbar_wait(&acc_empty[buf_i], ((tl >> 1) & 1u) ^ 1u, status, abort_flag)) break;
          tc_fence_after();
          const uint32_t acc = tmem + kAccCols * buf_i;
          bool ok = true;
          for (int kt = 0; kt < j.kt; ++kt, ++it) {
            const uint32_t s = it % kStages, use = it / kStages;
            if (!mbar_wait(&full[s], use & 1u, status, abort_flag)) { ok = false; break; }
            if (!mbar_wait(&peer_full[s], use & 1u, status, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint8_t* st = stage_base + s * STAGE_BYTES;
            const uint32_t sa = smem_addr(st), sb = sa + A_BYTES;
            const uint32_t ssfa = sb + B_BYTES, ssfb = ssfa + SFA_BYTES;
            const uint32_t sf = tmem + kSfCol + (it & 1u) * kSfBufCols;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              tc_copy_sf_pair(sf + 4 * ks, sdesc_sf_atom(ssfa + ks * kAtomBytes));
              tc_copy_sf_pair(sf + 16 + 4 * ks, sdesc_sf_atom(ssfb + ks * kAtomBytes));
            }
            const uint64_t da = sdesc_sw128(sa), db = sdesc_sw128(sb);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              tc_mma_nvf4_pair(acc, da + 2 * ks, db + 2 * ks, kIdesc, sf + 4 * ks, sf + 16 + 4 * ks,
                               (kt | ks) != 0 ? 1u : 0u);
            }
            tc_commit_pair(&empty[s], 3);
          }
          if (!ok) break;
          tc_commit_pair(&acc_full[buf_i], 3);
        }
        tc_commit_pair(mma_done, 1);
        volatile int never = 0;
        mbar_wait(mma_done, 0, status, &never);
      }
    }
  } else {
    regs_inc<kRegsEpi>();
    // ------------------------------------------------------------ epilogue
    // Every epilogue warp walks the same tile list and never leaves it early (a
    // failed wait only skips that tile's work), so the cluster-wide barrier at the
    // end is reached by all threads.
    const int ew = warp - 4;          // 0..15
    const int quad = warp & 3;        // TMEM lanes 32*quad .. 32*quad+31
    const int slice = ew >> 2;        // 32-column slice of the 128-column tile
    float* wbuf = epi_smem + ew * EPI_WARP_FLOATS;
    epilogue_ns<E, kOpts>(p, tmem, acc_full, acc_empty, rank, status, abort_flag, wbuf, scale_tab,
                          quad, slice, lane, first, step, total);
  }

  tc_fence_before();
  // both CTAs of a pair are done with the TMEM (the leader's MMAs completed before
  // its MMA thread got here) before either frees it
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
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

template <Epi E, uint32_t kOpts>
cudaError_t launch_impl(const NsParams& p, cudaStream_t st, int num_sms) {
  static unsigned long long attr_set = 0ull;   // one bit per device; a benign race
  static int max_pairs[64] = {};               // co-resident CTA pairs per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  auto kern = nvfp4_ns_pair_kernel<E, kOpts>;
  if (!(attr_set & (1ull << dev))) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set |= 1ull << dev;
  }
  // setmaxnreg.inc can only hand out what the block was launched with: refuse to
  // launch unless the compiled register count is exactly the split's budget
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if ((uint32_t)fa.numRegs != kRegsLaunch) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (max_pairs[dev] == 0) {
    cfg.gridDim = dim3(2 * (num_sms / 2), 1, 1);
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
    if (e != cudaSuccess) return e;
    if (n < 1) return cudaErrorInvalidConfiguration;
    max_pairs[dev] = n;
  }
  const int64_t units = p.prefix[p.count];
  const int64_t pairs = units < max_pairs[dev] ? (units > 0 ? units : 1) : max_pairs[dev];
  cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
  e = cudaLaunchKernelEx(&cfg, kern, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <uint32_t kOpts>
cudaError_t launch_ns_opts(Epi epi, const NsParams& p, cudaStream_t st, int num_sms) {
  cudaError_t e;
  switch (epi) {
    case Epi::GramX:
      if ((e = launch_impl<Epi::GramX, kOpts>(p, st, num_sms)) != cudaSuccess) return e;
      ns_bounds_kernel<Epi::GramX><<<p.count, 256, 0, st>>>(p);
      break;
    case Epi::GramA:
      if ((e = launch_impl<Epi::GramA, kOpts>(p, st, num_sms)) != cudaSuccess) return e;
      ns_bounds_kernel<Epi::GramA><<<p.count, 256, 0, st>>>(p);
      break;
    case Epi::Update:
      if ((e = launch_impl<Epi::Update, kOpts>(p, st, num_sms)) != cudaSuccess) return e;
      if (!p.last) ns_bounds_kernel<Epi::Update><<<p.count, 256, 0, st>>>(p);
      break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_ns(Epi epi, const NsParams& p, cudaStream_t st, int num_sms) {
  switch (p.opts & (kOptRht | kOpt46)) {
    case 0: return launch_ns_opts<0>(epi, p, st, num_sms);
    case kOpt46: return launch_ns_opts<kOpt46>(epi, p, st, num_sms);
    case kOptRht: return launch_ns_opts<kOptRht>(epi, p, st, num_sms);
    default: return launch_ns_opts<kOptRht | kOpt46>(epi, p, st, num_sms);
  }
}

}  // namespace fs4
