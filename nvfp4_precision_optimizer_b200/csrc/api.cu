// C ABI of libfs4 (declared in include/fs4.h): argument validation, workspace
// planning and the launch sequence of the direct NVFP4 Newton-Schulz step.
#include <cmath>
#include <cstring>
#include <mutex>

#include "../../include/fs4.h"
#include "fs4_device.cuh"
#include "fs4_internal.h"

using namespace fs4;

namespace {

struct DeviceInfo {
  bool valid = false;
  bool arch_ok = false;
  int num_sms = 0;
};

std::mutex g_dev_mu;
DeviceInfo g_dev[64];

fs4_status device_info(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FS4_ERR_CUDA;
  if (dev < 0 || dev >= 64) return FS4_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (!g_dev[dev].valid) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return FS4_ERR_CUDA;
    g_dev[dev].arch_ok = (major == 10 && minor == 0);
    g_dev[dev].num_sms = sms;
    g_dev[dev].valid = true;
  }
  *out = g_dev[dev];
  return out->arch_ok ? FS4_OK : FS4_ERR_ARCH;
}

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline fs4_status cuda_status(cudaError_t e) { return e == cudaSuccess ? FS4_OK : FS4_ERR_CUDA; }

// Byte range [lo, hi) covered by a rows x cols matrix with leading dimension ld.
inline void span(const void* base, int64_t rows, int64_t cols, int64_t ld, uintptr_t* lo,
                 uintptr_t* hi) {
  *lo = reinterpret_cast<uintptr_t>(base);
  *hi = *lo + (uintptr_t)(((rows - 1) * ld + cols) * 4);
}

struct Plan {
  int32_t count = 0;
  MatDesc mat[kMaxBatch];
  int64_t units_reduce[kMaxBatch], units_pre[kMaxBatch], units_gram[kMaxBatch], units_upd[kMaxBatch];
  int64_t zero_bytes = 0;   // header + state blocks, zeroed at the start of a call
  int64_t total_bytes = 0;
};

fs4_status validate_desc(const fs4_ns_desc& d, const fs4_nvfp4_state* st, bool sizing) {
  if (sizing) {   // workspace size / layout queries: shapes only
    if (d.m < 16 || d.n < 16 || d.m > FS4_MAX_DIM || d.n > FS4_MAX_DIM) return FS4_ERR_SHAPE;
    if (d.m % 16 || d.n % 16) return FS4_ERR_SHAPE;
    return FS4_OK;
  }
  if (st) {   // NVFP4 source: G is not read
    if (d.G || !st->codes || !st->scales || !st->s_g || st->mask > 0xFFFFu) return FS4_ERR_INVALID_ARG;
    if (!aligned(st->codes, 16) || !aligned(st->scales, 16) || !aligned(st->s_g, 4)) return FS4_ERR_INVALID_ARG;
  } else if (!d.G) {
    return FS4_ERR_INVALID_ARG;
  }
  if (!d.out) return FS4_ERR_INVALID_ARG;
  if (d.m < 16 || d.n < 16 || d.m > FS4_MAX_DIM || d.n > FS4_MAX_DIM) return FS4_ERR_SHAPE;
  if (d.m % 16 || d.n % 16) return FS4_ERR_SHAPE;
  if ((!st && d.ld < d.n) || d.ld_out < d.n) return FS4_ERR_INVALID_ARG;
  if (!std::isfinite(d.a) || !std::isfinite(d.b) || !std::isfinite(d.c)) return FS4_ERR_INVALID_ARG;
  if ((!st && !aligned(d.G, 4)) || !aligned(d.out, 4)) return FS4_ERR_INVALID_ARG;
  return FS4_OK;
}

// Lay out the workspace: [header | state blocks of all matrices | big buffers of all matrices].
fs4_status make_plan(int32_t count, const fs4_ns_desc* descs, Plan* pl,
                     const fs4_nvfp4_state* states = nullptr, bool sizing = false, bool bf16 = false) {
  if (count < 1 || count > kMaxBatch) return FS4_ERR_SHAPE;
  if (!descs) return FS4_ERR_INVALID_ARG;
  pl->count = count;
  int64_t off = kHeaderBytes;
  for (int i = 0; i < count; ++i) {
    const fs4_ns_desc& d = descs[i];
    const fs4_status s = validate_desc(d, states ? &states[i] : nullptr, sizing);
    if (s != FS4_OK) return s;
    MatDesc& md = pl->mat[i];
    md.G = d.G;
    md.out = d.out;
    md.ldg = states ? d.n : d.ld;
    md.qcodes = states ? states[i].codes : nullptr;
    md.qscales = states ? states[i].scales : nullptr;
    md.qsg = states ? states[i].s_g : nullptr;
    md.qmask = states ? states[i].mask : 0u;
    md.ldo = d.ld_out;
    md.tall = d.m > d.n ? 1 : 0;
    md.m = (int32_t)(md.tall ? d.n : d.m);
    md.n = (int32_t)(md.tall ? d.m : d.n);
    md.mp = (int32_t)align_up(md.m, kPad);
    md.np = (int32_t)align_up(md.n, kPad);
    md.a = d.a; md.b = d.b; md.c = d.c;
    md.state_off = off;
    off += state_block_bytes(md.mp, md.np);
    pl->units_reduce[i] = (d.m + 15) / 16;
    pl->units_pre[i] = (int64_t)(md.mp / 64) * (md.np / 64);
    const int64_t T = md.mp / 256;
    // GEMM units: 128 x 256 tiles (Gram products: on and above the 256-block diagonal)
    pl->units_gram[i] = T * (T + 1);
    pl->units_upd[i] = (int64_t)(md.mp / 128) * (md.np / 256);
  }
  pl->zero_bytes = align_up(off, 1024);
  off = pl->zero_bytes;
  for (int i = 0; i < count; ++i) {
    pl->mat[i].big_off = off;
    off += align_up(big_block_bytes(pl->mat[i].mp, pl->mat[i].np, bf16), 1024);
  }
  pl->total_bytes = off;
  if (sizing) return FS4_OK;
  // outputs must not overlap any input or any other output
  for (int i = 0; i < count; ++i) {
    uintptr_t olo, ohi;
    span(descs[i].out, descs[i].m, descs[i].n, descs[i].ld_out, &olo, &ohi);
    for (int k = 0; k < count; ++k) {
      uintptr_t glo, ghi;
      if (states) {   // the NVFP4 codes and scales are the inputs
        glo = reinterpret_cast<uintptr_t>(states[k].codes);
        ghi = glo + (uintptr_t)(descs[k].m * descs[k].n / 2);
        if (olo < ghi && glo < ohi) return FS4_ERR_ALIAS;
        glo = reinterpret_cast<uintptr_t>(states[k].scales);
        ghi = glo + (uintptr_t)(descs[k].m * descs[k].n / 16);
      } else {
        span(descs[k].G, descs[k].m, descs[k].n, descs[k].ld, &glo, &ghi);
      }
      if (olo < ghi && glo < ohi) return FS4_ERR_ALIAS;
      if (k != i) {
        span(descs[k].out, descs[k].m, descs[k].n, descs[k].ld_out, &glo, &ghi);
        if (olo < ghi && glo < ohi) return FS4_ERR_ALIAS;
      }
    }
  }
  return FS4_OK;
}

bool fill_prefix(NsParams& p, const int64_t* units) {
  int64_t acc = 0;
  p.prefix[0] = 0;
  for (int i = 0; i < p.count; ++i) {
    acc += units[i];
    if (acc > 0x7FFFFFFF) return false;
    p.prefix[i + 1] = (int32_t)acc;
  }
  return true;
}

// Reused parameter block: 19 KB, too large for the stack of every caller thread.
thread_local NsParams t_params;

fs4_status run_ns(const Plan& pl, int32_t K, float clip_k, uint32_t flags, const uint16_t* rht_masks,
                  uint8_t* ws,
                  cudaStream_t st, int num_sms, void* const* events = nullptr, bool bf16 = false) {
  int ev_i = 0;
  auto mark = [&]() -> bool {
    if (!events) return true;
    return cudaEventRecord(static_cast<cudaEvent_t>(events[ev_i++]), st) == cudaSuccess;
  };
  const int stop = (int)((flags >> 8) & 0xFF) - 1;   // -1: run everything
  NsParams& p = t_params;
  std::memset(&p, 0, sizeof(p));
  p.count = pl.count;
  p.clip_k = clip_k;
  p.status = reinterpret_cast<uint32_t*>(ws);
  p.ws = ws;
  p.opts = ((flags & FS4_NS_RHT) ? kOptRht : 0u) | ((flags & FS4_NS_ADAPTIVE46) ? kOpt46 : 0u) |
           ((flags & FS4_NS_CLIP_QUANTILE) ? kOptQuantile : 0u) |
           (pl.mat[0].qcodes ? kOptNvSrc : 0u) |  // a call's matrices are all FP32 or all NVFP4
           (bf16 ? kOptBf16 : 0u);
  if (flags & FS4_NS_RHT)
    for (int i = 0; i < 3 * K; ++i) p.rht[i] = rht_masks[i];
  std::memcpy(p.mat, pl.mat, sizeof(MatDesc) * pl.count);

  if (!mark()) return FS4_ERR_CUDA;
  cudaError_t e = cudaMemsetAsync(ws, 0, (size_t)pl.zero_bytes, st);
  if (e != cudaSuccess) return FS4_ERR_CUDA;
  if (!fill_prefix(p, pl.units_reduce)) return FS4_ERR_SHAPE;
  if ((e = launch_ns_reduce(p, st, num_sms)) != cudaSuccess) return FS4_ERR_CUDA;
  if ((p.opts & kOptQuantile) && (e = launch_ns_quantile(p, st, num_sms)) != cudaSuccess)
    return FS4_ERR_CUDA;
  if (!mark()) return FS4_ERR_CUDA;
  if (!fill_prefix(p, pl.units_pre)) return FS4_ERR_SHAPE;
  if ((e = launch_ns_preamble(p, st, num_sms)) != cudaSuccess) return FS4_ERR_CUDA;
  if (!mark()) return FS4_ERR_CUDA;
  if (stop == 0) return FS4_OK;
  // 8192-class batches (FLOP-weighted mean of the short side m at least 6144): the products'
  // mainloops outlast their epilogues, and the kernels variant with more scale-factor
  // copier threads is the faster one
  {
    double wsum = 0.0, wm = 0.0;
    for (int i = 0; i < pl.count; ++i) {
      const double m = (double)pl.mat[i].m, w = m * m * (double)pl.mat[i].n;
      wsum += w;
      wm += w * m;
    }
    if (wsum > 0.0 && wm >= 6144.0 * wsum) p.opts |= kOptWideK;
  }
  for (int k = 0; k < K; ++k) {
    p.iter = k;
    p.last = 0;
    if (!fill_prefix(p, pl.units_gram)) return FS4_ERR_SHAPE;
    p.stall = (k == 0 && (flags & FS4_TEST_STALL)) ? 1 : 0;
    if ((e = launch_gemm_ns(Epi::GramX, p, st, num_sms)) != cudaSuccess) return FS4_ERR_CUDA;
    p.stall = 0;
    if (!mark()) return FS4_ERR_CUDA;
    if (stop == 1 + 3 * k) return FS4_OK;
    p.dbg_b = (stop == 2 + 3 * k) ? 1 : 0;
    if ((e = launch_gemm_ns(Epi::GramA, p, st, num_sms)) != cudaSuccess) return FS4_ERR_CUDA;
    p.dbg_b = 0;
    if (!mark()) return FS4_ERR_CUDA;
    if (stop == 2 + 3 * k) return FS4_OK;
    p.last = (k == K - 1) ? 1 : 0;
    if (!fill_prefix(p, pl.units_upd)) return FS4_ERR_SHAPE;
    if ((e = launch_gemm_ns(Epi::Update, p, st, num_sms)) != cudaSuccess) return FS4_ERR_CUDA;
    if (!mark()) return FS4_ERR_CUDA;
    if (stop == 3 + 3 * k) return FS4_OK;
  }
  return FS4_OK;
}

}  // namespace

extern "C" {

size_t fs4_nvfp4_quantize_workspace_size(void) { return kHeaderBytes; }

size_t fs4_momentum_workspace_size(void) { return kHeaderBytes; }

fs4_status fs4_momentum_nvfp4(const float* g, int64_t rows, int64_t cols, int64_t ld,
                              float beta, const uint8_t* prev_codes,
                              const uint8_t* prev_scales, const float* prev_sg,
                              uint32_t prev_mask, uint8_t* codes, uint8_t* scales, float* s_g,
                              uint32_t mask, uint64_t seed, float* m_out, int64_t ld_out,
                              void* workspace, size_t workspace_bytes, void* stream) {
  if (!g || !codes || !scales || !s_g) return FS4_ERR_INVALID_ARG;
  const int nprev = (prev_codes != nullptr) + (prev_scales != nullptr) + (prev_sg != nullptr);
  if (nprev != 0 && nprev != 3) return FS4_ERR_INVALID_ARG;
  if (!std::isfinite(beta) || prev_mask > 0xFFFFu || mask > 0xFFFFu) return FS4_ERR_INVALID_ARG;
  if (rows < 1 || cols < 16 || rows > (1ll << 31) || cols > (1ll << 31) || cols % 16) return FS4_ERR_SHAPE;
  if (ld < cols || (m_out && ld_out < cols)) return FS4_ERR_INVALID_ARG;
  if (!aligned(g, 4) || (m_out && !aligned(m_out, 4)) || !aligned(codes, 16) || !aligned(scales, 16) ||
      !aligned(s_g, 4) || (prev_codes && (!aligned(prev_codes, 16) || !aligned(prev_sg, 4))))
    return FS4_ERR_INVALID_ARG;
  if (m_out) {
    uintptr_t glo, ghi, olo, ohi;
    span(g, rows, cols, ld, &glo, &ghi);
    span(m_out, rows, cols, ld_out, &olo, &ohi);
    if (olo < ghi && glo < ohi) return FS4_ERR_ALIAS;
  }
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < kHeaderBytes) return FS4_ERR_WORKSPACE;
  DeviceInfo di;
  const fs4_status ds = device_info(&di);
  if (ds != FS4_OK) return ds;
  return cuda_status(launch_momentum(g, rows, cols, ld, beta, prev_codes, prev_scales, prev_sg,
                                     prev_mask, codes, scales, s_g, mask, seed, m_out, ld_out,
                                     static_cast<uint8_t*>(workspace),
                                     static_cast<cudaStream_t>(stream), di.num_sms));
}

fs4_status fs4_nvfp4_quantize(const float* x, int64_t rows, int64_t cols, int64_t ld, int32_t axis,
                              uint8_t* codes, uint8_t* scales, float* s_g, uint32_t flags,
                              void* workspace, size_t workspace_bytes, void* stream) {
  if (!x || !codes || !scales || !s_g) return FS4_ERR_INVALID_ARG;
  if (axis != FS4_AXIS_ROW && axis != FS4_AXIS_COL) return FS4_ERR_INVALID_ARG;
  if (flags & ~(uint32_t)(FS4_SG_AMAX | FS4_LAYOUT_TILED | FS4_TEST_STALL)) return FS4_ERR_INVALID_ARG;
  if (rows < 1 || cols < 1 || rows > (1ll << 31) || cols > (1ll << 31)) return FS4_ERR_SHAPE;
  if ((axis == FS4_AXIS_ROW ? cols : rows) % 16) return FS4_ERR_SHAPE;
  if (ld < cols) return FS4_ERR_INVALID_ARG;
  if (!aligned(codes, 16) || !aligned(scales, 16) || !aligned(s_g, 4) || !aligned(x, 4))
    return FS4_ERR_INVALID_ARG;
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < kHeaderBytes) return FS4_ERR_WORKSPACE;
  DeviceInfo di;
  const fs4_status ds = device_info(&di);
  if (ds != FS4_OK) return ds;
  return cuda_status(launch_quantize(x, rows, cols, ld, axis, codes, scales, s_g, flags,
                                     static_cast<uint8_t*>(workspace),
                                     static_cast<cudaStream_t>(stream), di.num_sms));
}

size_t fs4_nvfp4_quantize_batched_workspace_size(int32_t count) {
  if (count < 1 || count > kMaxBatch) return 0;
  return quantize_batched_workspace_bytes(count);
}

fs4_status fs4_nvfp4_quantize_batched(int32_t count, const fs4_quant_desc* descs, uint32_t flags,
                                      void* workspace, size_t workspace_bytes, void* stream) {
  if (!descs) return FS4_ERR_INVALID_ARG;
  if (count < 1 || count > kMaxBatch) return FS4_ERR_SHAPE;
  if (flags & ~(uint32_t)(FS4_SG_AMAX | FS4_LAYOUT_TILED | FS4_TEST_STALL)) return FS4_ERR_INVALID_ARG;
  static thread_local QuantDesc qd[kMaxBatch];
  for (int i = 0; i < count; ++i) {
    const fs4_quant_desc& d = descs[i];
    if (!d.x || !d.codes || !d.scales || !d.s_g) return FS4_ERR_INVALID_ARG;
    if (d.axis != FS4_AXIS_ROW && d.axis != FS4_AXIS_COL) return FS4_ERR_INVALID_ARG;
    if (d.rows < 1 || d.cols < 1 || d.rows > (1ll << 31) || d.cols > (1ll << 31)) return FS4_ERR_SHAPE;
    if ((d.axis == FS4_AXIS_ROW ? d.cols : d.rows) % 16) return FS4_ERR_SHAPE;
    if (d.ld < d.cols) return FS4_ERR_INVALID_ARG;
    if (!aligned(d.codes, 16) || !aligned(d.scales, 16) || !aligned(d.s_g, 4) || !aligned(d.x, 4))
      return FS4_ERR_INVALID_ARG;
    qd[i].x = d.x; qd[i].rows = d.rows; qd[i].cols = d.cols; qd[i].ld = d.ld; qd[i].axis = d.axis;
    qd[i].codes = d.codes; qd[i].scales = d.scales; qd[i].s_g = d.s_g;
  }
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < quantize_batched_workspace_bytes(count))
    return FS4_ERR_WORKSPACE;
  DeviceInfo di;
  const fs4_status ds = device_info(&di);
  if (ds != FS4_OK) return ds;
  return cuda_status(launch_quantize_batched(count, qd, flags, static_cast<uint8_t*>(workspace),
                                             static_cast<cudaStream_t>(stream), di.num_sms));
}

fs4_status fs4_nvfp4_dequantize(const uint8_t* codes, const uint8_t* scales, const float* s_g,
                                int64_t rows, int64_t cols, float* y, int64_t ld, uint32_t flags,
                                void* stream) {
  if (!codes || !scales || !s_g || !y) return FS4_ERR_INVALID_ARG;
  if (flags & ~(uint32_t)FS4_LAYOUT_TILED) return FS4_ERR_INVALID_ARG;
  if (rows < 1 || cols < 1 || rows > (1ll << 31) || cols > (1ll << 31) || cols % 16) return FS4_ERR_SHAPE;
  if (ld < cols) return FS4_ERR_INVALID_ARG;
  if (!aligned(codes, 16) || !aligned(scales, 16) || !aligned(y, 4)) return FS4_ERR_INVALID_ARG;
  DeviceInfo di;
  const fs4_status ds = device_info(&di);
  if (ds != FS4_OK) return ds;
  return cuda_status(launch_dequantize(codes, scales, s_g, rows, cols, y, ld, flags,
                                       static_cast<cudaStream_t>(stream), di.num_sms));
}

fs4_status fs4_nvfp4_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_sg,
                          const uint8_t* b_codes, const uint8_t* b_scales, const float* b_sg,
                          int64_t M, int64_t N, int64_t K, float* d, int64_t ldd, void* workspace,
                          size_t workspace_bytes, void* stream) {
  if (!a_codes || !a_scales || !a_sg || !b_codes || !b_scales || !b_sg || !d) return FS4_ERR_INVALID_ARG;
  if (M < 1 || N < 1 || K < 1 || M > FS4_MAX_DIM || N > FS4_MAX_DIM || K > FS4_MAX_DIM) return FS4_ERR_SHAPE;
  if (ldd < N) return FS4_ERR_INVALID_ARG;
  if (!aligned(a_codes, 16) || !aligned(a_scales, 16) || !aligned(b_codes, 16) ||
      !aligned(b_scales, 16) || !aligned(d, 4))
    return FS4_ERR_INVALID_ARG;
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < kHeaderBytes) return FS4_ERR_WORKSPACE;
  DeviceInfo di;
  const fs4_status ds = device_info(&di);
  if (ds != FS4_OK) return ds;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(workspace, 0, 4, st) != cudaSuccess) return FS4_ERR_CUDA;
  GemmPlainArgs g{};
  g.a_codes = a_codes; g.a_scales = a_scales; g.a_sg = a_sg;
  g.b_codes = b_codes; g.b_scales = b_scales; g.b_sg = b_sg;
  g.M = (int32_t)M; g.N = (int32_t)N;
  g.Kp = (int32_t)align_up(K, 256);
  g.Mp = (int32_t)align_up(M, 128);
  g.Np = (int32_t)align_up(N, 128);
  g.d = d; g.ldd = ldd;
  g.status = static_cast<uint32_t*>(workspace);
  return cuda_status(launch_gemm_plain(g, st, di.num_sms));
}

size_t fs4_root_ns_batched_workspace_size(int32_t count, const fs4_ns_desc* descs) {
  static thread_local Plan pl;
  if (make_plan(count, descs, &pl, nullptr, true) != FS4_OK) return 0;
  return (size_t)pl.total_bytes;
}

static fs4_status batched_impl(int32_t count, const fs4_ns_desc* descs, int32_t K, float clip_k,
                               uint32_t flags, const uint16_t* rht_masks, void* workspace,
                               size_t workspace_bytes, void* stream, void* const* events,
                               int32_t n_events, const fs4_nvfp4_state* states, bool bf16);

size_t fs4_root_ns_bf16_batched_workspace_size(int32_t count, const fs4_ns_desc* descs) {
  static thread_local Plan pl;
  if (make_plan(count, descs, &pl, nullptr, true, true) != FS4_OK) return 0;
  return (size_t)pl.total_bytes;
}

fs4_status fs4_root_ns_bf16_batched(int32_t count, const fs4_ns_desc* descs, int32_t K, float clip_k,
                                    uint32_t flags, void* workspace, size_t workspace_bytes,
                                    void* stream) {
  return batched_impl(count, descs, K, clip_k, flags, nullptr, workspace, workspace_bytes, stream,
                      nullptr, 0, nullptr, true);
}

fs4_status fs4_root_ns_bf16_batched_timed(int32_t count, const fs4_ns_desc* descs, int32_t K,
                                          float clip_k, uint32_t flags, void* workspace,
                                          size_t workspace_bytes, void* stream,
                                          void* const* phase_events, int32_t n_events) {
  if (!phase_events) return FS4_ERR_INVALID_ARG;
  return batched_impl(count, descs, K, clip_k, flags, nullptr, workspace, workspace_bytes, stream,
                      phase_events, n_events, nullptr, true);
}

size_t fs4_root_ns_workspace_size(int64_t m, int64_t n) {
  if (m < 16 || n < 16 || m > FS4_MAX_DIM || n > FS4_MAX_DIM || m % 16 || n % 16) return 0;
  const int64_t mm = m < n ? m : n, nn = m < n ? n : m;
  const int64_t mp = align_up(mm, kPad), np = align_up(nn, kPad);
  return (size_t)(align_up(kHeaderBytes + state_block_bytes(mp, np), 1024) +
                  align_up(big_block_bytes(mp, np), 1024));
}

static fs4_status batched_impl(int32_t count, const fs4_ns_desc* descs, int32_t K, float clip_k,
                               uint32_t flags, const uint16_t* rht_masks, void* workspace,
                               size_t workspace_bytes, void* stream, void* const* events,
                               int32_t n_events, const fs4_nvfp4_state* states,
                               bool bf16) {
  if (K < 1 || K > FS4_MAX_ITERS) return FS4_ERR_SHAPE;
  if (!std::isfinite(clip_k)) return FS4_ERR_INVALID_ARG;
  if (flags & ~(uint32_t)(0xFF00u | FS4_TEST_STALL | FS4_NS_RHT | FS4_NS_ADAPTIVE46 |
                          FS4_NS_CLIP_QUANTILE))
    return FS4_ERR_INVALID_ARG;
  if ((flags & FS4_NS_CLIP_QUANTILE) && !(clip_k > 0.0f && clip_k <= 1.0f)) return FS4_ERR_INVALID_ARG;
  if ((flags & FS4_NS_RHT) && !rht_masks) return FS4_ERR_INVALID_ARG;
  if (bf16 && (flags & (FS4_NS_RHT | FS4_NS_ADAPTIVE46))) return FS4_ERR_INVALID_ARG;
  static thread_local Plan pl;
  const fs4_status s = make_plan(count, descs, &pl, states, false, bf16);
  if (s != FS4_OK) return s;
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < (size_t)pl.total_bytes)
    return FS4_ERR_WORKSPACE;
  // the workspace must not overlap any input or output either
  const uintptr_t wlo = reinterpret_cast<uintptr_t>(workspace), whi = wlo + (uintptr_t)pl.total_bytes;
  for (int i = 0; i < count; ++i) {
    uintptr_t lo, hi;
    if (states) {
      lo = reinterpret_cast<uintptr_t>(states[i].codes);
      hi = lo + (uintptr_t)(descs[i].m * descs[i].n / 2);
      if (lo < whi && wlo < hi) return FS4_ERR_ALIAS;
      lo = reinterpret_cast<uintptr_t>(states[i].scales);
      hi = lo + (uintptr_t)(descs[i].m * descs[i].n / 16);
    } else {
      span(descs[i].G, descs[i].m, descs[i].n, descs[i].ld, &lo, &hi);
    }
    if (lo < whi && wlo < hi) return FS4_ERR_ALIAS;
    span(descs[i].out, descs[i].m, descs[i].n, descs[i].ld_out, &lo, &hi);
    if (lo < whi && wlo < hi) return FS4_ERR_ALIAS;
  }
  if (events) {
    for (int32_t i = 0; i < 3 + 3 * K; ++i)
      if (i >= n_events || !events[i]) return FS4_ERR_INVALID_ARG;
  }
  DeviceInfo di;
  const fs4_status ds = device_info(&di);
  if (ds != FS4_OK) return ds;
  return run_ns(pl, K, clip_k, flags, rht_masks, static_cast<uint8_t*>(workspace),
                static_cast<cudaStream_t>(stream), di.num_sms, events, bf16);
}

fs4_status fs4_root_ns_batched_nvfp4(int32_t count, const fs4_ns_desc* descs,
                                     const fs4_nvfp4_state* states, int32_t K, float clip_k,
                                     uint32_t flags, const uint16_t* rht_masks, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  if (!states) return FS4_ERR_INVALID_ARG;
  return batched_impl(count, descs, K, clip_k, flags, rht_masks, workspace, workspace_bytes, stream,
                      nullptr, 0, states, false);
}

fs4_status fs4_root_ns_batched_nvfp4_timed(int32_t count, const fs4_ns_desc* descs,
                                           const fs4_nvfp4_state* states, int32_t K, float clip_k,
                                           uint32_t flags, const uint16_t* rht_masks,
                                           void* workspace, size_t workspace_bytes, void* stream,
                                           void* const* phase_events, int32_t n_events) {
  if (!states || !phase_events) return FS4_ERR_INVALID_ARG;
  return batched_impl(count, descs, K, clip_k, flags, rht_masks, workspace, workspace_bytes, stream,
                      phase_events, n_events, states, false);
}

fs4_status fs4_root_ns_batched(int32_t count, const fs4_ns_desc* descs, int32_t K, float clip_k,
                               uint32_t flags, void* workspace, size_t workspace_bytes,
                               void* stream) {
  return batched_impl(count, descs, K, clip_k, flags, nullptr, workspace, workspace_bytes, stream,
                      nullptr, 0, nullptr, false);
}

fs4_status fs4_root_ns_batched_ex(int32_t count, const fs4_ns_desc* descs, int32_t K, float clip_k,
                                  uint32_t flags, const uint16_t* rht_masks, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  return batched_impl(count, descs, K, clip_k, flags, rht_masks, workspace, workspace_bytes, stream,
                      nullptr, 0, nullptr, false);
}

fs4_status fs4_root_ns_batched_timed(int32_t count, const fs4_ns_desc* descs, int32_t K,
                                     float clip_k, uint32_t flags, const uint16_t* rht_masks,
                                     void* workspace, size_t workspace_bytes, void* stream,
                                     void* const* phase_events, int32_t n_events) {
  if (!phase_events) return FS4_ERR_INVALID_ARG;
  return batched_impl(count, descs, K, clip_k, flags, rht_masks, workspace, workspace_bytes, stream,
                      phase_events, n_events, nullptr, false);
}

fs4_status fs4_root_ns(const float* G, int64_t m, int64_t n, int64_t ld, float* out,
                       int64_t ld_out, int32_t K, float a, float b, float c, float clip_k,
                       uint32_t flags, void* workspace, size_t workspace_bytes, void* stream) {
  fs4_ns_desc d;
  d.G = G; d.out = out; d.m = m; d.n = n; d.ld = ld; d.ld_out = ld_out;
  d.a = a; d.b = b; d.c = c;
  return fs4_root_ns_batched(1, &d, K, clip_k, flags, workspace, workspace_bytes, stream);
}

fs4_status fs4_device_status(const void* workspace, void* stream) {
  if (!workspace) return FS4_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, workspace, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess) return FS4_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return FS4_ERR_CUDA;
  if (word & kStatusTimeout) return FS4_ERR_TIMEOUT;
  if (word & kStatusNonFinite) return FS4_ERR_NONFINITE;
  return FS4_OK;
}

const char* fs4_status_string(fs4_status s) {
  switch (s) {
    case FS4_OK: return "FS4_OK";
    case FS4_ERR_INVALID_ARG: return "FS4_ERR_INVALID_ARG";
    case FS4_ERR_SHAPE: return "FS4_ERR_SHAPE";
    case FS4_ERR_ALIAS: return "FS4_ERR_ALIAS";
    case FS4_ERR_WORKSPACE: return "FS4_ERR_WORKSPACE";
    case FS4_ERR_ARCH: return "FS4_ERR_ARCH";
    case FS4_ERR_CUDA: return "FS4_ERR_CUDA";
    case FS4_ERR_NONFINITE: return "FS4_ERR_NONFINITE";
    case FS4_ERR_TIMEOUT: return "FS4_ERR_TIMEOUT";
    default: return "FS4_ERR_UNKNOWN";
  }
}

static fs4_status layout_impl(int32_t count, const fs4_ns_desc* descs, int32_t index,
                              fs4_ns_layout* layout, bool bf16) {
  if (!layout) return FS4_ERR_INVALID_ARG;
  static thread_local Plan pl;
  const fs4_status s = make_plan(count, descs, &pl, nullptr, true, bf16);
  if (s != FS4_OK) return s;
  if (index < 0 || index >= count) return FS4_ERR_INVALID_ARG;
  const MatDesc& d = pl.mat[index];
  const MatLayout L = mat_layout(d.mp, d.np, d.state_off, d.big_off, bf16);
  layout->mp = d.mp;
  layout->np = d.np;
  layout->X = L.X;
  layout->A = L.A;
  for (int k = 0; k < 2; ++k) {
    layout->qX_codes[k] = L.qX[k]; layout->qX_scales[k] = L.sX[k];
    layout->qXT_codes[k] = L.qXT[k]; layout->qXT_scales[k] = L.sXT[k];
  }
  layout->qA_codes = L.qA; layout->qA_scales = L.sA;
  layout->qB_codes = L.qB; layout->qB_scales = L.sB;
  layout->scalars = L.state + (int64_t)offsetof(NsState, sg);
  return FS4_OK;
}

fs4_status fs4_root_ns_layout(int32_t count, const fs4_ns_desc* descs, int32_t index,
                              fs4_ns_layout* layout) {
  return layout_impl(count, descs, index, layout, false);
}

fs4_status fs4_root_ns_bf16_layout(int32_t count, const fs4_ns_desc* descs, int32_t index,
                                   fs4_ns_layout* layout) {
  return layout_impl(count, descs, index, layout, true);
}

}  // extern "C"
