// fs4_root_ns_noalloc: the single-matrix Newton-Schulz step for callers that
// cannot allocate device memory.
//
// Some callers have no way to obtain a workspace: plugins living inside a host
// framework that owns every device allocation and hands out none, or loops in
// which a run-time allocation is not permitted.  This entry point gives them the
// same step with the workspace taken from a fixed array compiled into the
// library.
//
// The array lives in every device that loads the library, for the life of the
// process.  Its address is looked up once per device (cudaGetSymbolAddress on
// the first call made with that device current; make that first call before any
// stream capture).  All calls share it: two calls whose work overlaps on the
// GPU (different streams, or different host threads) race on it.  Each call
// clears the parts that must start at zero before using them.
#include <mutex>

#include "../../include/fs4.h"
#include "fs4_internal.h"

namespace {

static __device__ __align__(256) uint8_t g_noalloc_scratch[FS4_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {};

// Device address of the scratch array on the current device (looked up once per device).
fs4_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FS4_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return FS4_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return FS4_OK;
}

}  // namespace

extern "C" fs4_status fs4_root_ns_noalloc(const float* G, int64_t m, int64_t n, int64_t ld,
                                          float* out, int64_t ld_out, int32_t K, float a, float b,
                                          float c, float clip_k, void* stream) {
  const size_t need = fs4_root_ns_workspace_size(m, n);
  if (need == 0) return FS4_ERR_SHAPE;
  if (need > (size_t)FS4_NOALLOC_SCRATCH_BYTES) return FS4_ERR_WORKSPACE;
  void* scratch = nullptr;
  const fs4_status s = noalloc_scratch(&scratch);
  if (s != FS4_OK) return s;
  return fs4_root_ns(G, m, n, ld, out, ld_out, K, a, b, c, clip_k, 0u, scratch,
                     (size_t)FS4_NOALLOC_SCRATCH_BYTES, stream);
}
