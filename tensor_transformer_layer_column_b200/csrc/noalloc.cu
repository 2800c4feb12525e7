// tp_layernorm_bwd_noalloc: the LayerNorm backward without a caller workspace.
//
// Some callers cannot allocate device memory at the point where they run the
// backward: code inside a custom allocator or memory-pool callback, runtimes
// that hand the library a fixed memory budget up front, or embedders that
// forbid cudaMalloc on their hot path.  This entry point serves them: its
// only scratch (the per-block dgamma/dbeta partial sums) lives in a
// file-scope device array that is part of the loaded library image, so the
// call itself allocates nothing.
//
// Costs of that choice, stated for the caller:
//  * every GPU that loads the library holds the array (4 MiB) until exit;
//  * every call shares the one array of its device, so calls whose kernels
//    may overlap on a GPU (different streams, or graphs replayed
//    concurrently) race on it and must be serialised by the caller;
//  * the first call on each device resolves the array's device address
//    (cudaGetSymbolAddress) with that device current; make that first call
//    outside any stream capture.
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"

namespace tp {

namespace {

// Per-block partial sums: the kernel writes nb * 2 * D floats, every one of
// them, before the reduction reads them, so nothing needs clearing between
// calls and the array keeps the last call's values.
constexpr size_t kStaticScratchFloats = 1u << 20;   // 4 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) float g_ln_bwd_scratch[kStaticScratchFloats];

std::mutex g_scratch_mu;
float* g_scratch_ptr[kMaxDevices] = {};

// Device address of this device's copy of the array.  In host code the name
// g_ln_bwd_scratch is only a host-side stand-in, never a device address.
tp_status scratch_for_current_device(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TP_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_ln_bwd_scratch) != cudaSuccess || p == nullptr)
      return TP_ERR_CUDA;
    g_scratch_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_scratch_ptr[dev];
  return TP_OK;
}

}  // namespace

}  // namespace tp

extern "C" tp_status tp_layernorm_bwd_noalloc(const tp_bf16* dy, const tp_bf16* x,
                                              const tp_bf16* gamma, const float* mean,
                                              const float* rstd, const tp_bf16* dres, int rows,
                                              int D, tp_bf16* dx, tp_bf16* dgamma, tp_bf16* dbeta,
                                              tp_stream stream) {
  using namespace tp;
  if (!dy || !x || !gamma || !mean || !rstd || !dx || rows < 0 || D <= 0) return TP_ERR_INVALID_ARG;
  if (D > 8192) return TP_ERR_UNSUPPORTED;   // beyond the kernel's and the scratch's width limit
  if (D % 8) return TP_ERR_MISALIGNED;
  for (const void* p : {(const void*)dy, (const void*)x, (const void*)gamma, (const void*)dres,
                        (const void*)dx})
    if (p && !al16(p)) return TP_ERR_MISALIGNED;
  float* scratch = nullptr;
  tp_status st = scratch_for_current_device(&scratch);
  if (st != TP_OK) return st;
  // Row blocks: the same count as the workspace entry point (2 per SM, at
  // most one per row), so both group rows alike and give identical dgamma /
  // dbeta; capped by what the array holds (2 * D partial floats per block,
  // 64 blocks at D = 8192, where the two may group rows differently).
  long long nb = layernorm_bwd_blocks(rows < 1 ? 1 : rows);
  const long long cap = (long long)(kStaticScratchFloats / (2 * (size_t)D));
  if (nb > cap) nb = cap;
  if (nb < 1) nb = 1;
  if ((size_t)nb * 2 * (size_t)D > kStaticScratchFloats) return TP_ERR_WORKSPACE;
  return launch_layernorm_bwd_blocks(dy, x, gamma, mean, rstd, dres, rows, D, dx, dgamma, dbeta,
                                     (int)nb, scratch, (cudaStream_t)stream);
}
