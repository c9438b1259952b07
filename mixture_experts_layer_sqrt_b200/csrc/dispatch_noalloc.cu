// moe_dispatch_noalloc: the dispatch stage without a caller-provided workspace.
//
// Some callers cannot allocate device memory on their call path: a plugin
// running inside an inference engine that hands it no workspace, a serving
// loop where cudaMalloc (which may synchronise the device) is forbidden, or a
// program whose device memory is entirely owned by another allocator.  For
// them this entry point takes the per-chunk histogram scratch from a
// fixed-size array in the library's own device memory instead of `ws`.
//
// The array lives in every GPU that loads the library until the process
// exits.  Its device address is looked up once per device, on the first call
// made with that device current; make that first call before any stream
// capture.  Every call shares the array: calls that overlap on the GPU (two
// streams, two host threads) race on it and must be serialised by the caller.
// The kernels overwrite every scratch entry they later read, so nothing needs
// clearing between calls.
#include <limits.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int kNoAllocScratchInts = MOE_DISPATCH_NOALLOC_MAX_SCRATCH_INTS;
static __device__ __align__(256) int32_t g_dispatch_scratch[kNoAllocScratchInts];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int32_t *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_dispatch_scratch on the current device (nullptr on error).
int32_t *scratch_on_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dispatch_scratch) != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = static_cast<int32_t *>(p);
  }
  return g_scratch_ptr[dev];
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_dispatch_noalloc(const MoEConfig *cfg, int T, const int32_t *topk_idx,
                                           const float *topk_w, const void *x, int32_t *expert_counts,
                                           int32_t *expert_offsets, int32_t *slot_row, int32_t *row_token,
                                           float *row_weight, void *x_perm, moe_stream_t stream) {
  using namespace moe;
  // The argument rules are those of moe_dispatch; the workspace size check is
  // replaced by the fixed scratch limit.
  const size_t need = moe_dispatch_workspace_size(cfg, T);
  if (need == 0) return MOE_ERR_INVALID_ARG;
  if ((long long)T * cfg->top_k > INT_MAX / 2) return MOE_ERR_UNSUPPORTED;
  if (!expert_counts || !expert_offsets) return MOE_ERR_INVALID_ARG;
  // x_perm == NULL builds the row maps only, and x may then be NULL too
  if (T > 0 && (!topk_idx || !topk_w || !slot_row || !row_token || !row_weight ||
                (x_perm && (!x || ((uintptr_t)x & 15u) || ((uintptr_t)x_perm & 15u)))))
    return MOE_ERR_INVALID_ARG;
  if ((long long)num_chunks(T) * cfg->num_experts > kNoAllocScratchInts) return MOE_ERR_UNSUPPORTED;
  int32_t *scratch = scratch_on_current_device();
  if (!scratch) return MOE_ERR_CUDA;
  return launch_dispatch(*cfg, T, topk_idx, topk_w, x, expert_counts, expert_offsets, slot_row, row_token,
                         row_weight, x_perm, scratch, (cudaStream_t)stream);
}
