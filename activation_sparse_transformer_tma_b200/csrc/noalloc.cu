// noalloc.cu -- the fused up + down projection for callers that cannot
// allocate device memory.
//
// twell_fused_updown needs a caller-provided workspace (its work plan and the
// partial rows of split tokens).  Some callers cannot provide one: a plugin
// called from a host framework whose call path forbids device allocation,
// or a serving process whose device memory was handed in full to its own pool
// at start-up, has no way to call cudaMalloc for it.
// twell_fused_updown_noalloc does the same work with its scratch in a
// file-scope device array of fixed size instead, so the caller passes only
// inputs and outputs.
//
// The array is part of the library's device image: every GPU on which the
// library's kernels are loaded holds kScratchBytes of it until the process
// exits.  Its device address is looked up once per device (first call on that
// device, with that device current) and cached for the life of the process;
// after cudaDeviceReset the cached address is stale, so the entry point must
// not be used across a device reset.
//
// Capacity: the plan of T tokens takes about 24 bytes per token (counts,
// split offsets and one work item each) plus the partial rows of split
// tokens.  T <= 696,848 fits for every supported d; the partial-row capacity
// is whatever the rest of the array holds.
#include <atomic>
#include <cstdint>
#include <mutex>

#include "tw_internal.h"

constexpr size_t kScratchBytes = size_t(16) << 20;  // 16 MiB

// Host code must not pass &g_fused_scratch to a kernel: on the host that name
// is a stand-in, not a device address.  The address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_fused_scratch[kScratchBytes];

namespace {

constexpr int kMaxDevices = 64;

std::mutex g_setup_mutex;
std::atomic<void*> g_scratch_ptr[kMaxDevices];

// Device address of g_fused_scratch on the current device, or nullptr.
void* scratch_on_current_device(cudaError_t* err) {
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDevices) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  void* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
  if (p) return p;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  p = g_scratch_ptr[dev].load(std::memory_order_relaxed);
  if (!p) {
    *err = cudaGetSymbolAddress(&p, g_fused_scratch);
    if (*err != cudaSuccess) return nullptr;
    g_scratch_ptr[dev].store(p, std::memory_order_release);
  }
  return p;
}

}  // namespace

extern "C" tw_status twell_fused_updown_noalloc(const void* x, const tw_twell* g,
                                                const void* Wu_t, const void* Wd, int32_t d,
                                                void* y, tw_dtype y_dtype, int32_t* dev_status,
                                                cudaStream_t stream) {
  // the same checks as twell_fused_updown: with T == 0 the token-sized
  // buffers may be NULL and nothing is launched
  tw_status st = tw::check_twell(g);
  if (st != TW_OK) return st;
  const bool any = g->T > 0;
  if ((any && (!x || !y)) || !Wu_t || !Wd || !tw::dtype_ok(y_dtype)) return TW_ERR_INVALID_ARG;
  if (d <= 0) return TW_ERR_INVALID_ARG;
  if (!tw::row_d_ok(d, g->dtype)) return TW_ERR_UNSUPPORTED;
  if (!tw::aligned16(x) || !tw::aligned16(Wu_t) || !tw::aligned16(Wd) || !tw::aligned16(y))
    return TW_ERR_ALIGNMENT;
  if (!any) return TW_OK;
  // the work plan of T tokens must fit the fixed scratch area
  if (!tw::fused_plan_fits(g->T, d, kScratchBytes)) return TW_ERR_UNSUPPORTED;
  cudaError_t err = cudaSuccess;
  void* scratch = scratch_on_current_device(&err);
  if (!scratch) return TW_ERR_CUDA;
  err = tw::launch_fused_updown_in_scratch(x, *g, Wu_t, Wd, d, y, y_dtype, scratch, kScratchBytes,
                                           dev_status, stream);
  return err == cudaSuccess ? TW_OK : TW_ERR_CUDA;
}
