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
// device, with that device current) and cached.
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

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" tw_status twell_fused_updown_noalloc(const void* x, const tw_twell* g,
                                                const void* Wu_t, const void* Wd, int32_t d,
                                                void* y, tw_dtype y_dtype, int32_t* dev_status,
                                                cudaStream_t stream) {
  if (!g || !x || !Wu_t || !Wd || !y) return TW_ERR_INVALID_ARG;
  if (g->T < 0 || g->F <= 0 || g->C < 0 || g->spill_cap < 0 || d <= 0) return TW_ERR_INVALID_ARG;
  if ((g->dtype != TW_F32 && g->dtype != TW_BF16) || (y_dtype != TW_F32 && y_dtype != TW_BF16))
    return TW_ERR_INVALID_ARG;
  if (g->W != 128 || g->F % 128 != 0 || g->C > 32 || g->F > 65536) return TW_ERR_UNSUPPORTED;
  if (!g->cnt || !g->spill_ref || !g->spill_n) return TW_ERR_INVALID_ARG;
  if (g->C > 0 && (!g->val || !g->idx)) return TW_ERR_INVALID_ARG;
  if (g->spill_cap > 0 && (!g->spill_tk || !g->spill_val)) return TW_ERR_INVALID_ARG;
  if (d % 8 != 0 || d > (g->dtype == TW_BF16 ? 2048 : 1024)) return TW_ERR_UNSUPPORTED;
  if (!al16(x) || !al16(Wu_t) || !al16(Wd) || !al16(y) || (g->val && !al16(g->val)) ||
      (g->idx && !al16(g->idx)) || (g->spill_val && !al16(g->spill_val)))
    return TW_ERR_ALIGNMENT;
  // the work plan of T tokens must fit the fixed scratch area
  if (!tw::fused_plan_fits(g->T, d, kScratchBytes)) return TW_ERR_UNSUPPORTED;
  if (g->T == 0) return TW_OK;
  cudaError_t err = cudaSuccess;
  void* scratch = scratch_on_current_device(&err);
  if (!scratch) return TW_ERR_CUDA;
  err = tw::launch_fused_updown_in_scratch(x, *g, Wu_t, Wd, d, y, y_dtype, scratch, kScratchBytes,
                                           dev_status, stream);
  return err == cudaSuccess ? TW_OK : TW_ERR_CUDA;
}
