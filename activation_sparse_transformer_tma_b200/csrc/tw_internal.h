// tw_internal.h -- host-side launchers shared between the library's .cu files.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "twell.h"

namespace tw {

// Device properties cached per device.
int num_sms();

// Raise `func`'s dynamic shared-memory limit to `bytes` on the current device.
// The attribute belongs to the device, so it is set once per (kernel, device)
// and remembered under a lock; a process that drives several GPUs gets it set
// on each of them.
cudaError_t set_smem_limit(const void* func, int bytes);

// Launch with the programmatic stream-serialization attribute: the kernel's
// CTAs may be scheduled while the previous kernel on the stream finishes, so
// its launch overlaps that kernel's tail.  Every kernel launched this way
// calls pdl_wait() (tw_common.cuh) before its first global memory access.
template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kern)(Params...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

// Host-side argument checks shared by the entry points (abi.cu).
bool row_d_ok(int d, tw_dtype t);
bool aligned16(const void* p);
bool dtype_ok(tw_dtype t);
tw_status check_twell(const tw_twell* g);

// Default upper bound on any single pipeline wait inside a kernel (ns).
constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;

// Test aid of the bounded waits: the wait limit armed by
// tw_test_withhold_next_gate_loads (0 if none), consumed by the next tile-GEMM
// gate launch.
unsigned long long take_withheld_gate_wait();

// tcgen05 bf16 gate GEMM with TwELL epilogue.  Shapes validated by caller.
cudaError_t launch_gate_twell_tc(const void* x, const void* Wg_t, int T, int d, int F,
                                 const tw_twell& out, void* dump, int32_t* status,
                                 cudaStream_t stream);
// The same GEMM and packing for small batches (1 <= T <= kFewMaxT): units on
// the MMA's M side, the reduction over d split across a thread-block cluster.
constexpr int kFewMaxT = 64;
cudaError_t launch_gate_twell_few(const void* x, const void* Wg_t, int T, int d, int F,
                                  const tw_twell& out, void* dump, int32_t* status,
                                  cudaStream_t stream);
// fp32 CUDA-core gate with the same TwELL packing.
cudaError_t launch_gate_twell_f32(const float* x, const float* Wg_t, int T, int d, int F,
                                  const tw_twell& out, float* dump, int32_t* status,
                                  cudaStream_t stream);
// The whole FFN of 1 <= T <= kDecodeStepMaxT tokens (bf16, W = 128) in one
// cooperative launch: gate + TwELL packing, then the fused up + down.
constexpr int kDecodeStepMaxT = 64;
size_t decode_ws_bytes(int T, int d, int F);
cudaError_t launch_decode_step(const void* x, const void* Wg_t, const void* Wu_t, const void* Wd,
                               int T, int d, int F, const tw_twell& out, void* dump, void* y,
                               tw_dtype y_dtype, void* ws, int32_t* status, cudaStream_t stream);
// Fused up+down over TwELL (plan + persistent gather kernel).
size_t fused_ws_bytes(int T, int d);
cudaError_t launch_fused_updown(const void* x, const tw_twell& g, const void* Wu_t,
                                const void* Wd, int d, void* y, tw_dtype y_dtype, void* ws,
                                int32_t* status, cudaStream_t stream);
// The same fused path with its work plan laid out in a fixed scratch area.
bool fused_plan_fits(int T, int d, size_t limit);
cudaError_t launch_fused_updown_in_scratch(const void* x, const tw_twell& g, const void* Wu_t,
                                           const void* Wd, int d, void* y, tw_dtype y_dtype,
                                           void* scratch, size_t scratch_bytes, int32_t* status,
                                           cudaStream_t stream);
// Dense comparator pieces (bf16, tcgen05).
cudaError_t launch_dense_gateup_tc(const void* x, const void* Wg_t, const void* Wu_t, int T,
                                   int d, int F, void* h, int32_t* status, cudaStream_t stream);
cudaError_t launch_dense_down_tc(const void* h, const void* Wd_dense, int T, int d, int F,
                                 void* y, int32_t* status, cudaStream_t stream);
// Dense training comparator (bf16, tcgen05): forward saves g, u, h [T][F]
// bf16 and writes y fp32; backward uses du, dz [T][F] bf16 scratch.
cudaError_t launch_dense_train_forward(const void* x, const void* Wg_t, const void* Wu_t,
                                       const void* Wd, int T, int d, int F, uint16_t* g,
                                       uint16_t* u, uint16_t* h, float* y, int32_t* status,
                                       cudaStream_t stream);
cudaError_t launch_dense_train_backward(const void* x, const void* dy, const void* Wg_t,
                                        const void* Wu_t, const void* Wd, int T, int d, int F,
                                        float lam, const uint16_t* g, const uint16_t* u,
                                        const uint16_t* h, uint16_t* du, uint16_t* dz, float* dx,
                                        float* dWg_t, float* dWu_t, float* dWd, int32_t* status,
                                        cudaStream_t stream);
// One active (t, j) entry of the hybrid backward, recorded for the
// weight-gradient pass: h = g u, du, dz.
struct Payload {
  int32_t t, j;  // token and unit
  float h, du, dz;
};

// Gather engine, hybrid modes (fused_updown.cu); ws holds fused_ws_bytes(T, d).
cudaError_t launch_hybrid_gather_forward(const void* x, const tw_hybrid& gu, const void* Wu_t,
                                         const void* Wd, int d, void* y, tw_dtype y_dtype,
                                         void* ws, int32_t* status, cudaStream_t stream);
cudaError_t launch_hybrid_gather_backward(const void* dy, const tw_hybrid& gu, const void* Wg_t,
                                          const void* Wu_t, const void* Wd, int d, float lam,
                                          const int32_t* e0, Payload* pay, void* dx,
                                          tw_dtype dx_dtype, void* ws, int32_t* status,
                                          cudaStream_t stream);

// Hybrid (training) kernels.
cudaError_t launch_twell_to_hybrid(const tw_twell& g, const tw_hybrid& out, int32_t* status,
                                   cudaStream_t stream);
size_t hybrid_forward_ws_bytes(int T, int d);
cudaError_t launch_hybrid_forward(const void* x, const tw_hybrid& gu, const void* Wu_t,
                                  const void* Wd, int d, void* y, tw_dtype y_dtype, void* ws,
                                  int32_t* status, cudaStream_t stream);
size_t hybrid_backward_ws_bytes(int T, int d, int F, int C_h, int backup_cap);
cudaError_t launch_hybrid_backward(const void* x, const void* dy, const tw_hybrid& gu,
                                   const void* Wg_t, const void* Wu_t, const void* Wd, int d,
                                   float lam, void* dx, tw_dtype dx_dtype, float* dWg_t,
                                   float* dWu_t, float* dWd, void* ws, size_t ws_bytes,
                                   int32_t* status, cudaStream_t stream);

// calibrate.cu: scattered whole-row gathers of a bf16 [rows][d] matrix
// (see tw_measure_row_gather in twell.h).
cudaError_t launch_row_gather(const void* mat, int rows, int d, long long n, unsigned seed,
                              uint32_t* checksum, cudaStream_t stream);
// Measurement aid: one front-to-back read of `bytes` (a multiple of 16).
cudaError_t launch_stream_read(const void* buf, long long bytes, uint32_t* checksum,
                               cudaStream_t stream);

}  // namespace tw
