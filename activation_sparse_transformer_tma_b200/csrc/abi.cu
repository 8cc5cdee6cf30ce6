// abi.cu -- extern "C" entry points of libtwell.so: argument validation
// (before any launch) and dispatch to the kernels.  The library never
// allocates device memory and never synchronises the caller's stream.
#include <atomic>
#include <cstdint>
#include <map>
#include <mutex>
#include <utility>

#include "tw_internal.h"

namespace tw {

int num_sms() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v <= 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      v = 1;
    cache[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

cudaError_t set_smem_limit(const void* func, int bytes) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> done;  // (kernel, device) -> bytes set
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  auto it = done.find({func, dev});
  if (it != done.end() && it->second >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done[{func, dev}] = bytes;
  return e;
}

namespace {
std::atomic<unsigned long long> g_withheld_gate_wait{0};
}  // namespace

unsigned long long take_withheld_gate_wait() { return g_withheld_gate_wait.exchange(0); }

}  // namespace tw

namespace {

constexpr int kTileW = 128;    // the tile width of the dense comparators' F tiles
constexpr int kMaxRowD = 2048;

// TwELL tile widths: 64, 128 (the default) or 256 (tile-local indices are
// uint8).  Any capacity C up to the tile width.
bool tile_width_ok(int W) { return W == 64 || W == 128 || W == 256; }

}  // namespace

namespace tw {

// Row width d: a multiple of 8, at most 2048 for bf16 rows and 1024 for fp32
// rows (the gather engine keeps one token's row slices and its fp32 output
// slices in the registers of one team of warps).
bool row_d_ok(int d, tw_dtype t) {
  return d % 8 == 0 && d <= (t == TW_BF16 ? kMaxRowD : kMaxRowD / 2);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool dtype_ok(tw_dtype t) { return t == TW_F32 || t == TW_BF16; }

// Shared checks of a TwELL descriptor.
tw_status check_twell(const tw_twell* g) {
  if (!g) return TW_ERR_INVALID_ARG;
  if (g->T < 0 || g->F <= 0 || g->C < 0 || g->spill_cap < 0 || !dtype_ok(g->dtype))
    return TW_ERR_INVALID_ARG;
  if (!tile_width_ok(g->W) || g->F % g->W != 0 || g->C > g->W) return TW_ERR_UNSUPPORTED;
  if (g->F > 65536) return TW_ERR_UNSUPPORTED;
  // arrays sized by T may be NULL for an empty batch
  if (!g->spill_n || (g->T > 0 && (!g->cnt || !g->spill_ref))) return TW_ERR_INVALID_ARG;
  if (g->T > 0 && g->C > 0 && (!g->val || !g->idx)) return TW_ERR_INVALID_ARG;
  if (g->spill_cap > 0 && (!g->spill_tk || !g->spill_val)) return TW_ERR_INVALID_ARG;
  if ((g->val && !aligned16(g->val)) || (g->idx && !aligned16(g->idx)) ||
      (g->spill_val && !aligned16(g->spill_val)))
    return TW_ERR_ALIGNMENT;
  return TW_OK;
}

}  // namespace tw

namespace {

using tw::aligned16;
using tw::check_twell;
using tw::dtype_ok;
using tw::row_d_ok;

tw_status from_cuda(cudaError_t e) { return e == cudaSuccess ? TW_OK : TW_ERR_CUDA; }

tw_status check_hybrid(const tw_hybrid* h) {
  if (!h) return TW_ERR_INVALID_ARG;
  if (h->T < 0 || h->F <= 0 || h->C_h < 0 || h->C_h > h->F || h->backup_cap < 0 ||
      !dtype_ok(h->dtype))
    return TW_ERR_INVALID_ARG;
  // unit histograms live in shared memory; dense rows are read 16 bytes at a time
  if (h->F > 51200 || h->F % 8 != 0) return TW_ERR_UNSUPPORTED;
  if ((size_t)h->T * (size_t)h->C_h + (size_t)h->backup_cap * (size_t)h->F > 0x7FFFFFFFull)
    return TW_ERR_UNSUPPORTED;  // entry numbers are int32
  // arrays sized by T may be NULL for an empty batch
  if (!h->n_backup || (h->T > 0 && (!h->row_nnz || !h->row_slot))) return TW_ERR_INVALID_ARG;
  if (h->T > 0 && h->C_h > 0 && (!h->ell_g || !h->ell_idx)) return TW_ERR_INVALID_ARG;
  if (h->backup_cap > 0 && (!h->backup_rows || !h->backup_g)) return TW_ERR_INVALID_ARG;
  return TW_OK;
}

}  // namespace

extern "C" {

tw_status tw_measure_row_gather(const void* mat, int32_t rows, int32_t d, int64_t n_gathers,
                                uint32_t seed, uint32_t* checksum, cudaStream_t stream) {
  if (rows < 1 || d < 8 || d > 2048 || d % 8 != 0 || n_gathers < 0 || !mat || !checksum)
    return TW_ERR_INVALID_ARG;
  if (!aligned16(mat)) return TW_ERR_ALIGNMENT;
  if (n_gathers == 0) return TW_OK;
  return from_cuda(
      tw::launch_row_gather(mat, rows, d, (long long)n_gathers, seed, checksum, stream));
}

tw_status tw_measure_stream_read(const void* buf, int64_t bytes, uint32_t* checksum,
                                 cudaStream_t stream) {
  if (bytes < 0 || bytes % 16 != 0 || !buf || !checksum) return TW_ERR_INVALID_ARG;
  if (!aligned16(buf)) return TW_ERR_ALIGNMENT;
  if (bytes == 0) return TW_OK;
  return from_cuda(tw::launch_stream_read(buf, (long long)bytes, checksum, stream));
}

const char* tw_status_string(tw_status s) {
  switch (s) {
    case TW_OK: return "TW_OK";
    case TW_ERR_INVALID_ARG: return "TW_ERR_INVALID_ARG";
    case TW_ERR_UNSUPPORTED: return "TW_ERR_UNSUPPORTED";
    case TW_ERR_ALIGNMENT: return "TW_ERR_ALIGNMENT";
    case TW_ERR_CUDA: return "TW_ERR_CUDA";
    case TW_ERR_SPILL_CAPACITY: return "TW_ERR_SPILL_CAPACITY";
    case TW_ERR_BACKUP_CAPACITY: return "TW_ERR_BACKUP_CAPACITY";
    case TW_ERR_TIMEOUT: return "TW_ERR_TIMEOUT";
    case TW_ERR_WORKSPACE: return "TW_ERR_WORKSPACE";
  }
  return "TW_UNKNOWN_STATUS";
}

int32_t twell_version(void) { return 100; }

void tw_test_withhold_next_gate_loads(uint64_t wait_limit_ns) {
  tw::g_withheld_gate_wait.store(wait_limit_ns > 0 ? wait_limit_ns : 1);
}

tw_status twell_gate_gemm(const void* x, const void* Wg_t, int32_t T, int32_t d, int32_t F,
                          tw_dtype dtype, const tw_twell* out, void* g_dense_dump,
                          int32_t* dev_status, cudaStream_t stream) {
  tw_status st = check_twell(out);
  if (st != TW_OK) return st;
  if ((T > 0 && !x) || !Wg_t) return TW_ERR_INVALID_ARG;
  if (T < 0 || d <= 0 || F <= 0 || out->T != T || out->F != F || out->dtype != dtype)
    return TW_ERR_INVALID_ARG;
  if (d % 8 != 0) return TW_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(Wg_t) || (g_dense_dump && !aligned16(g_dense_dump)))
    return TW_ERR_ALIGNMENT;
  if (T == 0) return from_cuda(cudaMemsetAsync(out->spill_n, 0, sizeof(int32_t), stream));
  if (dtype == TW_BF16) {
    if (d < 64) return TW_ERR_UNSUPPORTED;
    if (T <= tw::kFewMaxT && out->W == 128)
      return from_cuda(tw::launch_gate_twell_few(x, Wg_t, T, d, F, *out, g_dense_dump,
                                                 dev_status, stream));
    return from_cuda(tw::launch_gate_twell_tc(x, Wg_t, T, d, F, *out, g_dense_dump, dev_status,
                                              stream));
  }
  return from_cuda(tw::launch_gate_twell_f32(static_cast<const float*>(x),
                                             static_cast<const float*>(Wg_t), T, d, F, *out,
                                             static_cast<float*>(g_dense_dump), dev_status,
                                             stream));
}

size_t twell_fused_updown_workspace_size(int32_t T, int32_t d) {
  if (T < 0 || d <= 0) return 0;
  return tw::fused_ws_bytes(T, d);
}

tw_status twell_fused_updown(const void* x, const tw_twell* g, const void* Wu_t, const void* Wd,
                             int32_t d, void* y, tw_dtype y_dtype, void* ws, size_t ws_bytes,
                             int32_t* dev_status, cudaStream_t stream) {
  tw_status st = check_twell(g);
  if (st != TW_OK) return st;
  const bool any = g->T > 0;  // with no tokens x, y and ws are not touched
  if ((any && (!x || !y || !ws)) || !Wu_t || !Wd || !dtype_ok(y_dtype)) return TW_ERR_INVALID_ARG;
  if (d <= 0) return TW_ERR_INVALID_ARG;
  if (!row_d_ok(d, g->dtype)) return TW_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(Wu_t) || !aligned16(Wd) || !aligned16(y) || !aligned16(ws))
    return TW_ERR_ALIGNMENT;
  if (!any) return TW_OK;
  if (ws_bytes < tw::fused_ws_bytes(g->T, d)) return TW_ERR_WORKSPACE;
  return from_cuda(
      tw::launch_fused_updown(x, *g, Wu_t, Wd, d, y, y_dtype, ws, dev_status, stream));
}

tw_status twell_to_hybrid(const tw_twell* g, const tw_hybrid* out, int32_t* dev_status,
                          cudaStream_t stream) {
  tw_status st = check_twell(g);
  if (st != TW_OK) return st;
  st = check_hybrid(out);
  if (st != TW_OK) return st;
  if (out->T != g->T || out->F != g->F || out->dtype != g->dtype) return TW_ERR_INVALID_ARG;
  if (g->T == 0) return from_cuda(cudaMemsetAsync(out->n_backup, 0, sizeof(int32_t), stream));
  return from_cuda(tw::launch_twell_to_hybrid(*g, *out, dev_status, stream));
}

size_t hybrid_ffn_forward_workspace_size(int32_t T, int32_t d) {
  if (T < 0 || d <= 0) return 0;
  return tw::hybrid_forward_ws_bytes(T, d);
}

tw_status hybrid_ffn_forward(const void* x, const tw_hybrid* gu, const void* Wu_t,
                             const void* Wd, int32_t d, void* y, tw_dtype y_dtype, void* ws,
                             size_t ws_bytes, int32_t* dev_status, cudaStream_t stream) {
  tw_status st = check_hybrid(gu);
  if (st != TW_OK) return st;
  const bool any = gu->T > 0;  // with no tokens x, y, ws and ell_u are not touched
  if ((any && (!x || !y || !ws)) || !Wu_t || !Wd || !dtype_ok(y_dtype)) return TW_ERR_INVALID_ARG;
  if ((any && gu->C_h > 0 && !gu->ell_u) || (gu->backup_cap > 0 && !gu->backup_u))
    return TW_ERR_INVALID_ARG;
  if (d <= 0) return TW_ERR_INVALID_ARG;
  if (!row_d_ok(d, gu->dtype)) return TW_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(Wu_t) || !aligned16(Wd) || !aligned16(y) || !aligned16(ws))
    return TW_ERR_ALIGNMENT;
  if (any && ws_bytes < tw::hybrid_forward_ws_bytes(gu->T, d)) return TW_ERR_WORKSPACE;
  return from_cuda(
      tw::launch_hybrid_forward(x, *gu, Wu_t, Wd, d, y, y_dtype, ws, dev_status, stream));
}

size_t hybrid_ffn_backward_workspace_size(int32_t T, int32_t d, int32_t F, int32_t C_h,
                                          int32_t backup_cap) {
  if (T < 0 || F <= 0 || C_h < 0 || backup_cap < 0) return 0;
  return tw::hybrid_backward_ws_bytes(T, d, F, C_h, backup_cap);
}

tw_status hybrid_ffn_backward(const void* x, const void* dy, const tw_hybrid* gu,
                              const void* Wg_t, const void* Wu_t, const void* Wd, int32_t d,
                              float l1_lambda, void* dx, tw_dtype dx_dtype, float* dWg_t,
                              float* dWu_t, float* dWd, void* ws, size_t ws_bytes,
                              int32_t* dev_status, cudaStream_t stream) {
  tw_status st = check_hybrid(gu);
  if (st != TW_OK) return st;
  const bool any = gu->T > 0;  // with no tokens only the weight gradients are written
  if ((any && (!x || !dy || !dx || !ws)) || !Wg_t || !Wu_t || !Wd || !dWg_t || !dWu_t || !dWd ||
      !dtype_ok(dx_dtype))
    return TW_ERR_INVALID_ARG;
  if ((any && gu->C_h > 0 && !gu->ell_u) || (gu->backup_cap > 0 && !gu->backup_u))
    return TW_ERR_INVALID_ARG;
  if (d <= 0) return TW_ERR_INVALID_ARG;
  if (!row_d_ok(d, gu->dtype)) return TW_ERR_UNSUPPORTED;
  const void* ptrs[] = {x, dy, Wg_t, Wu_t, Wd, dx, dWg_t, dWu_t, dWd, ws};
  for (const void* p : ptrs)
    if (!aligned16(p)) return TW_ERR_ALIGNMENT;
  if (any && ws_bytes < tw::hybrid_backward_ws_bytes(gu->T, d, gu->F, gu->C_h, gu->backup_cap))
    return TW_ERR_WORKSPACE;
  return from_cuda(tw::launch_hybrid_backward(x, dy, *gu, Wg_t, Wu_t, Wd, d, l1_lambda, dx,
                                              dx_dtype, dWg_t, dWu_t, dWd, ws, ws_bytes,
                                              dev_status, stream));
}

tw_status dense_ffn_forward(const void* x, const void* Wg_t, const void* Wu_t,
                            const void* Wd_dense, int32_t T, int32_t d, int32_t F, void* h_ws,
                            void* y, int32_t* dev_status, cudaStream_t stream) {
  if (!x || !Wg_t || !Wu_t || !Wd_dense || !h_ws || !y) return TW_ERR_INVALID_ARG;
  if (T < 0 || d <= 0 || F <= 0) return TW_ERR_INVALID_ARG;
  if (d % 32 != 0 || d < 64 || F % kTileW != 0) return TW_ERR_UNSUPPORTED;
  const void* ptrs[] = {x, Wg_t, Wu_t, Wd_dense, h_ws, y};
  for (const void* p : ptrs)
    if (!aligned16(p)) return TW_ERR_ALIGNMENT;
  if (T == 0) return TW_OK;
  cudaError_t e = tw::launch_dense_gateup_tc(x, Wg_t, Wu_t, T, d, F, h_ws, dev_status, stream);
  if (e != cudaSuccess) return TW_ERR_CUDA;
  return from_cuda(tw::launch_dense_down_tc(h_ws, Wd_dense, T, d, F, y, dev_status, stream));
}

size_t twell_ffn_small_batch_workspace_size(int32_t T, int32_t d, int32_t F) {
  if (T < 0 || d <= 0 || F <= 0) return 0;
  return tw::decode_ws_bytes(T, d, F);
}

tw_status twell_ffn_small_batch(const void* x, const void* Wg_t, const void* Wu_t, const void* Wd,
                                int32_t T, int32_t d, int32_t F, const tw_twell* g,
                                void* g_dense_dump, void* y, tw_dtype y_dtype, void* ws,
                                size_t ws_bytes, int32_t* dev_status, cudaStream_t stream) {
  tw_status st = check_twell(g);
  if (st != TW_OK) return st;
  if (g->T != T || g->F != F || T < 0 || d <= 0) return TW_ERR_INVALID_ARG;
  if ((T > 0 && (!x || !y || !ws)) || !Wg_t || !Wu_t || !Wd || !dtype_ok(y_dtype))
    return TW_ERR_INVALID_ARG;
  if (g->dtype != TW_BF16 || g->W != 128 || T > tw::kDecodeStepMaxT || d % 8 != 0 || d < 64 ||
      d > kMaxRowD)
    return TW_ERR_UNSUPPORTED;
  const void* ptrs[] = {x, Wg_t, Wu_t, Wd, y, ws, g_dense_dump};
  for (const void* p : ptrs)
    if (!aligned16(p)) return TW_ERR_ALIGNMENT;
  if (T == 0) return from_cuda(cudaMemsetAsync(g->spill_n, 0, sizeof(int32_t), stream));
  if (ws_bytes < tw::decode_ws_bytes(T, d, F)) return TW_ERR_WORKSPACE;
  return from_cuda(tw::launch_decode_step(x, Wg_t, Wu_t, Wd, T, d, F, *g, g_dense_dump, y,
                                          y_dtype, ws, dev_status, stream));
}

// Workspace of the dense training comparator: g, u, h (saved by the forward
// for the backward) then du, dz (backward scratch), each [T][F] bf16.
static size_t dense_train_part(int32_t T, int32_t F) {
  return ((size_t)T * (size_t)F * 2 + 255) & ~size_t(255);
}

size_t dense_ffn_train_workspace_size(int32_t T, int32_t F) {
  if (T < 0 || F <= 0) return 0;
  return 5 * dense_train_part(T, F);
}

size_t dense_ffn_train_saved_bytes(int32_t T, int32_t F) {
  if (T < 0 || F <= 0) return 0;
  return 3 * dense_train_part(T, F);
}

static tw_status check_dense_train(int32_t T, int32_t d, int32_t F, const void* ws,
                                   size_t ws_bytes) {
  if (T < 0 || d <= 0 || F <= 0) return TW_ERR_INVALID_ARG;
  if (d % 32 != 0 || d < 64 || F % kTileW != 0) return TW_ERR_UNSUPPORTED;
  if (T > 0 && !ws) return TW_ERR_INVALID_ARG;
  if (!aligned16(ws)) return TW_ERR_ALIGNMENT;
  if (T > 0 && ws_bytes < 5 * dense_train_part(T, F)) return TW_ERR_WORKSPACE;
  return TW_OK;
}

tw_status dense_ffn_train_forward(const void* x, const void* Wg_t, const void* Wu_t,
                                  const void* Wd, int32_t T, int32_t d, int32_t F, void* ws,
                                  size_t ws_bytes, float* y, int32_t* dev_status,
                                  cudaStream_t stream) {
  tw_status st = check_dense_train(T, d, F, ws, ws_bytes);
  if (st != TW_OK) return st;
  if ((T > 0 && (!x || !y)) || !Wg_t || !Wu_t || !Wd) return TW_ERR_INVALID_ARG;
  const void* ptrs[] = {x, Wg_t, Wu_t, Wd, y};
  for (const void* p : ptrs)
    if (!aligned16(p)) return TW_ERR_ALIGNMENT;
  if (T == 0) return TW_OK;
  uint16_t* base = static_cast<uint16_t*>(ws);
  const size_t part = dense_train_part(T, F) / 2;
  return from_cuda(tw::launch_dense_train_forward(x, Wg_t, Wu_t, Wd, T, d, F, base,
                                                  base + part, base + 2 * part, y, dev_status,
                                                  stream));
}

tw_status dense_ffn_train_backward(const void* x, const void* dy, const void* Wg_t,
                                   const void* Wu_t, const void* Wd, int32_t T, int32_t d,
                                   int32_t F, float l1_lambda, void* ws, size_t ws_bytes,
                                   float* dx, float* dWg_t, float* dWu_t, float* dWd,
                                   int32_t* dev_status, cudaStream_t stream) {
  tw_status st = check_dense_train(T, d, F, ws, ws_bytes);
  if (st != TW_OK) return st;
  if ((T > 0 && (!x || !dy || !dx)) || !Wg_t || !Wu_t || !Wd || !dWg_t || !dWu_t || !dWd)
    return TW_ERR_INVALID_ARG;
  const void* ptrs[] = {x, dy, Wg_t, Wu_t, Wd, dx, dWg_t, dWu_t, dWd};
  for (const void* p : ptrs)
    if (!aligned16(p)) return TW_ERR_ALIGNMENT;
  if (T == 0) {  // no tokens: zero weight gradients
    const size_t b = sizeof(float) * (size_t)F * d;
    cudaError_t e = cudaMemsetAsync(dWg_t, 0, b, stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(dWu_t, 0, b, stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(dWd, 0, b, stream);
    return from_cuda(e);
  }
  uint16_t* base = static_cast<uint16_t*>(ws);
  const size_t part = dense_train_part(T, F) / 2;
  return from_cuda(tw::launch_dense_train_backward(
      x, dy, Wg_t, Wu_t, Wd, T, d, F, l1_lambda, base, base + part, base + 2 * part,
      base + 3 * part, base + 4 * part, dx, dWg_t, dWu_t, dWd, dev_status, stream));
}

}  // extern "C"
