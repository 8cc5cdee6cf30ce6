// gate_f32.cu -- full-precision fp32 gate projection with TwELL packing, on
// the CUDA cores ("Sparser, Faster, Lighter Transformer Language Models",
// technical summary, section 2.1).  TF32 tensor cores would not reach fp32
// accuracy, so the fp32 path uses FMA with a fixed accumulation order
// (i = 0 .. d-1).  One CTA computes one 128-token x W-unit tile of z in
// shared memory (W the TwELL tile width), then each thread packs its own
// token row.
#include "tw_common.cuh"
#include "tw_internal.h"

namespace tw {
namespace {

constexpr int ROWS = 128;   // tokens per CTA
constexpr int KC = 64;      // reduction chunk staged in shared memory
constexpr int UC = 32;      // units per register chunk
constexpr int XS_LD = KC + 1;

// TILE: the TwELL tile width W (64, 128 or 256).
template <int TILE>
constexpr size_t smem_f32() {
  return sizeof(float) *
         ((size_t)ROWS * XS_LD + (size_t)UC * XS_LD + (size_t)ROWS * (TILE + 1));
}

template <int TILE>
__global__ void __launch_bounds__(ROWS)
    gate_twell_f32_kernel(const float* __restrict__ x, const float* __restrict__ Wg_t, int T,
                          int d, int F, int C, float* val, uint8_t* idx, uint8_t* cnt,
                          int32_t* spill_ref, int spill_cap, int32_t* spill_tk, float* spill_val,
                          int32_t* spill_n, float* dump, int32_t* status) {
  constexpr int SEG_LD = TILE + 1;
  extern __shared__ float sh[];
  float* xs = sh;                      // [ROWS][XS_LD]
  float* wsm = xs + ROWS * XS_LD;      // [UC][XS_LD]
  float* seg = wsm + UC * XS_LD;       // [ROWS][SEG_LD]
  const int k = blockIdx.y;
  const int t0 = blockIdx.x * ROWS;
  const int tid = threadIdx.x;
  const int t = t0 + tid;
  const bool row_ok = t < T;

  for (int cc = 0; cc < TILE / UC; ++cc) {
    float acc[UC];
#pragma unroll
    for (int u = 0; u < UC; ++u) acc[u] = 0.f;
    for (int i0 = 0; i0 < d; i0 += KC) {
      for (int e = tid; e < ROWS * KC; e += ROWS) {
        const int r = e / KC, c = e % KC, gi = i0 + c;
        xs[r * XS_LD + c] = (t0 + r < T && gi < d) ? x[(size_t)(t0 + r) * d + gi] : 0.f;
      }
      for (int e = tid; e < UC * KC; e += ROWS) {
        const int u = e / KC, c = e % KC, gi = i0 + c;
        const int j = k * TILE + cc * UC + u;
        wsm[u * XS_LD + c] = gi < d ? Wg_t[(size_t)j * d + gi] : 0.f;
      }
      __syncthreads();
      for (int c = 0; c < KC; ++c) {
        const float xv = xs[tid * XS_LD + c];
#pragma unroll
        for (int u = 0; u < UC; ++u) acc[u] = fmaf(xv, wsm[u * XS_LD + c], acc[u]);
      }
      __syncthreads();
    }
#pragma unroll
    for (int u = 0; u < UC; ++u) seg[tid * SEG_LD + cc * UC + u] = acc[u];
  }
  if (!row_ok) return;

  const size_t kt = (size_t)k * T + t;
  int n = 0;
  for (int c = 0; c < TILE; ++c) {
    const float z = seg[tid * SEG_LD + c];
    const float g = z > 0.f ? z : 0.f;
    if (dump) dump[(size_t)t * F + (size_t)k * TILE + c] = g;
    if (g != 0.f) {
      if (n < C) {
        val[kt * C + n] = g;
        idx[kt * C + n] = (uint8_t)c;
      }
      ++n;
    }
  }
  for (int s = n; s < C; ++s) {
    val[kt * C + s] = 0.f;
    idx[kt * C + s] = 0;
  }
  // a full 256-wide tile has no uint8 count: stored as 255 and flagged
  if (n > 255) set_status(status, 1 << TW_ERR_UNSUPPORTED);
  cnt[kt] = (uint8_t)(n < 255 ? n : 255);
  if (n > C) {
    const int slot = atomicAdd(spill_n, 1);
    if (slot < spill_cap) {
      spill_ref[kt] = slot;
      spill_tk[2 * (size_t)slot] = t;
      spill_tk[2 * (size_t)slot + 1] = k;
      for (int c = 0; c < TILE; ++c) {
        const float z = seg[tid * SEG_LD + c];
        spill_val[(size_t)slot * TILE + c] = z > 0.f ? z : 0.f;
      }
    } else {
      spill_ref[kt] = -1;
      set_status(status, kStatusSpill);
    }
  }
}

}  // namespace

namespace {

template <int TILE>
cudaError_t launch_f32_w(const float* x, const float* Wg_t, int T, int d, int F,
                         const tw_twell& out, float* dump, int32_t* status, cudaStream_t stream) {
  cudaError_t e = set_smem_limit(reinterpret_cast<const void*>(gate_twell_f32_kernel<TILE>),
                                 (int)smem_f32<TILE>());
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(out.spill_n, 0, sizeof(int32_t), stream);
  if (e != cudaSuccess) return e;
  dim3 grid((T + ROWS - 1) / ROWS, F / TILE);
  gate_twell_f32_kernel<TILE><<<grid, ROWS, smem_f32<TILE>(), stream>>>(
      x, Wg_t, T, d, F, out.C, static_cast<float*>(out.val), out.idx, out.cnt, out.spill_ref,
      out.spill_cap, out.spill_tk, static_cast<float*>(out.spill_val), out.spill_n, dump, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gate_twell_f32(const float* x, const float* Wg_t, int T, int d, int F,
                                  const tw_twell& out, float* dump, int32_t* status,
                                  cudaStream_t stream) {
  if (out.W == 64) return launch_f32_w<64>(x, Wg_t, T, d, F, out, dump, status, stream);
  if (out.W == 256) return launch_f32_w<256>(x, Wg_t, T, d, F, out, dump, status, stream);
  return launch_f32_w<128>(x, Wg_t, T, d, F, out, dump, status, stream);
}

}  // namespace tw
