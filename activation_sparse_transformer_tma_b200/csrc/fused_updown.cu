// fused_updown.cu -- fused up + down projection over a TwELL gate tensor
// ("Sparser, Faster, Lighter Transformer Language Models", technical summary,
// section 2.2): weights are read only for the non-zero activations; for each
// active unit j of token t a dot product u = x_t . Wu_t[j] and a scaled row
// y_t += (g_tj u) Wd[j] are accumulated, all in fp32, and no dense
// intermediate is written to memory.
//
// One warp owns one token.  x_t stays in registers (packed), y_t accumulates
// in fp32 registers; each lane owns 16-byte column slices, so every weight
// row is gathered with fully coalesced 16-byte loads (512 contiguous bytes
// per warp instruction).  The dot product is finished with warp shuffles.
// Active units are found from the tile-major TwELL counts with a ballot over
// 32 tiles at a time; slot entries are broadcast lane-to-lane by shuffles.
#include "tw_common.cuh"
#include "tw_internal.h"

namespace tw {
namespace {

template <typename T>
struct Lane;

// bf16: 8 values per 16-byte slice.
template <>
struct Lane<uint16_t> {
  static constexpr int E = 8;
  using Raw = uint4;
  TW_DEV static Raw zero() { return make_uint4(0, 0, 0, 0); }
  TW_DEV static void widen(const Raw& r, float (&f)[8]) {
    f[0] = bf16_lo(r.x); f[1] = bf16_hi(r.x);
    f[2] = bf16_lo(r.y); f[3] = bf16_hi(r.y);
    f[4] = bf16_lo(r.z); f[5] = bf16_hi(r.z);
    f[6] = bf16_lo(r.w); f[7] = bf16_hi(r.w);
  }
  TW_DEV static float scalar(uint16_t v) { return bf16_to_f32(v); }
};

// fp32: 4 values per 16-byte slice.
template <>
struct Lane<float> {
  static constexpr int E = 4;
  using Raw = float4;
  TW_DEV static Raw zero() { return make_float4(0.f, 0.f, 0.f, 0.f); }
  TW_DEV static void widen(const Raw& r, float (&f)[4]) {
    f[0] = r.x; f[1] = r.y; f[2] = r.z; f[3] = r.w;
  }
  TW_DEV static float scalar(float v) { return v; }
};

template <typename Raw>
TW_DEV Raw ldg_nc(const void* p) {
  return __ldg(reinterpret_cast<const Raw*>(p));
}

template <typename Tin>
struct FusedArgs {
  const Tin* x;
  const Tin* val;
  const uint8_t* idx;
  const uint8_t* cnt;
  const int32_t* spill_ref;
  const Tin* spill_val;
  const Tin* Wu_t;
  const Tin* Wd;
  void* y;
  int32_t* status;
  int T, d, F, C, spill_cap;
};

// Accumulates one active unit (g, j) into acc.
template <typename Tin, int NCH, bool kTogether>
TW_DEV void unit_contrib(const FusedArgs<Tin>& a, const typename Lane<Tin>::Raw (&xr)[NCH],
                         float (&acc)[NCH][Lane<Tin>::E], float gv, int j, int lane) {
  using L = Lane<Tin>;
  constexpr int E = L::E;
  constexpr int SPAN = 32 * E;
  const Tin* wu = a.Wu_t + (size_t)j * a.d;
  const Tin* wd = a.Wd + (size_t)j * a.d;
  typename L::Raw ru[NCH], rd[NCH];
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    const int col = c * SPAN + lane * E;
    ru[c] = col < a.d ? ldg_nc<typename L::Raw>(wu + col) : L::zero();
    if (kTogether) rd[c] = col < a.d ? ldg_nc<typename L::Raw>(wd + col) : L::zero();
  }
  float part = 0.f;
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    float xf[E], wf[E];
    L::widen(xr[c], xf);
    L::widen(ru[c], wf);
#pragma unroll
    for (int e = 0; e < E; ++e) part = fmaf(xf[e], wf[e], part);
  }
  if (!kTogether) {
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const int col = c * SPAN + lane * E;
      rd[c] = col < a.d ? ldg_nc<typename L::Raw>(wd + col) : L::zero();
    }
  }
  const float h = gv * warp_sum(part);
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    float wf[E];
    L::widen(rd[c], wf);
#pragma unroll
    for (int e = 0; e < E; ++e) acc[c][e] = fmaf(h, wf[e], acc[c][e]);
  }
}

template <typename Tin, int NCH, bool kTogether, bool kOutBf16>
__global__ void __launch_bounds__(256) fused_updown_kernel(const FusedArgs<Tin> a) {
  using L = Lane<Tin>;
  constexpr int E = L::E;
  constexpr int SPAN = 32 * E;
  constexpr int W = 128;
  const int lane = threadIdx.x & 31;
  const int t = (int)((blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5);
  if (t >= a.T) return;  // whole warp

  typename L::Raw xr[NCH];
  const Tin* xt = a.x + (size_t)t * a.d;
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    const int col = c * SPAN + lane * E;
    xr[c] = col < a.d ? ldg_nc<typename L::Raw>(xt + col) : L::zero();
  }
  float acc[NCH][E];
#pragma unroll
  for (int c = 0; c < NCH; ++c)
#pragma unroll
    for (int e = 0; e < E; ++e) acc[c][e] = 0.f;

  const int K = a.F / W;
  for (int kb = 0; kb < K; kb += 32) {
    const int k = kb + lane;
    const int n = k < K ? (int)a.cnt[(size_t)k * a.T + t] : 0;
    unsigned act = __ballot_sync(0xFFFFFFFFu, n > 0);
    while (act) {
      const int b = __ffs(act) - 1;
      act &= act - 1;
      const int nk = __shfl_sync(0xFFFFFFFFu, n, b);
      const int kk = kb + b;
      const size_t kt = (size_t)kk * a.T + t;
      if (nk <= a.C) {
        float gl = 0.f;
        int jl = 0;
        if (lane < nk) {
          gl = L::scalar(a.val[kt * a.C + lane]);
          jl = kk * W + a.idx[kt * a.C + lane];
        }
        for (int s = 0; s < nk; ++s) {
          const float gv = __shfl_sync(0xFFFFFFFFu, gl, s);
          const int j = __shfl_sync(0xFFFFFFFFu, jl, s);
          unit_contrib<Tin, NCH, kTogether>(a, xr, acc, gv, j, lane);
        }
      } else {
        const int ref = a.spill_ref[kt];
        if (ref < 0 || ref >= a.spill_cap) {
          // The spill entry was dropped for lack of capacity (already flagged
          // by the producer); only the C slots of this tile are available.
          if (lane == 0) set_status(a.status, kStatusSpill);
          float gl = 0.f;
          int jl = 0;
          if (lane < a.C) {
            gl = L::scalar(a.val[kt * a.C + lane]);
            jl = kk * W + a.idx[kt * a.C + lane];
          }
          for (int s = 0; s < a.C; ++s)
            unit_contrib<Tin, NCH, kTogether>(a, xr, acc, __shfl_sync(0xFFFFFFFFu, gl, s),
                                              __shfl_sync(0xFFFFFFFFu, jl, s), lane);
          continue;
        }
        const Tin* seg = a.spill_val + (size_t)ref * W;
#pragma unroll 1
        for (int part = 0; part < W / 32; ++part) {
          const float v = L::scalar(seg[part * 32 + lane]);
          unsigned m = __ballot_sync(0xFFFFFFFFu, v != 0.f);
          while (m) {
            const int s = __ffs(m) - 1;
            m &= m - 1;
            const float gv = __shfl_sync(0xFFFFFFFFu, v, s);
            unit_contrib<Tin, NCH, kTogether>(a, xr, acc, gv, kk * W + part * 32 + s, lane);
          }
        }
      }
    }
  }

#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    const int col = c * SPAN + lane * E;
    if (col >= a.d) continue;
    if (kOutBf16) {
      uint16_t* yt = static_cast<uint16_t*>(a.y) + (size_t)t * a.d + col;
      if constexpr (E == 8) {
        uint4 w = make_uint4(pack_bf16x2(acc[c][0], acc[c][1]), pack_bf16x2(acc[c][2], acc[c][3]),
                             pack_bf16x2(acc[c][4], acc[c][5]), pack_bf16x2(acc[c][6], acc[c][7]));
        *reinterpret_cast<uint4*>(yt) = w;
      } else {
        uint2 w = make_uint2(pack_bf16x2(acc[c][0], acc[c][1]), pack_bf16x2(acc[c][2], acc[c][3]));
        *reinterpret_cast<uint2*>(yt) = w;
      }
    } else {
      float* yt = static_cast<float*>(a.y) + (size_t)t * a.d + col;
#pragma unroll
      for (int q = 0; q < E / 4; ++q)
        reinterpret_cast<float4*>(yt)[q] =
            make_float4(acc[c][4 * q], acc[c][4 * q + 1], acc[c][4 * q + 2], acc[c][4 * q + 3]);
    }
  }
}

template <typename Tin, int NCH, bool kTogether>
cudaError_t launch_nch(const FusedArgs<Tin>& a, tw_dtype y_dtype, cudaStream_t stream) {
  const int warps_per_block = 8;
  const size_t blocks = ((size_t)a.T + warps_per_block - 1) / warps_per_block;
  if (blocks == 0) return cudaSuccess;
  if (y_dtype == TW_BF16)
    fused_updown_kernel<Tin, NCH, kTogether, true><<<(unsigned)blocks, 32 * warps_per_block, 0, stream>>>(a);
  else
    fused_updown_kernel<Tin, NCH, kTogether, false><<<(unsigned)blocks, 32 * warps_per_block, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fused_updown(const void* x, const tw_twell& g, const void* Wu_t,
                                const void* Wd, int d, void* y, tw_dtype y_dtype,
                                int32_t* status, cudaStream_t stream) {
  if (g.dtype == TW_BF16) {
    FusedArgs<uint16_t> a{static_cast<const uint16_t*>(x), static_cast<const uint16_t*>(g.val),
                          g.idx, g.cnt, g.spill_ref, static_cast<const uint16_t*>(g.spill_val),
                          static_cast<const uint16_t*>(Wu_t), static_cast<const uint16_t*>(Wd),
                          y, status, g.T, d, g.F, g.C, g.spill_cap};
    if (d <= 256) return launch_nch<uint16_t, 1, true>(a, y_dtype, stream);
    if (d <= 512) return launch_nch<uint16_t, 2, true>(a, y_dtype, stream);
    if (d <= 1024) return launch_nch<uint16_t, 4, true>(a, y_dtype, stream);
    return launch_nch<uint16_t, 8, true>(a, y_dtype, stream);
  }
  FusedArgs<float> a{static_cast<const float*>(x), static_cast<const float*>(g.val), g.idx, g.cnt,
                     g.spill_ref, static_cast<const float*>(g.spill_val),
                     static_cast<const float*>(Wu_t), static_cast<const float*>(Wd), y, status,
                     g.T, d, g.F, g.C, g.spill_cap};
  if (d <= 128) return launch_nch<float, 1, true>(a, y_dtype, stream);
  if (d <= 256) return launch_nch<float, 2, true>(a, y_dtype, stream);
  if (d <= 512) return launch_nch<float, 4, true>(a, y_dtype, stream);
  if (d <= 1024) return launch_nch<float, 8, false>(a, y_dtype, stream);
  return launch_nch<float, 16, false>(a, y_dtype, stream);
}

}  // namespace tw
