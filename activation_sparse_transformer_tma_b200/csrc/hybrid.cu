// hybrid.cu -- training-side kernels for the hybrid sparse format
// ("Sparser, Faster, Lighter Transformer Language Models", technical summary,
// sections 2.3 and 2.4):
//   * TwELL -> hybrid: each token row becomes a compact ELL row (global unit
//     indices, ascending) when it has at most C_h non-zeros, otherwise a dense
//     backup row; backup slots follow ascending token order;
//   * hybrid forward and the per-token pass of the backward (dh, du, dz, dx
//     with the L1 term) run on the gather engine of fused_updown.cu;
//   * the weight gradients are summed per unit from the backward's per-entry
//     records after a deterministic, token-ordered transposition (stable
//     counting sort by unit; no float atomics).
#include "pdl.cuh"
#include "tw_common.cuh"
#include "tw_internal.h"

namespace tw {
namespace {

constexpr unsigned FULL = 0xFFFFFFFFu;

template <typename T>
TW_DEV float ld_scalar(const T* p, size_t i);
template <>
TW_DEV float ld_scalar<uint16_t>(const uint16_t* p, size_t i) { return bf16_to_f32(p[i]); }
template <>
TW_DEV float ld_scalar<float>(const float* p, size_t i) { return p[i]; }

// The V = 16 / sizeof(T) values of row[cl .. cl + V) widened exactly to
// fp32 (zeros past n).  row + cl must be 16-byte aligned (n % V == 0).
template <typename T>
TW_DEV void load_vec(const T* row, int cl, int n, float (&v)[16 / sizeof(T)]) {
  const uint4 r = cl < n ? *reinterpret_cast<const uint4*>(row + cl) : make_uint4(0, 0, 0, 0);
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
  if constexpr (sizeof(T) == 2) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(w[i]);
  }
}

template <typename T>
TW_DEV void st_scalar(T* p, size_t i, float v);
template <>
TW_DEV void st_scalar<uint16_t>(uint16_t* p, size_t i, float v) { p[i] = f32_to_bf16(v); }
template <>
TW_DEV void st_scalar<float>(float* p, size_t i, float v) { p[i] = v; }

TW_DEV unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Row vectors of length d held by one warp: lane owns 16-byte slices.
template <typename T>
struct Slice;
template <>
struct Slice<uint16_t> {
  static constexpr int E = 8;
  using Raw = uint4;
  TW_DEV static Raw load(const uint16_t* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }
  TW_DEV static Raw zero() { return make_uint4(0, 0, 0, 0); }
  TW_DEV static void widen(const Raw& r, float (&f)[8]) {
    f[0] = bf16_lo(r.x); f[1] = bf16_hi(r.x); f[2] = bf16_lo(r.y); f[3] = bf16_hi(r.y);
    f[4] = bf16_lo(r.z); f[5] = bf16_hi(r.z); f[6] = bf16_lo(r.w); f[7] = bf16_hi(r.w);
  }
};
template <>
struct Slice<float> {
  static constexpr int E = 4;
  using Raw = float4;
  TW_DEV static Raw load(const float* p) { return __ldg(reinterpret_cast<const float4*>(p)); }
  TW_DEV static Raw zero() { return make_float4(0.f, 0.f, 0.f, 0.f); }
  TW_DEV static void widen(const Raw& r, float (&f)[4]) { f[0] = r.x; f[1] = r.y; f[2] = r.z; f[3] = r.w; }
};

template <typename V>
struct HView {
  int T, F, C_h, backup_cap;
  const V* ell_g;
  V* ell_u;
  const uint16_t* ell_idx;
  const int32_t* row_nnz;
  const int32_t* row_slot;
  const V* backup_g;
  V* backup_u;
};

// Bit i set when value i of the 16-byte chunk r is non-zero (as a float
// compare would say: -0 is zero, NaN is not).
template <typename T>
TW_DEV unsigned nonzero_mask(const uint4& r) {
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
  unsigned m = 0;
  if constexpr (sizeof(T) == 2) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      m |= ((w[i] & 0x7FFFu) != 0u ? 1u : 0u) << (2 * i);
      m |= ((w[i] & 0x7FFF0000u) != 0u ? 1u : 0u) << (2 * i + 1);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) m |= ((w[i] & 0x7FFFFFFFu) != 0u ? 1u : 0u) << i;
  }
  return m;
}

constexpr int kDenseGroup = 8;  // 16-byte chunks per lane loaded together

// Enumerates the active entries of token t in ascending unit order.
//  * ELL row: ell_fn(valid, j, rank) once per lane for 32 entries at a time.
//  * backup row: dense_fn(cl, mask, rank0) for this lane's V = 16 / sizeof(T)
//    columns [cl, cl + V) that hold a non-zero: bit i of mask marks column
//    cl + i, whose rank among the row's non-zeros is
//    rank0 + popc(mask & ((1 << i) - 1)).  The row is read kDenseGroup
//    chunks per lane at a time (one load latency per group, not per chunk);
//    ranks come from a warp scan of the per-lane counts.
// Rows whose backup slot was dropped for lack of capacity have no entries.
template <typename T, class EllFn, class DenseFn>
TW_DEV void for_each_chunk(const HView<T>& h, int t, int slot, int nnz, int lane, EllFn&& ell_fn,
                           DenseFn&& dense_fn) {
  if (slot < 0) {
    for (int s0 = 0; s0 < nnz; s0 += 32) {
      const int s = s0 + lane;
      const bool v = s < nnz;
      const size_t pos = (size_t)t * h.C_h + (v ? s : 0);
      const int j = v ? (int)h.ell_idx[pos] : 0;
      ell_fn(v, j, s);
    }
  } else if (slot < h.backup_cap) {
    constexpr int V = 16 / (int)sizeof(T);
    const T* row = h.backup_g + (size_t)slot * h.F;
    int base = 0;
    for (int c0 = 0; c0 < h.F; c0 += 32 * V * kDenseGroup) {
      uint4 r[kDenseGroup];
#pragma unroll
      for (int q = 0; q < kDenseGroup; ++q) {
        const int cl = c0 + (q * 32 + lane) * V;
        r[q] = cl < h.F ? *reinterpret_cast<const uint4*>(row + cl) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int q = 0; q < kDenseGroup; ++q) {
        const int cl = c0 + (q * 32 + lane) * V;
        const unsigned mask = nonzero_mask<T>(r[q]);
        const int nz = __popc(mask);
        int incl = nz;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int u = __shfl_up_sync(FULL, incl, o);
          if (lane >= o) incl += u;
        }
        const int total = __shfl_sync(FULL, incl, 31);
        if (mask != 0u) dense_fn(cl, mask, base + incl - nz);
        base += total;
      }
    }
  }
}

// --------------------------------------------------------- TwELL -> hybrid --
// Warp per token: row_nnz, and the ELL row when nnz <= C_h.
template <typename T>
__global__ void __launch_bounds__(256)
    hyb_rows_kernel(int Tn, int F, int W, int C, const uint8_t* cnt, const T* val, const uint8_t* idx,
                    const int32_t* spill_ref, int spill_cap, const T* spill_val, int C_h,
                    T* ell_g, uint16_t* ell_idx, int32_t* row_nnz, int32_t* status) {
  pdl_wait();
  pdl_launch_next();
  const int lane = threadIdx.x & 31;
  const int t = (int)((blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5);
  if (t >= Tn) return;
  const int K = F / W;
  int total = 0;
  for (int kb = 0; kb < K; kb += 32) {
    const int k = kb + lane;
    total += k < K ? (int)cnt[(size_t)k * Tn + t] : 0;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) total += __shfl_xor_sync(FULL, total, o);
  if (lane == 0) row_nnz[t] = total;
  const size_t rbase = (size_t)t * C_h;
  if (total > C_h) {  // backup row: its ELL slots hold (+0, 0); g is filled after the scan
    for (int s = lane; s < C_h; s += 32) {
      ell_g[rbase + s] = T(0);
      ell_idx[rbase + s] = 0;
    }
    return;
  }

  int pos = 0;  // next ELL position of this row
  for (int kb = 0; kb < K; kb += 32) {
    const int k = kb + lane;
    const int n = k < K ? (int)cnt[(size_t)k * Tn + t] : 0;
    // exclusive prefix of counts over the 32 tiles
    int incl = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(FULL, incl, o);
      if (lane >= o) incl += v;
    }
    const int excl = incl - n;
    // tiles within capacity: each lane copies its own tile's slots, eight
    // loads in flight before the stores
    if (n > 0 && n <= C) {
      const size_t kt = (size_t)k * Tn + t;
      const size_t q0 = rbase + pos + excl;
      for (int s0 = 0; s0 < n; s0 += 8) {
        T v[8];
        uint8_t ix[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (s0 + i < n) {
            v[i] = val[kt * C + s0 + i];
            ix[i] = idx[kt * C + s0 + i];
          }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (s0 + i < n) {
            ell_g[q0 + s0 + i] = v[i];
            ell_idx[q0 + s0 + i] = (uint16_t)(k * W + ix[i]);
          }
        }
      }
    }
    // overflowing tiles: the warp reads each one's spilled segment
    unsigned act = __ballot_sync(FULL, n > C);
    while (act) {
      const int b = __ffs(act) - 1;
      act &= act - 1;
      const int nk = __shfl_sync(FULL, n, b);
      const int p0 = pos + __shfl_sync(FULL, excl, b);
      const int kk = kb + b;
      const size_t kt = (size_t)kk * Tn + t;
      {
        const int ref = spill_ref[kt];
        if (ref < 0 || ref >= spill_cap) {
          // Dropped spill entry: only the C slots are known.
          if (lane == 0) set_status(status, kStatusSpill);
          for (int s = lane; s < C; s += 32) {
            ell_g[rbase + p0 + s] = val[kt * C + s];
            ell_idx[rbase + p0 + s] = (uint16_t)(kk * W + idx[kt * C + s]);
          }
          for (int s = C + lane; s < nk; s += 32) {  // keep the row's slots defined
            ell_g[rbase + p0 + s] = T(0);
            ell_idx[rbase + p0 + s] = 0;
          }
          continue;
        }
        int r = 0;
        for (int part = 0; part < W / 32; ++part) {
          const T v = spill_val[(size_t)ref * W + part * 32 + lane];
          const bool nz = ld_scalar<T>(&v, 0) != 0.f;
          const unsigned m = __ballot_sync(FULL, nz);
          if (nz) {
            const int q = p0 + r + __popc(m & lanemask_lt());
            ell_g[rbase + q] = v;
            ell_idx[rbase + q] = (uint16_t)(kk * W + part * 32 + lane);
          }
          r += __popc(m);
        }
      }
    }
    pos += __shfl_sync(FULL, incl, 31);
  }
  for (int s = total + lane; s < C_h; s += 32) {
    ell_g[rbase + s] = T(0);
    ell_idx[rbase + s] = 0;
  }
}

// Single-CTA exclusive scan over n int32 values.
//  mode 0 (backup slots): flag = in[i] > thr; out[i] = flag ? slot : -1;
//          aux[slot] = i for slot < cap; *total = number of flags.
//  mode 1 (offsets): out[i] = exclusive prefix of in[]; out[n] = total.
//  mode 2 (entry offsets): as mode 1, counting in[i] only for rows whose slot
//          aux[i] is below cap (ELL rows and stored backup rows).
constexpr int SCAN_THREADS = 1024;
__global__ void __launch_bounds__(SCAN_THREADS)
    scan_kernel(int mode, int n, const int32_t* in, int thr, int32_t* out, int32_t* aux, int cap,
                int32_t* total, int32_t* status, int32_t* zero, int nzero) {
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t carry;
  pdl_wait();
  pdl_launch_next();
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  // a counter array of a later kernel, cleared here instead of by a memset
  for (int i = tid; i < nzero; i += SCAN_THREADS) zero[i] = 0;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < n; base += SCAN_THREADS) {
    const int i = base + tid;
    int v = 0;
    if (i < n) {
      if (mode == 0) v = in[i] > thr ? 1 : 0;
      else if (mode == 1) v = in[i];
      else v = aux[i] < cap ? in[i] : 0;
    }
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(FULL, incl, o);
      if (lane >= o) incl += u;
    }
    if (lane == 31) warp_sums[wid] = incl;
    __syncthreads();
    if (wid == 0) {
      int s = warp_sums[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(FULL, s, o);
        if (lane >= o) s += u;
      }
      warp_sums[lane] = s;  // inclusive over warps
    }
    __syncthreads();
    const int excl = carry + (wid > 0 ? warp_sums[wid - 1] : 0) + incl - v;
    if (i < n) {
      if (mode == 0) {
        out[i] = v ? excl : -1;
        if (v && excl < cap) aux[excl] = i;
      } else {
        out[i] = excl;
      }
    }
    __syncthreads();
    if (tid == 0) carry += warp_sums[31];
    __syncthreads();
  }
  if (tid == 0) {
    if (mode == 0) {
      *total = carry;
      if (carry > cap) set_status(status, kStatusBackup);
    } else {
      out[n] = carry;
    }
  }
}

// Warp per backup slot: dense g row from TwELL (zero fill, then scatter).
template <typename T, int W>
__global__ void __launch_bounds__(256)
    hyb_backup_kernel(int Tn, int F, int C, const uint8_t* cnt, const T* val, const uint8_t* idx,
                      const int32_t* spill_ref, int spill_cap, const T* spill_val,
                      const int32_t* backup_rows, const int32_t* n_backup, int backup_cap,
                      T* backup_g) {
  pdl_wait();
  pdl_launch_next();
  const int lane = threadIdx.x & 31;
  const int slot = (int)((blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5);
  const int nb = min(*n_backup, backup_cap);
  if (slot >= nb) return;
  const int t = backup_rows[slot];
  T* row = backup_g + (size_t)slot * F;
  uint4* row4 = reinterpret_cast<uint4*>(row);
  for (int i = lane; i < F * (int)sizeof(T) / 16; i += 32) row4[i] = make_uint4(0, 0, 0, 0);
  __syncwarp();
  // lane k handles tile k (its slots); spilled tiles are copied by the warp
  const int K = F / W;
  for (int kb = 0; kb < K; kb += 32) {
    const int k = kb + lane;
    const size_t kt = (size_t)k * Tn + t;
    const int n = k < K ? cnt[kt] : 0;
    int ref = -1;
    if (n > C) {
      ref = spill_ref[kt];
      if (ref >= spill_cap) ref = -1;
    }
    if (n > 0 && ref < 0) {  // the slots, eight loads in flight before the stores
      const int m = n < C ? n : C;
      for (int s0 = 0; s0 < m; s0 += 8) {
        T v[8];
        uint8_t ix[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (s0 + i < m) {
            v[i] = val[kt * C + s0 + i];
            ix[i] = idx[kt * C + s0 + i];
          }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (s0 + i < m) row[k * W + ix[i]] = v[i];
      }
    }
    // spilled tiles: the warp copies four segments at a time, all loads first
    unsigned sp = __ballot_sync(FULL, ref >= 0);
    while (sp) {
      int src[4], rb[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        src[q] = sp ? __ffs(sp) - 1 : -1;
        if (sp) sp &= sp - 1;
        rb[q] = __shfl_sync(FULL, ref, src[q] < 0 ? 0 : src[q]);
      }
      T v[4][W / 32];
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int c = 0; c < W / 32; ++c)
          if (src[q] >= 0) v[q][c] = spill_val[(size_t)rb[q] * W + c * 32 + lane];
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int c = 0; c < W / 32; ++c)
          if (src[q] >= 0) row[(kb + src[q]) * W + c * 32 + lane] = v[q][c];
    }
  }
}

// ------------------------------------------------ hybrid forward/backward --
// The per-token passes of the hybrid forward (u on the pattern, y) and of the
// backward (dh, du, dz, dx and the per-entry record) run on the gather engine
// (fused_updown.cu), which splits heavy rows and streams the weight rows
// through shared memory.  The weight gradients below use its records.

// The records of the backward are in token-major order (entry e0[t] + rank),
// and each carries its unit.  The weight gradients sum them per unit in
// ascending token order, i.e. ascending record index, so each unit's records
// are gathered into a unit-major list and sorted there:
//   1. hyb_ucount_kernel  records per unit (one atomic per record);
//   2. scan_kernel        exclusive prefix of the counts -> unit_off;
//   3. hyb_place_kernel   each record's index at its unit's next place (the
//                         order inside a unit is arbitrary here);
//   4. hyb_wgrad_kernel   one CTA per unit sorts its segment (bitonic: in one
//                         warp's registers up to 64 records, in shared
//                         memory up to kSegSmem; longer segments as sorted
//                         runs merged by rank into a scratch list) and sums
//                         in that order.
// Every pass is flat over the records, so a heavy backup row costs no one
// thread or warp more than its share.
constexpr int kSegSmem = 2048;  // records of a unit sorted in shared memory
constexpr int kPaySmem = 512;   // records of a unit whose payloads are staged in shared memory

__global__ void __launch_bounds__(256)
    hyb_ucount_kernel(const Payload* pay, const int32_t* e_total, int32_t* ucnt) {
  pdl_wait();
  pdl_launch_next();
  const int n = *e_total;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n; e += gridDim.x * blockDim.x)
    atomicAdd(&ucnt[pay[e].j], 1);
}

__global__ void __launch_bounds__(256)
    hyb_place_kernel(const Payload* pay, const int32_t* e_total, const int32_t* unit_off,
                     int32_t* cursor, int32_t* list) {
  pdl_wait();
  pdl_launch_next();
  const int n = *e_total;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n; e += gridDim.x * blockDim.x) {
    const int j = pay[e].j;
    list[unit_off[j] + atomicAdd(&cursor[j], 1)] = e;
  }
}

// Ascending bitonic sort of v[0, P) in shared memory (P a power of two <= the
// array), all threads of the CTA.
TW_DEV void block_bitonic(int32_t* v, int P) {
  for (int k = 2; k <= P; k <<= 1) {
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      for (int i = threadIdx.x; i < P; i += blockDim.x) {
        const int o = i ^ jj;
        if (o > i) {
          const int32_t a = v[i], b = v[o];
          if ((a > b) == ((i & k) == 0)) {
            v[i] = b;
            v[o] = a;
          }
        }
      }
      __syncthreads();
    }
  }
}

// Ascending bitonic sort of 64 values held by one warp, two per lane: a at
// position lane, b at position lane + 32.  All in registers and shuffles.
TW_DEV void warp_bitonic64(int32_t& a, int32_t& b, int lane) {
#pragma unroll
  for (int k = 2; k <= 64; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j == 32) {  // partners in the same lane; k == 64, ascending everywhere
        const int32_t lo = min(a, b), hi = max(a, b);
        a = lo;
        b = hi;
      } else {
        const int32_t pa = __shfl_xor_sync(FULL, a, j), pb = __shfl_xor_sync(FULL, b, j);
        const bool lower = (lane & j) == 0;
        const bool asc_a = (lane & k) == 0, asc_b = ((lane + 32) & k) == 0;
        a = (asc_a == lower) ? min(a, pa) : max(a, pa);
        b = (asc_b == lower) ? min(b, pb) : max(b, pb);
      }
    }
  }
}

// Weight gradients of one unit per CTA, records summed in token order.
template <typename T>
__global__ void __launch_bounds__(256)
    hyb_wgrad_kernel(int F, int d, const T* x, const T* dy, const int32_t* unit_off,
                     int32_t* list, int32_t* sorted, const Payload* pay, float* dWg_t,
                     float* dWu_t, float* dWd) {
  using S = Slice<T>;
  constexpr int E = S::E;
  __shared__ int32_t seg[kSegSmem];
  pdl_wait();
  pdl_launch_next();
  const int j = blockIdx.x;
  const int b = unit_off[j], n = unit_off[j + 1] - b;
  const bool small = n <= kSegSmem;
  if (n <= 64) {  // most units: one warp sorts in registers
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      int32_t va = lane < n ? list[b + lane] : INT32_MAX;
      int32_t vb = lane + 32 < n ? list[b + lane + 32] : INT32_MAX;
      warp_bitonic64(va, vb, lane);
      seg[lane] = va;
      seg[lane + 32] = vb;
    }
    __syncthreads();
  } else if (small) {
    int P = 1;
    while (P < n) P <<= 1;
    for (int i = threadIdx.x; i < P; i += blockDim.x) seg[i] = i < n ? list[b + i] : INT32_MAX;
    __syncthreads();
    block_bitonic(seg, P);
  } else {
    // sorted runs of kSegSmem records, written back in place
    for (int r0 = 0; r0 < n; r0 += kSegSmem) {
      const int len = min(kSegSmem, n - r0);
      for (int i = threadIdx.x; i < kSegSmem; i += blockDim.x)
        seg[i] = i < len ? list[b + r0 + i] : INT32_MAX;
      __syncthreads();
      block_bitonic(seg, kSegSmem);
      for (int i = threadIdx.x; i < len; i += blockDim.x) list[b + r0 + i] = seg[i];
      __syncthreads();
    }
    // final place of a record: its rank in its own run plus, in every other
    // run, the number of smaller records (indices are distinct)
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      const int32_t v = list[b + i];
      const int own = i / kSegSmem;
      int pos = i - own * kSegSmem;
      for (int r = 0; r * kSegSmem < n; ++r) {
        if (r == own) continue;
        int lo = r * kSegSmem, hi = min(n, lo + kSegSmem);
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (list[b + mid] < v) lo = mid + 1;
          else hi = mid;
        }
        pos += lo - r * kSegSmem;
      }
      sorted[b + pos] = v;
    }
    __syncthreads();
  }
  const int32_t* order = small ? seg : sorted + b;
  // the payloads of a unit with few records, in summation order, fetched in
  // one parallel pass: the summation loop then waits on the token rows only
  __shared__ Payload pls[kPaySmem];
  const bool staged = n <= kPaySmem;
  if (staged) {
    for (int i = threadIdx.x; i < n; i += blockDim.x) pls[i] = pay[order[i]];
    __syncthreads();
  }
  // column pairs on the paired fp32 FMA (each half is one fma.rn.f32, so
  // the sums are those of scalar FMAs in the same order)
  constexpr int E2 = E / 2;
  const int stride = blockDim.x * E;
  for (int col = threadIdx.x * E; col < d; col += stride) {
    float2 ad[E2], au[E2], ag[E2];
#pragma unroll
    for (int e = 0; e < E2; ++e) ad[e] = au[e] = ag[e] = make_float2(0.f, 0.f);
#pragma unroll 8
    for (int q = 0; q < n; ++q) {
      const Payload p = staged ? pls[q] : pay[order[q]];
      float xf[E], df[E];
      S::widen(S::load(x + (size_t)p.t * d + col), xf);
      S::widen(S::load(dy + (size_t)p.t * d + col), df);
      const float2 h2 = make_float2(p.h, p.h), du2 = make_float2(p.du, p.du),
                   dz2 = make_float2(p.dz, p.dz);
#pragma unroll
      for (int e = 0; e < E2; ++e) {
        const float2 x2 = make_float2(xf[2 * e], xf[2 * e + 1]);
        ad[e] = __ffma2_rn(h2, make_float2(df[2 * e], df[2 * e + 1]), ad[e]);
        au[e] = __ffma2_rn(du2, x2, au[e]);
        ag[e] = __ffma2_rn(dz2, x2, ag[e]);
      }
    }
    const size_t o = (size_t)j * d + col;
#pragma unroll
    for (int e = 0; e < E2; e += 2) {
      *reinterpret_cast<float4*>(dWd + o + 2 * e) = make_float4(ad[e].x, ad[e].y, ad[e + 1].x, ad[e + 1].y);
      *reinterpret_cast<float4*>(dWu_t + o + 2 * e) = make_float4(au[e].x, au[e].y, au[e + 1].x, au[e + 1].y);
      *reinterpret_cast<float4*>(dWg_t + o + 2 * e) = make_float4(ag[e].x, ag[e].y, ag[e + 1].x, ag[e + 1].y);
    }
  }
}

// ------------------------------------------------------------ workspace ----
struct BwdWs {  // the gather engine's own workspace follows these arrays
  int32_t* e0;        // [T+1], e0[T] = number of records
  Payload* pay;       // [Emax]
  int32_t* ucnt;      // [F] records per unit, then [F] placement cursors (zeroed together)
  int32_t* cursor;
  int32_t* unit_off;  // [F+1]
  int32_t* list;      // [Emax] unit-major record indices
  int32_t* sorted;    // [Emax] scratch for segments longer than kSegSmem
  size_t bytes;
};

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

BwdWs carve(void* base, int T, int F, int C_h, int backup_cap) {
  const size_t emax = (size_t)T * C_h + (size_t)backup_cap * F;
  BwdWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  const size_t o_e0 = take(sizeof(int32_t) * ((size_t)T + 1));
  const size_t o_pay = take(sizeof(Payload) * (emax > 0 ? emax : 1));
  const size_t o_cnt = take(sizeof(int32_t) * 2 * (size_t)F);
  const size_t o_off = take(sizeof(int32_t) * ((size_t)F + 1));
  const size_t o_list = take(sizeof(int32_t) * (emax > 0 ? emax : 1));
  const size_t o_sorted = take(sizeof(int32_t) * (emax > 0 ? emax : 1));
  w.bytes = off;
  if (base) {
    char* p = static_cast<char*>(base);
    w.e0 = reinterpret_cast<int32_t*>(p + o_e0);
    w.pay = reinterpret_cast<Payload*>(p + o_pay);
    w.ucnt = reinterpret_cast<int32_t*>(p + o_cnt);
    w.cursor = w.ucnt + F;
    w.unit_off = reinterpret_cast<int32_t*>(p + o_off);
    w.list = reinterpret_cast<int32_t*>(p + o_list);
    w.sorted = reinterpret_cast<int32_t*>(p + o_sorted);
  }
  return w;
}

template <typename T>
HView<T> view_of(const tw_hybrid& g) {
  HView<T> h;
  h.T = g.T;
  h.F = g.F;
  h.C_h = g.C_h;
  h.backup_cap = g.backup_cap;
  h.ell_g = static_cast<const T*>(g.ell_g);
  h.ell_u = static_cast<T*>(g.ell_u);
  h.ell_idx = g.ell_idx;
  h.row_nnz = g.row_nnz;
  h.row_slot = g.row_slot;
  h.backup_g = static_cast<const T*>(g.backup_g);
  h.backup_u = static_cast<T*>(g.backup_u);
  return h;
}

unsigned warp_blocks(int n) { return (unsigned)(((size_t)n + 7) / 8); }

template <typename T>
cudaError_t to_hybrid_t(const tw_twell& g, const tw_hybrid& o, int32_t* status, cudaStream_t s) {
  if (g.T == 0) return cudaSuccess;
  cudaError_t e = launch_pdl(
      hyb_rows_kernel<T>, dim3(warp_blocks(g.T)), dim3(256), 0, s, g.T, g.F, g.W, g.C,
      (const uint8_t*)g.cnt, static_cast<const T*>(g.val), (const uint8_t*)g.idx,
      (const int32_t*)g.spill_ref, g.spill_cap, static_cast<const T*>(g.spill_val), o.C_h,
      static_cast<T*>(o.ell_g), o.ell_idx, o.row_nnz, status);
  if (e != cudaSuccess) return e;
  e = launch_pdl(scan_kernel, dim3(1), dim3(SCAN_THREADS), 0, s, 0, g.T, (const int32_t*)o.row_nnz,
                 o.C_h, o.row_slot, o.backup_rows, o.backup_cap, o.n_backup, status,
                 (int32_t*)nullptr, 0);
  if (e != cudaSuccess) return e;
  if (o.backup_cap > 0) {
    auto kern = g.W == 64 ? hyb_backup_kernel<T, 64>
                          : (g.W == 256 ? hyb_backup_kernel<T, 256> : hyb_backup_kernel<T, 128>);
    e = launch_pdl(kern, dim3(warp_blocks(o.backup_cap)), dim3(256), 0, s, g.T, g.F, g.C,
                   (const uint8_t*)g.cnt, static_cast<const T*>(g.val), (const uint8_t*)g.idx,
                   (const int32_t*)g.spill_ref, g.spill_cap, static_cast<const T*>(g.spill_val),
                   (const int32_t*)o.backup_rows, (const int32_t*)o.n_backup, o.backup_cap,
                   static_cast<T*>(o.backup_g));
  }
  return e;
}

template <typename T>
cudaError_t backward_t(const void* x, const void* dy, const tw_hybrid& gu, const void* Wg_t,
                       const void* Wu_t, const void* Wd, int d, float lam, void* dx,
                       tw_dtype dx_dtype, float* dWg_t, float* dWu_t, float* dWd, void* ws,
                       int32_t* status, cudaStream_t s) {
  const BwdWs w = carve(ws, gu.T, gu.F, gu.C_h, gu.backup_cap);
  void* engine_ws = static_cast<char*>(ws) + w.bytes;
  // entry offsets of every token (token-major order); the per-unit record
  // counts and placement cursors of the weight-gradient pass are cleared here
  cudaError_t e = launch_pdl(scan_kernel, dim3(1), dim3(SCAN_THREADS), 0, s, 2, gu.T,
                             (const int32_t*)gu.row_nnz, 0, w.e0, gu.row_slot, gu.backup_cap,
                             (int32_t*)nullptr, status, w.ucnt, 2 * gu.F);
  if (e != cudaSuccess) return e;
  // per-token pass: dh, du, dz, dx and one record per entry
  e = launch_hybrid_gather_backward(dy, gu, Wg_t, Wu_t, Wd, d, lam, w.e0, w.pay, dx, dx_dtype,
                                    engine_ws, status, s);
  if (e != cudaSuccess) return e;
  // weight gradients: records grouped by unit, then each unit sorted and summed
  const int grid = num_sms() * 8;
  const int32_t* e_total = w.e0 + gu.T;
  e = launch_pdl(hyb_ucount_kernel, dim3(grid), dim3(256), 0, s, (const Payload*)w.pay, e_total,
                 w.ucnt);
  if (e != cudaSuccess) return e;
  e = launch_pdl(scan_kernel, dim3(1), dim3(SCAN_THREADS), 0, s, 1, gu.F, (const int32_t*)w.ucnt,
                 0, w.unit_off, (int32_t*)nullptr, 0, (int32_t*)nullptr, status,
                 (int32_t*)nullptr, 0);
  if (e != cudaSuccess) return e;
  e = launch_pdl(hyb_place_kernel, dim3(grid), dim3(256), 0, s, (const Payload*)w.pay, e_total,
                 (const int32_t*)w.unit_off, w.cursor, w.list);
  if (e != cudaSuccess) return e;
  return launch_pdl(hyb_wgrad_kernel<T>, dim3(gu.F), dim3(256), 0, s, gu.F, d,
                    static_cast<const T*>(x), static_cast<const T*>(dy),
                    (const int32_t*)w.unit_off, w.list, w.sorted, (const Payload*)w.pay, dWg_t,
                    dWu_t, dWd);
}

}  // namespace

cudaError_t launch_twell_to_hybrid(const tw_twell& g, const tw_hybrid& out, int32_t* status,
                                   cudaStream_t stream) {
  return g.dtype == TW_BF16 ? to_hybrid_t<uint16_t>(g, out, status, stream)
                            : to_hybrid_t<float>(g, out, status, stream);
}

size_t hybrid_forward_ws_bytes(int T, int d) { return fused_ws_bytes(T, d); }

cudaError_t launch_hybrid_forward(const void* x, const tw_hybrid& gu, const void* Wu_t,
                                  const void* Wd, int d, void* y, tw_dtype y_dtype, void* ws,
                                  int32_t* status, cudaStream_t stream) {
  if (gu.T == 0) return cudaSuccess;
  return launch_hybrid_gather_forward(x, gu, Wu_t, Wd, d, y, y_dtype, ws, status, stream);
}

size_t hybrid_backward_ws_bytes(int T, int d, int F, int C_h, int backup_cap) {
  return carve(nullptr, T, F, C_h, backup_cap).bytes + fused_ws_bytes(T, d);
}

cudaError_t launch_hybrid_backward(const void* x, const void* dy, const tw_hybrid& gu,
                                   const void* Wg_t, const void* Wu_t, const void* Wd, int d,
                                   float lam, void* dx, tw_dtype dx_dtype, float* dWg_t,
                                   float* dWu_t, float* dWd, void* ws, size_t ws_bytes,
                                   int32_t* status, cudaStream_t stream) {
  (void)ws_bytes;
  if (gu.T == 0) {
    cudaMemsetAsync(dWg_t, 0, sizeof(float) * (size_t)gu.F * d, stream);
    cudaMemsetAsync(dWu_t, 0, sizeof(float) * (size_t)gu.F * d, stream);
    cudaMemsetAsync(dWd, 0, sizeof(float) * (size_t)gu.F * d, stream);
    return cudaGetLastError();
  }
  return gu.dtype == TW_BF16
             ? backward_t<uint16_t>(x, dy, gu, Wg_t, Wu_t, Wd, d, lam, dx, dx_dtype, dWg_t, dWu_t,
                                    dWd, ws, status, stream)
             : backward_t<float>(x, dy, gu, Wg_t, Wu_t, Wd, d, lam, dx, dx_dtype, dWg_t, dWu_t,
                                 dWd, ws, status, stream);
}

}  // namespace tw
