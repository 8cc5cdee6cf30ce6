// fused_updown.cu -- fused up + down projection over a TwELL gate tensor
// ("Sparser, Faster, Lighter Transformer Language Models", technical summary,
// section 2.2): weights are read only for the non-zero activations; for each
// active unit j of token t a dot product u = x_t . Wu_t[j] and a scaled row
// y_t += (g_tj u) Wd[j] are accumulated in fp32.  No dense intermediate is
// written to memory.
//
// Work decomposition.  Per-token activity is very uneven (a few tokens carry
// tens of times the median number of active units), so a token with more
// than kPart active units is split into parts of kPart entries:
//   1. plan_count_kernel   nnz_t = sum of the TwELL tile counts of token t;
//   2. plan_scan_kernel    (one CTA) parts per token, partial-buffer slots for
//                          split tokens (bounded by the workspace), the work
//                          item list and its length;
//   3. fused_kernel        persistent warps take work items from a ticket
//                          counter.  An item is a whole token or one part.
// A split token's parts write fp32 partial rows to the workspace; the part
// that finishes last (atomic counter per token) sums them in part order, so
// y is deterministic.
//
// Data movement.  Each warp owns a ring of shared-memory stages; lane 0
// gathers the Wu and Wd rows of upcoming entries with 1-D bulk copies
// (cp.async.bulk, completion on one mbarrier per stage, no multicast) while
// the warp computes on earlier stages, so several KB per warp are in flight.
// Every lane owns 16-byte column slices: conflict-free shared loads.  x_t
// stays packed in registers; the bf16 dot product uses the mixed-precision
// fma (bf16 inputs, fp32 accumulator), the axpy uses packed fp32x2 fma.
#include "tw_common.cuh"
#include "tw_internal.h"

namespace tw {
namespace {

constexpr unsigned FULL = 0xFFFFFFFFu;
constexpr int W = 128;            // TwELL tile width
constexpr int kPart = 64;         // entries per part of a split token
constexpr int kWarps = 6;         // warps per CTA of the fused kernel
constexpr int kRingBytes = 32768; // shared-memory ring per warp
constexpr int kListCap = 64;      // entry window collected at a time

// --------------------------------------------------------------- workspace --
struct FusedWs {
  int32_t* hdr;        // [0] item ticket, [1] number of items
  int32_t* nnz;        // [T]
  int32_t* item_off;   // [T+1]
  int32_t* slot_off;   // [T] first partial slot of a split token, -1 if whole
  int32_t* done;       // [T] parts finished (split tokens)
  int32_t* item_token; // [max_items]
  float* partial;      // [parts_cap][d]
  int parts_cap, max_items;
  size_t bytes;
  size_t zero_bytes;   // prefix (hdr .. done) cleared before every call
};

size_t al256(size_t v) { return (v + 255) & ~size_t(255); }

FusedWs carve(void* base, int T, int d) {
  FusedWs w{};
  w.parts_cap = T / 2 + 256;
  w.max_items = T + w.parts_cap;
  size_t off = 0;
  auto take = [&](size_t b) { size_t o = off; off = al256(off + b); return o; };
  const size_t o_hdr = take(4 * sizeof(int32_t));
  const size_t o_done = take(sizeof(int32_t) * (size_t)T);
  w.zero_bytes = off;
  const size_t o_nnz = take(sizeof(int32_t) * (size_t)T);
  const size_t o_off = take(sizeof(int32_t) * ((size_t)T + 1));
  const size_t o_slot = take(sizeof(int32_t) * (size_t)T);
  const size_t o_item = take(sizeof(int32_t) * (size_t)w.max_items);
  const size_t o_part = take(sizeof(float) * (size_t)w.parts_cap * d);
  w.bytes = off;
  if (base) {
    char* p = static_cast<char*>(base);
    w.hdr = reinterpret_cast<int32_t*>(p + o_hdr);
    w.done = reinterpret_cast<int32_t*>(p + o_done);
    w.nnz = reinterpret_cast<int32_t*>(p + o_nnz);
    w.item_off = reinterpret_cast<int32_t*>(p + o_off);
    w.slot_off = reinterpret_cast<int32_t*>(p + o_slot);
    w.item_token = reinterpret_cast<int32_t*>(p + o_item);
    w.partial = reinterpret_cast<float*>(p + o_part);
  }
  return w;
}

// -------------------------------------------------------------------- plan --
__global__ void plan_count_kernel(int T, int K, const uint8_t* __restrict__ cnt, int32_t* nnz) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  int s = 0;
  for (int k = 0; k < K; ++k) s += cnt[(size_t)k * T + t];
  nnz[t] = s;
}

constexpr int kScanThreads = 1024;

// Block-wide exclusive scan of one value per thread; returns the prefix and
// writes the block total to *total.
TW_DEV int block_exclusive_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(FULL, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) warp_sums[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    int s = lane < (int)(blockDim.x >> 5) ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(FULL, s, o);
      if (lane >= o) s += u;
    }
    warp_sums[lane] = s;
  }
  __syncthreads();
  const int excl = (wid > 0 ? warp_sums[wid - 1] : 0) + incl - v;
  *total = warp_sums[(blockDim.x >> 5) - 1];
  __syncthreads();
  return excl;
}

// One CTA: parts per token, partial slots (bounded), item offsets, item list.
__global__ void __launch_bounds__(kScanThreads)
    plan_scan_kernel(int T, const int32_t* __restrict__ nnz, int parts_cap, int max_items,
                     int32_t* slot_off, int32_t* item_off, int32_t* item_token, int32_t* hdr) {
  __shared__ int warp_sums[32];
  __shared__ int carry_slots, carry_items;
  if (threadIdx.x == 0) carry_slots = carry_items = 0;
  __syncthreads();
  // pass 1: partial slots of split tokens, in token order, within capacity
  for (int base = 0; base < T; base += kScanThreads) {
    const int t = base + threadIdx.x;
    const int n = t < T ? nnz[t] : 0;
    const int parts = n > kPart ? (n + kPart - 1) / kPart : 0;
    int tot;
    const int ex = block_exclusive_scan(parts, warp_sums, &tot) + carry_slots;
    if (t < T) slot_off[t] = (parts > 0 && ex + parts <= parts_cap) ? ex : -1;
    if (threadIdx.x == 0) carry_slots += tot;
    __syncthreads();
  }
  // pass 2: items (a token whose split did not fit is one item)
  for (int base = 0; base < T; base += kScanThreads) {
    const int t = base + threadIdx.x;
    int parts = 0;
    if (t < T) {
      const int n = nnz[t];
      parts = (slot_off[t] >= 0) ? (n + kPart - 1) / kPart : 1;
    }
    int tot;
    const int ex = block_exclusive_scan(parts, warp_sums, &tot) + carry_items;
    if (t < T) {
      item_off[t] = ex;
      for (int p = 0; p < parts && ex + p < max_items; ++p) item_token[ex + p] = t;
    }
    if (threadIdx.x == 0) carry_items += tot;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    item_off[T] = carry_items;
    hdr[1] = carry_items < max_items ? carry_items : max_items;
  }
}

// ----------------------------------------------------------- element types --
template <typename T>
struct Elem;

template <>
struct Elem<uint16_t> {  // bf16
  static constexpr int E = 8;  // values per 16-byte slice
  TW_DEV static float scalar(uint16_t v) { return bf16_to_f32(v); }
  // acc0 += x.lo*w.lo, acc1 += x.hi*w.hi for every bf16 pair of a slice
  TW_DEV static void dot(const uint4& x, const uint4& w, float& a0, float& a1) {
    dot_pair(x.x, w.x, a0, a1);
    dot_pair(x.y, w.y, a0, a1);
    dot_pair(x.z, w.z, a0, a1);
    dot_pair(x.w, w.w, a0, a1);
  }
  TW_DEV static void dot_pair(uint32_t xp, uint32_t wp, float& a0, float& a1) {
    asm("{\n\t.reg .b16 xl, xh, wl, wh;\n\t"
        "mov.b32 {xl, xh}, %2;\n\t"
        "mov.b32 {wl, wh}, %3;\n\t"
        "fma.rn.f32.bf16 %0, xl, wl, %0;\n\t"
        "fma.rn.f32.bf16 %1, xh, wh, %1;\n\t}"
        : "+f"(a0), "+f"(a1)
        : "r"(xp), "r"(wp));
  }
  // acc[0..7] += h * w[0..7]
  TW_DEV static void axpy(float h, const uint4& w, float* acc) {
    axpy_pair(h, w.x, acc[0], acc[1]);
    axpy_pair(h, w.y, acc[2], acc[3]);
    axpy_pair(h, w.z, acc[4], acc[5]);
    axpy_pair(h, w.w, acc[6], acc[7]);
  }
  TW_DEV static void axpy_pair(float h, uint32_t wp, float& a0, float& a1) {
    const float w0 = bf16_lo(wp), w1 = bf16_hi(wp);
    asm("{\n\t.reg .b64 hh, ww, aa;\n\t"
        "mov.b64 hh, {%2, %2};\n\t"
        "mov.b64 ww, {%3, %4};\n\t"
        "mov.b64 aa, {%0, %1};\n\t"
        "fma.rn.f32x2 aa, hh, ww, aa;\n\t"
        "mov.b64 {%0, %1}, aa;\n\t}"
        : "+f"(a0), "+f"(a1)
        : "f"(h), "f"(w0), "f"(w1));
  }
};

template <>
struct Elem<float> {
  static constexpr int E = 4;
  TW_DEV static float scalar(float v) { return v; }
  TW_DEV static void dot(const uint4& x, const uint4& w, float& a0, float& a1) {
    a0 = fmaf(__uint_as_float(x.x), __uint_as_float(w.x), a0);
    a1 = fmaf(__uint_as_float(x.y), __uint_as_float(w.y), a1);
    a0 = fmaf(__uint_as_float(x.z), __uint_as_float(w.z), a0);
    a1 = fmaf(__uint_as_float(x.w), __uint_as_float(w.w), a1);
  }
  TW_DEV static void axpy(float h, const uint4& w, float* acc) {
    acc[0] = fmaf(h, __uint_as_float(w.x), acc[0]);
    acc[1] = fmaf(h, __uint_as_float(w.y), acc[1]);
    acc[2] = fmaf(h, __uint_as_float(w.z), acc[2]);
    acc[3] = fmaf(h, __uint_as_float(w.w), acc[3]);
  }
};

TW_DEV void bulk_g2s(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes),
        "r"(smem_u32(bar))
      : "memory");
}
TW_DEV void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
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
  FusedWs ws;
  int stages;        // ring depth per warp
  int stage_bytes;   // 2 rows
  unsigned long long timeout_ns;
};

struct WarpSmem {
  uint64_t* bar;     // [stages]
  float* g;          // [kListCap]
  int32_t* j;        // [kListCap]
  uint8_t* ring;     // [stages][stage_bytes]
};

// Collect the entries of token t with ordinal in [lo, hi) (tile-major order,
// ascending within a tile) into the warp's list.  Returns the number written.
template <typename Tin>
TW_DEV int collect(const FusedArgs<Tin>& a, int t, int lo, int hi, const WarpSmem& s, int lane) {
  const int K = a.F / W;
  int base = 0;  // ordinal of the first entry of tile kb
  for (int kb = 0; kb < K && base < hi; kb += 32) {
    const int k = kb + lane;
    const int n = k < K ? (int)a.cnt[(size_t)k * a.T + t] : 0;
    int incl = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(FULL, incl, o);
      if (lane >= o) incl += u;
    }
    const int tb = base + incl - n;  // first ordinal of tile k
    unsigned act = __ballot_sync(FULL, n > 0 && tb < hi && tb + n > lo);
    while (act) {
      const int b = __ffs(act) - 1;
      act &= act - 1;
      const int nk = __shfl_sync(FULL, n, b);
      const int o0 = __shfl_sync(FULL, tb, b);
      const int kk = kb + b;
      const size_t kt = (size_t)kk * a.T + t;
      int ref = -1;
      if (nk > a.C) {
        ref = a.spill_ref[kt];
        if (ref < 0 || ref >= a.spill_cap) {
          // dropped spill entry (capacity, already flagged by the producer):
          // only the C slots are known; the rest of the tile is skipped
          if (lane == 0) set_status(a.status, kStatusSpill);
          ref = -1;
        }
      }
      if (ref < 0) {
        const int m = nk <= a.C ? nk : a.C;
        for (int s0 = 0; s0 < nk; s0 += 32) {
          const int sl = s0 + lane;
          const int o = o0 + sl;
          if (sl < nk && o >= lo && o < hi) {
            // ordinals past the known slots contribute nothing (g = 0)
            s.g[o - lo] = sl < m ? Elem<Tin>::scalar(a.val[kt * a.C + sl]) : 0.f;
            s.j[o - lo] = sl < m ? kk * W + a.idx[kt * a.C + sl] : kk * W;
          }
        }
      } else {
        const Tin* seg = a.spill_val + (size_t)ref * W;
        int r = 0;
#pragma unroll 1
        for (int part = 0; part < W / 32; ++part) {
          const float v = Elem<Tin>::scalar(seg[part * 32 + lane]);
          const unsigned m = __ballot_sync(FULL, v != 0.f);
          const int o = o0 + r + __popc(m & ((1u << lane) - 1u));
          if (v != 0.f && o >= lo && o < hi) {
            s.g[o - lo] = v;
            s.j[o - lo] = kk * W + part * 32 + lane;
          }
          r += __popc(m);
        }
      }
    }
    base += __shfl_sync(FULL, incl, 31);
  }
  __syncwarp();
  const int got = (base < hi ? base : hi) - lo;
  return got > 0 ? got : 0;
}

template <typename Tin, int NCH, bool kOutBf16>
__global__ void __launch_bounds__(32 * kWarps, 1) fused_kernel(const FusedArgs<Tin> a) {
  using L = Elem<Tin>;
  constexpr int E = L::E;
  constexpr int SPAN = 32 * E;  // columns covered by one warp-wide 16-byte slice
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const int lane = threadIdx.x & 31;
  const int wid = threadIdx.x >> 5;
  const int d = a.d;
  const uint32_t row_bytes = (uint32_t)d * sizeof(Tin);

  // per-warp shared memory: barriers, entry list, ring
  const size_t per_warp = 128 + kListCap * 8 + (size_t)a.stages * a.stage_bytes;
  uint8_t* mine = smem_raw + (size_t)wid * per_warp;
  WarpSmem s;
  s.bar = reinterpret_cast<uint64_t*>(mine);
  s.g = reinterpret_cast<float*>(mine + 128);
  s.j = reinterpret_cast<int32_t*>(mine + 128 + kListCap * 4);
  s.ring = mine + 128 + kListCap * 8;
  if (lane == 0) {
    for (int i = 0; i < a.stages; ++i) mbar_init(&s.bar[i], 1);
    fence_mbar_init();
  }
  __syncwarp();
  int never = 0;
  uint32_t issued = 0, consumed = 0;  // bulk-copy stages issued / waited, this warp
  bool failed = false;

  for (;;) {
    int item = 0;
    if (lane == 0) item = atomicAdd(&a.ws.hdr[0], 1);
    item = __shfl_sync(FULL, item, 0);
    if (item >= a.ws.hdr[1]) break;
    const int t = a.ws.item_token[item];
    const int p = item - a.ws.item_off[t];
    const int nnz = a.ws.nnz[t];
    const bool split = a.ws.slot_off[t] >= 0;
    const int lo = split ? p * kPart : 0;
    const int hi = split ? min(nnz, lo + kPart) : nnz;

    uint4 xr[NCH];
    const Tin* xt = a.x + (size_t)t * d;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const int col = c * SPAN + lane * E;
      xr[c] = col < d ? __ldg(reinterpret_cast<const uint4*>(xt + col)) : make_uint4(0, 0, 0, 0);
    }
    float acc[NCH][E];
#pragma unroll
    for (int c = 0; c < NCH; ++c)
#pragma unroll
      for (int e = 0; e < E; ++e) acc[c][e] = 0.f;

    for (int w0 = lo; w0 < hi && !failed; w0 += kListCap) {
      const int n = collect(a, t, w0, min(hi, w0 + kListCap), s, lane);
      // prologue: fill the ring
      const int pre = n < a.stages ? n : a.stages;
      if (lane == 0) {
        for (int e = 0; e < pre; ++e) {
          const uint32_t st = (issued + e) % a.stages;
          uint8_t* dst = s.ring + (size_t)st * a.stage_bytes;
          const int j = s.j[e];
          fence_proxy_async_smem();
          mbar_arrive_expect_tx(&s.bar[st], 2 * row_bytes);
          bulk_g2s(dst, a.Wu_t + (size_t)j * d, row_bytes, &s.bar[st]);
          bulk_g2s(dst + row_bytes, a.Wd + (size_t)j * d, row_bytes, &s.bar[st]);
        }
      }
      uint32_t base_issue = issued;
      issued += pre;
      for (int e = 0; e < n; ++e) {
        const uint32_t seq = base_issue + e;
        const uint32_t st = seq % a.stages;
        const uint32_t ph = (seq / a.stages) & 1u;
        bool ok = mbar_wait(&s.bar[st], ph, &never, a.timeout_ns);
        ok = __all_sync(FULL, ok);
        if (!ok) {
          failed = true;
          break;
        }
        consumed = seq + 1;
        const uint8_t* stage = s.ring + (size_t)st * a.stage_bytes;
        const uint4* wu = reinterpret_cast<const uint4*>(stage);
        const uint4* wd = reinterpret_cast<const uint4*>(stage + row_bytes);
        float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          const int col = c * SPAN + lane * E;
          if (col < d) {
            const uint4 w = wu[col / E];
            if (c & 1) L::dot(xr[c], w, p2, p3);
            else L::dot(xr[c], w, p0, p1);
          }
        }
        const float u = warp_sum((p0 + p1) + (p2 + p3));
        const float h = s.g[e] * u;
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          const int col = c * SPAN + lane * E;
          if (col < d) L::axpy(h, wd[col / E], acc[c]);
        }
        __syncwarp();  // every lane is done with this stage
        const int nxt = e + a.stages;
        if (lane == 0 && nxt < n) {
          const int j = s.j[nxt];
          uint8_t* dst = s.ring + (size_t)st * a.stage_bytes;
          fence_proxy_async_smem();
          mbar_arrive_expect_tx(&s.bar[st], 2 * row_bytes);
          bulk_g2s(dst, a.Wu_t + (size_t)j * d, row_bytes, &s.bar[st]);
          bulk_g2s(dst + row_bytes, a.Wd + (size_t)j * d, row_bytes, &s.bar[st]);
        }
        if (nxt < n) ++issued;
      }
      __syncwarp();
    }
    if (failed) break;

    // ------------------------------------------------------------ output --
    float* out_row = nullptr;
    if (split) out_row = a.ws.partial + (size_t)(a.ws.slot_off[t] + p) * d;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const int col = c * SPAN + lane * E;
      if (col >= d) continue;
      if (split) {
#pragma unroll
        for (int q = 0; q < E / 4; ++q)
          reinterpret_cast<float4*>(out_row + col)[q] =
              make_float4(acc[c][4 * q], acc[c][4 * q + 1], acc[c][4 * q + 2], acc[c][4 * q + 3]);
      } else if (kOutBf16) {
        uint16_t* yt = static_cast<uint16_t*>(a.y) + (size_t)t * d + col;
#pragma unroll
        for (int q = 0; q < E / 2; ++q)
          reinterpret_cast<uint32_t*>(yt)[q] = pack_bf16x2(acc[c][2 * q], acc[c][2 * q + 1]);
      } else {
        float* yt = static_cast<float*>(a.y) + (size_t)t * d + col;
#pragma unroll
        for (int q = 0; q < E / 4; ++q)
          reinterpret_cast<float4*>(yt)[q] =
              make_float4(acc[c][4 * q], acc[c][4 * q + 1], acc[c][4 * q + 2], acc[c][4 * q + 3]);
      }
    }
    if (split) {
      // the last part to finish sums the partial rows in part order
      __threadfence();
      __syncwarp();
      const int parts = a.ws.item_off[t + 1] - a.ws.item_off[t];
      int prev = 0;
      if (lane == 0) prev = atomicAdd(&a.ws.done[t], 1);
      prev = __shfl_sync(FULL, prev, 0);
      if (prev == parts - 1) {
        __threadfence();
        const float* part0 = a.ws.partial + (size_t)a.ws.slot_off[t] * d;
        for (int col = lane * 4; col < d; col += 128) {
          float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int q = 0; q < parts; ++q) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(part0 + (size_t)q * d + col));
            sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
          }
          if (kOutBf16) {
            uint16_t* yt = static_cast<uint16_t*>(a.y) + (size_t)t * d + col;
            reinterpret_cast<uint2*>(yt)[0] = make_uint2(pack_bf16x2(sum.x, sum.y),
                                                         pack_bf16x2(sum.z, sum.w));
          } else {
            *reinterpret_cast<float4*>(static_cast<float*>(a.y) + (size_t)t * d + col) = sum;
          }
        }
      }
    }
  }

  if (failed) {
    if (lane == 0) set_status(a.status, kStatusTimeout);
    // let the copies still in flight land before the CTA may exit
    for (uint32_t q = consumed; q < issued; ++q)
      mbar_wait(&s.bar[q % a.stages], (q / a.stages) & 1u, &never, a.timeout_ns);
  }
}

template <typename Tin, int NCH>
cudaError_t launch_t(FusedArgs<Tin> a, tw_dtype y_dtype, cudaStream_t stream) {
  a.stage_bytes = 2 * a.d * (int)sizeof(Tin);
  a.stages = kRingBytes / a.stage_bytes;
  if (a.stages > 8) a.stages = 8;
  if (a.stages < 2) a.stages = 2;
  const size_t per_warp = 128 + kListCap * 8 + (size_t)a.stages * a.stage_bytes;
  const size_t smem = per_warp * kWarps;
  auto kern_bf = fused_kernel<Tin, NCH, true>;
  auto kern_f = fused_kernel<Tin, NCH, false>;
  auto kern = y_dtype == TW_BF16 ? kern_bf : kern_f;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 32 * kWarps, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  kern<<<num_sms() * per_sm, 32 * kWarps, smem, stream>>>(a);
  return cudaGetLastError();
}

// Layout of the same work plan inside a fixed scratch area of `limit` bytes:
// the split capacity shrinks to what fits (tokens past it stay unsplit).
// Returns false when even the unsplit plan does not fit.
bool carve_within(void* base, int T, int d, size_t limit, FusedWs* out) {
  const int full_cap = T / 2 + 256;
  int lo = 0, hi = full_cap;  // largest parts_cap whose layout fits
  auto layout = [&](int cap) {
    FusedWs w{};
    w.parts_cap = cap;
    w.max_items = T + cap;
    size_t off = 0;
    auto take = [&](size_t b) { size_t o = off; off = al256(off + b); return o; };
    const size_t o_hdr = take(4 * sizeof(int32_t));
    const size_t o_done = take(sizeof(int32_t) * (size_t)T);
    w.zero_bytes = off;
    const size_t o_nnz = take(sizeof(int32_t) * (size_t)T);
    const size_t o_off = take(sizeof(int32_t) * ((size_t)T + 1));
    const size_t o_slot = take(sizeof(int32_t) * (size_t)T);
    const size_t o_item = take(sizeof(int32_t) * (size_t)w.max_items);
    const size_t o_part = take(sizeof(float) * (size_t)(cap > 0 ? cap : 1) * d);
    w.bytes = off;
    if (base) {
      char* p = static_cast<char*>(base);
      w.hdr = reinterpret_cast<int32_t*>(p + o_hdr);
      w.done = reinterpret_cast<int32_t*>(p + o_done);
      w.nnz = reinterpret_cast<int32_t*>(p + o_nnz);
      w.item_off = reinterpret_cast<int32_t*>(p + o_off);
      w.slot_off = reinterpret_cast<int32_t*>(p + o_slot);
      w.item_token = reinterpret_cast<int32_t*>(p + o_item);
      w.partial = reinterpret_cast<float*>(p + o_part);
    }
    return w;
  };
  if (layout(0).bytes > limit) return false;
  while (lo < hi) {
    const int mid = lo + (hi - lo + 1) / 2;
    if (layout(mid).bytes <= limit) lo = mid;
    else hi = mid - 1;
  }
  *out = layout(lo);
  return true;
}

}  // namespace

size_t fused_ws_bytes(int T, int d) { return carve(nullptr, T, d).bytes; }

bool fused_plan_fits(int T, int d, size_t limit) {
  FusedWs w;
  return carve_within(nullptr, T, d, limit, &w);
}

cudaError_t launch_fused_updown_in_scratch(const void* x, const tw_twell& g, const void* Wu_t,
                                           const void* Wd, int d, void* y, tw_dtype y_dtype,
                                           void* scratch, size_t scratch_bytes, int32_t* status,
                                           cudaStream_t stream) {
  FusedWs w;
  if (!carve_within(scratch, g.T, d, scratch_bytes, &w)) return cudaErrorInvalidValue;
  cudaError_t e = cudaMemsetAsync(scratch, 0, w.zero_bytes, stream);
  if (e != cudaSuccess) return e;
  const int K = g.F / W;
  plan_count_kernel<<<(g.T + 255) / 256, 256, 0, stream>>>(g.T, K, g.cnt, w.nnz);
  plan_scan_kernel<<<1, kScanThreads, 0, stream>>>(g.T, w.nnz, w.parts_cap, w.max_items,
                                                   w.slot_off, w.item_off, w.item_token, w.hdr);
  if (g.dtype == TW_BF16) {
    FusedArgs<uint16_t> a{static_cast<const uint16_t*>(x), static_cast<const uint16_t*>(g.val),
                          g.idx, g.cnt, g.spill_ref, static_cast<const uint16_t*>(g.spill_val),
                          static_cast<const uint16_t*>(Wu_t), static_cast<const uint16_t*>(Wd),
                          y, status, g.T, d, g.F, g.C, g.spill_cap, w, 0, 0, kWaitTimeoutNs};
    if (d <= 256) return launch_t<uint16_t, 1>(a, y_dtype, stream);
    if (d <= 512) return launch_t<uint16_t, 2>(a, y_dtype, stream);
    if (d <= 1024) return launch_t<uint16_t, 4>(a, y_dtype, stream);
    return launch_t<uint16_t, 8>(a, y_dtype, stream);
  }
  FusedArgs<float> a{static_cast<const float*>(x), static_cast<const float*>(g.val), g.idx, g.cnt,
                     g.spill_ref, static_cast<const float*>(g.spill_val),
                     static_cast<const float*>(Wu_t), static_cast<const float*>(Wd), y, status,
                     g.T, d, g.F, g.C, g.spill_cap, w, 0, 0, kWaitTimeoutNs};
  if (d <= 128) return launch_t<float, 1>(a, y_dtype, stream);
  if (d <= 256) return launch_t<float, 2>(a, y_dtype, stream);
  if (d <= 512) return launch_t<float, 4>(a, y_dtype, stream);
  if (d <= 1024) return launch_t<float, 8>(a, y_dtype, stream);
  return launch_t<float, 16>(a, y_dtype, stream);
}

cudaError_t launch_fused_updown(const void* x, const tw_twell& g, const void* Wu_t,
                                const void* Wd, int d, void* y, tw_dtype y_dtype, void* ws,
                                int32_t* status, cudaStream_t stream) {
  const FusedWs w = carve(ws, g.T, d);
  cudaError_t e = cudaMemsetAsync(ws, 0, w.zero_bytes, stream);
  if (e != cudaSuccess) return e;
  const int K = g.F / W;
  plan_count_kernel<<<(g.T + 255) / 256, 256, 0, stream>>>(g.T, K, g.cnt, w.nnz);
  plan_scan_kernel<<<1, kScanThreads, 0, stream>>>(g.T, w.nnz, w.parts_cap, w.max_items,
                                                   w.slot_off, w.item_off, w.item_token, w.hdr);
  if (g.dtype == TW_BF16) {
    FusedArgs<uint16_t> a{static_cast<const uint16_t*>(x), static_cast<const uint16_t*>(g.val),
                          g.idx, g.cnt, g.spill_ref, static_cast<const uint16_t*>(g.spill_val),
                          static_cast<const uint16_t*>(Wu_t), static_cast<const uint16_t*>(Wd),
                          y, status, g.T, d, g.F, g.C, g.spill_cap, w, 0, 0, kWaitTimeoutNs};
    if (d <= 256) return launch_t<uint16_t, 1>(a, y_dtype, stream);
    if (d <= 512) return launch_t<uint16_t, 2>(a, y_dtype, stream);
    if (d <= 1024) return launch_t<uint16_t, 4>(a, y_dtype, stream);
    return launch_t<uint16_t, 8>(a, y_dtype, stream);
  }
  FusedArgs<float> a{static_cast<const float*>(x), static_cast<const float*>(g.val), g.idx, g.cnt,
                     g.spill_ref, static_cast<const float*>(g.spill_val),
                     static_cast<const float*>(Wu_t), static_cast<const float*>(Wd), y, status,
                     g.T, d, g.F, g.C, g.spill_cap, w, 0, 0, kWaitTimeoutNs};
  if (d <= 128) return launch_t<float, 1>(a, y_dtype, stream);
  if (d <= 256) return launch_t<float, 2>(a, y_dtype, stream);
  if (d <= 512) return launch_t<float, 4>(a, y_dtype, stream);
  if (d <= 1024) return launch_t<float, 8>(a, y_dtype, stream);
  return launch_t<float, 16>(a, y_dtype, stream);
}

}  // namespace tw
