// fused_updown.cu -- the gather engine: per-token work over a sparse
// activation pattern, where each active (t, j) gathers rows j of dense
// weights, forms one dot product with a row of the token and adds scaled
// weight rows to an fp32 output row of the token.  Three modes:
//
//   kModeTwell   inference ("Sparser, Faster, Lighter Transformer Language
//                Models", technical summary, section 2.2), entries from TwELL:
//                  u = x_t . Wu_t[j],  y_t += (g u) Wd[j];
//   kModeHybFwd  training forward on the hybrid pattern (sections 2.3-2.4):
//                  the same, and u is saved (rounded) at the entry;
//   kModeHybBwd  training backward on the hybrid pattern (section 2.4):
//                  dh = dy_t . Wd[j],  du = dh g,  dz = dh u + lambda,
//                  dx_t += du Wu_t[j] + dz Wg_t[j],  and (t, g u, du, dz) is
//                  recorded for the weight-gradient pass.
// No dense intermediate is written to memory.
//
// Work decomposition.  Per-token activity is very uneven (a few tokens carry
// tens of times the median number of active units), so a token with more
// than `part` active units is split into parts:
//   1. plan_count_*        entries per token, and per-block partials;
//   2. plan_scan_kernel    (one CTA) the part size (adapted to the total work),
//                          partial-buffer rows for split tokens (bounded by
//                          the workspace), one descriptor {t, first entry,
//                          end entry, partial row} per work item; when the
//                          part size is the largest and every split fits,
//                          only the block partials are scanned and
//                          plan_write_kernel writes the same plan in parallel;
//   3. gather_kernel       persistent teams take work items from a ticket
//                          counter (the next ticket is fetched while the
//                          current item runs).
// The launches are programmatic dependent launches: each kernel's start-up
// overlaps the previous kernel's tail, and waits for its results before its
// first global access.  The planner clears the ticket and the arrival
// counters, so a call needs no memset.
// A split token's parts are added up a binary tree over the part index
// through fp32 partial rows in the workspace (one arrival counter per tree
// node); the tree's shape is fixed by the number of parts, so the output is
// deterministic, and its depth, not the number of parts, sets the time the
// last part spends on the sum.
//
// Teams.  An item is processed by a team of kTeam warps; warp w of the team
// owns one contiguous range of the d columns (the token's row and the output
// of that range live in its registers).  A window of up to kListCap entries
// runs in two phases: each warp forms its partial dot products of all the
// window's entries, two at a time, and leaves them in shared memory; after
// one named barrier each warp adds the team's partials in warp order, derives
// the entry's scalars and updates its own columns.  Entry lists alternate
// between two buffers and the next item's descriptor is published during the
// current item, so a window costs two team barriers (list written, partials
// written) and an item none of its own.
//
// Data movement.  Weight rows are gathered with plain 16-byte vector loads
// straight into registers (each lane owns 16-byte column slices, so a warp's
// load of a row slice is fully coalesced).  In each phase two register sets
// hold the rows of two entry pairs; a set is reloaded with the rows of the
// pair after next as soon as it has been consumed, so loads stay in flight
// through the phase.  (Bulk copies into shared memory were the first design;
// the copy engine spends a roughly fixed time per copy, which bounded that
// version by the number of row slices, not by bytes.)
//
// Arithmetic.  bf16 dot products use the mixed-precision FMA (bf16 operands,
// fp32 accumulator); the scaled-row updates widen bf16 pairs exactly and use
// packed fp32x2 FMA.
#include "pdl.cuh"
#include "tw_common.cuh"
#include "tw_internal.h"

namespace tw {
namespace {

constexpr unsigned FULL = 0xFFFFFFFFu;
constexpr int kPart = 64;          // entries per part of a split token (upper bound)
constexpr int kMinPart = 8;        // lower bound of the part size
// Items of split tokens and unsplit tokens with at least kHeavy entries are
// handed out first: with the long items taken early, the last items of the
// launch are short and the teams finish close together.
constexpr int kHeavy = 32;
constexpr int kTeam = 2;           // warps per work item
constexpr int kTeams = 8;          // teams per CTA
constexpr int kListCap = 64;       // entry window collected at a time
constexpr int kCountBlock = 256;   // tokens per block of the count kernels

enum : int { kModeTwell = 0, kModeHybFwd = 1, kModeHybBwd = 2 };

// --------------------------------------------------------------- workspace --
struct FusedWs {
  int32_t* hdr;        // [0] item ticket, [1] number of items, [2] part size, [3] fast plan
  int32_t* done;       // [parts_cap] arrivals per internal node of a split token's sum tree
  int32_t* nnz;        // [T]
  int32_t* slot_off;   // [T] first partial row of a split token, -1 if whole
  int4* item_desc;     // [max_items] {t, lo, hi, partial row or -1}
  int4* bpart;         // [nb] per block of kCountBlock tokens: entries, split parts and items
                       // with the largest part size; the planner's fast path scans them
  float* partial;      // [parts_cap][d]
  int parts_cap, max_items;
  size_t bytes;        // hdr[0] and done are cleared by the planner (plan_scan_kernel)
};

size_t al256(size_t v) { return (v + 255) & ~size_t(255); }

// Layout of the workspace for T tokens of width d with room for `cap`
// partial rows; pointers are set when base is not null.
FusedWs layout(void* base, int T, int d, int cap) {
  FusedWs w{};
  w.parts_cap = cap;
  w.max_items = T + cap;
  size_t off = 0;
  auto take = [&](size_t b) { size_t o = off; off = al256(off + b); return o; };
  const size_t o_hdr = take(4 * sizeof(int32_t));
  const size_t o_done = take(sizeof(int32_t) * (size_t)(cap > 0 ? cap : 1));
  const size_t o_nnz = take(sizeof(int32_t) * (size_t)T);
  const size_t o_slot = take(sizeof(int32_t) * (size_t)T);
  const size_t o_desc = take(sizeof(int4) * (size_t)w.max_items);
  const size_t o_bpart = take(sizeof(int4) * ((size_t)T / kCountBlock + 1));
  const size_t o_part = take(sizeof(float) * (size_t)(cap > 0 ? cap : 1) * d);
  w.bytes = off;
  if (base) {
    char* p = static_cast<char*>(base);
    w.hdr = reinterpret_cast<int32_t*>(p + o_hdr);
    w.done = reinterpret_cast<int32_t*>(p + o_done);
    w.nnz = reinterpret_cast<int32_t*>(p + o_nnz);
    w.slot_off = reinterpret_cast<int32_t*>(p + o_slot);
    w.item_desc = reinterpret_cast<int4*>(p + o_desc);
    w.bpart = reinterpret_cast<int4*>(p + o_bpart);
    w.partial = reinterpret_cast<float*>(p + o_part);
  }
  return w;
}

FusedWs carve(void* base, int T, int d) { return layout(base, T, d, T / 2 + 1024); }

// The same plan inside a fixed scratch area of `limit` bytes: the split
// capacity shrinks to what fits (tokens past it stay unsplit).  Returns false
// when even the unsplit plan does not fit.
bool carve_within(void* base, int T, int d, size_t limit, FusedWs* out) {
  if (layout(nullptr, T, d, 0).bytes > limit) return false;
  int lo = 0, hi = T / 2 + 1024;  // largest capacity whose layout fits
  while (lo < hi) {
    const int mid = lo + (hi - lo + 1) / 2;
    if (layout(nullptr, T, d, mid).bytes <= limit) lo = mid;
    else hi = mid - 1;
  }
  *out = layout(base, T, d, lo);
  return true;
}

// -------------------------------------------------------------------- plan --
// Per-block partials for the planner's fast path: entries, split parts, work
// items and heavy items (see kHeavy) of the block's tokens with the part size
// kPart (thread 0 writes).
TW_DEV void count_block_partials(int n, bool valid, int4* bpart) {
  __shared__ int red[4][kCountBlock / 32];
  const int parts = n > kPart ? (n + kPart - 1) / kPart : 0;
  int v[4] = {n, parts, valid ? (parts > 0 ? parts : 1) : 0,
              valid ? (parts > 0 ? parts : (n >= kHeavy ? 1 : 0)) : 0};
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v[i] += __shfl_xor_sync(FULL, v[i], o);
    if (lane == 0) red[i][wid] = v[i];
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int4 r = make_int4(0, 0, 0, 0);
    for (int w2 = 0; w2 < kCountBlock / 32; ++w2) {
      r.x += red[0][w2];
      r.y += red[1][w2];
      r.z += red[2][w2];
      r.w += red[3][w2];
    }
    bpart[blockIdx.x] = r;
  }
}

__global__ void __launch_bounds__(kCountBlock)
    plan_count_twell_kernel(int T, int K, const uint8_t* __restrict__ cnt, int32_t* nnz,
                            int4* bpart) {
  pdl_wait();  // the counts come from the gate
  pdl_launch_next();
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  int s = 0;
  if (t < T) {
    for (int k = 0; k < K; ++k) s += cnt[(size_t)k * T + t];
    nnz[t] = s;
  }
  count_block_partials(s, t < T, bpart);
}

// Hybrid rows: the row's non-zero count, or 0 for a backup row that was not
// stored (capacity exceeded, flagged by the conversion).
__global__ void __launch_bounds__(kCountBlock)
    plan_count_hybrid_kernel(int T, const int32_t* __restrict__ row_nnz,
                             const int32_t* __restrict__ row_slot, int cap, int32_t* nnz,
                             int4* bpart) {
  pdl_wait();
  pdl_launch_next();
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  int s = 0;
  if (t < T) {
    s = row_slot[t] >= cap ? 0 : row_nnz[t];
    nnz[t] = s;
  }
  count_block_partials(s, t < T, bpart);
}

constexpr int kScanThreads = 1024;

// Block-wide exclusive scan of one value per thread; *total gets the sum.
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

// Largest T whose per-token counts are staged in shared memory by the planner
// (with one padding word per run of tokens).
constexpr int kScanSmemTokens = 40960;
size_t plan_scan_smem(int T) {
  if (T > kScanSmemTokens) return 0;
  const int run = (T + kScanThreads - 1) / kScanThreads;
  return sizeof(int32_t) * ((size_t)T + T / (run > 0 ? run : 1) + 1);
}

// One CTA: the part size, partial rows of split tokens (in token order,
// within capacity), then one descriptor per work item: heavy items (see
// kHeavy) first, then the others, each group in token order.  The part size is
// kPart, lowered to about two items per team when there are few entries in
// all (small batches), but not below kMinPart; it is stored in hdr[2].
// Each thread owns a contiguous run of tokens, so each of the three passes
// needs a single block-wide scan.  The counts are first copied into shared
// memory with coalesced loads (a padding word after every run keeps the
// threads' strided reads free of bank conflicts); beyond kScanSmemTokens the
// passes read them from global memory.
__global__ void __launch_bounds__(kScanThreads)
    plan_scan_kernel(int T, const int32_t* __restrict__ nnz, int parts_cap, int max_items,
                     int n_teams, int32_t* slot_off, int4* item_desc, int32_t* hdr, int4* bpart,
                     int nb, int32_t* done) {
  __shared__ int warp_sums[32];
  __shared__ int part_sh;
  extern __shared__ int32_t staged[];
  pdl_wait();
  pdl_launch_next();
  // the engine's item ticket and the arrival counters of split tokens' sum
  // trees start at zero (the gather kernel, two launches on, uses them)
  if (threadIdx.x == 0) hdr[0] = 0;
  for (int i = threadIdx.x; i < parts_cap; i += kScanThreads) done[i] = 0;
  // Fast path, from the count kernels' per-block partials: when there is
  // enough work for the largest part size and every split token fits the
  // partial rows, the plan below would use part = kPart and split every token
  // with more entries.  Then only the block partials are scanned here (into
  // per-block offsets of split parts and items) and plan_write_kernel writes
  // the same plan with one thread per token.
  {
    int e = 0, sp = 0, it = 0, hv = 0;
    for (int b = threadIdx.x; b < nb; b += kScanThreads) {
      const int4 v = bpart[b];
      e += v.x;
      sp += v.y;
      it += v.z;
      hv += v.w;
    }
    int te, tsp, tit, thv;
    block_exclusive_scan(e, warp_sums, &te);
    block_exclusive_scan(sp, warp_sums, &tsp);
    block_exclusive_scan(it, warp_sums, &tit);
    block_exclusive_scan(hv, warp_sums, &thv);
    if (te / (2 * n_teams) >= kPart && tsp <= parts_cap) {
      // per block: first split part, first heavy item, first other item
      int carry_s = 0, carry_h = 0, carry_l = 0;
      for (int b0 = 0; b0 < nb; b0 += kScanThreads) {
        const int b = b0 + threadIdx.x;
        const int4 v = b < nb ? bpart[b] : make_int4(0, 0, 0, 0);
        int ts2, th2, tl2;
        const int xs = block_exclusive_scan(v.y, warp_sums, &ts2);
        const int xh = block_exclusive_scan(v.w, warp_sums, &th2);
        const int xl = block_exclusive_scan(v.z - v.w, warp_sums, &tl2);
        if (b < nb) bpart[b] = make_int4(carry_s + xs, carry_h + xh, thv + carry_l + xl, 0);
        carry_s += ts2;
        carry_h += th2;
        carry_l += tl2;
      }
      if (threadIdx.x == 0) {
        hdr[1] = tit < max_items ? tit : max_items;
        hdr[2] = kPart;
        hdr[3] = 1;
      }
      return;
    }
    if (threadIdx.x == 0) hdr[3] = 0;
  }
  const int run = (T + kScanThreads - 1) / kScanThreads;
  const int t0 = threadIdx.x * run;
  const int t1 = min(T, t0 + run);
  const bool in_smem = T <= kScanSmemTokens;
  if (in_smem) {
#pragma unroll 8
    for (int i = threadIdx.x; i < T; i += kScanThreads) staged[i + i / run] = nnz[i];
    __syncthreads();
  }
  auto count = [&](int t) { return in_smem ? staged[t + t / run] : nnz[t]; };
  // pass 0: total number of entries -> part size
  int local = 0;
  for (int t = t0; t < t1; ++t) local += count(t);
  int total;
  block_exclusive_scan(local, warp_sums, &total);
  if (threadIdx.x == 0) {
    const int p = total / (2 * n_teams);
    part_sh = p < kMinPart ? kMinPart : (p > kPart ? kPart : p);
    hdr[2] = part_sh;
  }
  __syncthreads();
  const int part = part_sh;
  // pass 1: partial rows of split tokens, in token order; a token whose rows
  // would pass the capacity (and every later one) stays unsplit
  local = 0;
  for (int t = t0; t < t1; ++t) {
    const int n = count(t);
    local += n > part ? (n + part - 1) / part : 0;
  }
  int tot;
  const int ex1 = block_exclusive_scan(local, warp_sums, &tot);
  // pass 2: one descriptor per work item, heavy items first (the slot
  // decision of pass 1 is recomputed from the same running offset)
  int local_h = 0, local_l = 0;
  int ex = ex1;
  for (int t = t0; t < t1; ++t) {
    const int n = count(t);
    const int parts = n > part ? (n + part - 1) / part : 0;
    const bool split = parts > 0 && ex + parts <= parts_cap;
    slot_off[t] = split ? ex : -1;
    if (split)
      local_h += parts;
    else if (n >= kHeavy)
      ++local_h;
    else
      ++local_l;
    ex += parts;
  }
  int tot_h, tot_l;
  int exh = block_exclusive_scan(local_h, warp_sums, &tot_h);
  int exl = tot_h + block_exclusive_scan(local_l, warp_sums, &tot_l);
  ex = ex1;
  for (int t = t0; t < t1; ++t) {
    const int n = count(t);
    const int parts = n > part ? (n + part - 1) / part : 0;
    const bool split = parts > 0 && ex + parts <= parts_cap;
    if (!split) {
      int& at = n >= kHeavy ? exh : exl;
      if (at < max_items) item_desc[at] = make_int4(t, 0, n, -1);
      ++at;
    } else {
      for (int q = 0; q < parts && exh + q < max_items; ++q)
        item_desc[exh + q] = make_int4(t, q * part, min(n, (q + 1) * part), ex + q);
      exh += parts;
    }
    ex += parts;
  }
  tot = tot_h + tot_l;
  if (threadIdx.x == 0) hdr[1] = tot < max_items ? tot : max_items;
}

// The fast-path plan, one thread per token: split parts and items of the
// token from its count, block-local offsets from a block scan plus the
// block's offsets from the planner.  The same plan as the single-CTA path
// with part = kPart.  Does nothing unless the planner took the fast path.
__global__ void __launch_bounds__(kCountBlock)
    plan_write_kernel(int T, const int32_t* __restrict__ nnz, int max_items, int32_t* slot_off,
                      int4* item_desc, const int32_t* hdr, const int4* bpart) {
  __shared__ int warp_sums[32];
  pdl_wait();
  pdl_launch_next();
  if (hdr[3] == 0) return;  // uniform
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  const int n = t < T ? nnz[t] : 0;
  const int parts = n > kPart ? (n + kPart - 1) / kPart : 0;
  const int items = t < T ? (parts > 0 ? parts : 1) : 0;
  const int heavy = t < T ? (parts > 0 ? parts : (n >= kHeavy ? 1 : 0)) : 0;
  int tot;
  const int xs = block_exclusive_scan(parts, warp_sums, &tot);
  const int xh = block_exclusive_scan(heavy, warp_sums, &tot);
  const int xl = block_exclusive_scan(items - heavy, warp_sums, &tot);
  if (t >= T) return;
  const int4 off = bpart[blockIdx.x];  // first split part, heavy item, other item
  const int so = parts > 0 ? off.x + xs : -1;
  slot_off[t] = so;
  const int base = off.y + xh;
  if (parts == 0) {
    const int at = heavy ? base : off.z + xl;
    if (at < max_items) item_desc[at] = make_int4(t, 0, n, -1);
  } else {
    for (int q = 0; q < parts && base + q < max_items; ++q)
      item_desc[base + q] = make_int4(t, q * kPart, min(n, (q + 1) * kPart), so + q);
  }
}

// ------------------------------------------------------------- arithmetic --
// Rows are handled as 16-byte slices of E values = P pairs.
TW_DEV float2 bf16_pair(uint32_t p) {  // exact widening of two packed bf16
  return make_float2(__uint_as_float(p << 16), __uint_as_float(p & 0xFFFF0000u));
}

template <typename T>
struct Elem;

template <>
struct Elem<uint16_t> {       // bf16
  static constexpr int E = 8;  // values per 16-byte slice
  static constexpr int P = 4;  // pairs per slice
  TW_DEV static float scalar(uint16_t v) { return bf16_to_f32(v); }
  TW_DEV static void store(uint16_t* p, float v) { *p = f32_to_bf16(v); }
  TW_DEV static void pairs(const uint4& r, float2 (&w)[P]) {
    w[0] = bf16_pair(r.x); w[1] = bf16_pair(r.y); w[2] = bf16_pair(r.z); w[3] = bf16_pair(r.w);
  }
  // a[0..3] += x . w over one slice with the mixed-precision FMA (bf16
  // inputs, fp32 accumulator; the bf16 product is exact in fp32).
  TW_DEV static void dot(const uint4& x, const uint4& w, float (&a)[4]) {
    dot_pair(x.x, w.x, a[0], a[1]);
    dot_pair(x.y, w.y, a[2], a[3]);
    dot_pair(x.z, w.z, a[0], a[1]);
    dot_pair(x.w, w.w, a[2], a[3]);
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
};

template <>
struct Elem<float> {
  static constexpr int E = 4;
  static constexpr int P = 2;
  TW_DEV static float scalar(float v) { return v; }
  TW_DEV static void store(float* p, float v) { *p = v; }
  TW_DEV static void pairs(const uint4& r, float2 (&w)[P]) {
    w[0] = make_float2(__uint_as_float(r.x), __uint_as_float(r.y));
    w[1] = make_float2(__uint_as_float(r.z), __uint_as_float(r.w));
  }
  TW_DEV static void dot(const uint4& x, const uint4& w, float (&a)[4]) {
    a[0] = fmaf(__uint_as_float(x.x), __uint_as_float(w.x), a[0]);
    a[1] = fmaf(__uint_as_float(x.y), __uint_as_float(w.y), a[1]);
    a[2] = fmaf(__uint_as_float(x.z), __uint_as_float(w.z), a[2]);
    a[3] = fmaf(__uint_as_float(x.w), __uint_as_float(w.w), a[3]);
  }
};

// Sum over the warp of p0 and of p1 with five shuffle steps; lane 0 stores
// the first sum to *s0 and lane 16 the second to *s1.
TW_DEV void warp_sum2(float p0, float p1, int lane, float* s0, float* s1) {
  const bool hi = (lane & 16) != 0;
  float v = hi ? p1 : p0;
  v += __shfl_xor_sync(FULL, hi ? p0 : p1, 16);
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
  if (lane == 0) *s0 = v;
  if (lane == 16) *s1 = v;
}

// This warp's partial dot products of the token row (xr) with the rows of
// two entries (w[0], w[1]), all held in registers as this lane's 16-byte
// slices of the warp's column range; a missing second entry is all zeros.
// dot2_issue leaves four running sums per entry in each lane (bf16: the
// mixed-precision FMA, whose bf16 products are exact in fp32); dot2_reduce
// turns them into the two warp sums, so independent work can be placed
// between the two.  (The tensor pipe was tried for these dot products, with
// the rows of two entries as the A fragment of an m16n8k16 MMA and the
// diagonal of D kept: the chains of dependent MMAs made it slower.)
template <typename Tin, int NCHW>
TW_DEV void dot2_issue(const uint4 (&xr)[NCHW], const uint4 (&w)[2][NCHW], float (&D)[2][4]) {
#pragma unroll
  for (int e = 0; e < 2; ++e)
#pragma unroll
    for (int i = 0; i < 4; ++i) D[e][i] = 0.f;
#pragma unroll
  for (int c = 0; c < NCHW; ++c) {
    Elem<Tin>::dot(xr[c], w[0][c], D[0]);
    Elem<Tin>::dot(xr[c], w[1][c], D[1]);
  }
}

template <typename Tin>
TW_DEV void dot2_reduce(const float (&D)[2][4], int lane, float* v0, float* v1) {
  const float p0 = (D[0][0] + D[0][1]) + (D[0][2] + D[0][3]);
  const float p1 = (D[1][0] + D[1][1]) + (D[1][2] + D[1][3]);
  warp_sum2(p0, p1, lane, v0, v1);
}

// Rows j0 and (when `two`) j1 of a row-major [F][d] weight, this lane's
// slices of columns [c0, c0 + my_cols), into registers (zeros elsewhere).
// Read-only 16-byte load that asks L2 to keep the line (weight rows are
// gathered again by other tokens; activations and outputs stream past them).
TW_DEV uint4 ldg_keep(const uint4* p, uint64_t policy) {
  uint4 r;
  asm("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p), "l"(policy));
  return r;
}
TW_DEV uint64_t policy_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

//
// kFull: every lane's slices lie inside the row (d is exactly kTeam warps'
// slices), so no load is predicated; a missing second entry then re-reads
// the first entry's row, which its zero coefficient leaves without effect.
template <typename Tin, int NCHW, bool kFull>
TW_DEV void load_rows2(uint4 (&w)[2][NCHW], const Tin* base, int j0, int j1, bool two, int d,
                       int c0, int my_cols, int lane, uint64_t pol) {
  constexpr int E = Elem<Tin>::E;
  constexpr int SPAN = 32 * E;
  const uint4* p0 = reinterpret_cast<const uint4*>(base + (size_t)j0 * d + c0);
  if constexpr (kFull) {
    const uint4* p1 = reinterpret_cast<const uint4*>(base + (size_t)(two ? j1 : j0) * d + c0);
#pragma unroll
    for (int c = 0; c < NCHW; ++c) {
      w[0][c] = ldg_keep(p0 + c * 32 + lane, pol);
      w[1][c] = ldg_keep(p1 + c * 32 + lane, pol);
    }
  } else {
    const uint4* p1 = reinterpret_cast<const uint4*>(base + (size_t)j1 * d + c0);
#pragma unroll
    for (int c = 0; c < NCHW; ++c) {
      const int lc = c * SPAN + lane * E;
      const bool in = lc < my_cols;
      w[0][c] = in ? ldg_keep(p0 + lc / E, pol) : make_uint4(0, 0, 0, 0);
      w[1][c] = in && two ? ldg_keep(p1 + lc / E, pol) : make_uint4(0, 0, 0, 0);
    }
  }
}

// Named barrier over the kTeam warps of one team (ids 1..kTeams; 0 is
// __syncthreads).  Every warp of a team executes the same sequence of these.
TW_DEV void team_bar(int team) {
  asm volatile("bar.sync %0, %1;" ::"r"(team + 1), "r"(kTeam * 32) : "memory");
}
TW_DEV unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

template <typename Tin>
struct GatherArgs {
  // TwELL entry source
  const uint8_t* cnt;
  const Tin* val;
  const uint8_t* idx;
  const int32_t* spill_ref;
  const Tin* spill_val;
  int W, C, spill_cap;  // tile width, capacity, spill entries
  int staged;           // TwELL data and token rows are prefetched (see StageSmem)
  // hybrid entry source
  const Tin* ell_g;
  Tin* ell_u;
  const uint16_t* ell_idx;
  const int32_t* row_slot;
  const Tin* backup_g;
  Tin* backup_u;
  int C_h, backup_cap;
  // shapes
  int T, F, d;
  // token rows and gathered weight rows
  const Tin* xin;   // x (inference, forward) or dy (backward)
  const Tin* rdot;  // Wu_t (inference, forward) or Wd (backward)
  const Tin* rax1;  // Wd (inference, forward) or Wu_t (backward)
  const Tin* rax2;  // Wg_t (backward)
  float lam;
  const int32_t* e0;
  Payload* pay;
  void* out;
  int32_t* status;
  FusedWs ws;
};

// Asynchronous copies from global into shared memory; each thread waits for
// its own copies (cp_async_wait_all) before it reads them.
TW_DEV void cp_async16(void* smem, const void* gmem, bool valid) {
  const uint32_t sa = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(sa), "l"(gmem),
               "r"(valid ? 16 : 0)
               : "memory");
}
TW_DEV void cp_async8(void* smem, const void* gmem) {
  const uint32_t sa = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(sa), "l"(gmem) : "memory");
}
TW_DEV void cp_async4(void* smem, const void* gmem) {
  const uint32_t sa = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(sa), "l"(gmem) : "memory");
}
TW_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
TW_DEV void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// The next item's TwELL data and token row, copied into shared memory while
// the current item runs (TwELL mode, when a tile's C slots are 16 bytes, the
// token has at most kStageTiles tiles and the count array can be read in
// aligned 4-byte words).  Lane l of a warp copies, for tile k = 32 r + l of
// every round r, the count word into the warp's own cnt row, and for the
// rounds the warp writes (see collect_twell) the slots, indices and spill
// reference; and its own slices of the token row.  So every thread later
// reads only what it copied itself.
constexpr int kStageTiles = 64;
template <int NCHW>
struct StageSmem {
  uint32_t cnt[kTeam][kStageTiles];
  uint4 val[kStageTiles];
  uint2 idx[kStageTiles];
  int32_t ref[kStageTiles];
  uint4 x[kTeam][NCHW][32];
};

// One window's entry list.
struct EntryList {
  float g[kListCap];
  int32_t j[kListCap];
  int32_t pos[kListCap];  // hybrid position of the entry (u is saved / read there)
  float u[kListCap];      // saved u of the entry (backward)
  alignas(16) float part[kListCap][kTeam];  // each warp's partial dot product per entry
                                           // (a pair's partials are 16 bytes)
};

// Shared state of one team.  Lists alternate by window parity and
// descriptors by item parity, so no barrier is needed before either is
// rewritten: a buffer is written again two windows (items) later, after both
// warps have passed the barriers of the window (item) in between.
struct TeamSmem {
  EntryList list[2];
  int4 desc[2];           // item descriptors, published one item ahead
  int n[2];               // entries in the window, by window parity (hybrid modes)
  int prev;               // arrival count at a sum-tree node, broadcast to the team
};

// TwELL: the entries of token t with ordinal in [lo, hi) (tile-major order,
// ascending within a tile) into a list; returns how many.  Each lane owns one
// tile of a round of 32 tiles, so the slots of all active tiles of a round are
// read at once; spilled tiles are read by the whole warp.  The rounds are
// dealt out to `nwho` warps (this one is `who`): every warp scans every
// round's counts, so all know each entry's ordinal and the total, and each
// writes the entries of its own rounds.
//
// The data of a round are loaded one round ahead and in one go: the count
// and, for a round this warp writes, the tile's slots (one 16-byte load when
// C slots are 16 bytes) with their indices and the spill reference, whether
// or not the tile has entries.  So a list costs one dependent trip to memory
// (two for a token with a spilled tile) instead of one per step.
//
// With `st` (see StageSmem) the round data come from this warp's copies in
// shared memory instead.
template <typename Tin, int NCHW = 1>
TW_DEV int collect_twell(const GatherArgs<Tin>& a, int t, int lo, int hi, float* sg, int32_t* sj,
                         int lane, int who, int nwho, const StageSmem<NCHW>* st = nullptr) {
  constexpr int E = Elem<Tin>::E;  // slots in 16 bytes
  const int W = a.W;
  const int K = a.F / W;
  const int C = a.C;
  const bool vec = C == E;  // a tile's slots are one 16-byte load
  struct Round {
    int n, ref;
    uint4 v;
    uint2 ix;
  };
  auto fetch = [&](int kb) {
    Round r{0, -1, make_uint4(0, 0, 0, 0), make_uint2(0, 0)};
    const int k = kb + lane;
    if (k < K && st) {
      const size_t kt = (size_t)k * a.T + t;
      r.n = (int)((st->cnt[who][k] >> (8 * (unsigned)(kt & 3))) & 0xFFu);
      if (((kb >> 5) % nwho) == who) {
        r.v = st->val[k];
        r.ix = st->idx[k];
        r.ref = st->ref[k];
      }
    } else if (k < K) {
      const size_t kt = (size_t)k * a.T + t;
      r.n = a.cnt[kt];
      if (vec && ((kb >> 5) % nwho) == who) {
        r.v = __ldg(reinterpret_cast<const uint4*>(a.val + kt * C));
        if constexpr (E == 8)
          r.ix = __ldg(reinterpret_cast<const uint2*>(a.idx + kt * C));
        else
          r.ix.x = __ldg(reinterpret_cast<const uint32_t*>(a.idx + kt * C));
        r.ref = a.spill_ref[kt];
      }
    }
    return r;
  };
  int base = 0;  // ordinal of the first entry of tile kb
  Round nxt = fetch(0);
  for (int kb = 0; kb < K && base < hi; kb += 32) {
    const int k = kb + lane;
    const Round cur = nxt;
    if (kb + 32 < K) nxt = fetch(kb + 32);
    const bool mine = ((kb >> 5) % nwho) == who;
    const int n = cur.n;
    int incl = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(FULL, incl, o);
      if (lane >= o) incl += u;
    }
    const int tb = base + incl - n;  // first ordinal of tile k
    const bool over = mine && n > 0 && tb < hi && tb + n > lo;
    const size_t kt = (size_t)k * a.T + t;
    int ref = -1;
    if (over && n > C) {
      ref = vec ? cur.ref : a.spill_ref[kt];
      if (ref < 0 || ref >= a.spill_cap) {
        // dropped spill entry (capacity, flagged by the producer): only the
        // C slots are known; the other entries of the tile contribute 0
        set_status(a.status, kStatusSpill);
        ref = -1;
      }
    }
    if (over && ref < 0) {
      const int m = n <= C ? n : C;
      const int s0 = lo > tb ? lo - tb : 0;
      const int s1 = hi - tb < n ? hi - tb : n;
      if (vec) {
        const uint32_t vw[4] = {cur.v.x, cur.v.y, cur.v.z, cur.v.w};
#pragma unroll
        for (int sl = 0; sl < E; ++sl) {
          if (sl >= s0 && sl < s1) {
            float gv;
            if constexpr (sizeof(Tin) == 2)
              gv = __uint_as_float((sl & 1) ? (vw[sl >> 1] & 0xFFFF0000u) : (vw[sl >> 1] << 16));
            else
              gv = __uint_as_float(vw[sl]);
            const uint32_t iw = sl < 4 ? cur.ix.x : cur.ix.y;
            const int ix = (int)((iw >> (8 * (sl & 3))) & 0xFFu);
            const int o = tb + sl - lo;
            sg[o] = sl < m ? gv : 0.f;
            sj[o] = sl < m ? k * W + ix : k * W;
          }
        }
        for (int sl = s0 > E ? s0 : E; sl < s1; ++sl) {  // past the slots: a dropped spill
          sg[tb + sl - lo] = 0.f;
          sj[tb + sl - lo] = k * W;
        }
      } else {
#pragma unroll 4
        for (int sl = s0; sl < s1; ++sl) {
          const int o = tb + sl - lo;
          sg[o] = sl < m ? Elem<Tin>::scalar(a.val[kt * C + sl]) : 0.f;
          sj[o] = sl < m ? k * W + a.idx[kt * C + sl] : k * W;
        }
      }
    }
    unsigned sp = __ballot_sync(FULL, ref >= 0);
    while (sp) {
      const int b = __ffs(sp) - 1;
      sp &= sp - 1;
      const int rb = __shfl_sync(FULL, ref, b);
      const int o0 = __shfl_sync(FULL, tb, b);
      const Tin* seg = a.spill_val + (size_t)rb * W;
      // all parts of the segment first (W <= 256: at most 8 per lane)
      float v[8];
#pragma unroll
      for (int part = 0; part < 8; ++part)
        v[part] = part < W / 32 ? Elem<Tin>::scalar(seg[part * 32 + lane]) : 0.f;
      int r = 0;
#pragma unroll
      for (int part = 0; part < 8; ++part) {
        if (part >= W / 32) break;
        const unsigned m = __ballot_sync(FULL, v[part] != 0.f);
        const int o = o0 + r + __popc(m & lanemask_lt());
        if (v[part] != 0.f && o >= lo && o < hi) {
          sg[o - lo] = v[part];
          sj[o - lo] = (kb + b) * W + part * 32 + lane;
        }
        r += __popc(m);
      }
    }
    base += __shfl_sync(FULL, incl, 31);
  }
  const int got = (base < hi ? base : hi) - lo;
  return got > 0 ? got : 0;
}

// Hybrid: the entries of token t with ordinal in [lo, hi): ELL slots in order,
// or the non-zeros of its backup row in ascending unit order.
template <typename Tin, int MODE>
TW_DEV int collect_hybrid(const GatherArgs<Tin>& a, int t, int lo, int hi, EntryList& s,
                          int lane) {
  const int slot = a.row_slot[t];
  if (slot < 0) {
    for (int e0 = lo; e0 < hi; e0 += 32) {
      const int e = e0 + lane;
      if (e < hi) {
        const size_t pos = (size_t)t * a.C_h + e;
        s.g[e - lo] = Elem<Tin>::scalar(a.ell_g[pos]);
        s.j[e - lo] = a.ell_idx[pos];
        s.pos[e - lo] = (int)pos;
        if (MODE == kModeHybBwd) s.u[e - lo] = Elem<Tin>::scalar(a.ell_u[pos]);
      }
    }
  } else {
    // dense row, 32 * NQ * V columns per round: lane l owns NQ * V contiguous
    // columns (NQ independent 16-byte loads), so one warp scan of the lanes'
    // non-zero counts ranks them in column order
    constexpr int V = 16 / (int)sizeof(Tin);  // values per 16-byte load
    constexpr int NQ = 2;                     // loads per lane per round
    constexpr int NV = NQ * V;                // values per lane per round (<= 32)
    const Tin* row = a.backup_g + (size_t)slot * a.F;
    int base = 0;
    for (int c0 = 0; c0 < a.F && base < hi; c0 += 32 * NV) {
      const int cl = c0 + lane * NV;  // this lane's first column
      uint4 raw[NQ];
#pragma unroll
      for (int q = 0; q < NQ; ++q)
        raw[q] = cl + q * V < a.F ? *reinterpret_cast<const uint4*>(row + cl + q * V)
                                  : make_uint4(0, 0, 0, 0);
      unsigned mask = 0;  // bit i: column cl + i is non-zero
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const uint32_t w[4] = {raw[q].x, raw[q].y, raw[q].z, raw[q].w};
#pragma unroll
        for (int i = 0; i < V; ++i) {
          const bool nzv = sizeof(Tin) == 2 ? ((w[i >> 1] >> (16 * (i & 1))) & 0x7FFFu) != 0
                                            : (w[i] & 0x7FFFFFFFu) != 0;
          mask |= (nzv ? 1u : 0u) << (q * V + i);
        }
      }
      const int nz = __popc(mask);
      int incl = nz;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(FULL, incl, o);
        if (lane >= o) incl += u;
      }
      const int first = base + incl - nz;  // rank of this lane's first non-zero
      if (nz > 0 && first < hi && first + nz > lo) {
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          unsigned mq = (mask >> (q * V)) & ((1u << V) - 1u);
          while (mq) {
            const int i = __ffs(mq) - 1;
            mq &= mq - 1;
            const int bit = q * V + i;
            const int r = first + __popc(mask & ((1u << bit) - 1u));
            if (r >= lo && r < hi) {
              const uint32_t wd = (i >> (sizeof(Tin) == 2 ? 1 : 0)) == 0   ? raw[q].x
                                  : (i >> (sizeof(Tin) == 2 ? 1 : 0)) == 1 ? raw[q].y
                                  : (i >> (sizeof(Tin) == 2 ? 1 : 0)) == 2 ? raw[q].z
                                                                           : raw[q].w;
              float v;
              if constexpr (sizeof(Tin) == 2)
                v = __uint_as_float((i & 1) ? (wd & 0xFFFF0000u) : (wd << 16));
              else
                v = __uint_as_float(wd);
              const size_t pos = (size_t)slot * a.F + cl + bit;
              s.g[r - lo] = v;
              s.j[r - lo] = cl + bit;
              s.pos[r - lo] = (int)pos;
              if (MODE == kModeHybBwd) s.u[r - lo] = Elem<Tin>::scalar(a.backup_u[pos]);
            }
          }
        }
      }
      base += __shfl_sync(FULL, incl, 31);
    }
  }
  return hi - lo;
}

// NCHW: 16-byte column slices per lane for one warp of a team.
// Teams per CTA: fewer for the widest rows, whose register sets of row slices
// need more than 128 registers per thread (three sets in the backward).
template <int NCHW, int MODE>
constexpr int teams_for() { return NCHW < 4 ? kTeams : (MODE == kModeHybBwd ? 4 : 6); }

// Dynamic shared memory of a gather launch: StageSmem per team (TwELL mode
// with staging).
template <int NCHW, int MODE>
constexpr size_t gather_smem_bytes() {
  return MODE == kModeTwell ? sizeof(StageSmem<NCHW>) * teams_for<NCHW, MODE>() : 0;
}

// kFull: d is exactly the kTeam warps' slices (see load_rows2).
template <typename Tin, int NCHW, bool kOutBf16, int MODE, bool kFull>
__global__ void __launch_bounds__(32 * kTeam * teams_for<NCHW, MODE>(), 1)
    gather_kernel(const GatherArgs<Tin> a) {
  using L = Elem<Tin>;
  constexpr int E = L::E;
  constexpr int P = L::P;
  constexpr int SPAN = 32 * E;       // columns of one warp-wide slice
  constexpr int COLS = NCHW * SPAN;  // columns owned by one warp
  constexpr bool kBwd = MODE == kModeHybBwd;
  __shared__ TeamSmem team_smem[teams_for<NCHW, MODE>()];
  const int lane = threadIdx.x & 31;
  const int wid = threadIdx.x >> 5;
  const int team = wid / kTeam;
  const int tw = wid % kTeam;  // this warp's place in its team
  const int d = a.d;
  const int c0 = tw * COLS;    // first column of this warp
  const int my_cols = d - c0 < COLS ? (d - c0 > 0 ? d - c0 : 0) : COLS;
  TeamSmem& ts = team_smem[team];
  pdl_wait();  // the plan comes from the previous launch
  pdl_launch_next();
  const int n_items = a.ws.hdr[1];
  const bool leader = tw == 0;
  const uint64_t pol = policy_evict_last();

  // Items come from a ticket counter.  The leader publishes the descriptor
  // of the team's next item while the current one runs (before the team
  // barrier in the middle of its first window), so an item starts without a
  // barrier of its own.
  int ticket = 0;
  auto publish = [&](int slot) {
    if (leader && lane == 0) {
      ts.desc[slot] = ticket < n_items ? a.ws.item_desc[ticket] : make_int4(-1, 0, 0, -1);
      if (ticket < n_items) ticket = atomicAdd(&a.ws.hdr[0], 1);
    }
  };
  if (leader && lane == 0) ticket = atomicAdd(&a.ws.hdr[0], 1);
  publish(0);
  team_bar(team);

  // TwELL mode: the next item's data are copied into shared memory while the
  // current item's updates run (see StageSmem); this is the first item's.
  // Dynamic shared memory: the teams' StageSmem (TwELL mode); see
  // gather_smem_bytes.
  extern __shared__ __align__(16) unsigned char stage_smem[];
  StageSmem<NCHW>& sg = reinterpret_cast<StageSmem<NCHW>*>(stage_smem)[team];
  const bool staged = MODE == kModeTwell && a.staged != 0;
  auto stage = [&](int tn) {
    const int K = a.F / a.W;
    for (int kb = 0; kb < K; kb += 32) {
      const int k = kb + lane;
      if (k < K) {
        const size_t kt = (size_t)k * a.T + tn;
        cp_async4(&sg.cnt[tw][k], a.cnt + (kt & ~size_t(3)));
        if (((kb >> 5) % kTeam) == tw) {
          cp_async16(&sg.val[k], a.val + kt * a.C, true);
          if constexpr (E == 8)
            cp_async8(&sg.idx[k], a.idx + kt * a.C);
          else
            cp_async4(&sg.idx[k].x, a.idx + kt * a.C);
          cp_async4(&sg.ref[k], a.spill_ref + kt);
        }
      }
    }
    const Tin* xn = a.xin + (size_t)tn * d;
#pragma unroll
    for (int c = 0; c < NCHW; ++c) {
      const int col = c0 + c * SPAN + lane * E;
      const bool ok = kFull || col < d;
      cp_async16(&sg.x[tw][c][lane], ok ? xn + col : xn, ok);
    }
    cp_async_commit();
  };
  if (staged && ts.desc[0].x >= 0) stage(ts.desc[0].x);

  uint32_t win = 0;  // windows processed by the team: the list parity
  for (uint32_t it = 0;; ++it) {
    const int4 desc = ts.desc[it & 1];
    if (desc.x < 0) break;
    const int t = desc.x, lo = desc.y, hi = desc.z, prow = desc.w;
    const bool to_backup = MODE == kModeHybFwd && a.row_slot[t] >= 0;
    bool published = false;
    // after the item's last partials barrier: the next item's staged copies
    auto stage_next = [&]() {
      if (staged) {
        const int4 nd = ts.desc[(it + 1) & 1];
        if (nd.x >= 0) stage(nd.x);
      }
    };

    uint4 xr[NCHW];  // the token's row slices, kept in the input format
    float2 acc[NCHW][P];
    const Tin* xt = a.xin + (size_t)t * d;
    if (staged) cp_async_wait_all();
#pragma unroll
    for (int c = 0; c < NCHW; ++c) {
      const int col = c0 + c * SPAN + lane * E;
      if (staged)
        xr[c] = sg.x[tw][c][lane];
      else
        xr[c] = kFull || col < d ? __ldcs(reinterpret_cast<const uint4*>(xt + col))
                                 : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int q = 0; q < P; ++q) acc[c][q] = make_float2(0.f, 0.f);
    }

    for (int w0 = lo; w0 < hi; w0 += kListCap, ++win) {
      EntryList& ls = ts.list[win & 1];
      const int w1 = min(hi, w0 + kListCap);
      int n;
      if constexpr (MODE == kModeTwell) {
        n = collect_twell<Tin, NCHW>(a, t, w0, w1, ls.g, ls.j, lane, tw, kTeam,
                                     staged ? &sg : nullptr);
        team_bar(team);  // the list is written
      } else {
        if (leader) {
          const int m = collect_hybrid<Tin, MODE>(a, t, w0, w1, ls, lane);
          if (lane == 0) ts.n[win & 1] = m;
        }
        team_bar(team);  // the list is written
        n = ts.n[win & 1];
      }
      const int npairs = (n + 1) / 2;
      // rows of a missing second entry are zeros, so both rows always update
      auto update = [&](const uint4 (&R)[2][NCHW], float sa, float sb) {
        const float2 ha = make_float2(sa, sa), hb = make_float2(sb, sb);
#pragma unroll
        for (int c = 0; c < NCHW; ++c) {
          float2 w[P];
          L::pairs(R[0][c], w);
#pragma unroll
          for (int q = 0; q < P; ++q) acc[c][q] = __ffma2_rn(ha, w[q], acc[c][q]);
          L::pairs(R[1][c], w);
#pragma unroll
          for (int q = 0; q < P; ++q) acc[c][q] = __ffma2_rn(hb, w[q], acc[c][q]);
        }
      };
      // rows of the entry pair pp (its first entry always exists)
      auto load = [&](uint4 (&R)[2][NCHW], const Tin* base, int pp) {
        const int2 jj = *reinterpret_cast<const int2*>(&ls.j[2 * pp]);
        const bool two = 2 * pp + 1 < n;
        load_rows2<Tin, NCHW, kFull>(R, base, jj.x, two ? jj.y : 0, two, d, c0, my_cols, lane,
                                     pol);
      };
      {
        // Two phases per window.  Phase 1: this warp's partial dot products of
        // every entry pair, two pairs of dot rows in flight, no team barrier
        // between pairs.  One team barrier.  Phase 2: the scalars of each
        // entry from the team's partials (added in warp order) -- h, or in
        // the backward du and dz with the entry's record -- and the row
        // updates, two pairs of update rows in flight.  Outside the backward,
        // a register set freed by the last dot pairs takes the rows of the
        // first update pairs at once (pair q in set q & 1, as in phase 2).
        uint4 S0[2][NCHW], S1[2][NCHW];
        if (npairs > 0) load(S0, a.rdot, 0);
        if (npairs > 1) load(S1, a.rdot, 1);
        auto dots = [&](uint4 (&R)[2][NCHW], int pp) {
          float D[2][4];
          dot2_issue<Tin, NCHW>(xr, R, D);
          if (pp + 2 < npairs)
            load(R, a.rdot, pp + 2);
          else if (!kBwd && (pp & 1) < npairs)
            load(R, a.rax1, pp & 1);
          dot2_reduce<Tin>(D, lane, &ls.part[2 * pp][tw], &ls.part[2 * pp + 1][tw]);
        };
        for (int pp = 0; pp < npairs; pp += 2) {
          dots(S0, pp);
          if (pp + 1 < npairs) dots(S1, pp + 1);
        }
        if (!published) {  // the next item's descriptor, behind the barrier below
          publish((it + 1) & 1);
          published = true;
        }
        if constexpr (kBwd) {
          // S0, S1: Wu_t rows (du); T0, T1: Wg_t rows (dz)
          uint4 T0[2][NCHW], T1[2][NCHW];
          if (npairs > 0) {
            load(S0, a.rax1, 0);
            load(T0, a.rax2, 0);
          }
          if (npairs > 1) {
            load(S1, a.rax1, 1);
            load(T1, a.rax2, 1);
          }
          team_bar(team);  // the partials (and the next descriptor) are written
          auto coef = [&](int e, float& du, float& dz) {
            du = dz = 0.f;
            if (e >= n) return;
            float dh = 0.f;
#pragma unroll
            for (int q = 0; q < kTeam; ++q) dh += ls.part[e][q];
            const float gv = ls.g[e], uv = ls.u[e];
            du = dh * gv;
            dz = fmaf(dh, uv, a.lam);
            if (leader && lane == 0) {
              Payload pl;
              pl.t = t;
              pl.j = ls.j[e];
              pl.h = gv * uv;
              pl.du = du;
              pl.dz = dz;
              a.pay[a.e0[t] + w0 + e] = pl;
            }
          };
          auto upd2 = [&](uint4 (&RU)[2][NCHW], uint4 (&RG)[2][NCHW], int pp) {
            float dua, dza, dub, dzb;
            coef(2 * pp, dua, dza);
            coef(2 * pp + 1, dub, dzb);
            update(RU, dua, dub);
            if (pp + 2 < npairs) load(RU, a.rax1, pp + 2);
            update(RG, dza, dzb);
            if (pp + 2 < npairs) load(RG, a.rax2, pp + 2);
          };
          for (int pp = 0; pp < npairs; pp += 2) {
            upd2(S0, T0, pp);
            if (pp + 1 < npairs) upd2(S1, T1, pp + 1);
          }
          continue;
        }
        team_bar(team);  // the partials (and the next descriptor) are written
        if (w1 == hi) stage_next();
        // h of the pair's entries: u from the team's partials (added in warp
        // order), times g; 0 for a missing second entry
        static_assert(kTeam == 2, "a pair's partials are read as one float4");
        auto upd = [&](uint4 (&R)[2][NCHW], int pp) {
          const float4 pt = *reinterpret_cast<const float4*>(&ls.part[2 * pp][0]);
          const float2 gg = *reinterpret_cast<const float2*>(&ls.g[2 * pp]);
          const bool two = 2 * pp + 1 < n;
          const float ua = pt.x + pt.y, ub = pt.z + pt.w;
          if (MODE == kModeHybFwd && leader && lane == 0) {
            Tin* dst = to_backup ? a.backup_u : a.ell_u;
            L::store(dst + ls.pos[2 * pp], ua);
            if (two) L::store(dst + ls.pos[2 * pp + 1], ub);
          }
          update(R, gg.x * ua, two ? gg.y * ub : 0.f);
          if (pp + 2 < npairs) load(R, a.rax1, pp + 2);
        };
        for (int pp = 0; pp < npairs; pp += 2) {
          upd(S0, pp);
          if (pp + 1 < npairs) upd(S1, pp + 1);
        }
      }
    }
    if (!published) {  // an item without entries
      publish((it + 1) & 1);
      team_bar(team);
      stage_next();
    }

    // ------------------------------------------------------------ output --
    // A split token's parts are summed up a binary tree over the part index:
    // node [L, L + 2s) adds its children [L, L + s) and [L + s, L + 2s), and
    // a node's sum is published in the partial row of its first part L.  Of
    // two children, the one that finishes second (arrival counter per
    // internal node, keyed by its right child's first part) loads the
    // other's row into its registers and goes up; the first one stops.
    // Floating-point addition is commutative, so every node's sum, and y, is
    // the same whichever part finishes first.  The team that completes the
    // root writes the output row.
    bool complete = true;
    if (prow >= 0) {
      const int part = a.ws.hdr[2];
      const int parts = (a.ws.nnz[t] + part - 1) / part;
      const int leaf = lo / part;
      const int row0 = prow - leaf;  // the token's first partial row
      int node = leaf;
      for (int span = 1; span < parts; span *= 2) {
        const int left = node & ~(2 * span - 1);
        const int right = left + span;
        if (right >= parts) {  // no right sibling: the node is its own parent
          node = left;
          continue;
        }
        float* mine = a.ws.partial + (size_t)(row0 + node) * d;
#pragma unroll
        for (int c = 0; c < NCHW; ++c) {
          const int col = c0 + c * SPAN + lane * E;
          if (col >= d) continue;
#pragma unroll
          for (int q = 0; q < P / 2; ++q)
            reinterpret_cast<float4*>(mine + col)[q] =
                make_float4(acc[c][2 * q].x, acc[c][2 * q].y, acc[c][2 * q + 1].x,
                            acc[c][2 * q + 1].y);
        }
        __threadfence();
        team_bar(team);  // both halves of the row are written
        if (leader && lane == 0) ts.prev = atomicAdd(&a.ws.done[row0 + right], 1);
        team_bar(team);
        if (ts.prev == 0) {  // the sibling is still running; it goes on
          complete = false;
          break;
        }
        __threadfence();
        const float* other = a.ws.partial + (size_t)(row0 + (node == left ? right : left)) * d;
        float4 sib[NCHW][P / 2];
#pragma unroll
        for (int c = 0; c < NCHW; ++c) {
          const int col = c0 + c * SPAN + lane * E;
#pragma unroll
          for (int q = 0; q < P / 2; ++q)
            sib[c][q] = col < d ? __ldcg(reinterpret_cast<const float4*>(other + col) + q)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int c = 0; c < NCHW; ++c)
#pragma unroll
          for (int q = 0; q < P / 2; ++q) {
            acc[c][2 * q].x += sib[c][q].x;
            acc[c][2 * q].y += sib[c][q].y;
            acc[c][2 * q + 1].x += sib[c][q].z;
            acc[c][2 * q + 1].y += sib[c][q].w;
          }
        node = left;
      }
    }
    if (complete) {
#pragma unroll
      for (int c = 0; c < NCHW; ++c) {
        const int col = c0 + c * SPAN + lane * E;
        if (col >= d) continue;
        if (!kOutBf16) {
          float* dst = static_cast<float*>(a.out) + (size_t)t * d + col;
#pragma unroll
          for (int q = 0; q < P / 2; ++q)
            __stcs(reinterpret_cast<float4*>(dst) + q,
                   make_float4(acc[c][2 * q].x, acc[c][2 * q].y, acc[c][2 * q + 1].x,
                               acc[c][2 * q + 1].y));
        } else {
          uint16_t* yt = static_cast<uint16_t*>(a.out) + (size_t)t * d + col;
#pragma unroll
          for (int q = 0; q < P; ++q)
            reinterpret_cast<uint32_t*>(yt)[q] = pack_bf16x2(acc[c][q].x, acc[c][q].y);
        }
      }
    }
  }
}

template <typename Tin, int NCHW, int MODE>
cudaError_t launch_nchw(GatherArgs<Tin> a, bool out_bf16, cudaStream_t stream) {
  const bool full = a.d == kTeam * NCHW * 32 * Elem<Tin>::E;
  auto kern = full ? (out_bf16 ? gather_kernel<Tin, NCHW, true, MODE, true>
                               : gather_kernel<Tin, NCHW, false, MODE, true>)
                   : (out_bf16 ? gather_kernel<Tin, NCHW, true, MODE, false>
                               : gather_kernel<Tin, NCHW, false, MODE, false>);
  constexpr int threads = 32 * kTeam * teams_for<NCHW, MODE>();
  const size_t dyn = a.staged ? gather_smem_bytes<NCHW, MODE>() : 0;
  cudaError_t e = cudaSuccess;
  if (dyn > 0) {
    e = set_smem_limit(reinterpret_cast<const void*>(kern), (int)dyn);
    if (e != cudaSuccess) return e;
  }
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, dyn);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  return launch_pdl(kern, dim3(num_sms() * per_sm), dim3(threads), dyn, stream, a);
}

// Small batches (T <= kDecodeMaxT, decoding): one CTA per token, no work
// plan.  The work per token is small and its rows come from HBM, so the
// aim is to have as many row loads in flight as possible:
//   warp 0 collects a window of the token's entries into shared memory;
//   each warp takes every kDecWarps-th entry, two at a time, and forms
//     h = g * (x_t . Wu_t[j]) with a warp reduction;
//   each thread then accumulates its own columns of y over all entries of
//     the window, eight rows of Wd in flight.
// Entries are summed in their (tile-major) order, so y is deterministic.
// One CTA per token leaves a token with hundreds of entries (heavy-tailed
// activity) to a single CTA: at 16 tokens of the 2B decoding workload, with
// a 425-entry token, that took 120 us, so the planned path (which splits
// heavy tokens) takes over above 8 tokens.
constexpr int kDecWarps = 8;
constexpr int kDecodeMaxT = 8;

template <typename Tin, bool kOutBf16>
__global__ void __launch_bounds__(32 * kDecWarps) decode_kernel(const GatherArgs<Tin> a) {
  using L = Elem<Tin>;
  constexpr int E = L::E;
  constexpr int P = L::P;
  constexpr int SPAN = 32 * E;   // columns of one warp-wide slice
  constexpr int NCH = 8;         // slices per lane: d <= 8 * SPAN (the validated maximum)
  __shared__ EntryList lst;
  __shared__ int lst_n;
  __shared__ float hsh[kListCap];
  const int t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = a.d;
  const Tin* xt = a.xin + (size_t)t * d;
  uint4 xr[NCH];  // the whole token row in every warp, for the dot products
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    const int cc = c * SPAN + lane * E;
    xr[c] = cc < d ? __ldg(reinterpret_cast<const uint4*>(xt + cc)) : make_uint4(0, 0, 0, 0);
  }
  const int col = threadIdx.x * E;  // this thread's output columns
  float2 acc[P];
#pragma unroll
  for (int q = 0; q < P; ++q) acc[q] = make_float2(0.f, 0.f);

  for (int w0 = 0;; w0 += kListCap) {
    if (warp == 0) {
      const int n = collect_twell(a, t, w0, w0 + kListCap, lst.g, lst.j, lane, 0, 1);
      if (lane == 0) lst_n = n;
    }
    __syncthreads();
    const int n = lst_n;
    // h of each entry: two entries per warp at a time
    for (int e = warp; e < n; e += 2 * kDecWarps) {
      const int e2 = e + kDecWarps;
      const bool two = e2 < n;
      const uint4* r0 = reinterpret_cast<const uint4*>(a.rdot + (size_t)lst.j[e] * d);
      const uint4* r1 = reinterpret_cast<const uint4*>(a.rdot + (size_t)(two ? lst.j[e2] : 0) * d);
      uint4 w0v[NCH], w1v[NCH];
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        const int cc = c * SPAN + lane * E;
        w0v[c] = cc < d ? __ldg(r0 + cc / E) : make_uint4(0, 0, 0, 0);
        w1v[c] = cc < d && two ? __ldg(r1 + cc / E) : make_uint4(0, 0, 0, 0);
      }
      float p0[4] = {0.f, 0.f, 0.f, 0.f}, p1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        L::dot(xr[c], w0v[c], p0);
        L::dot(xr[c], w1v[c], p1);
      }
      const float u0 = warp_sum((p0[0] + p0[1]) + (p0[2] + p0[3]));
      const float u1 = warp_sum((p1[0] + p1[1]) + (p1[2] + p1[3]));
      if (lane == 0) {
        hsh[e] = lst.g[e] * u0;
        if (two) hsh[e2] = lst.g[e2] * u1;
      }
    }
    __syncthreads();
    // y columns of this thread over the window's entries
    if (col < d) {
      for (int e0 = 0; e0 < n; e0 += 8) {
        uint4 w[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          w[u] = e0 + u < n ? __ldg(reinterpret_cast<const uint4*>(a.rax1 + (size_t)lst.j[e0 + u] * d + col))
                            : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (e0 + u >= n) break;
          const float h = hsh[e0 + u];
          const float2 hh = make_float2(h, h);
          float2 wv[P];
          L::pairs(w[u], wv);
#pragma unroll
          for (int q = 0; q < P; ++q) acc[q] = __ffma2_rn(hh, wv[q], acc[q]);
        }
      }
    }
    __syncthreads();  // the window's list and h are reused
    if (n < kListCap) break;
  }
  if (col < d) {
    if (kOutBf16) {
      uint16_t* yt = static_cast<uint16_t*>(a.out) + (size_t)t * d + col;
#pragma unroll
      for (int q = 0; q < P; ++q)
        reinterpret_cast<uint32_t*>(yt)[q] = pack_bf16x2(acc[q].x, acc[q].y);
    } else {
      float* yt = static_cast<float*>(a.out) + (size_t)t * d + col;
#pragma unroll
      for (int q = 0; q < P / 2; ++q)
        reinterpret_cast<float4*>(yt)[q] = make_float4(acc[2 * q].x, acc[2 * q].y,
                                                       acc[2 * q + 1].x, acc[2 * q + 1].y);
    }
  }
}

template <typename Tin, int MODE>
cudaError_t launch_mode(const GatherArgs<Tin>& a, bool out_bf16, cudaStream_t stream) {
  // chunks of one 16-byte slice per lane, split over the kTeam warps
  constexpr int SPAN = 32 * Elem<Tin>::E;
  const int nch = (a.d + SPAN - 1) / SPAN;
  const int per = (nch + kTeam - 1) / kTeam;
  if (per <= 1) return launch_nchw<Tin, 1, MODE>(a, out_bf16, stream);
  if (per <= 2) return launch_nchw<Tin, 2, MODE>(a, out_bf16, stream);
  if (per <= 4) return launch_nchw<Tin, 4, MODE>(a, out_bf16, stream);
  return cudaErrorInvalidValue;  // d beyond the validated maximum
}

// Plan the items from the counts in w.nnz (filled by `count`, which launches
// the count kernel and returns its launch status), run the engine.  The four
// launches are programmatic dependent launches (launch_pdl).
template <typename Tin, int MODE, class CountFn>
cudaError_t run_engine(GatherArgs<Tin> a, bool out_bf16, void* base, CountFn count,
                       cudaStream_t stream) {
  const int n_teams = num_sms() * kTeams;  // workers taking items
  cudaError_t e = count();
  if (e != cudaSuccess) return e;
  const size_t scan_smem = plan_scan_smem(a.T);
  if (scan_smem > 48 * 1024) {
    e = set_smem_limit(reinterpret_cast<const void*>(plan_scan_kernel),
                       (int)plan_scan_smem(kScanSmemTokens));
    if (e != cudaSuccess) return e;
  }
  const int nb = (a.T + kCountBlock - 1) / kCountBlock;
  e = launch_pdl(plan_scan_kernel, dim3(1), dim3(kScanThreads), scan_smem, stream, a.T,
                 (const int32_t*)a.ws.nnz, a.ws.parts_cap, a.ws.max_items, n_teams, a.ws.slot_off,
                 a.ws.item_desc, a.ws.hdr, a.ws.bpart, nb, a.ws.done);
  if (e != cudaSuccess) return e;
  e = launch_pdl(plan_write_kernel, dim3(nb), dim3(kCountBlock), 0, stream, a.T,
                 (const int32_t*)a.ws.nnz, a.ws.max_items, a.ws.slot_off, a.ws.item_desc,
                 (const int32_t*)a.ws.hdr, (const int4*)a.ws.bpart);
  if (e != cudaSuccess) return e;
  return launch_mode<Tin, MODE>(a, out_bf16, stream);
}

template <typename Tin>
cudaError_t twell_fused_t(const void* x, const tw_twell& g, const void* Wu_t, const void* Wd, int d,
                          void* y, tw_dtype y_dtype, void* base, const FusedWs& w,
                          int32_t* status, cudaStream_t stream) {
  GatherArgs<Tin> a{};
  a.cnt = g.cnt;
  a.val = static_cast<const Tin*>(g.val);
  a.idx = g.idx;
  a.spill_ref = g.spill_ref;
  a.spill_val = static_cast<const Tin*>(g.spill_val);
  a.W = g.W;
  a.C = g.C;
  a.spill_cap = g.spill_cap;
  a.T = g.T;
  a.F = g.F;
  a.d = d;
  a.xin = static_cast<const Tin*>(x);
  a.rdot = static_cast<const Tin*>(Wu_t);
  a.rax1 = static_cast<const Tin*>(Wd);
  a.out = y;
  a.status = status;
  a.ws = w;
  const int T = g.T, K = g.F / g.W;
  // prefetching the next item's TwELL data needs 16-byte slot rows, at most
  // kStageTiles tiles and count words that stay inside the count array
  a.staged = g.C == Elem<Tin>::E && K <= kStageTiles && T % 4 == 0 &&
             reinterpret_cast<uintptr_t>(g.cnt) % 4 == 0;
  // A handful of tokens: one CTA per token, no plan.  Above that the planned
  // path wins, because it splits the heavy tokens of the batch over teams
  // (at T = 64 of the 2B workload: 50 us planned, 282 us one CTA per token).
  if (T <= kDecodeMaxT) {
    auto kern = y_dtype == TW_BF16 ? decode_kernel<Tin, true> : decode_kernel<Tin, false>;
    kern<<<T, 32 * kDecWarps, 0, stream>>>(a);
    return cudaGetLastError();
  }
  return run_engine<Tin, kModeTwell>(
      a, y_dtype == TW_BF16, base,
      [&] {
        return launch_pdl(plan_count_twell_kernel, dim3((T + kCountBlock - 1) / kCountBlock),
                          dim3(kCountBlock), 0, stream, T, K, (const uint8_t*)g.cnt, w.nnz,
                          w.bpart);
      },
      stream);
}

cudaError_t twell_fused(const void* x, const tw_twell& g, const void* Wu_t, const void* Wd, int d,
                        void* y, tw_dtype y_dtype, void* base, const FusedWs& w, int32_t* status,
                        cudaStream_t stream) {
  return g.dtype == TW_BF16
             ? twell_fused_t<uint16_t>(x, g, Wu_t, Wd, d, y, y_dtype, base, w, status, stream)
             : twell_fused_t<float>(x, g, Wu_t, Wd, d, y, y_dtype, base, w, status, stream);
}

template <typename Tin, int MODE>
cudaError_t hybrid_t(const void* xin, const tw_hybrid& h, const void* rdot, const void* rax1,
                     const void* rax2, int d, float lam, const int32_t* e0, Payload* pay,
                     void* out, tw_dtype out_dtype, void* base, int32_t* status,
                     cudaStream_t stream) {
  const FusedWs w = carve(base, h.T, d);
  GatherArgs<Tin> a{};
  a.ell_g = static_cast<const Tin*>(h.ell_g);
  a.ell_u = static_cast<Tin*>(h.ell_u);
  a.ell_idx = h.ell_idx;
  a.row_slot = h.row_slot;
  a.backup_g = static_cast<const Tin*>(h.backup_g);
  a.backup_u = static_cast<Tin*>(h.backup_u);
  a.C_h = h.C_h;
  a.backup_cap = h.backup_cap;
  a.T = h.T;
  a.F = h.F;
  a.d = d;
  a.xin = static_cast<const Tin*>(xin);
  a.rdot = static_cast<const Tin*>(rdot);
  a.rax1 = static_cast<const Tin*>(rax1);
  a.rax2 = static_cast<const Tin*>(rax2);
  a.lam = lam;
  a.e0 = e0;
  a.pay = pay;
  a.out = out;
  a.status = status;
  a.ws = w;
  const int T = h.T;
  return run_engine<Tin, MODE>(
      a, out_dtype == TW_BF16, base,
      [&] {
        return launch_pdl(plan_count_hybrid_kernel, dim3((T + kCountBlock - 1) / kCountBlock),
                          dim3(kCountBlock), 0, stream, T, (const int32_t*)h.row_nnz,
                          (const int32_t*)h.row_slot, h.backup_cap, w.nnz, w.bpart);
      },
      stream);
}

}  // namespace

size_t fused_ws_bytes(int T, int d) { return carve(nullptr, T, d).bytes; }

cudaError_t launch_fused_updown(const void* x, const tw_twell& g, const void* Wu_t,
                                const void* Wd, int d, void* y, tw_dtype y_dtype, void* ws,
                                int32_t* status, cudaStream_t stream) {
  return twell_fused(x, g, Wu_t, Wd, d, y, y_dtype, ws, carve(ws, g.T, d), status, stream);
}

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
  return twell_fused(x, g, Wu_t, Wd, d, y, y_dtype, scratch, w, status, stream);
}

namespace {

// u is +0 off the pattern: clears ell_u and the stored rows of backup_u (the
// first min(*n_backup, cap), the rows a backup slot holds), 16 bytes per
// store with a byte tail, before the engine writes the pattern's entries.
__global__ void __launch_bounds__(256)
    hyb_zero_u_kernel(uint8_t* ell_u, size_t ell_bytes, uint8_t* backup_u, size_t row_bytes,
                      const int32_t* n_backup, int cap) {
  pdl_wait();
  pdl_launch_next();
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  const size_t i0 = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  auto clear = [&](uint8_t* p, size_t bytes) {
    const size_t n16 = bytes / 16;
    for (size_t i = i0; i < n16; i += stride) reinterpret_cast<uint4*>(p)[i] = make_uint4(0, 0, 0, 0);
    for (size_t b = n16 * 16 + i0; b < bytes; b += stride) p[b] = 0;
  };
  if (ell_u != nullptr) clear(ell_u, ell_bytes);
  if (backup_u != nullptr) {
    const int nb = min(*n_backup, cap);
    clear(backup_u, (size_t)(nb > 0 ? nb : 0) * row_bytes);
  }
}

}  // namespace

cudaError_t launch_hybrid_gather_forward(const void* x, const tw_hybrid& gu, const void* Wu_t,
                                         const void* Wd, int d, void* y, tw_dtype y_dtype,
                                         void* ws, int32_t* status, cudaStream_t stream) {
  // u is defined as +0 off the pattern: clear both u arrays, the engine then
  // writes the pattern's entries
  const size_t esz = gu.dtype == TW_BF16 ? 2 : 4;
  if (gu.C_h > 0 || gu.backup_cap > 0) {
    cudaError_t e = launch_pdl(
        hyb_zero_u_kernel, dim3(num_sms() * 4), dim3(256), 0, stream,
        gu.C_h > 0 ? static_cast<uint8_t*>(gu.ell_u) : (uint8_t*)nullptr,
        esz * (size_t)gu.T * gu.C_h,
        gu.backup_cap > 0 ? static_cast<uint8_t*>(gu.backup_u) : (uint8_t*)nullptr,
        esz * (size_t)gu.F, (const int32_t*)gu.n_backup, gu.backup_cap);
    if (e != cudaSuccess) return e;
  }
  return gu.dtype == TW_BF16
             ? hybrid_t<uint16_t, kModeHybFwd>(x, gu, Wu_t, Wd, nullptr, d, 0.f, nullptr, nullptr,
                                               y, y_dtype, ws, status, stream)
             : hybrid_t<float, kModeHybFwd>(x, gu, Wu_t, Wd, nullptr, d, 0.f, nullptr, nullptr, y,
                                            y_dtype, ws, status, stream);
}

cudaError_t launch_hybrid_gather_backward(const void* dy, const tw_hybrid& gu, const void* Wg_t,
                                          const void* Wu_t, const void* Wd, int d, float lam,
                                          const int32_t* e0, Payload* pay, void* dx,
                                          tw_dtype dx_dtype, void* ws, int32_t* status,
                                          cudaStream_t stream) {
  return gu.dtype == TW_BF16
             ? hybrid_t<uint16_t, kModeHybBwd>(dy, gu, Wd, Wu_t, Wg_t, d, lam, e0, pay, dx,
                                               dx_dtype, ws, status, stream)
             : hybrid_t<float, kModeHybBwd>(dy, gu, Wd, Wu_t, Wg_t, d, lam, e0, pay, dx, dx_dtype,
                                            ws, status, stream);
}

}  // namespace tw
