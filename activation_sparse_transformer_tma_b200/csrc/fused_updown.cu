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
//   1. plan_count_*        entries per token;
//   2. plan_scan_kernel    (one CTA) the part size (adapted to the total work),
//                          partial-buffer rows for split tokens (bounded by
//                          the workspace), one descriptor {t, first entry,
//                          end entry, partial row} per work item;
//   3. gather_kernel       persistent teams take work items from a ticket
//                          counter (the next ticket is fetched while the
//                          current item runs).
// A split token's parts write fp32 partial rows to the workspace; the part
// that finishes last (atomic counter per token) sums them in part order, so
// the output is deterministic.
//
// Teams.  An item is processed by a team of kTeam warps; warp w of the team
// owns one contiguous range of the d columns (the token's row and the output
// of that range live in its registers).  Per entry every warp forms its
// partial dot product, the partials meet in shared memory behind a named
// barrier and are added in warp order, and every warp updates its own
// columns.
//
// Data movement.  Each warp owns a ring of shared-memory stages; lane 0
// gathers its column range of the weight rows of upcoming entries with 1-D
// bulk copies (cp.async.bulk, completion on one mbarrier per stage, no
// multicast) while the warp computes on earlier stages.  Every lane owns
// 16-byte column slices: conflict-free shared loads.  bf16 dot products use
// the mixed-precision FMA (bf16 inputs, fp32 accumulator); the scaled-row
// updates widen bf16 pairs exactly and use packed fp32x2 FMA.
#include "tw_common.cuh"
#include "tw_internal.h"

namespace tw {
namespace {

constexpr unsigned FULL = 0xFFFFFFFFu;
constexpr int W = 128;             // TwELL tile width
constexpr int kPart = 64;          // entries per part of a split token (upper bound)
constexpr int kMinPart = 8;        // lower bound of the part size
constexpr int kTeam = 2;           // warps per work item
constexpr int kTeams = 8;          // teams per CTA
constexpr int kWarps = kTeam * kTeams;
constexpr int kRingBytes = 12288;  // shared-memory ring per warp
constexpr int kListCap = 64;       // entry window collected at a time

enum : int { kModeTwell = 0, kModeHybFwd = 1, kModeHybBwd = 2 };

// --------------------------------------------------------------- workspace --
struct FusedWs {
  int32_t* hdr;        // [0] item ticket, [1] number of items, [2] part size
  int32_t* done;       // [T] parts finished (split tokens)
  int32_t* nnz;        // [T]
  int32_t* slot_off;   // [T] first partial row of a split token, -1 if whole
  int4* item_desc;     // [max_items] {t, lo, hi, partial row or -1}
  float* partial;      // [parts_cap][d]
  int parts_cap, max_items;
  size_t bytes;
  size_t zero_bytes;   // prefix (hdr, done) cleared before every call
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
  const size_t o_done = take(sizeof(int32_t) * (size_t)T);
  w.zero_bytes = off;
  const size_t o_nnz = take(sizeof(int32_t) * (size_t)T);
  const size_t o_slot = take(sizeof(int32_t) * (size_t)T);
  const size_t o_desc = take(sizeof(int4) * (size_t)w.max_items);
  const size_t o_part = take(sizeof(float) * (size_t)(cap > 0 ? cap : 1) * d);
  w.bytes = off;
  if (base) {
    char* p = static_cast<char*>(base);
    w.hdr = reinterpret_cast<int32_t*>(p + o_hdr);
    w.done = reinterpret_cast<int32_t*>(p + o_done);
    w.nnz = reinterpret_cast<int32_t*>(p + o_nnz);
    w.slot_off = reinterpret_cast<int32_t*>(p + o_slot);
    w.item_desc = reinterpret_cast<int4*>(p + o_desc);
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
__global__ void plan_count_twell_kernel(int T, int K, const uint8_t* __restrict__ cnt,
                                        int32_t* nnz) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  int s = 0;
  for (int k = 0; k < K; ++k) s += cnt[(size_t)k * T + t];
  nnz[t] = s;
}

// Hybrid rows: the row's non-zero count, or 0 for a backup row that was not
// stored (capacity exceeded, flagged by the conversion).
__global__ void plan_count_hybrid_kernel(int T, const int32_t* __restrict__ row_nnz,
                                         const int32_t* __restrict__ row_slot, int cap,
                                         int32_t* nnz) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  nnz[t] = row_slot[t] >= cap ? 0 : row_nnz[t];
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

// One CTA: the part size, partial rows of split tokens (in token order,
// within capacity), then one descriptor per work item.  The part size is
// kPart, lowered to about two items per team when there are few entries in
// all (small batches), but not below kMinPart; it is stored in hdr[2].
// Each thread owns a contiguous run of tokens, so each of the three passes
// needs a single block-wide scan.
__global__ void __launch_bounds__(kScanThreads)
    plan_scan_kernel(int T, const int32_t* __restrict__ nnz, int parts_cap, int max_items,
                     int n_teams, int32_t* slot_off, int4* item_desc, int32_t* hdr) {
  __shared__ int warp_sums[32];
  __shared__ int part_sh;
  const int run = (T + kScanThreads - 1) / kScanThreads;
  const int t0 = threadIdx.x * run;
  const int t1 = min(T, t0 + run);
  // pass 0: total number of entries -> part size
  int local = 0;
  for (int t = t0; t < t1; ++t) local += nnz[t];
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
    const int n = nnz[t];
    local += n > part ? (n + part - 1) / part : 0;
  }
  int tot;
  int ex = block_exclusive_scan(local, warp_sums, &tot);
  for (int t = t0; t < t1; ++t) {
    const int n = nnz[t];
    const int parts = n > part ? (n + part - 1) / part : 0;
    slot_off[t] = (parts > 0 && ex + parts <= parts_cap) ? ex : -1;
    ex += parts;
  }
  // pass 2: one descriptor per work item
  local = 0;
  for (int t = t0; t < t1; ++t)
    local += slot_off[t] >= 0 ? (nnz[t] + part - 1) / part : 1;
  ex = block_exclusive_scan(local, warp_sums, &tot);
  for (int t = t0; t < t1; ++t) {
    const int n = nnz[t], so = slot_off[t];
    if (so < 0) {
      if (ex < max_items) item_desc[ex] = make_int4(t, 0, n, -1);
      ++ex;
    } else {
      const int parts = (n + part - 1) / part;
      for (int p = 0; p < parts && ex + p < max_items; ++p)
        item_desc[ex + p] = make_int4(t, p * part, min(n, (p + 1) * part), so + p);
      ex += parts;
    }
  }
  if (threadIdx.x == 0) hdr[1] = tot < max_items ? tot : max_items;
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
  int C, spill_cap;
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
  int stages;       // ring depth per warp
  int slice_bytes;  // bytes of one row's column range of one warp (max over warps)
  unsigned long long timeout_ns;
};

// Shared state of one team.
struct TeamSmem {
  float g[kListCap];
  int32_t j[kListCap];
  int32_t pos[kListCap];  // hybrid position of the entry (u is saved / read there)
  float u[kListCap];      // saved u of the entry (backward)
  float red[2][kTeam];    // partial dot products, double-buffered by entry parity
  int ok[2][kTeam];       // wait results, same buffering
  int4 desc[2];           // current item, double-buffered by item parity
  int n;                  // entries in the current window
  int prev;               // split-token finisher broadcast
};

// TwELL: the entries of token t with ordinal in [lo, hi) (tile-major order,
// ascending within a tile) into the team's list; returns how many.  Each lane
// owns one tile, so the slots of all active tiles are read in one round;
// spilled tiles are read by the whole warp.
template <typename Tin>
TW_DEV int collect_twell(const GatherArgs<Tin>& a, int t, int lo, int hi, TeamSmem& s, int lane) {
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
    const bool over = n > 0 && tb < hi && tb + n > lo;
    const size_t kt = (size_t)k * a.T + t;
    int ref = -1;
    if (over && n > a.C) {
      ref = a.spill_ref[kt];
      if (ref < 0 || ref >= a.spill_cap) {
        // dropped spill entry (capacity, flagged by the producer): only the
        // C slots are known; the other entries of the tile contribute 0
        set_status(a.status, kStatusSpill);
        ref = -1;
      }
    }
    if (over && ref < 0) {
      const int m = n <= a.C ? n : a.C;
      const int s0 = lo > tb ? lo - tb : 0;
      const int s1 = hi - tb < n ? hi - tb : n;
#pragma unroll 4
      for (int sl = s0; sl < s1; ++sl) {
        const int o = tb + sl - lo;
        s.g[o] = sl < m ? Elem<Tin>::scalar(a.val[kt * a.C + sl]) : 0.f;
        s.j[o] = sl < m ? k * W + a.idx[kt * a.C + sl] : k * W;
      }
    }
    unsigned sp = __ballot_sync(FULL, ref >= 0);
    while (sp) {
      const int b = __ffs(sp) - 1;
      sp &= sp - 1;
      const int rb = __shfl_sync(FULL, ref, b);
      const int o0 = __shfl_sync(FULL, tb, b);
      const Tin* seg = a.spill_val + (size_t)rb * W;
      int r = 0;
#pragma unroll 1
      for (int part = 0; part < W / 32; ++part) {
        const float v = Elem<Tin>::scalar(seg[part * 32 + lane]);
        const unsigned m = __ballot_sync(FULL, v != 0.f);
        const int o = o0 + r + __popc(m & lanemask_lt());
        if (v != 0.f && o >= lo && o < hi) {
          s.g[o - lo] = v;
          s.j[o - lo] = (kb + b) * W + part * 32 + lane;
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
TW_DEV int collect_hybrid(const GatherArgs<Tin>& a, int t, int lo, int hi, TeamSmem& s,
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
    int base = 0;
    for (int c0 = 0; c0 < a.F && base < hi; c0 += 32) {
      const int c = c0 + lane;
      const size_t pos = (size_t)slot * a.F + c;
      const float v = c < a.F ? Elem<Tin>::scalar(a.backup_g[pos]) : 0.f;
      const unsigned m = __ballot_sync(FULL, v != 0.f);
      const int r = base + __popc(m & lanemask_lt());
      if (v != 0.f && r >= lo && r < hi) {
        s.g[r - lo] = v;
        s.j[r - lo] = c;
        s.pos[r - lo] = (int)pos;
        if (MODE == kModeHybBwd) s.u[r - lo] = Elem<Tin>::scalar(a.backup_u[pos]);
      }
      base += __popc(m);
    }
  }
  return hi - lo;
}

// NCHW: 16-byte column slices per lane for one warp of a team.
template <typename Tin, int NCHW, bool kOutBf16, int MODE>
__global__ void __launch_bounds__(32 * kWarps, 1) gather_kernel(const GatherArgs<Tin> a) {
  using L = Elem<Tin>;
  constexpr int E = L::E;
  constexpr int P = L::P;
  constexpr int SPAN = 32 * E;             // columns of one warp-wide slice
  constexpr int COLS = NCHW * SPAN;        // columns owned by one warp
  constexpr int NROWS = MODE == kModeHybBwd ? 3 : 2;  // weight rows per entry
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const int lane = threadIdx.x & 31;
  const int wid = threadIdx.x >> 5;
  const int team = wid / kTeam;
  const int tw = wid % kTeam;              // this warp's place in its team
  const int d = a.d;
  const int c0 = tw * COLS;                // first column of this warp
  const int my_cols = d - c0 < COLS ? (d - c0 > 0 ? d - c0 : 0) : COLS;
  const uint32_t my_bytes = (uint32_t)my_cols * sizeof(Tin);
  const size_t stage_bytes = (size_t)NROWS * a.slice_bytes;

  // shared memory: [kTeams] TeamSmem, then per warp: barriers + ring
  TeamSmem& ts = reinterpret_cast<TeamSmem*>(smem_raw)[team];
  const size_t team_bytes = (sizeof(TeamSmem) * kTeams + 127) & ~size_t(127);
  const size_t per_warp = 128 + (size_t)a.stages * stage_bytes;
  uint8_t* mine = smem_raw + team_bytes + (size_t)wid * per_warp;
  uint64_t* bar = reinterpret_cast<uint64_t*>(mine);
  uint8_t* ring = mine + 128;
  if (lane == 0) {
    for (int i = 0; i < a.stages; ++i) mbar_init(&bar[i], 1);
    fence_mbar_init();
  }
  __syncwarp();

  int never = 0;
  // Ring position of this warp, advanced incrementally (no division):
  // cst/cph next stage to wait on and its phase parity, pst next stage to
  // fill, inflight stages filled but not yet waited on.
  uint32_t cst = 0, cph = 0, pst = 0, inflight = 0;
  bool failed = false;
  const int n_items = a.ws.hdr[1];
  const bool leader = tw == 0;

  auto issue = [&](int j) {
    uint8_t* dst = ring + (size_t)pst * stage_bytes;
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(&bar[pst], NROWS * my_bytes);
    bulk_g2s(dst, a.rdot + (size_t)j * d + c0, my_bytes, &bar[pst]);
    bulk_g2s(dst + a.slice_bytes, a.rax1 + (size_t)j * d + c0, my_bytes, &bar[pst]);
    if (MODE == kModeHybBwd)
      bulk_g2s(dst + 2 * a.slice_bytes, a.rax2 + (size_t)j * d + c0, my_bytes, &bar[pst]);
  };

  int ticket = 0;
  if (leader && lane == 0) ticket = atomicAdd(&a.ws.hdr[0], 1);
  for (uint32_t it = 0;; ++it) {
    // The descriptor slot alternates between items: the partner reads slot
    // it&1 after this barrier, and the leader next writes it two items later,
    // behind barriers the partner has passed.
    if (leader && lane == 0) {
      const int item = ticket;
      ts.desc[it & 1] = item < n_items ? a.ws.item_desc[item] : make_int4(-1, 0, 0, -1);
      if (item < n_items) ticket = atomicAdd(&a.ws.hdr[0], 1);  // next, fetched early
    }
    team_bar(team);
    const int4 desc = ts.desc[it & 1];
    if (desc.x < 0) break;
    const int t = desc.x, lo = desc.y, hi = desc.z, prow = desc.w;
    const bool to_backup = MODE == kModeHybFwd && a.row_slot[t] >= 0;

    uint4 xr[NCHW];  // the token's row slices, kept in the input format
    float2 acc[NCHW][P];
    const Tin* xt = a.xin + (size_t)t * d;
#pragma unroll
    for (int c = 0; c < NCHW; ++c) {
      const int col = c0 + c * SPAN + lane * E;
      xr[c] = col < d ? __ldg(reinterpret_cast<const uint4*>(xt + col)) : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int q = 0; q < P; ++q) acc[c][q] = make_float2(0.f, 0.f);
    }

    for (int w0 = lo; w0 < hi && !failed; w0 += kListCap) {
      if (leader) {
        const int w1 = min(hi, w0 + kListCap);
        const int n = MODE == kModeTwell ? collect_twell(a, t, w0, w1, ts, lane)
                                         : collect_hybrid<Tin, MODE>(a, t, w0, w1, ts, lane);
        if (lane == 0) ts.n = n;
      }
      team_bar(team);
      const int n = ts.n;
      const int pre = n < a.stages ? n : a.stages;
      for (int e = 0; e < pre; ++e) {
        if (lane == 0 && my_bytes) issue(ts.j[e]);
        pst = pst + 1 == (uint32_t)a.stages ? 0u : pst + 1;
        ++inflight;
      }
      for (int e = 0; e < n; ++e) {
        const uint32_t st = cst;
        bool ok = true;
        if (my_bytes) ok = mbar_wait(&bar[st], cph, &never, a.timeout_ns);
        ok = __all_sync(FULL, ok);
        const uint8_t* stage = ring + (size_t)st * stage_bytes;
        const uint4* rd = reinterpret_cast<const uint4*>(stage);
        const uint4* r1 = reinterpret_cast<const uint4*>(stage + a.slice_bytes);
        const uint4* r2 = reinterpret_cast<const uint4*>(stage + 2 * a.slice_bytes);
        float pa[4] = {0.f, 0.f, 0.f, 0.f};
        float pb[4] = {0.f, 0.f, 0.f, 0.f};
        if (ok) {
#pragma unroll
          for (int c = 0; c < NCHW; ++c) {
            const int lc = c * SPAN + lane * E;  // column within this warp's range
            if (lc < my_cols) {
              if (c & 1) L::dot(xr[c], rd[lc / E], pb);
              else L::dot(xr[c], rd[lc / E], pa);
            }
          }
        }
        const float part = warp_sum(((pa[0] + pb[0]) + (pa[1] + pb[1])) +
                                    ((pa[2] + pb[2]) + (pa[3] + pb[3])));
        const int rb = e & 1;  // exchange buffer of this entry
        if (lane == 0) {
          ts.red[rb][tw] = part;
          ts.ok[rb][tw] = ok ? 1 : 0;
        }
        team_bar(team);  // unconditional: every warp of the team reaches it
        float dotv = 0.f;
        bool all_ok = true;
#pragma unroll
        for (int q = 0; q < kTeam; ++q) {
          dotv += ts.red[rb][q];
          all_ok = all_ok && ts.ok[rb][q] != 0;
        }
        if (!all_ok) {  // the same decision in every warp of the team
          failed = true;
          break;
        }
        --inflight;
        if (++cst == (uint32_t)a.stages) {
          cst = 0;
          cph ^= 1u;
        }
        const float gv = ts.g[e];
        float s1, s2 = 0.f;
        if (MODE == kModeHybBwd) {
          const float uv = ts.u[e];
          s1 = dotv * gv;                    // du
          s2 = fmaf(dotv, uv, a.lam);        // dz
          if (leader && lane == 0) {
            Payload p;
            p.t = t;
            p.h = gv * uv;
            p.du = s1;
            p.dz = s2;
            a.pay[a.e0[t] + w0 + e] = p;
          }
        } else {
          s1 = gv * dotv;                    // h
          if (MODE == kModeHybFwd && leader && lane == 0)
            L::store((to_backup ? a.backup_u : a.ell_u) + ts.pos[e], dotv);
        }
        const float2 h1 = make_float2(s1, s1);
        const float2 h2 = make_float2(s2, s2);
#pragma unroll
        for (int c = 0; c < NCHW; ++c) {
          const int lc = c * SPAN + lane * E;
          if (lc < my_cols) {
            float2 w[P];
            L::pairs(r1[lc / E], w);
#pragma unroll
            for (int q = 0; q < P; ++q) acc[c][q] = __ffma2_rn(h1, w[q], acc[c][q]);
            if (MODE == kModeHybBwd) {
              L::pairs(r2[lc / E], w);
#pragma unroll
              for (int q = 0; q < P; ++q) acc[c][q] = __ffma2_rn(h2, w[q], acc[c][q]);
            }
          }
        }
        __syncwarp();  // every lane is done with this stage
        const int nxt = e + a.stages;
        if (nxt < n) {  // refill the stage just freed (the ring was full)
          if (lane == 0 && my_bytes) issue(ts.j[nxt]);
          pst = pst + 1 == (uint32_t)a.stages ? 0u : pst + 1;
          ++inflight;
        }
      }
      team_bar(team);  // the list may be overwritten by the next window
    }
    if (failed) break;

    // ------------------------------------------------------------ output --
    const bool split = prow >= 0;
    float* out_row = split ? a.ws.partial + (size_t)prow * d : nullptr;
#pragma unroll
    for (int c = 0; c < NCHW; ++c) {
      const int col = c0 + c * SPAN + lane * E;
      if (col >= d) continue;
      if (split || !kOutBf16) {
        float* dst = split ? out_row + col : static_cast<float*>(a.out) + (size_t)t * d + col;
#pragma unroll
        for (int q = 0; q < P / 2; ++q)
          reinterpret_cast<float4*>(dst)[q] = make_float4(acc[c][2 * q].x, acc[c][2 * q].y,
                                                          acc[c][2 * q + 1].x, acc[c][2 * q + 1].y);
      } else {
        uint16_t* yt = static_cast<uint16_t*>(a.out) + (size_t)t * d + col;
#pragma unroll
        for (int q = 0; q < P; ++q)
          reinterpret_cast<uint32_t*>(yt)[q] = pack_bf16x2(acc[c][q].x, acc[c][q].y);
      }
    }
    if (split) {
      // the last part to finish sums the partial rows in part order
      __threadfence();
      team_bar(team);  // both halves of this part's row are written
      const int part = a.ws.hdr[2];
      const int parts = (a.ws.nnz[t] + part - 1) / part;
      if (leader && lane == 0) ts.prev = atomicAdd(&a.ws.done[t], 1);
      team_bar(team);
      if (ts.prev == parts - 1) {
        __threadfence();
        const float* part0 = a.ws.partial + (size_t)(prow - lo / part) * d;
        for (int col = c0 + lane * 4; col < c0 + my_cols; col += 128) {
          float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int q = 0; q < parts; ++q) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(part0 + (size_t)q * d + col));
            sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
          }
          if (kOutBf16) {
            uint16_t* yt = static_cast<uint16_t*>(a.out) + (size_t)t * d + col;
            reinterpret_cast<uint2*>(yt)[0] = make_uint2(pack_bf16x2(sum.x, sum.y),
                                                         pack_bf16x2(sum.z, sum.w));
          } else {
            *reinterpret_cast<float4*>(static_cast<float*>(a.out) + (size_t)t * d + col) = sum;
          }
        }
      }
    }
  }

  if (failed) {
    if (lane == 0) set_status(a.status, kStatusTimeout);
    // let the copies still in flight land before the CTA may exit
    for (uint32_t q = 0; q < inflight; ++q) {
      if (my_bytes) mbar_wait(&bar[cst], cph, &never, a.timeout_ns);
      if (++cst == (uint32_t)a.stages) {
        cst = 0;
        cph ^= 1u;
      }
    }
  }
}

template <typename Tin, int NCHW, int MODE>
cudaError_t launch_nchw(GatherArgs<Tin> a, bool out_bf16, cudaStream_t stream) {
  constexpr int SPAN = 32 * Elem<Tin>::E;
  constexpr int NROWS = MODE == kModeHybBwd ? 3 : 2;
  a.slice_bytes = NCHW * SPAN * (int)sizeof(Tin);
  a.stages = kRingBytes / (NROWS * a.slice_bytes);
  if (a.stages > 8) a.stages = 8;
  if (a.stages < 2) a.stages = 2;
  const size_t team_bytes = (sizeof(TeamSmem) * kTeams + 127) & ~size_t(127);
  const size_t per_warp = 128 + (size_t)a.stages * NROWS * a.slice_bytes;
  const size_t smem = team_bytes + per_warp * kWarps;
  auto kern = out_bf16 ? gather_kernel<Tin, NCHW, true, MODE> : gather_kernel<Tin, NCHW, false, MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 32 * kWarps, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  kern<<<num_sms() * per_sm, 32 * kWarps, smem, stream>>>(a);
  return cudaGetLastError();
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
  if constexpr (sizeof(Tin) == 4) return launch_nchw<Tin, 8, MODE>(a, out_bf16, stream);
  return cudaErrorInvalidValue;  // d beyond the validated maximum
}

// Clear the workspace prefix, plan the items from the counts in w.nnz (filled
// by `count`), run the engine.
template <typename Tin, int MODE, class CountFn>
cudaError_t run_engine(GatherArgs<Tin> a, bool out_bf16, void* base, CountFn count,
                       cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(base, 0, a.ws.zero_bytes, stream);
  if (e != cudaSuccess) return e;
  count();
  plan_scan_kernel<<<1, kScanThreads, 0, stream>>>(a.T, a.ws.nnz, a.ws.parts_cap,
                                                   a.ws.max_items, num_sms() * kTeams,
                                                   a.ws.slot_off, a.ws.item_desc, a.ws.hdr);
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
  a.timeout_ns = kWaitTimeoutNs;
  const int T = g.T, K = g.F / W;
  return run_engine<Tin, kModeTwell>(
      a, y_dtype == TW_BF16, base,
      [&] { plan_count_twell_kernel<<<(T + 255) / 256, 256, 0, stream>>>(T, K, g.cnt, w.nnz); },
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
  a.timeout_ns = kWaitTimeoutNs;
  const int T = h.T;
  return run_engine<Tin, MODE>(
      a, out_dtype == TW_BF16, base,
      [&] {
        plan_count_hybrid_kernel<<<(T + 255) / 256, 256, 0, stream>>>(T, h.row_nnz, h.row_slot,
                                                                       h.backup_cap, w.nnz);
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

cudaError_t launch_hybrid_gather_forward(const void* x, const tw_hybrid& gu, const void* Wu_t,
                                         const void* Wd, int d, void* y, tw_dtype y_dtype,
                                         void* ws, int32_t* status, cudaStream_t stream) {
  // u is defined as +0 off the pattern: clear both u arrays, the engine then
  // writes the pattern's entries
  cudaError_t e = cudaSuccess;
  const size_t esz = gu.dtype == TW_BF16 ? 2 : 4;
  if (gu.C_h > 0) e = cudaMemsetAsync(gu.ell_u, 0, esz * (size_t)gu.T * gu.C_h, stream);
  if (e == cudaSuccess && gu.backup_cap > 0)
    e = cudaMemsetAsync(gu.backup_u, 0, esz * (size_t)gu.backup_cap * gu.F, stream);
  if (e != cudaSuccess) return e;
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
