// decode_step.cu -- the whole gated FFN of a small batch (1 <= T <= 64
// tokens, decoding) in ONE persistent, cooperative launch: the gate
// projection with its TwELL packing ("Sparser, Faster, Lighter Transformer
// Language Models", technical summary, section 2.1) and the fused up + down
// projection over the active units (section 2.2).
//
// With a handful of tokens the step is bound by streaming Wg from HBM
// (d x F bf16, 33.5 MB at d = 2048, F = 8192) plus a few dozen gathered
// weight rows per token; the separate launches of the gate and the fused
// kernels (and their set-up) cost more than the data movement itself.  Here
// one grid, one CTA of 16 warps per SM, runs its phases separated by grid
// barriers:
//
//   A  gate: work items of 16 units x 256 columns of d.  Each CTA serves one
//      slice of d and stages that slice of every token's x in shared memory;
//      its warps take the slice's unit groups, stream their 16 Wg rows
//      (16-byte loads, all eight 32-column steps in flight) and multiply
//      them with x on the tensor pipe: mma.sync
//      m16n8k16 with the units on M and the tokens on N, one 8-token column
//      tile per MMA.  The reduction over d is split into slices: each item
//      writes fp32 partial sums zpart[slice][t][u], which the next phase
//      adds in slice order.
//
// Up to 16 tokens:
//   B  packing and dot products: each (tile k, token t) gets one or more
//      warps.  Every one of them adds the slices in a fixed order, applies
//      ReLU and rounds g to bf16; the first packs the tile's TwELL slots
//      exactly as the gate GEMM's epilogue does (ascending units, count,
//      padding, lossless spill of the whole segment past C).  The warps then
//      split the tile's non-zeros (two at a time per warp): for an entry
//      (j, g) a warp forms u = x_t . Wu_t[j] (fp32) and stores h = g u and j
//      at the entry's place in the tile (stride W per tile, ascending).
//      Each warp then asks L2 for the Wd rows of its entries, so phase C
//      finds them there.
//   C  updates: one CTA per (token, 256-column slice of d); warp w takes the
//      tiles k = w (mod 16) in rounds of four (one load trip for the round's
//      counts and first eight entries per tile), accumulates h Wd[j] over its
//      columns in fp32, and the CTA adds the warps' partial rows in warp
//      order.
//
// 17 to 64 tokens, where a heavy token's tiles would hold single warps up
// for long:
//   B  packing only, one warp per (tile, token), as above; every non-zero's
//      unit j and g go to its place in the tile's row of a per-token list.
//      (Requesting its Wu and Wd rows into L2 here made the next grid
//      barrier wait behind that traffic and cost more than it saved.)
//   C  dot products: every CTA builds the same per-token prefix sums of the
//      tile counts; the grid's warps then take the entry pairs of all tokens
//      in turn, ask L2 for the pair's Wd rows, form u = x_t . Wu_t[j] over
//      the whole row and store h = g u.
//   D  updates: tasks (token, chunk of up to kChunk entries, 256-column
//      slice), one warp each, which accumulates h Wd[j] over the chunk's
//      entries in order, 8 columns per lane in fp32.  A token with one chunk
//      writes y; the chunks of a longer token write partial rows.
//   E  (only when some token was split) each split token's y is the sum of
//      its chunks' partial rows in chunk order.
//
// y is deterministic in both.
//
#include "tw_common.cuh"
#include "tw_internal.h"

namespace tw {
namespace {

constexpr unsigned FULL = 0xFFFFFFFFu;
constexpr int kWarpsD = 16;
constexpr int kThreadsD = 32 * kWarpsD;
constexpr int kW = 128;          // TwELL tile width of this path
constexpr int kSlice = 256;      // columns of d per gate work item
constexpr int kSteps = kSlice / 32;
// A CTA of phase A serves one 256-column slice of d and stages just that
// slice of every token, at a row stride of kSliceRow 16-byte
// chunks (32 used): the 64-byte pad puts the two token rows read by one
// quarter-warp on disjoint banks.
constexpr int kSliceRow = 36;
constexpr int kChunk = 32;       // entries per phase-D task (one warp) of a token
constexpr int kChunkRows = 512;  // partial rows in the workspace

struct DecodeArgs {
  const uint16_t* x;
  const uint16_t* Wg;
  const uint16_t* Wu;
  const uint16_t* Wd;
  int T, d, F, C, S;  // S: slices of d
  // TwELL output
  uint16_t* val;
  uint8_t* idx;
  uint8_t* cnt;
  int32_t* spill_ref;
  int spill_cap;
  int32_t* spill_tk;
  uint16_t* spill_val;
  int32_t* spill_n;
  uint16_t* dump;
  // y
  void* y;
  int y_bf16;
  // workspace
  int32_t* bar;    // [0] arrivals, [1] departures
  float* zpart;    // [S][T][F]
  int32_t* jtile;  // [T][F]: units of the non-zeros of tile k at [k * W, k * W + cnt)
  float* htile;    // [T][F]: their g (phase B), then h = g u (phase C)
  float* prow;     // [kChunkRows][d]: partial rows of the chunks of split tokens
  int32_t* status;
  unsigned long long timeout_ns;
};

TW_DEV void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                     uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

TW_DEV int ld_acquire(const int32_t* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// The bf16 g of the four units lane, lane + 32, lane + 64, lane + 96 of tile
// k for token t: the nsl slices' fp32 partial sums added in slice order, ReLU
// (-0 -> +0), then rounding.  The partials were written by other CTAs before
// the grid barrier, so they are read from L2 (.cg), and a batch of slices is
// loaded before its first add: these loads are the phase's latency.
TW_DEV void tile_g(const DecodeArgs& a, int nsl, int t, int k, int lane, uint16_t (&gv)[4]) {
  constexpr int kBatch = 8;  // slices loaded together (d <= 2048 is one batch)
  const float* zp = a.zpart + (size_t)t * a.F + k * kW + lane;
  const size_t sstride = (size_t)a.T * a.F;
  float z[4] = {0.f, 0.f, 0.f, 0.f};
  for (int s0 = 0; s0 < nsl; s0 += kBatch) {
    float p[kBatch][4];
#pragma unroll
    for (int s = 0; s < kBatch; ++s)
#pragma unroll
      for (int i = 0; i < 4; ++i)
        p[s][i] = s0 + s < nsl ? __ldcg(zp + (size_t)(s0 + s) * sstride + 32 * i) : 0.f;
#pragma unroll
    for (int s = 0; s < kBatch; ++s)
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (s0 + s < nsl) z[i] += p[s][i];
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float zr = (int32_t)__float_as_uint(z[i]) > 0 ? z[i] : 0.0f;
    gv[i] = f32_to_bf16(zr);
  }
}

// 8 columns of token t's x from column col (zeros past T or d).
TW_DEV uint4 xrow_g(const DecodeArgs& a, int t, int col) {
  if (t >= a.T || col >= a.d) return make_uint4(0, 0, 0, 0);
  return __ldg(reinterpret_cast<const uint4*>(a.x + (size_t)t * a.d + col));
}

// Asks L2 for a weight row (d bf16) ahead of its use, one 128-byte line per
// lane and step, so that the phase after the next barrier finds it there.
TW_DEV void prefetch_row_l2(const uint16_t* row, int d, int lane) {
  for (int c = lane * 64; c < d; c += 32 * 64)
    asm volatile("prefetch.global.L2 [%0];" ::"l"(row + c));
}

// Grid-wide barrier number `b` (1-based) of this launch.  Bounded: a CTA that
// has waited longer than timeout_ns flags TW_ERR_TIMEOUT and goes on.
TW_DEV void grid_barrier(const DecodeArgs& a, int b) {
  __syncthreads();
  if (threadIdx.x == 0) {
    // release: the CTA's writes (ordered before this thread by the CTA
    // barrier) become visible before the arrival does
    asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(&a.bar[0]) : "memory");
    const int target = b * (int)gridDim.x;
    uint64_t t0 = 0;
    for (uint32_t i = 0; ld_acquire(&a.bar[0]) < target; ++i) {
      __nanosleep(32);
      if ((i & 63u) == 63u) {
        const uint64_t now = globaltimer_ns();
        if (t0 == 0) {
          t0 = now;
        } else if (now - t0 > a.timeout_ns) {
          set_status(a.status, kStatusTimeout);
          break;
        }
      }
    }
  }
  __syncthreads();
}

// NT: 8-token column tiles of the gate MMAs (1, 2, 4 or 8: T <= 8 * NT).
template <int NT>
__global__ void __launch_bounds__(kThreadsD, 1) decode_step_kernel(const DecodeArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int T = a.T, d = a.d, F = a.F, K = F / kW;
  // x slice of phase A: [8 * NT][kSliceRow]
  uint4* xsl = reinterpret_cast<uint4*>(smem);
  const size_t x_bytes = (size_t)8 * NT * kSliceRow * 16;
  // after it: the warps' partial rows of phase C (up to 16 tokens) or the
  // plan tables of phases C and D (more)
  float* red = reinterpret_cast<float*>(smem + x_bytes);  // [16][256]
  int* tbl = reinterpret_cast<int*>(red);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = gridDim.x * kWarpsD;
  const int gw = blockIdx.x * kWarpsD + warp;
  // 16 bytes of token t's x at column col (zeros past T or d); x is a few
  // KB per token and stays in L1 and L2
  auto xrow = [&](int t, int col) -> uint4 { return xrow_g(a, t, col); };
  // 8 values of y for token t at column col, in y's dtype
  auto store_y = [&](int t, int col, const float (&v)[8]) {
    if (a.y_bf16) {
      uint16_t* yt = static_cast<uint16_t*>(a.y) + (size_t)t * d + col;
      *reinterpret_cast<uint4*>(yt) =
          make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                     pack_bf16x2(v[6], v[7]));
    } else {
      float4* yt = reinterpret_cast<float4*>(static_cast<float*>(a.y) + (size_t)t * d + col);
      yt[0] = make_float4(v[0], v[1], v[2], v[3]);
      yt[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
  };
  if (blockIdx.x == 0 && threadIdx.x == 0) *a.spill_n = 0;  // before any spill (phase B)
  __syncthreads();

  // ------------------------------------------------------------ A: gate --
  {
    // Work items of 16 units x 256 columns; each CTA serves one slice of d
    // (staged for every token) and its warps take that slice's unit groups.
    // mma.sync m16n8k16 with the units on M and the tokens on N; each item
    // writes fp32 partial sums zpart[slice][t][u].
    const int g = lane >> 2, q = lane & 3;
    const int S = a.S;
    const int s_cta = blockIdx.x % S;
    const int ncs = ((int)gridDim.x - s_cta + S - 1) / S;  // CTAs serving slice s_cta
    {
      const int cs = s_cta * kSlice;
      for (int i = threadIdx.x; i < 8 * NT * 32; i += kThreadsD) {
        const int t = i >> 5, col = cs + (i & 31) * 8;
        xsl[t * kSliceRow + (i & 31)] =
            t < T && col < d ? __ldg(reinterpret_cast<const uint4*>(a.x + (size_t)t * d + col))
                             : make_uint4(0, 0, 0, 0);
      }
      __syncthreads();
    }
    constexpr int kStepsA = kSteps;  // Wg row steps in flight: all eight
    for (int item = (blockIdx.x / S) * kWarpsD + warp; item < F / 16; item += ncs * kWarpsD) {
      const int u0 = item * 16, c0 = s_cta * kSlice;
      const uint16_t* r_lo = a.Wg + (size_t)(u0 + g) * d;
      const uint16_t* r_hi = a.Wg + (size_t)(u0 + g + 8) * d;
      float D[NT][4];
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int i = 0; i < 4; ++i) D[n][i] = 0.f;
#pragma unroll
      for (int i0 = 0; i0 < kSteps; i0 += kStepsA) {
        uint4 alo[kStepsA], ahi[kStepsA];
#pragma unroll
        for (int i = 0; i < kStepsA; ++i) {
          const int col = c0 + (i0 + i) * 32 + 8 * q;
          const bool in = col < d;
          alo[i] = in ? __ldcs(reinterpret_cast<const uint4*>(r_lo + col)) : make_uint4(0, 0, 0, 0);
          ahi[i] = in ? __ldcs(reinterpret_cast<const uint4*>(r_hi + col)) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int i = 0; i < kStepsA; ++i) {
          // The 8 columns a lane loaded take the k-indices of its A fragment
          // (the same permutation of k for every unit row and token column),
          // so the products pair Wg[u][col] with x[t][col].
#pragma unroll
          for (int n = 0; n < NT; ++n) {
            const uint4 xb = xsl[(8 * n + g) * kSliceRow + (i0 + i) * 4 + q];
            mma16816(D[n], alo[i].x, ahi[i].x, alo[i].y, ahi[i].y, xb.x, xb.y);
            mma16816(D[n], alo[i].z, ahi[i].z, alo[i].w, ahi[i].w, xb.z, xb.w);
          }
        }
      }
      // D[m][n]: lane (g, q) holds (g, 2q), (g, 2q+1), (g+8, 2q), (g+8, 2q+1)
      float* zp = a.zpart + (size_t)s_cta * T * F;
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const int t0 = 8 * n + 2 * q;
        if (t0 < T) {
          zp[(size_t)t0 * F + u0 + g] = D[n][0];
          zp[(size_t)t0 * F + u0 + g + 8] = D[n][2];
        }
        if (t0 + 1 < T) {
          zp[(size_t)(t0 + 1) * F + u0 + g] = D[n][1];
          zp[(size_t)(t0 + 1) * F + u0 + g + 8] = D[n][3];
        }
      }
    }
  }
  grid_barrier(a, 1);

  if constexpr (NT < 4) {
    // up to 16 tokens: packing with the dot products, then updates (B, C)
  // -------------------------------------- B: TwELL pack, h = g (x_t . Wu_t[j]) --
  {
    const unsigned lt = (1u << lane) - 1u;
    const int n_it = K * T;
    const int m = nwarps >= n_it ? nwarps / n_it : 1;  // warps per (tile, token)
    const int sub = nwarps >= n_it ? gw / n_it : 0;
    for (int item = nwarps >= n_it ? gw % n_it : gw; sub < m && item < n_it;
         item += nwarps >= n_it ? n_it : nwarps) {
      const int k = item / T, t = item % T;
      uint16_t gv[4];
      tile_g(a, a.S, t, k, lane, gv);
      unsigned bal[4];
      int n = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        bal[i] = __ballot_sync(FULL, gv[i] != 0);
        n += __popc(bal[i]);
      }
      const size_t off = (size_t)k * T + t;
      const int C = a.C;
      if (sub == 0) {  // the tile's TwELL slots, count, padding and spill
        int before = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int pos = before + __popc(bal[i] & lt);
          if (gv[i] != 0 && pos < C) {
            a.val[off * C + pos] = gv[i];
            a.idx[off * C + pos] = (uint8_t)(lane + 32 * i);
          }
          before += __popc(bal[i]);
          if (a.dump) a.dump[(size_t)t * F + k * kW + lane + 32 * i] = gv[i];
        }
        for (int sl = lane; sl < C; sl += 32) {
          if (sl >= n) {
            a.val[off * C + sl] = 0;
            a.idx[off * C + sl] = 0;
          }
        }
        if (lane == 0) a.cnt[off] = (uint8_t)n;
        if (n > C) {  // uniform across the warp
          int slot = 0;
          if (lane == 0) slot = atomicAdd(a.spill_n, 1);
          slot = __shfl_sync(FULL, slot, 0);
          if (slot < a.spill_cap) {
            if (lane == 0) {
              a.spill_ref[off] = slot;
              a.spill_tk[2 * (size_t)slot] = t;
              a.spill_tk[2 * (size_t)slot + 1] = k;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) a.spill_val[(size_t)slot * kW + lane + 32 * i] = gv[i];
          } else if (lane == 0) {
            a.spill_ref[off] = -1;
            set_status(a.status, kStatusSpill);
          }
        }
      }
      // the tile's non-zeros, ascending; entry p goes to the warp with
      // p % m == sub, which lists (unit, g) of its entries in its slice of
      // `red` and forms their dot products two at a time
      float* lst = red + warp * kSlice;  // 128 (unit, g) pairs
      int before = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int pos = before + __popc(bal[i] & lt);
        if (gv[i] != 0 && pos % m == sub) {
          const int r = pos / m;
          lst[2 * r] = __int_as_float(k * kW + lane + 32 * i);
          lst[2 * r + 1] = bf16_to_f32(gv[i]);
        }
        before += __popc(bal[i]);
      }
      __syncwarp();
      const int nh = sub < n ? (n - sub + m - 1) / m : 0;  // entries of this warp
      for (int r = 2; r < nh; ++r)  // the Wu rows of this warp's later pairs
        prefetch_row_l2(a.Wu + (size_t)__float_as_int(lst[2 * r]) * d, d, lane);
      for (int r0 = 0; r0 < nh; r0 += 2) {
        const bool two = r0 + 1 < nh;
        const int j0 = __float_as_int(lst[2 * r0]);
        const int j1 = two ? __float_as_int(lst[2 * r0 + 2]) : j0;
        const uint16_t* w0 = a.Wu + (size_t)j0 * d;
        const uint16_t* w1 = a.Wu + (size_t)j1 * d;
        float p[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll 8
        for (int c = lane * 8; c < d; c += 256) {
          const uint4 xv = xrow(t, c);
          const uint4 wa = __ldg(reinterpret_cast<const uint4*>(w0 + c));
          const uint4 wb = two ? __ldg(reinterpret_cast<const uint4*>(w1 + c)) : make_uint4(0, 0, 0, 0);
          p[0][0] = fmaf(bf16_lo(xv.x), bf16_lo(wa.x), p[0][0]);
          p[0][1] = fmaf(bf16_hi(xv.x), bf16_hi(wa.x), p[0][1]);
          p[0][2] = fmaf(bf16_lo(xv.y), bf16_lo(wa.y), p[0][2]);
          p[0][3] = fmaf(bf16_hi(xv.y), bf16_hi(wa.y), p[0][3]);
          p[0][0] = fmaf(bf16_lo(xv.z), bf16_lo(wa.z), p[0][0]);
          p[0][1] = fmaf(bf16_hi(xv.z), bf16_hi(wa.z), p[0][1]);
          p[0][2] = fmaf(bf16_lo(xv.w), bf16_lo(wa.w), p[0][2]);
          p[0][3] = fmaf(bf16_hi(xv.w), bf16_hi(wa.w), p[0][3]);
          p[1][0] = fmaf(bf16_lo(xv.x), bf16_lo(wb.x), p[1][0]);
          p[1][1] = fmaf(bf16_hi(xv.x), bf16_hi(wb.x), p[1][1]);
          p[1][2] = fmaf(bf16_lo(xv.y), bf16_lo(wb.y), p[1][2]);
          p[1][3] = fmaf(bf16_hi(xv.y), bf16_hi(wb.y), p[1][3]);
          p[1][0] = fmaf(bf16_lo(xv.z), bf16_lo(wb.z), p[1][0]);
          p[1][1] = fmaf(bf16_hi(xv.z), bf16_hi(wb.z), p[1][1]);
          p[1][2] = fmaf(bf16_lo(xv.w), bf16_lo(wb.w), p[1][2]);
          p[1][3] = fmaf(bf16_hi(xv.w), bf16_hi(wb.w), p[1][3]);
        }
        const float u0 = warp_sum((p[0][0] + p[0][1]) + (p[0][2] + p[0][3]));
        const float u1 = warp_sum((p[1][0] + p[1][1]) + (p[1][2] + p[1][3]));
        if (lane == 0) {
          const int pos0 = r0 * m + sub;
          a.jtile[(size_t)t * F + k * kW + pos0] = j0;
          a.htile[(size_t)t * F + k * kW + pos0] = lst[2 * r0 + 1] * u0;
          if (two) {
            const int pos1 = (r0 + 1) * m + sub;
            a.jtile[(size_t)t * F + k * kW + pos1] = j1;
            a.htile[(size_t)t * F + k * kW + pos1] = lst[2 * r0 + 3] * u1;
          }
        }
      }
      for (int r = 0; r < nh; ++r)  // the Wd rows phase C gathers for these entries
        prefetch_row_l2(a.Wd + (size_t)__float_as_int(lst[2 * r]) * d, d, lane);
      __syncwarp();  // the list is rewritten by the warp's next item
    }
  }
    grid_barrier(a, 2);

  // --------------------------------------------------- C: y_t = sum h Wd[j] --
  {
    const int nsl = (d + kSlice - 1) / kSlice;
    for (int task = blockIdx.x; task < T * nsl; task += gridDim.x) {
      const int t = task / nsl, sl = task % nsl;
      const int col = sl * kSlice + lane * 8;
      const bool in = col < d;
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
      // acc += h Wd[j][col, col + 8)
      auto axpy8 = [&](float h, const uint4& w) {
        acc[0] = fmaf(h, bf16_lo(w.x), acc[0]);
        acc[1] = fmaf(h, bf16_hi(w.x), acc[1]);
        acc[2] = fmaf(h, bf16_lo(w.y), acc[2]);
        acc[3] = fmaf(h, bf16_hi(w.y), acc[3]);
        acc[4] = fmaf(h, bf16_lo(w.z), acc[4]);
        acc[5] = fmaf(h, bf16_hi(w.z), acc[5]);
        acc[6] = fmaf(h, bf16_lo(w.w), acc[6]);
        acc[7] = fmaf(h, bf16_hi(w.w), acc[7]);
      };
      constexpr int kB = 8;  // entries whose rows are loaded together
      // Rounds of four of the warp's tiles (k = warp + 16 i).  Lane l loads
      // the count of tile kb + 16 (l / 8) and that tile's entry l % 8 (unit
      // and h; past the count they are not used), so a round's lists cost one
      // trip.  The entries are taken in tile order, kB rows in flight; the
      // entries past the eighth of a tile follow, tile by tile, 32 to a trip.
      for (int kb = warp; kb < K; kb += 4 * kWarpsD) {
        const int kl = kb + kWarpsD * (lane >> 3), bl = lane & 7;
        int nl = 0, jl = 0;
        float hl = 0.f;
        if (kl < K) {
          nl = a.cnt[(size_t)kl * T + t];
          const size_t e = (size_t)t * F + kl * kW + bl;
          jl = a.jtile[e];
          hl = a.htile[e];
        }
        unsigned live = __ballot_sync(FULL, bl < nl);
        while (live != 0) {
          int jj[kB];
          float hh[kB];
          bool vb[kB];
#pragma unroll
          for (int b = 0; b < kB; ++b) {
            vb[b] = live != 0;
            const int src = vb[b] ? __ffs(live) - 1 : 0;
            jj[b] = __shfl_sync(FULL, jl, src);
            hh[b] = __shfl_sync(FULL, hl, src);
            live &= live - 1u;
          }
          uint4 wv[kB];
#pragma unroll
          for (int b = 0; b < kB; ++b)
            wv[b] = in && vb[b] ? __ldg(reinterpret_cast<const uint4*>(a.Wd + (size_t)jj[b] * d + col))
                                : make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int b = 0; b < kB; ++b)
            if (vb[b]) axpy8(hh[b], wv[b]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int n = __shfl_sync(FULL, nl, 8 * i);
          const int k = kb + kWarpsD * i;
          if (n <= kB) continue;  // (zero past K)
          const size_t e0 = (size_t)t * F + k * kW;
          for (int s0 = kB; s0 < n; s0 += 32) {  // lane l loads entry s0 + l
            const int m = min(32, n - s0);
            int jo = 0;
            float ho = 0.f;
            if (lane < m) {
              jo = a.jtile[e0 + s0 + lane];
              ho = a.htile[e0 + s0 + lane];
            }
            for (int b0 = 0; b0 < m; b0 += kB) {
              int jj[kB];
              float hh[kB];
#pragma unroll
              for (int b = 0; b < kB; ++b) {
                jj[b] = __shfl_sync(FULL, jo, (b0 + b) & 31);
                hh[b] = __shfl_sync(FULL, ho, (b0 + b) & 31);
              }
              uint4 wv[kB];
#pragma unroll
              for (int b = 0; b < kB; ++b)
                wv[b] = in && b0 + b < m ? __ldg(reinterpret_cast<const uint4*>(
                                               a.Wd + (size_t)jj[b] * d + col))
                                         : make_uint4(0, 0, 0, 0);
#pragma unroll
              for (int b = 0; b < kB; ++b)
                if (b0 + b < m) axpy8(hh[b], wv[b]);
            }
          }
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) red[warp * kSlice + lane * 8 + i] = acc[i];
      __syncthreads();
      if (warp == 0 && in) {
        float v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = red[lane * 8 + i];
        for (int w = 1; w < kWarpsD; ++w)
#pragma unroll
          for (int i = 0; i < 8; ++i) v[i] += red[w * kSlice + lane * 8 + i];
        if (a.y_bf16) {
          uint16_t* yt = static_cast<uint16_t*>(a.y) + (size_t)t * d + col;
          *reinterpret_cast<uint4*>(yt) =
              make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                         pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
        } else {
          float4* yt = reinterpret_cast<float4*>(static_cast<float*>(a.y) + (size_t)t * d + col);
          yt[0] = make_float4(v[0], v[1], v[2], v[3]);
          yt[1] = make_float4(v[4], v[5], v[6], v[7]);
        }
      }
      __syncthreads();  // red is reused by the next task
    }
  }

  } else {
    // 17 to 64 tokens: packing, then dot products and updates spread evenly
    // over the grid (B to E)
  // ------------------------------- B: TwELL pack, and (unit, g) per entry --
  {
    const unsigned lt = (1u << lane) - 1u;
    const int n_it = K * T;
    for (int item = gw; item < n_it; item += nwarps) {
      const int k = item / T, t = item % T;
      uint16_t gv[4];
      tile_g(a, a.S, t, k, lane, gv);
      unsigned bal[4];
      int n = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        bal[i] = __ballot_sync(FULL, gv[i] != 0);
        n += __popc(bal[i]);
      }
      const size_t off = (size_t)k * T + t;
      const int C = a.C;
      {  // the tile's TwELL slots, count, padding and spill
        int before = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int pos = before + __popc(bal[i] & lt);
          if (gv[i] != 0 && pos < C) {
            a.val[off * C + pos] = gv[i];
            a.idx[off * C + pos] = (uint8_t)(lane + 32 * i);
          }
          before += __popc(bal[i]);
          if (a.dump) a.dump[(size_t)t * F + k * kW + lane + 32 * i] = gv[i];
        }
        for (int sl = lane; sl < C; sl += 32) {
          if (sl >= n) {
            a.val[off * C + sl] = 0;
            a.idx[off * C + sl] = 0;
          }
        }
        if (lane == 0) a.cnt[off] = (uint8_t)n;
        if (n > C) {  // uniform across the warp
          int slot = 0;
          if (lane == 0) slot = atomicAdd(a.spill_n, 1);
          slot = __shfl_sync(FULL, slot, 0);
          if (slot < a.spill_cap) {
            if (lane == 0) {
              a.spill_ref[off] = slot;
              a.spill_tk[2 * (size_t)slot] = t;
              a.spill_tk[2 * (size_t)slot + 1] = k;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) a.spill_val[(size_t)slot * kW + lane + 32 * i] = gv[i];
          } else if (lane == 0) {
            a.spill_ref[off] = -1;
            set_status(a.status, kStatusSpill);
          }
        }
      }
      // the tile's non-zeros, ascending: unit and g at [t][k * W + pos]
      {
        int before = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int pos = before + __popc(bal[i] & lt);
          if (gv[i] != 0) {
            const size_t e = (size_t)t * F + k * kW + pos;
            a.jtile[e] = k * kW + lane + 32 * i;
            a.htile[e] = bf16_to_f32(gv[i]);
          }
          before += __popc(bal[i]);
        }
      }
    }
  }
  grid_barrier(a, 2);

  // ----------------------------------------------- per-CTA plan of C and D --
  // pre[t][k]: entries of token t in tiles before k (so E_t = pre[t][K]);
  // every CTA builds the same tables from the counts.  Phase C takes entry
  // pairs of each token, phase D tasks (token, chunk of kChunk entries,
  // 256-column slice); a token with more than kChunk entries is split into
  // chunks with partial rows (in token order while the rows last; a token
  // past them keeps one task per slice).
  int* pre = tbl;  // [T][K + 1]
  int* tab = pre + (size_t)T * (K + 1);  // pair_off[T + 1], nch[T], row_off[T], task_off[T + 1]
  int* pair_off = tab;
  int* nch = pair_off + (T + 1);
  int* row_off = nch + T;
  int* task_off = row_off + T;
  __shared__ int any_split;
  const int nsl = (d + kSlice - 1) / kSlice;
  // the counts [K][T] into pre[t][k + 1] with one pass of all threads, then
  // each token's running sum over its tiles in place
  for (int i = threadIdx.x; i < K * T; i += kThreadsD) {
    const int k = i / T, t = i % T;
    pre[(size_t)t * (K + 1) + k + 1] = a.cnt[i];
  }
  __syncthreads();
  for (int t = warp; t < T; t += kWarpsD) {
    int base = 0;
    if (lane == 0) pre[(size_t)t * (K + 1)] = 0;
    for (int kb = 0; kb < K; kb += 32) {
      const int k = kb + lane;
      const int n = k < K ? pre[(size_t)t * (K + 1) + k + 1] : 0;
      int incl = n;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(FULL, incl, o);
        if (lane >= o) incl += u;
      }
      if (k < K) pre[(size_t)t * (K + 1) + k + 1] = base + incl;
      base += __shfl_sync(FULL, incl, 31);
    }
  }
  __syncthreads();
  // warp 0, 32 tokens per round: running offsets of the pairs, the chunk
  // rows (a token asks for its chunks' rows in token order; it is split if
  // they fit, and once the rows asked for pass the capacity no later token
  // is) and the tasks
  if (warp == 0) {
    int po = 0, ro = 0, to = 0;
    bool split_any = false;
    auto incl_scan = [&](int v) {
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(FULL, v, o);
        if (lane >= o) v += u;
      }
      return v;
    };
    for (int t0 = 0; t0 < T; t0 += 32) {
      const int t = t0 + lane;
      const int E = t < T ? pre[(size_t)t * (K + 1) + K] : 0;
      const int pairs = (E + 1) / 2;
      const int c_all = (E + kChunk - 1) / kChunk;
      const int want = c_all > 1 ? c_all : 0;
      const int ip = incl_scan(pairs), iw = incl_scan(want);
      const int xw = ro + iw - want;
      const bool split = c_all > 1 && xw + c_all <= kChunkRows;
      const int c = split ? c_all : 1;
      const int tasks = t < T ? c * nsl : 0;
      const int itk = incl_scan(tasks);
      if (t < T) {
        pair_off[t] = po + ip - pairs;
        row_off[t] = split ? xw : -1;
        nch[t] = c;
        task_off[t] = to + itk - tasks;
      }
      split_any = split_any || __any_sync(FULL, split);
      po += __shfl_sync(FULL, ip, 31);
      ro += __shfl_sync(FULL, iw, 31);
      to += __shfl_sync(FULL, itk, 31);
    }
    if (lane == 0) {
      pair_off[T] = po;
      task_off[T] = to;
      any_split = split_any ? 1 : 0;
    }
  }
  __syncthreads();
  // entry e of token t: its tile k and place (largest k with pre[t][k] <= e)
  auto locate = [&](int t, int e, int& k, int& pos) {
    const int* pt = pre + (size_t)t * (K + 1);
    int lo = 0, hi = K;  // pt[lo] <= e < pt[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (pt[mid] <= e)
        lo = mid;
      else
        hi = mid;
    }
    k = lo;
    pos = e - pt[lo];
  };
  // the token whose range [off[t], off[t + 1]) holds q (off[0] <= q < off[T])
  auto owner = [&](const int* off, int q) {
    int lo = 0, hi = T;  // off[lo] <= q < off[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (off[mid] <= q)
        lo = mid;
      else
        hi = mid;
    }
    return lo;
  };

  // ---------------------------------- C: h = g (x_t . Wu_t[j]) per entry --
  {
    const int P = pair_off[T];
    for (int q = gw; q < P; q += nwarps) {
      const int t = owner(pair_off, q);
      const int E = pre[(size_t)t * (K + 1) + K];
      const int e0 = 2 * (q - pair_off[t]);
      const bool two = e0 + 1 < E;
      int k0, p0, k1, p1;
      locate(t, e0, k0, p0);
      if (two) {
        locate(t, e0 + 1, k1, p1);
      } else {
        k1 = k0;
        p1 = p0;
      }
      const size_t i0 = (size_t)t * F + k0 * kW + p0, i1 = (size_t)t * F + k1 * kW + p1;
      const int j0 = a.jtile[i0], j1 = a.jtile[i1];
      // the pair's Wd rows, which phase D gathers, are requested into L2
      // first: their DRAM reads overlap these dot products, and the next
      // grid barrier (whose release waits for them) comes after the Wu rows
      // anyway
      prefetch_row_l2(a.Wd + (size_t)j0 * d, d, lane);
      if (two) prefetch_row_l2(a.Wd + (size_t)j1 * d, d, lane);
      const uint16_t* w0 = a.Wu + (size_t)j0 * d;
      const uint16_t* w1 = a.Wu + (size_t)j1 * d;
      float pp[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll 8
      for (int c = lane * 8; c < d; c += 256) {
        const uint4 xv = xrow(t, c);
        const uint4 wa = __ldg(reinterpret_cast<const uint4*>(w0 + c));
        const uint4 wb = __ldg(reinterpret_cast<const uint4*>(w1 + c));
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
        const uint32_t aw[4] = {wa.x, wa.y, wa.z, wa.w};
        const uint32_t bw[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          pp[0][r] = fmaf(bf16_lo(xw[r]), bf16_lo(aw[r]), pp[0][r]);
          pp[0][r] = fmaf(bf16_hi(xw[r]), bf16_hi(aw[r]), pp[0][r]);
          pp[1][r] = fmaf(bf16_lo(xw[r]), bf16_lo(bw[r]), pp[1][r]);
          pp[1][r] = fmaf(bf16_hi(xw[r]), bf16_hi(bw[r]), pp[1][r]);
        }
      }
      const float u0 = warp_sum((pp[0][0] + pp[0][1]) + (pp[0][2] + pp[0][3]));
      const float u1 = warp_sum((pp[1][0] + pp[1][1]) + (pp[1][2] + pp[1][3]));
      if (lane == 0) {
        a.htile[i0] = a.htile[i0] * u0;  // g -> h = g u
        if (two) a.htile[i1] = a.htile[i1] * u1;
      }
    }
  }
  grid_barrier(a, 3);

  // --------------------- D: y_t (or a chunk's partial row) = sum h Wd[j] --
  {
    const int n_tasks = task_off[T];
    for (int task = gw; task < n_tasks; task += nwarps) {
      const int t = owner(task_off, task);
      const int r = task - task_off[t];
      const int c = r / nsl, sl = r % nsl;
      const int E = pre[(size_t)t * (K + 1) + K];
      const int lo = nch[t] > 1 ? c * kChunk : 0;
      const int hi = nch[t] > 1 ? min(E, lo + kChunk) : E;
      const int col = sl * kSlice + lane * 8;
      const bool in = col < d;
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
      // 32 entries at a time: lane l locates entry e0 + l and loads its unit
      // and h; the warp takes them in order by shuffles, with the Wd slices
      // of 8 entries in flight
      for (int e0 = lo; e0 < hi; e0 += 32) {
        const int ne = min(32, hi - e0);
        int jl = 0;
        float hl = 0.f;
        if (lane < ne) {
          int k, pos;
          locate(t, e0 + lane, k, pos);
          const size_t ix = (size_t)t * F + k * kW + pos;
          jl = a.jtile[ix];
          hl = a.htile[ix];
        }
        for (int b0 = 0; b0 < ne; b0 += 8) {
          constexpr int kB = 8;  // (16 in flight per lane measured slower)
          uint4 wv[kB];
#pragma unroll
          for (int b = 0; b < kB; ++b) {
            const int jb = __shfl_sync(FULL, jl, (b0 + b) & 31);
            wv[b] = in && b0 + b < ne
                        ? __ldg(reinterpret_cast<const uint4*>(a.Wd + (size_t)jb * d + col))
                        : make_uint4(0, 0, 0, 0);
          }
#pragma unroll
          for (int b = 0; b < kB; ++b) {
            const float hs = __shfl_sync(FULL, hl, (b0 + b) & 31);
            const float hb = b0 + b < ne ? hs : 0.f;
            acc[0] = fmaf(hb, bf16_lo(wv[b].x), acc[0]);
            acc[1] = fmaf(hb, bf16_hi(wv[b].x), acc[1]);
            acc[2] = fmaf(hb, bf16_lo(wv[b].y), acc[2]);
            acc[3] = fmaf(hb, bf16_hi(wv[b].y), acc[3]);
            acc[4] = fmaf(hb, bf16_lo(wv[b].z), acc[4]);
            acc[5] = fmaf(hb, bf16_hi(wv[b].z), acc[5]);
            acc[6] = fmaf(hb, bf16_lo(wv[b].w), acc[6]);
            acc[7] = fmaf(hb, bf16_hi(wv[b].w), acc[7]);
          }
        }
      }
      if (in) {
        if (nch[t] > 1) {
          float4* pr = reinterpret_cast<float4*>(a.prow + (size_t)(row_off[t] + c) * d + col);
          pr[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
          pr[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        } else {
          store_y(t, col, acc);
        }
      }
    }
  }

  // ------------------- E: the chunks of split tokens, added in chunk order --
  if (any_split) {  // the same in every CTA
    grid_barrier(a, 4);
    for (int task = gw; task < T * nsl; task += nwarps) {
      const int t = task / nsl, sl = task % nsl;
      const int col = sl * kSlice + lane * 8;
      if (nch[t] <= 1 || col >= d) continue;
      float v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = 0.f;
      // eight chunks' rows loaded before they are added, in chunk order
      constexpr int kCB = 8;
      const int nc = nch[t];
      for (int c0 = 0; c0 < nc; c0 += kCB) {
        float4 p[kCB][2];
#pragma unroll
        for (int c = 0; c < kCB; ++c) {
          const float4* pr =
              reinterpret_cast<const float4*>(a.prow + (size_t)(row_off[t] + c0 + c) * d + col);
          p[c][0] = c0 + c < nc ? __ldcg(pr) : make_float4(0.f, 0.f, 0.f, 0.f);
          p[c][1] = c0 + c < nc ? __ldcg(pr + 1) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int c = 0; c < kCB; ++c) {
          if (c0 + c < nc) {
            v[0] += p[c][0].x;
            v[1] += p[c][0].y;
            v[2] += p[c][0].z;
            v[3] += p[c][0].w;
            v[4] += p[c][1].x;
            v[5] += p[c][1].y;
            v[6] += p[c][1].z;
            v[7] += p[c][1].w;
          }
        }
      }
      store_y(t, col, v);
    }
  }

  }

  // leave the barrier counters at zero for the next call: the last CTA to
  // depart (all CTAs have passed every barrier) resets them
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const int prev = atomicAdd(&a.bar[1], 1);
    if (prev == (int)gridDim.x - 1) {
      atomicExch(&a.bar[0], 0);
      atomicExch(&a.bar[1], 0);
    }
  }
}

size_t al256(size_t v) { return (v + 255) & ~size_t(255); }

// Workspace layout for (T, d, F); pointers set when base is not null.
size_t decode_layout(void* base, int T, int d, int F, DecodeArgs* a) {
  const int S = (d + kSlice - 1) / kSlice;
  size_t off = 0;
  auto take = [&](size_t b) { const size_t o = off; off = al256(off + b); return o; };
  const size_t o_bar = take(2 * sizeof(int32_t));
  const size_t o_z = take(sizeof(float) * (size_t)S * T * F);
  const size_t o_jt = take(sizeof(int32_t) * (size_t)T * F);
  const size_t o_ht = take(sizeof(float) * (size_t)T * F);
  const size_t o_pr = take(sizeof(float) * (size_t)kChunkRows * d);
  if (base && a) {
    char* p = static_cast<char*>(base);
    a->S = S;
    a->bar = reinterpret_cast<int32_t*>(p + o_bar);
    a->zpart = reinterpret_cast<float*>(p + o_z);
    a->jtile = reinterpret_cast<int32_t*>(p + o_jt);
    a->htile = reinterpret_cast<float*>(p + o_ht);
    a->prow = reinterpret_cast<float*>(p + o_pr);
  }
  return off;
}

}  // namespace

size_t decode_ws_bytes(int T, int d, int F) { return decode_layout(nullptr, T, d, F, nullptr); }

cudaError_t launch_decode_step(const void* x, const void* Wg_t, const void* Wu_t, const void* Wd,
                               int T, int d, int F, const tw_twell& out, void* dump, void* y,
                               tw_dtype y_dtype, void* ws, int32_t* status, cudaStream_t stream) {
  DecodeArgs a{};
  decode_layout(ws, T, d, F, &a);
  a.x = static_cast<const uint16_t*>(x);
  a.Wg = static_cast<const uint16_t*>(Wg_t);
  a.Wu = static_cast<const uint16_t*>(Wu_t);
  a.Wd = static_cast<const uint16_t*>(Wd);
  a.T = T;
  a.d = d;
  a.F = F;
  a.C = out.C;
  a.val = static_cast<uint16_t*>(out.val);
  a.idx = out.idx;
  a.cnt = out.cnt;
  a.spill_ref = out.spill_ref;
  a.spill_cap = out.spill_cap;
  a.spill_tk = out.spill_tk;
  a.spill_val = static_cast<uint16_t*>(out.spill_val);
  a.spill_n = out.spill_n;
  a.dump = static_cast<uint16_t*>(dump);
  a.y = y;
  a.y_bf16 = y_dtype == TW_BF16;
  a.status = status;
  a.timeout_ns = kWaitTimeoutNs;
  const int NT = T <= 8 ? 1 : T <= 16 ? 2 : T <= 32 ? 4 : 8;
  const size_t xs_bytes = (size_t)8 * NT * kSliceRow * 16;
  const int K = F / kW;
  const size_t smem =
      xs_bytes + (NT < 4 ? sizeof(float) * kWarpsD * kSlice
                         : sizeof(int) * ((size_t)T * (K + 1) + 4 * (size_t)T + 2));
  const void* kern = NT == 1 ? reinterpret_cast<const void*>(decode_step_kernel<1>)
                     : NT == 2 ? reinterpret_cast<const void*>(decode_step_kernel<2>)
                     : NT == 4 ? reinterpret_cast<const void*>(decode_step_kernel<4>)
                               : reinterpret_cast<const void*>(decode_step_kernel<8>);
  cudaError_t e = set_smem_limit(kern, (int)smem);
  if (e != cudaSuccess) return e;
  void* args[] = {&a};
  return cudaLaunchCooperativeKernel(kern, dim3(num_sms()), dim3(kThreadsD), args, smem, stream);
}

}  // namespace tw
