// gemm_tc.cu -- persistent, warp-specialised tcgen05 GEMM for sm_100a with
// three fused epilogues:
//   * TwELL packing of g = ReLU(x Wg)   ("Sparser, Faster, Lighter Transformer
//     Language Models", technical summary, section 2.1: the sparse format is
//     produced directly in the matmul epilogue, staged in shared memory);
//   * h = ReLU(x Wg) * (x Wu) for the dense comparator (one GEMM over the
//     gate and up weights, both halves of a 256-wide tile);
//   * a plain bf16 store (the comparator's down projection).
//
// Pipeline (one CTA per SM, 192 threads):
//   warp 0      TMA producer: x and weight tiles -> 4-stage shared-memory ring
//               (128-byte swizzle, one mbarrier per stage, no multicast);
//   warp 1      allocates 512 TMEM columns (two 128x256 fp32 accumulators) and
//               issues tcgen05.mma (M=128, N=256, K=16) from one thread;
//   warps 2..5  epilogue: tcgen05.ld one TMEM lane (= one token row) per
//               thread, so the TwELL packing of a row is thread-local.
// The epilogue of tile i overlaps the main loop of tile i+1 (double-buffered
// accumulator).  The launch is a programmatic dependent launch: barrier and
// TMEM set-up overlap the previous kernel's tail.  Every wait is bounded: on timeout the CTA raises an abort
// flag, flags TW_ERR_TIMEOUT, drains its in-flight copies and MMAs, frees its
// TMEM and returns.
#include "tmap.h"
#include "pdl.cuh"
#include "tw_common.cuh"
#include "tw_internal.h"

namespace tw {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;  // 64 bf16 = 128 B = one swizzle atom row
constexpr int A_BYTES = BM * BK * 2;
constexpr int NUM_THREADS = 192;
constexpr int EPI_SLOTS = 32;  // TwELL slots per row staged in shared memory

// Tile widths: BN = 256 with a 4-stage ring, or BN = 128 with a 6-stage ring
// when there are too few 256-wide tiles to occupy every SM (small T).
template <int BN>
struct Shape {
  static constexpr int STAGES = BN == 256 ? 4 : 6;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = 2 * BN;  // two accumulators
};

// Per-thread staging of the TwELL epilogue.
struct EpiStage {
  alignas(16) uint16_t slot_val[128 * EPI_SLOTS];  // read back with 16-byte loads
  alignas(16) uint8_t slot_idx[128 * EPI_SLOTS];   // read back with 8-byte loads
};
static_assert(offsetof(EpiStage, slot_val) % 16 == 0 && offsetof(EpiStage, slot_idx) % 16 == 0,
              "epilogue staging must be 16-byte aligned");

template <int STAGES>
struct SmemTail {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int never;
  EpiStage epi;
};

template <int BN>
constexpr size_t smem_bytes() {
  return 1024 + (size_t)Shape<BN>::STAGES * Shape<BN>::STAGE_BYTES +
         sizeof(SmemTail<Shape<BN>::STAGES>);
}
static_assert(smem_bytes<256>() <= 227 * 1024 && smem_bytes<128>() <= 227 * 1024,
              "shared memory budget");

// ReLU on fp32 bits: negative numbers and -0 (sign bit set) become +0.
TW_DEV uint32_t relu_bits(uint32_t b) { return (int32_t)b > 0 ? b : 0u; }

// ------------------------------------------------------------ epilogues ----
// Operand layout flags every epilogue type carries:
//   kDualB  B tile = two halves from two weights (gate and up), BN = 256;
//   kAMN    A is MN-major: A[m][k] read from a [K][M] row-major tensor;
//   kBMN    B is MN-major: B[n][k] read from a [K][N] row-major tensor;
//   kDualK  the reduction runs over (A0, B0) and then (A1, B1), K/2 each.
struct OperandsKK {
  static constexpr bool kDualB = false, kAMN = false, kBMN = false, kDualK = false;
};

struct EpiTwell : OperandsKK {
  int T, F, W, C, spill_cap;  // W: TwELL tile width (64, 128 or 256; BN % W == 0)
  uint16_t* val;
  uint8_t* idx;
  uint8_t* cnt;
  int32_t* spill_ref;
  int32_t* spill_tk;
  uint16_t* spill_val;
  int32_t* spill_n;
  uint16_t* dump;
  int32_t* status;

  // taddr: TMEM address of this warp's lane block at column 0 of the tile;
  // the tile holds KT TwELL tiles of 128 columns.  Capacities up to
  // EPI_SLOTS are staged per thread in shared memory and stored with vector
  // stores; larger ones (up to the tile width) stage their first EPI_SLOTS
  // slots the same way and write the rest straight to global memory.
  template <int KT>
  TW_DEV void run(uint32_t taddr, int row, int nb, int ethread, EpiStage* st) const {
    if (C <= EPI_SLOTS) run_c<KT, false>(taddr, row, nb, ethread, st);
    else run_c<KT, true>(taddr, row, nb, ethread, st);
  }

  // Slot n (< C) of the packed row: staged, or (kWide, n >= EPI_SLOTS) direct.
  template <bool kWide>
  TW_DEV void put(uint16_t* sv, uint8_t* si, size_t kt_off, bool row_ok, int n, uint16_t v,
                  uint8_t j) const {
    if (!kWide || n < EPI_SLOTS) {
      sv[n] = v;
      si[n] = j;
    } else if (row_ok) {
      val[kt_off * C + n] = v;
      idx[kt_off * C + n] = j;
    }
  }

  template <int KT, bool kWide>
  TW_DEV void run_c(uint32_t taddr, int row, int nb, int ethread, EpiStage* st) const {
    const bool row_ok = row < T;
    const int K = F / W;
    const int ntile = KT * 128 / W;  // TwELL tiles in this accumulator tile
    const int nchunk = W / 32;       // 32-column TMEM loads per TwELL tile
    const int CS = kWide ? EPI_SLOTS : C;  // slots staged in shared memory
    uint16_t* sv = st->slot_val + ethread * EPI_SLOTS;
    uint8_t* si = st->slot_idx + ethread * EPI_SLOTS;
#pragma unroll 1
    for (int kt = 0; kt < ntile; ++kt) {
      const int k = nb * ntile + kt;
      if (k >= K) break;  // uniform across the CTA
      const size_t kt_off = (size_t)k * T + row;
      for (int s = 0; s < CS; ++s) {
        sv[s] = 0;
        si[s] = 0;
      }
      int n = 0;
#pragma unroll 1
      for (int c = 0; c < nchunk; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(taddr + kt * W + c * 32, r);
        tmem_ld_wait();
        uint32_t packed[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint32_t p = pack_bf16x2(__uint_as_float(relu_bits(r[2 * i])),
                                         __uint_as_float(relu_bits(r[2 * i + 1])));
          packed[i] = p;
          if (p != 0u) {
            if ((p & 0xFFFFu) != 0u) {
              if (n < C)
                put<kWide>(sv, si, kt_off, row_ok, n, (uint16_t)(p & 0xFFFFu),
                           (uint8_t)(c * 32 + 2 * i));
              ++n;
            }
            if ((p >> 16) != 0u) {
              if (n < C)
                put<kWide>(sv, si, kt_off, row_ok, n, (uint16_t)(p >> 16),
                           (uint8_t)(c * 32 + 2 * i + 1));
              ++n;
            }
          }
        }
        if (dump != nullptr && row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(dump + (size_t)row * F + (size_t)k * W + c * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
        }
      }
      if (row_ok) {
        // a full 256-wide tile has no uint8 count: stored as 255 and flagged
        if (n > 255) set_status(status, 1 << TW_ERR_UNSUPPORTED);
        cnt[kt_off] = (uint8_t)(n < 255 ? n : 255);
        if ((C & 7) == 0) {
          uint4* dv = reinterpret_cast<uint4*>(val + kt_off * C);
          uint2* di = reinterpret_cast<uint2*>(idx + kt_off * C);
          const uint4* svv = reinterpret_cast<const uint4*>(sv);
          const uint2* sii = reinterpret_cast<const uint2*>(si);
          for (int s = 0; s < CS / 8; ++s) {
            dv[s] = svv[s];
            di[s] = sii[s];
          }
        } else {
          for (int s = 0; s < CS; ++s) {
            val[kt_off * C + s] = sv[s];
            idx[kt_off * C + s] = si[s];
          }
        }
        if (kWide) {  // padding past the count beyond the staged slots
          for (int s = n > EPI_SLOTS ? n : EPI_SLOTS; s < C; ++s) {
            val[kt_off * C + s] = 0;
            idx[kt_off * C + s] = 0;
          }
        }
      }
      const bool spill = row_ok && n > C;
      if (__any_sync(0xFFFFFFFFu, spill)) {
        int slot = -1;
        if (spill) {
          slot = atomicAdd(spill_n, 1);
          if (slot < spill_cap) {
            spill_ref[(size_t)k * T + row] = slot;
            spill_tk[2 * (size_t)slot] = row;
            spill_tk[2 * (size_t)slot + 1] = k;
          } else {
            spill_ref[(size_t)k * T + row] = -1;
            set_status(status, kStatusSpill);
            slot = -1;
          }
        }
#pragma unroll 1
        for (int c = 0; c < nchunk; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(taddr + kt * W + c * 32, r);
          tmem_ld_wait();
          if (slot >= 0) {
            uint4* dst = reinterpret_cast<uint4*>(spill_val + (size_t)slot * W + c * 32);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e)
                w[e] = pack_bf16x2(__uint_as_float(relu_bits(r[8 * q + 2 * e])),
                                   __uint_as_float(relu_bits(r[8 * q + 2 * e + 1])));
              dst[q] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
      }
    }
  }
};

struct EpiGateUp {
  static constexpr bool kDualB = true, kAMN = false, kBMN = false, kDualK = false;
  int T, F;
  uint16_t* h;
  template <int KT>
  TW_DEV void run(uint32_t taddr, int row, int nb, int, EpiStage*) const {
    static_assert(KT == 2, "gate and up halves of a 256-wide tile");
    const bool row_ok = row < T;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t zr[32], ur[32];
      tmem_ld_32x32b_x32(taddr + c * 32, zr);
      tmem_ld_32x32b_x32(taddr + 128 + c * 32, ur);
      tmem_ld_wait();
      if (row_ok) {
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float h0 = __uint_as_float(relu_bits(zr[2 * i])) * __uint_as_float(ur[2 * i]);
          const float h1 =
              __uint_as_float(relu_bits(zr[2 * i + 1])) * __uint_as_float(ur[2 * i + 1]);
          w[i] = pack_bf16x2(h0, h1);
        }
        uint4* dst = reinterpret_cast<uint4*>(h + (size_t)row * F + (size_t)nb * 128 + c * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q) dst[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
      }
    }
  }
};

struct EpiStore : OperandsKK {
  int T, N;
  uint16_t* y;
  template <int KT>
  TW_DEV void run(uint32_t taddr, int row, int nb, int, EpiStage*) const {
    const bool row_ok = row < T;
#pragma unroll 1
    for (int c = 0; c < KT * 4; ++c) {
      const int col0 = nb * KT * 128 + c * 32;
      if (col0 >= N) break;  // uniform
      uint32_t r[32];
      tmem_ld_32x32b_x32(taddr + c * 32, r);
      tmem_ld_wait();
      if (row_ok) {
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          w[i] = pack_bf16x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
        uint4* dst = reinterpret_cast<uint4*>(y + (size_t)row * N + col0);
#pragma unroll
        for (int q = 0; q < 4; ++q) dst[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
      }
    }
  }
};

// Dense training comparator, forward: z = x Wg and u = x Wu in the two halves
// of a 256-wide tile; saves g = ReLU(z) and u (bf16, the activations the
// backward needs) and h = g u (bf16, the down projection's operand), all
// [T][F].  g is rounded to bf16 first, as the sparse path stores it.
struct EpiTrainGateUp {
  static constexpr bool kDualB = true, kAMN = false, kBMN = false, kDualK = false;
  int T, F;
  uint16_t* g;
  uint16_t* u;
  uint16_t* h;
  template <int KT>
  TW_DEV void run(uint32_t taddr, int row, int nb, int, EpiStage*) const {
    static_assert(KT == 2, "gate and up halves of a 256-wide tile");
    const bool row_ok = row < T;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t zr[32], ur[32];
      tmem_ld_32x32b_x32(taddr + c * 32, zr);
      tmem_ld_32x32b_x32(taddr + 128 + c * 32, ur);
      tmem_ld_wait();
      if (row_ok) {
        uint32_t wg[16], wu[16], wh[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          wg[i] = pack_bf16x2(__uint_as_float(relu_bits(zr[2 * i])),
                              __uint_as_float(relu_bits(zr[2 * i + 1])));
          wu[i] = pack_bf16x2(__uint_as_float(ur[2 * i]), __uint_as_float(ur[2 * i + 1]));
          wh[i] = pack_bf16x2(bf16_lo(wg[i]) * __uint_as_float(ur[2 * i]),
                              bf16_hi(wg[i]) * __uint_as_float(ur[2 * i + 1]));
        }
        const size_t off = (size_t)row * F + (size_t)nb * 128 + c * 32;
        uint4* dg = reinterpret_cast<uint4*>(g + off);
        uint4* du = reinterpret_cast<uint4*>(u + off);
        uint4* dh = reinterpret_cast<uint4*>(h + off);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          dg[q] = make_uint4(wg[4 * q], wg[4 * q + 1], wg[4 * q + 2], wg[4 * q + 3]);
          du[q] = make_uint4(wu[4 * q], wu[4 * q + 1], wu[4 * q + 2], wu[4 * q + 3]);
          dh[q] = make_uint4(wh[4 * q], wh[4 * q + 1], wh[4 * q + 2], wh[4 * q + 3]);
        }
      }
    }
  }
};

// Dense training comparator, backward through the gate: dh = dy Wd^T from
// TMEM; with the saved g and u, du = dh g and dz = (dh u + lambda) where
// g > 0 (ReLU'(0) = 0, and the L1 term's sign(g) is 1 on g > 0), both stored
// bf16 [T][F] as the operands of the dx and weight-gradient GEMMs.
struct EpiBwdGate : OperandsKK {
  int T, F;
  float lam;
  const uint16_t* g;
  const uint16_t* u;
  uint16_t* du;
  uint16_t* dz;
  template <int KT>
  TW_DEV void run(uint32_t taddr, int row, int nb, int, EpiStage*) const {
    const bool row_ok = row < T;
#pragma unroll 1
    for (int c = 0; c < KT * 4; ++c) {
      if (nb * KT * 128 + c * 32 >= F) break;  // uniform: a last tile past F
      uint32_t r[32];
      tmem_ld_32x32b_x32(taddr + c * 32, r);
      tmem_ld_wait();
      if (row_ok) {
        const size_t off = (size_t)row * F + (size_t)nb * KT * 128 + c * 32;
        const uint4* gp = reinterpret_cast<const uint4*>(g + off);
        const uint4* up = reinterpret_cast<const uint4*>(u + off);
        uint32_t gw[16], uw[16], wdu[16], wdz[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 a = gp[q], b = up[q];
          gw[4 * q] = a.x; gw[4 * q + 1] = a.y; gw[4 * q + 2] = a.z; gw[4 * q + 3] = a.w;
          uw[4 * q] = b.x; uw[4 * q + 1] = b.y; uw[4 * q + 2] = b.z; uw[4 * q + 3] = b.w;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float dh0 = __uint_as_float(r[2 * i]), dh1 = __uint_as_float(r[2 * i + 1]);
          const float g0 = bf16_lo(gw[i]), g1 = bf16_hi(gw[i]);
          const float u0 = bf16_lo(uw[i]), u1 = bf16_hi(uw[i]);
          wdu[i] = pack_bf16x2(dh0 * g0, dh1 * g1);
          wdz[i] = pack_bf16x2(g0 > 0.f ? fmaf(dh0, u0, lam) : 0.f,
                               g1 > 0.f ? fmaf(dh1, u1, lam) : 0.f);
        }
        uint4* pu = reinterpret_cast<uint4*>(du + off);
        uint4* pz = reinterpret_cast<uint4*>(dz + off);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          pu[q] = make_uint4(wdu[4 * q], wdu[4 * q + 1], wdu[4 * q + 2], wdu[4 * q + 3]);
          pz[q] = make_uint4(wdz[4 * q], wdz[4 * q + 1], wdz[4 * q + 2], wdz[4 * q + 3]);
        }
      }
    }
  }
};

// fp32 store of an [M][N] result (y and dx of the dense training FFN, and
// the weight gradients), with the operand layout as template flags.
template <bool AMN, bool BMN, bool DUALK>
struct EpiStoreF32 {
  static constexpr bool kDualB = false, kAMN = AMN, kBMN = BMN, kDualK = DUALK;
  int M, N;
  float* out;
  template <int KT>
  TW_DEV void run(uint32_t taddr, int row, int nb, int, EpiStage*) const {
    const bool row_ok = row < M;
#pragma unroll 1
    for (int c = 0; c < KT * 4; ++c) {
      const int col0 = nb * KT * 128 + c * 32;
      if (col0 >= N) break;  // uniform
      uint32_t r[32];
      tmem_ld_32x32b_x32(taddr + c * 32, r);
      tmem_ld_wait();
      if (row_ok) {
        float4* dst = reinterpret_cast<float4*>(out + (size_t)row * N + col0);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          dst[q] = make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                               __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
      }
    }
  }
};

// --------------------------------------------------------------- kernel ----
template <class Epi, int BN>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                   const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmA1,
                   int Kdim, int n_tiles_n,
                   int num_tiles, uint32_t a_bytes, const Epi epi, int32_t* status,
                   unsigned long long timeout_ns, int withhold_loads) {
  constexpr int STAGES = Shape<BN>::STAGES;
  constexpr int STAGE_BYTES = Shape<BN>::STAGE_BYTES;
  constexpr int B_BYTES = Shape<BN>::B_BYTES;
  constexpr int TMEM_COLS = Shape<BN>::TMEM_COLS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  auto* sm = reinterpret_cast<SmemTail<STAGES>*>(smem + (size_t)STAGES * STAGE_BYTES);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int kblocks = (Kdim + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sm->full[s], 1);
      mbar_init(&sm->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sm->tmem_full[a], 1);
      mbar_init(&sm->tmem_empty[a], 128);
    }
    mbar_init(&sm->drain, 1);
    sm->abort = 0;
    sm->never = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    if (Epi::kDualB || Epi::kDualK) tma_prefetch_desc(&tmB1);
    if (Epi::kDualK) tma_prefetch_desc(&tmA1);
  }
  if (warp == 1) {
    tmem_alloc(&sm->tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = sm->tmem_base;
  volatile int* abort = &sm->abort;
  // set-up above overlaps the previous kernel's tail (programmatic dependent
  // launch); its results are visible from here on
  pdl_wait();
  pdl_launch_next();

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------- TMA producer --
      uint32_t it = 0;
      bool ok = true;
      // withhold_loads (a test of the bounded waits): issue nothing and raise
      // nothing, so the MMA issuer's first wait can never complete and must
      // run out by its time limit
      for (int tile = blockIdx.x; tile < num_tiles && ok && !withhold_loads;
           tile += gridDim.x) {
        const int m_blk = tile / n_tiles_n;
        const int n_blk = tile % n_tiles_n;
        for (int kb = 0; kb < kblocks; ++kb) {
          const uint32_t s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait(&sm->empty[s], ph ^ 1u, abort, timeout_ns)) {
            ok = false;
            break;
          }
          uint8_t* a = smem + (size_t)s * STAGE_BYTES;
          uint8_t* b = a + A_BYTES;
          // the x box may be narrower than the 128-row tile (one small m-tile);
          // rows past it are stale and only reach output rows that are not stored
          mbar_arrive_expect_tx(&sm->full[s], a_bytes + B_BYTES);
          // dual K: the second half of the k-blocks reads (A1, B1)
          const bool second = Epi::kDualK && kb >= kblocks / 2;
          const CUtensorMap* ta = second ? &tmA1 : &tmA;
          const CUtensorMap* tb = second ? &tmB1 : &tmB0;
          const int kc = (second ? kb - kblocks / 2 : kb) * BK;
          if (Epi::kAMN) {  // two 64 x 64 boxes: rows are k, columns m
            tma_load_2d(a, ta, &sm->full[s], m_blk * BM, kc);
            tma_load_2d(a + A_BYTES / 2, ta, &sm->full[s], m_blk * BM + 64, kc);
          } else {
            tma_load_2d(a, ta, &sm->full[s], kc, m_blk * BM);
          }
          if (Epi::kDualB) {
            tma_load_2d(b, &tmB0, &sm->full[s], kc, n_blk * (BN / 2));
            tma_load_2d(b + B_BYTES / 2, &tmB1, &sm->full[s], kc, n_blk * (BN / 2));
          } else if (Epi::kBMN) {  // BN / 64 boxes of 64 x 64: rows are k, columns n
#pragma unroll
            for (int h = 0; h < BN / 64; ++h)
              tma_load_2d(b + h * (BK * 64 * 2), tb, &sm->full[s], n_blk * BN + h * 64, kc);
          } else {
            tma_load_2d(b, tb, &sm->full[s], kc, n_blk * BN);
          }
          ++it;
        }
      }
      if (!ok) {
        *abort = 1;
        set_status(status, kStatusTimeout);
        // Let the copies already issued land before the CTA can exit.
        const uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0u;
        for (uint32_t i = first; i < it; ++i)
          mbar_wait(&sm->full[i % STAGES], (i / STAGES) & 1u, &sm->never, kWaitTimeoutNs);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------ MMA issuer --
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, Epi::kAMN, Epi::kBMN);
      uint32_t it = 0, tl = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++tl) {
        const uint32_t acc = tl & 1u;
        const uint32_t aph = (tl >> 1) & 1u;
        if (!mbar_wait(&sm->tmem_empty[acc], aph ^ 1u, abort, timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < kblocks; ++kb) {
          const uint32_t s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait(&sm->full[s], ph, abort, timeout_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + (size_t)s * STAGE_BYTES);
          const uint32_t b_base = a_base + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            // K-major: the next 16 k start 32 B along the swizzled row; MN-major:
            // 16 k-rows (2048 B) further, the boxes of 64 MN-elements 8 KB apart
            const uint64_t ad = Epi::kAMN ? sdesc_mnmajor_sw128(a_base + kk * 2048, BK * 64 * 2)
                                          : sdesc_kmajor_sw128(a_base + kk * 32);
            const uint64_t bd = Epi::kBMN ? sdesc_mnmajor_sw128(b_base + kk * 2048, BK * 64 * 2)
                                          : sdesc_kmajor_sw128(b_base + kk * 32);
            umma_f16_ss(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&sm->empty[s]);
          ++it;
        }
        if (!ok) break;
        umma_commit(&sm->tmem_full[acc]);
      }
      if (!ok) {
        *abort = 1;
        set_status(status, kStatusTimeout);
      }
      // Every MMA this thread issued has completed once `drain` flips.
      umma_commit(&sm->drain);
      mbar_wait(&sm->drain, 0, &sm->never, kWaitTimeoutNs);
    }
  } else {
    // ------------------------------------------------------- epilogue -----
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int ethread = q * 32 + lane;
    uint32_t tl = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++tl) {
      const int m_blk = tile / n_tiles_n;
      const int n_blk = tile % n_tiles_n;
      const uint32_t acc = tl & 1u;
      const uint32_t ph = (tl >> 1) & 1u;
      bool ok = mbar_wait(&sm->tmem_full[acc], ph, abort, timeout_ns);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) {
        *abort = 1;
        if (lane == 0) set_status(status, kStatusTimeout);
        break;
      }
      tc_fence_after();
      const int row = m_blk * BM + q * 32 + lane;
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN;
      epi.template run<BN / 128>(taddr, row, n_blk, ethread, &sm->epi);
      tc_fence_before();
      mbar_arrive(&sm->tmem_empty[acc]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ----------------------------------------------------------------- host ----
// Row-major bf16 matrix [rows][cols]; boxes of 64 columns x box_rows rows.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  return make_tmap_bf16(m, base, rows, cols, BK, box_rows);
}

template <class Epi, int BN>
cudaError_t launch(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1, int Kdim,
                   int n_tiles_m, int n_tiles_n, const Epi& epi, int32_t* status,
                   cudaStream_t stream, uint32_t a_bytes = A_BYTES,
                   const CUtensorMap* a1 = nullptr, unsigned long long withheld_wait_ns = 0) {
  cudaError_t e = set_smem_limit(reinterpret_cast<const void*>(gemm_tc_kernel<Epi, BN>),
                                 (int)smem_bytes<BN>());
  if (e != cudaSuccess) return e;
  const int num_tiles = n_tiles_m * n_tiles_n;
  if (num_tiles == 0) return cudaSuccess;
  const int grid = num_tiles < num_sms() ? num_tiles : num_sms();
  return launch_pdl(gemm_tc_kernel<Epi, BN>, dim3(grid), dim3(NUM_THREADS), smem_bytes<BN>(),
                    stream, a, b0, b1, a1 ? *a1 : a, Kdim, n_tiles_n, num_tiles, a_bytes, epi,
                    status, withheld_wait_ns ? withheld_wait_ns : kWaitTimeoutNs,
                    withheld_wait_ns ? 1 : 0);
}

}  // namespace

cudaError_t launch_gate_twell_tc(const void* x, const void* Wg_t, int T, int d, int F,
                                 const tw_twell& out, void* dump, int32_t* status,
                                 cudaStream_t stream) {
  // 128-wide tiles when 256-wide ones would leave SMs idle (small T); a
  // 256-wide TwELL tile needs the 256-wide accumulator
  const int m_tiles = (T + BM - 1) / BM;
  const bool narrow = out.W <= 128 && (long long)m_tiles * ((F + 255) / 256) < num_sms();
  // with a single m-tile, load only the x rows that exist (rounded up to 16)
  const uint32_t a_rows = T < BM ? (uint32_t)((T + 15) / 16 * 16) : (uint32_t)BM;
  CUtensorMap ma, mb;
  if (!make_map(&ma, x, T, d, a_rows) || !make_map(&mb, Wg_t, F, d, narrow ? 128 : 256))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaMemsetAsync(out.spill_n, 0, sizeof(int32_t), stream);
  if (e != cudaSuccess) return e;
  EpiTwell epi;
  epi.T = T;
  epi.F = F;
  epi.W = out.W;
  epi.C = out.C;
  epi.spill_cap = out.spill_cap;
  epi.val = static_cast<uint16_t*>(out.val);
  epi.idx = out.idx;
  epi.cnt = out.cnt;
  epi.spill_ref = out.spill_ref;
  epi.spill_tk = out.spill_tk;
  epi.spill_val = static_cast<uint16_t*>(out.spill_val);
  epi.spill_n = out.spill_n;
  epi.dump = static_cast<uint16_t*>(dump);
  epi.status = status;
  const uint32_t a_bytes = a_rows * BK * 2;
  const unsigned long long withheld = take_withheld_gate_wait();
  return narrow ? launch<EpiTwell, 128>(ma, mb, mb, d, m_tiles, F / 128, epi, status, stream,
                                        a_bytes, nullptr, withheld)
                : launch<EpiTwell, 256>(ma, mb, mb, d, m_tiles, (F + 255) / 256, epi, status,
                                        stream, a_bytes, nullptr, withheld);
}

cudaError_t launch_dense_gateup_tc(const void* x, const void* Wg_t, const void* Wu_t, int T,
                                   int d, int F, void* h, int32_t* status, cudaStream_t stream) {
  CUtensorMap ma, mg, mu;
  if (!make_map(&ma, x, T, d, BM) || !make_map(&mg, Wg_t, F, d, 128) ||
      !make_map(&mu, Wu_t, F, d, 128))
    return cudaErrorInvalidValue;
  EpiGateUp epi;
  epi.T = T;
  epi.F = F;
  epi.h = static_cast<uint16_t*>(h);
  return launch<EpiGateUp, 256>(ma, mg, mu, d, (T + BM - 1) / BM, F / 128, epi, status, stream);
}

cudaError_t launch_dense_down_tc(const void* h, const void* Wd_dense, int T, int d, int F,
                                 void* y, int32_t* status, cudaStream_t stream) {
  CUtensorMap ma, mb;
  if (!make_map(&ma, h, T, F, BM) || !make_map(&mb, Wd_dense, d, F, 256))
    return cudaErrorInvalidValue;
  EpiStore epi;
  epi.T = T;
  epi.N = d;
  epi.y = static_cast<uint16_t*>(y);
  return launch<EpiStore, 256>(ma, mb, mb, F, (T + BM - 1) / BM, (d + 255) / 256, epi, status,
                               stream);
}

namespace {

// MN-major operand map: a [K][MN] row-major bf16 tensor in 64 x 64 boxes.
bool make_map_mn(CUtensorMap* m, const void* base, uint64_t k_rows, uint64_t mn_cols) {
  return make_tmap_bf16(m, base, k_rows, mn_cols, 64, 64);
}

}  // namespace

// Dense training comparator, forward: g, u, h saved in ws; y = h Wd (fp32).
cudaError_t launch_dense_train_forward(const void* x, const void* Wg_t, const void* Wu_t,
                                       const void* Wd, int T, int d, int F, uint16_t* g,
                                       uint16_t* u, uint16_t* h, float* y, int32_t* status,
                                       cudaStream_t stream) {
  const int m_tiles = (T + BM - 1) / BM;
  CUtensorMap mx, mg, mu, mh, mwd;
  if (!make_map(&mx, x, T, d, BM) || !make_map(&mg, Wg_t, F, d, 128) ||
      !make_map(&mu, Wu_t, F, d, 128) || !make_map(&mh, h, T, F, BM) ||
      !make_map_mn(&mwd, Wd, F, d))
    return cudaErrorInvalidValue;
  EpiTrainGateUp e1;
  e1.T = T;
  e1.F = F;
  e1.g = g;
  e1.u = u;
  e1.h = h;
  cudaError_t e = launch<EpiTrainGateUp, 256>(mx, mg, mu, d, m_tiles, F / 128, e1, status, stream);
  if (e != cudaSuccess) return e;
  EpiStoreF32<false, true, false> e2;  // y[t][i] = sum_j h[t][j] Wd[j][i]
  e2.M = T;
  e2.N = d;
  e2.out = y;
  return launch<EpiStoreF32<false, true, false>, 256>(mh, mwd, mwd, F, m_tiles, (d + 255) / 256,
                                                      e2, status, stream);
}

// Dense training comparator, backward: du, dz in ws; dx (fp32) and the three
// weight gradients (fp32, [F][d]).
cudaError_t launch_dense_train_backward(const void* x, const void* dy, const void* Wg_t,
                                        const void* Wu_t, const void* Wd, int T, int d, int F,
                                        float lam, const uint16_t* g, const uint16_t* u,
                                        const uint16_t* h, uint16_t* du, uint16_t* dz, float* dx,
                                        float* dWg_t, float* dWu_t, float* dWd, int32_t* status,
                                        cudaStream_t stream) {
  const int m_tiles = (T + BM - 1) / BM;
  const int d_tiles = (d + 255) / 256;
  CUtensorMap mdy, mwd_k, mdu, mdz, mwu_mn, mwg_mn, mh_mn, mdu_mn, mdz_mn, mdy_mn, mx_mn;
  if (!make_map(&mdy, dy, T, d, BM) || !make_map(&mwd_k, Wd, F, d, 256) ||
      !make_map(&mdu, du, T, F, BM) || !make_map(&mdz, dz, T, F, BM) ||
      !make_map_mn(&mwu_mn, Wu_t, F, d) || !make_map_mn(&mwg_mn, Wg_t, F, d) ||
      !make_map_mn(&mh_mn, h, T, F) || !make_map_mn(&mdu_mn, du, T, F) ||
      !make_map_mn(&mdz_mn, dz, T, F) || !make_map_mn(&mdy_mn, dy, T, d) ||
      !make_map_mn(&mx_mn, x, T, d))
    return cudaErrorInvalidValue;
  // dh = dy Wd^T, then du and dz in the epilogue
  EpiBwdGate e1;
  e1.T = T;
  e1.F = F;
  e1.lam = lam;
  e1.g = g;
  e1.u = u;
  e1.du = du;
  e1.dz = dz;
  cudaError_t e =
      launch<EpiBwdGate, 256>(mdy, mwd_k, mwd_k, d, m_tiles, (F + 255) / 256, e1, status, stream);
  if (e != cudaSuccess) return e;
  // dx = du Wu_t + dz Wg_t: one accumulator over K = 2F
  EpiStoreF32<false, true, true> e2;
  e2.M = T;
  e2.N = d;
  e2.out = dx;
  e = launch<EpiStoreF32<false, true, true>, 256>(mdu, mwu_mn, mwg_mn, 2 * F, m_tiles, d_tiles, e2,
                                                  status, stream, A_BYTES, &mdz);
  if (e != cudaSuccess) return e;
  // weight gradients over K = T: dWd = h^T dy, dWu_t = du^T x, dWg_t = dz^T x
  const int f_tiles = F / BM;
  EpiStoreF32<true, true, false> e3;
  e3.M = F;
  e3.N = d;
  e3.out = dWd;
  e = launch<EpiStoreF32<true, true, false>, 256>(mh_mn, mdy_mn, mdy_mn, T, f_tiles, d_tiles, e3,
                                                  status, stream);
  if (e != cudaSuccess) return e;
  e3.out = dWu_t;
  e = launch<EpiStoreF32<true, true, false>, 256>(mdu_mn, mx_mn, mx_mn, T, f_tiles, d_tiles, e3,
                                                  status, stream);
  if (e != cudaSuccess) return e;
  e3.out = dWg_t;
  return launch<EpiStoreF32<true, true, false>, 256>(mdz_mn, mx_mn, mx_mn, T, f_tiles, d_tiles,
                                                     e3, status, stream);
}

}  // namespace tw
