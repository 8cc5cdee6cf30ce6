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
// accumulator).  Every wait is bounded: on timeout the CTA raises an abort
// flag, flags TW_ERR_TIMEOUT, drains its in-flight copies and MMAs, frees its
// TMEM and returns.
#include "tmap.h"
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
struct EpiTwell {
  static constexpr bool kDualB = false;
  int T, F, C, spill_cap;
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
    const int K = F / 128;
    const int CS = kWide ? EPI_SLOTS : C;  // slots staged in shared memory
    uint16_t* sv = st->slot_val + ethread * EPI_SLOTS;
    uint8_t* si = st->slot_idx + ethread * EPI_SLOTS;
#pragma unroll 1
    for (int kt = 0; kt < KT; ++kt) {
      const int k = nb * KT + kt;
      if (k >= K) break;  // uniform across the CTA
      const size_t kt_off = (size_t)k * T + row;
      for (int s = 0; s < CS; ++s) {
        sv[s] = 0;
        si[s] = 0;
      }
      int n = 0;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(taddr + kt * 128 + c * 32, r);
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
          uint4* dst = reinterpret_cast<uint4*>(dump + (size_t)row * F + (size_t)k * 128 + c * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
        }
      }
      if (row_ok) {
        cnt[kt_off] = (uint8_t)n;
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
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(taddr + kt * 128 + c * 32, r);
          tmem_ld_wait();
          if (slot >= 0) {
            uint4* dst = reinterpret_cast<uint4*>(spill_val + (size_t)slot * 128 + c * 32);
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
  static constexpr bool kDualB = true;
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

struct EpiStore {
  static constexpr bool kDualB = false;
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

// --------------------------------------------------------------- kernel ----
template <class Epi, int BN>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                   const __grid_constant__ CUtensorMap tmB1, int Kdim, int n_tiles_n,
                   int num_tiles, uint32_t a_bytes, const Epi epi, int32_t* status,
                   unsigned long long timeout_ns) {
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
    if (Epi::kDualB) tma_prefetch_desc(&tmB1);
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

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------- TMA producer --
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
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
          tma_load_2d(a, &tmA, &sm->full[s], kb * BK, m_blk * BM);
          if (Epi::kDualB) {
            tma_load_2d(b, &tmB0, &sm->full[s], kb * BK, n_blk * (BN / 2));
            tma_load_2d(b + B_BYTES / 2, &tmB1, &sm->full[s], kb * BK, n_blk * (BN / 2));
          } else {
            tma_load_2d(b, &tmB0, &sm->full[s], kb * BK, n_blk * BN);
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
          mbar_wait(&sm->full[i % STAGES], (i / STAGES) & 1u, &sm->never, timeout_ns);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------ MMA issuer --
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN);
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
            umma_f16_ss(d_tmem, sdesc_kmajor_sw128(a_base + kk * 32),
                        sdesc_kmajor_sw128(b_base + kk * 32), idesc, (kb | kk) != 0 ? 1u : 0u);
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
      mbar_wait(&sm->drain, 0, &sm->never, timeout_ns);
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
                   cudaStream_t stream, uint32_t a_bytes = A_BYTES) {
  cudaError_t e = set_smem_limit(reinterpret_cast<const void*>(gemm_tc_kernel<Epi, BN>),
                                 (int)smem_bytes<BN>());
  if (e != cudaSuccess) return e;
  const int num_tiles = n_tiles_m * n_tiles_n;
  if (num_tiles == 0) return cudaSuccess;
  const int grid = num_tiles < num_sms() ? num_tiles : num_sms();
  gemm_tc_kernel<Epi, BN><<<grid, NUM_THREADS, smem_bytes<BN>(), stream>>>(
      a, b0, b1, Kdim, n_tiles_n, num_tiles, a_bytes, epi, status, kWaitTimeoutNs);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gate_twell_tc(const void* x, const void* Wg_t, int T, int d, int F,
                                 const tw_twell& out, void* dump, int32_t* status,
                                 cudaStream_t stream) {
  // 128-wide tiles when 256-wide ones would leave SMs idle (small T)
  const int m_tiles = (T + BM - 1) / BM;
  const bool narrow = (long long)m_tiles * ((F + 255) / 256) < num_sms();
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
  return narrow ? launch<EpiTwell, 128>(ma, mb, mb, d, m_tiles, F / 128, epi, status, stream,
                                        a_bytes)
                : launch<EpiTwell, 256>(ma, mb, mb, d, m_tiles, (F + 255) / 256, epi, status,
                                        stream, a_bytes);
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

}  // namespace tw
