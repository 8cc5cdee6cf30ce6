// gate_few.cu -- the gate GEMM with its TwELL epilogue for small batches
// (T <= kFewMaxT tokens), on tcgen05 with the operand roles swapped.
//
// With few tokens the gate is a matrix-vector product bound by streaming Wg
// (d x F bf16) from HBM ("Sparser, Faster, Lighter Transformer Language
// Models", technical summary, section 2.1, for what the epilogue produces).
// The tile GEMM of gemm_tc.cu puts 128 tokens on the MMA's M side; here a
// 128-unit tile of Wg_t is the M side and the T tokens, rounded up to 16, are
// the N side, so the tensor core spends nothing on absent token rows.
//
// F/128 unit tiles alone do not occupy the SMs (64 tiles at F = 8192), so the
// reduction over d is split across a thread-block cluster of S CTAs.  Each
// rank streams its share of the 64-column k-blocks through a TMA ring into
// its own TMEM accumulator; ranks 1..S-1 then write their fp32 partials into
// rank 0's shared memory (distributed shared memory) and arrive on a rank-0
// mbarrier, and rank 0 adds them in rank order, so the result does not depend
// on timing.  Rank 0 then applies ReLU, rounds to bf16 and packs TwELL.
//
// In this layout a TMEM lane is a unit and a column is a token.  Rank 0
// stages the bf16 g of 16 tokens in shared memory; then each epilogue warp
// packs whole tokens: four ballots over the tile's 128 units and a prefix
// count put the k-th non-zero in ascending unit order in slot k, slots past
// the count are zero, and a tile with more than C non-zeros spills all 128
// values, as the tile GEMM's epilogue does (one spill-slot atomic per warp
// and chunk).
//
// Roles (192 threads): warp 0 lane 0 issues TMA, warp 1 allocates TMEM and
// lane 0 issues the MMAs, warps 2..5 read TMEM (warp w owns lanes 32*(w%4)..).
// Every mbarrier wait is bounded; the two cluster barriers (after set-up and
// before exit) are reached by every thread after bounded work only.
#include "tmap.h"
#include "tw_common.cuh"
#include "tw_internal.h"

namespace tw {
namespace {

constexpr int kBK = 64;                    // bf16 columns per k-block (one 128-B swizzle row)
constexpr int kUnits = 128;                // units per tile (MMA M)
constexpr int kWBytes = kUnits * kBK * 2;  // Wg_t tile bytes per stage
constexpr int kMaxStages = 16;
constexpr int kThreads = 192;
constexpr int kMaxCluster = 8;                 // portable cluster size
constexpr size_t kPartMax = 64 * 1024;         // partial-sum buffers on rank 0
constexpr size_t kSmemMax = 227 * 1024;

struct FewTail {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t mma_done;
  uint64_t red_full;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int never;
  uint16_t g[16][kUnits];  // g of the current 16 tokens
};

struct FewOut {
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
};

struct FewShape {
  int N;            // tokens rounded up to 16 (MMA N, x box rows)
  int kblocks;      // ceil(d / 64)
  int stages;       // ring depth
  int stage_bytes;  // kWBytes + N * 128
  uint32_t tmem_cols;
  unsigned long long timeout_ns;
};

// 32 lanes x 16 consecutive 32-bit columns of tensor memory -> 16 registers
// per thread (thread i of the warp gets lane base+i).  Warp-collective.
TW_DEV void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
TW_DEV uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
TW_DEV uint32_t cluster_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
// All threads of all CTAs of the cluster; orders shared-memory writes
// (including mbarrier initialisation) before the other CTAs' later accesses.
TW_DEV void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
// Address of the same shared-memory offset in CTA `rank` of this cluster.
TW_DEV uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
TW_DEV void st_cluster_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
TW_DEV void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
// Bounded wait whose completion acquires at cluster scope (remote arrivals).
TW_DEV bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, volatile int* abort,
                              uint64_t timeout_ns) {
  uint64_t t0 = 0;
  for (uint32_t i = 0;; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(20000u)
        : "memory");
    if (ok) return true;
    if ((i & 31u) == 31u) {
      if (*abort) return false;
      const uint64_t now = globaltimer_ns();
      if (t0 == 0) t0 = now;
      else if (now - t0 > timeout_ns) return false;
    }
  }
}
TW_DEV void epi_bar(int id) { asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory"); }

__global__ void __launch_bounds__(kThreads, 1)
    gate_few_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                    const FewShape sh, const FewOut out) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  // 1024-byte aligned ring (128-byte swizzle atoms).  The offset is applied to
  // the shared array itself, so every pointer below stays a shared-space
  // pointer to the compiler (shared loads and stores, not generic ones).
  uint8_t* ring = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t S = cluster_size();
  const uint32_t rank = cluster_rank();
  float* part = reinterpret_cast<float*>(ring + (size_t)sh.stages * sh.stage_bytes);
  auto* tl = reinterpret_cast<FewTail*>(reinterpret_cast<uint8_t*>(part) +
                                        (size_t)(S - 1) * sh.N * kUnits * sizeof(float));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int k = blockIdx.x / S;  // unit tile
  const int kb0 = (int)(rank * sh.kblocks / S);
  const int kb1 = (int)((rank + 1) * sh.kblocks / S);

  if (threadIdx.x == 0) {
    for (int s = 0; s < sh.stages; ++s) {
      mbar_init(&tl->full[s], 1);
      mbar_init(&tl->empty[s], 1);
    }
    mbar_init(&tl->mma_done, 1);
    mbar_init(&tl->red_full, S > 1 ? (S - 1) * 128 : 1);  // used only when S > 1
    mbar_init(&tl->drain, 1);
    tl->abort = 0;
    tl->never = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(&tl->tmem_base, sh.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (S > 1) cluster_sync();  // rank 0's barriers are initialised before remote arrivals
  const uint32_t tmem_base = tl->tmem_base;
  volatile int* abort = &tl->abort;
  int32_t* status = out.status;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ TMA producer --
      uint32_t it = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb, ++it) {
        const uint32_t s = it % sh.stages;
        const uint32_t ph = (it / sh.stages) & 1u;
        if (!mbar_wait(&tl->empty[s], ph ^ 1u, abort, sh.timeout_ns)) {
          ok = false;
          break;
        }
        uint8_t* w = ring + (size_t)s * sh.stage_bytes;
        mbar_arrive_expect_tx(&tl->full[s], (uint32_t)sh.stage_bytes);
        tma_load_2d(w, &tmW, &tl->full[s], kb * kBK, k * kUnits);
        tma_load_2d(w + kWBytes, &tmX, &tl->full[s], kb * kBK, 0);
      }
      if (!ok) {
        *abort = 1;
        set_status(status, kStatusTimeout);
        const uint32_t first = it > (uint32_t)sh.stages ? it - sh.stages : 0u;
        for (uint32_t i = first; i < it; ++i)
          mbar_wait(&tl->full[i % sh.stages], (i / sh.stages) & 1u, &tl->never, sh.timeout_ns);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // -------------------------------------------------------- MMA issuer --
      const uint32_t idesc = idesc_bf16_f32(kUnits, sh.N);
      uint32_t it = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb, ++it) {
        const uint32_t s = it % sh.stages;
        const uint32_t ph = (it / sh.stages) & 1u;
        if (!mbar_wait(&tl->full[s], ph, abort, sh.timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_base = smem_u32(ring + (size_t)s * sh.stage_bytes);
        const uint32_t b_base = a_base + kWBytes;
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk)
          umma_f16_ss(tmem_base, sdesc_kmajor_sw128(a_base + kk * 32),
                      sdesc_kmajor_sw128(b_base + kk * 32), idesc, (it | kk) != 0 ? 1u : 0u);
        umma_commit(&tl->empty[s]);
      }
      if (ok) {
        umma_commit(&tl->mma_done);
      } else {
        *abort = 1;
        set_status(status, kStatusTimeout);
      }
      umma_commit(&tl->drain);
      mbar_wait(&tl->drain, 0, &tl->never, sh.timeout_ns);
    }
  } else {
    // ---------------------------------------------------------- epilogue --
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int u = q * 32 + lane;
    const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16);
    bool ok = mbar_wait(&tl->mma_done, 0, abort, sh.timeout_ns);
    ok = __all_sync(0xFFFFFFFFu, ok);
    if (ok) tc_fence_after();
    if (rank != 0) {
      if (ok) {
        // partial [t][u] into rank 0's buffer for this rank
        const uint32_t dst = map_to_rank(smem_u32(part), 0) +
                             (uint32_t)(((rank - 1) * sh.N * kUnits + u) * sizeof(float));
        for (int t0 = 0; t0 < sh.N; t0 += 16) {
          uint32_t r[16];
          tmem_ld_32x32b_x16(taddr + t0, r);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i)
            st_cluster_u32(dst + (uint32_t)((t0 + i) * kUnits * sizeof(float)), r[i]);
        }
        mbar_arrive_remote(map_to_rank(smem_u32(&tl->red_full), 0));
      } else {
        *abort = 1;
        if (lane == 0) set_status(status, kStatusTimeout);
      }
    } else {
      if (ok && S > 1) {
        ok = mbar_wait_cluster(&tl->red_full, 0, abort, sh.timeout_ns);
        ok = __all_sync(0xFFFFFFFFu, ok);
      }
      if (!ok) {
        *abort = 1;
        if (lane == 0) set_status(status, kStatusTimeout);
      } else {
        const int T = out.T, C = out.C;
        const uint32_t lt = (1u << lane) - 1u;
        for (int t0 = 0; t0 < T; t0 += 16) {
          // g of 16 tokens (thread = unit): ReLU of the rank-ordered sum,
          // rounded to bf16, staged in shared memory
          uint32_t r[16];
          tmem_ld_32x32b_x16(taddr + t0, r);
          tmem_ld_wait();
          float z[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) z[i] = __uint_as_float(r[i]);
          // the ranks' partials, in rank order; the 16 loads of a rank are
          // issued together (one shared-memory latency per rank, not per token)
          for (uint32_t p = 1; p < S; ++p) {
            const float* src = part + ((size_t)(p - 1) * sh.N + t0) * kUnits + u;
            float v[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = src[i * kUnits];
#pragma unroll
            for (int i = 0; i < 16; ++i) z[i] += v[i];
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float zr = (int32_t)__float_as_uint(z[i]) > 0 ? z[i] : 0.0f;  // ReLU, -0 -> +0
            tl->g[i][u] = f32_to_bf16(zr);
          }
          epi_bar(1);
          // packing (warp = token): warp q takes tokens q, q+4, q+8, q+12 of
          // the chunk; lane l holds units l, l+32, l+64, l+96
          uint16_t gv[4][4];
          uint32_t bal[4][4];
          int n[4];
          bool sp[4];
#pragma unroll
          for (int a = 0; a < 4; ++a) {
            const int i = q + 4 * a;
            n[a] = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              gv[a][j] = tl->g[i][lane + 32 * j];
              bal[a][j] = __ballot_sync(0xFFFFFFFFu, gv[a][j] != 0);
              n[a] += __popc(bal[a][j]);
            }
            sp[a] = t0 + i < T && n[a] > C;
          }
          // spill slots for this warp's overflowing tiles: one atomic
          const int nsp = (int)sp[0] + (int)sp[1] + (int)sp[2] + (int)sp[3];
          int base = 0;
          if (nsp > 0 && lane == 0) base = atomicAdd(out.spill_n, nsp);
          base = __shfl_sync(0xFFFFFFFFu, base, 0);
#pragma unroll
          for (int a = 0; a < 4; ++a) {
            const int t = t0 + q + 4 * a;
            if (t >= T) break;  // uniform across the warp
            const size_t off = (size_t)k * T + t;
            int before = 0;  // non-zeros in the unit blocks below block j
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int pos = before + __popc(bal[a][j] & lt);
              if (gv[a][j] != 0 && pos < C) {
                out.val[off * C + pos] = gv[a][j];
                out.idx[off * C + pos] = (uint8_t)(lane + 32 * j);
              }
              before += __popc(bal[a][j]);
            }
            for (int sl = lane; sl < C; sl += 32) {  // padding past the count
              if (sl >= n[a]) {
                out.val[off * C + sl] = 0;
                out.idx[off * C + sl] = 0;
              }
            }
            if (lane == 0) out.cnt[off] = (uint8_t)n[a];
            if (out.dump != nullptr) {
#pragma unroll
              for (int j = 0; j < 4; ++j)
                out.dump[(size_t)t * out.F + (size_t)k * kUnits + lane + 32 * j] = gv[a][j];
            }
            if (sp[a]) {  // uniform across the warp
              int slot = base;
              base += 1;
              if (slot < out.spill_cap) {
                if (lane == 0) {
                  out.spill_ref[off] = slot;
                  out.spill_tk[2 * (size_t)slot] = t;
                  out.spill_tk[2 * (size_t)slot + 1] = k;
                }
#pragma unroll
                for (int j = 0; j < 4; ++j)
                  out.spill_val[(size_t)slot * kUnits + lane + 32 * j] = gv[a][j];
              } else if (lane == 0) {
                out.spill_ref[off] = -1;
                set_status(status, kStatusSpill);
              }
            }
          }
          epi_bar(1);  // g is rewritten by the next chunk
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, sh.tmem_cols);
  }
  // rank 0's shared memory stays live until every rank has finished with it
  if (S > 1) cluster_sync();
}

}  // namespace

cudaError_t launch_gate_twell_few(const void* x, const void* Wg_t, int T, int d, int F,
                                  const tw_twell& out, void* dump, int32_t* status,
                                  cudaStream_t stream) {
  if (T < 1 || T > kFewMaxT) return cudaErrorInvalidValue;
  FewShape sh;
  sh.N = (T + 15) / 16 * 16;
  sh.kblocks = (d + kBK - 1) / kBK;
  sh.stage_bytes = kWBytes + sh.N * kBK * 2;
  sh.tmem_cols = sh.N <= 32 ? 32u : sh.N <= 64 ? 64u : 128u;
  sh.timeout_ns = kWaitTimeoutNs;
  const int K = F / kUnits;
  // the widest split that keeps one CTA per SM, at least one k-block per
  // rank, and rank 0's partial buffers within kPartMax
  int S = 1;
  for (int s = 2; s <= kMaxCluster; s *= 2)
    if ((long long)K * s <= num_sms() && s <= sh.kblocks &&
        (size_t)(s - 1) * sh.N * kUnits * sizeof(float) <= kPartMax)
      S = s;
  const size_t fixed = 1024 + (size_t)(S - 1) * sh.N * kUnits * sizeof(float) + sizeof(FewTail);
  int stages = (int)((kSmemMax - fixed) / sh.stage_bytes);
  const int per_rank = (sh.kblocks + S - 1) / S;
  stages = stages < kMaxStages ? stages : kMaxStages;
  stages = stages < per_rank ? stages : per_rank;
  if (stages < 1) return cudaErrorInvalidValue;
  sh.stages = stages;
  const size_t smem = fixed + (size_t)stages * sh.stage_bytes;

  cudaError_t e =
      set_smem_limit(reinterpret_cast<const void*>(gate_few_kernel), (int)kSmemMax);
  if (e != cudaSuccess) return e;
  CUtensorMap mw, mx;
  if (!make_tmap_bf16(&mw, Wg_t, F, d, kBK, kUnits) || !make_tmap_bf16(&mx, x, T, d, kBK, sh.N))
    return cudaErrorInvalidValue;
  e = cudaMemsetAsync(out.spill_n, 0, sizeof(int32_t), stream);
  if (e != cudaSuccess) return e;

  FewOut o;
  o.T = T;
  o.F = F;
  o.C = out.C;
  o.spill_cap = out.spill_cap;
  o.val = static_cast<uint16_t*>(out.val);
  o.idx = out.idx;
  o.cnt = out.cnt;
  o.spill_ref = out.spill_ref;
  o.spill_tk = out.spill_tk;
  o.spill_val = static_cast<uint16_t*>(out.spill_val);
  o.spill_n = out.spill_n;
  o.dump = static_cast<uint16_t*>(dump);
  o.status = status;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(K * S));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gate_few_kernel, mw, mx, sh, o);
}

}  // namespace tw
