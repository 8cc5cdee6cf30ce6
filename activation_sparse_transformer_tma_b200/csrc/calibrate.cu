// calibrate.cu -- measurement aids, not part of the FFN.
//
// Row gather: the rate at which the SMs pull whole rows of a bf16 matrix in
// scattered order with 16-byte vector loads, the access pattern of the fused
// up + down projection ("Sparser, Faster, Lighter Transformer Language
// Models", technical summary, section 2.2: the weights of the active units
// only are loaded).  Timed on a matrix that stays in L2, it is the
// gathered-row term of that kernel's roofline.
//
// Stream read: one launch that reads a buffer once, front to back, with
// 16-byte loads (eight in flight per thread, two CTAs of 512 threads per
// SM).  Timed cold on the bytes of a small-batch step (Wg, 33.5 MB at the
// 2B shape), it is what a launch that only streams those bytes takes, launch
// and ramp included: the floor for the gate of a few tokens.
//
// Row i is splitmix64((seed << 32) ^ i) mod rows.  splitmix64 is the
// counter-based generator of Steele, Lea and Flood ("Fast splittable
// pseudorandom number generators", OOPSLA 2014); a test restates it on the
// host.  The XOR of every 32-bit word read goes to one device word, so the
// loads cannot be dropped and the result does not depend on their order.
#include "tw_common.cuh"
#include "tw_internal.h"

namespace tw {
namespace {

constexpr int kWarpsG = 16;
constexpr int kChunksMax = 2048 / 256;  // 16-byte chunks per lane of a row (d <= 2048)

TW_DEV uint64_t splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Each warp takes gathers w, w + W, ... (W warps in all), two rows at a time
// in flight; lane l reads the 16-byte chunks l, l + 32, ... of a row.
__global__ void __launch_bounds__(32 * kWarpsG, 1)
    row_gather_kernel(const uint4* __restrict__ mat, int rows, int chunks, long long n,
                      unsigned seed, uint32_t* checksum) {
  const int lane = threadIdx.x & 31;
  const long long gw = (long long)blockIdx.x * kWarpsG + (threadIdx.x >> 5);
  const long long nw = (long long)gridDim.x * kWarpsG;
  const uint64_t base = (uint64_t)seed << 32;
  uint32_t acc = 0;
  for (long long i0 = 2 * gw; i0 < n; i0 += 2 * nw) {
    uint4 v[2][kChunksMax];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const long long i = i0 + r;
      const bool ok = i < n;
      const long long row = ok ? (long long)(splitmix64(base ^ (uint64_t)i) % (uint64_t)rows) : 0;
      const uint4* p = mat + row * chunks;
#pragma unroll
      for (int c = 0; c < kChunksMax; ++c) {
        const int ch = c * 32 + lane;
        v[r][c] = ok && ch < chunks ? __ldg(p + ch) : make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int c = 0; c < kChunksMax; ++c) acc ^= v[r][c].x ^ v[r][c].y ^ v[r][c].z ^ v[r][c].w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xFFFFFFFFu, acc, o);
  if (lane == 0) atomicXor(checksum, acc);
}

constexpr int kStreamThreads = 512;
constexpr int kStreamUnroll = 8;

// Grid-stride over the 16-byte chunks, kStreamUnroll loads in flight per
// thread; the XOR of every word goes to one device word, one atomic per CTA.
__global__ void __launch_bounds__(kStreamThreads)
    stream_read_kernel(const uint4* __restrict__ p, long long n16, uint32_t* checksum) {
  __shared__ uint32_t wx[kStreamThreads / 32];
  const long long stride = (long long)gridDim.x * kStreamThreads;
  long long i = (long long)blockIdx.x * kStreamThreads + threadIdx.x;
  uint32_t acc = 0;
  for (; i + (kStreamUnroll - 1) * stride < n16; i += kStreamUnroll * stride) {
    uint4 v[kStreamUnroll];
#pragma unroll
    for (int u = 0; u < kStreamUnroll; ++u) v[u] = __ldcs(p + i + u * stride);
#pragma unroll
    for (int u = 0; u < kStreamUnroll; ++u) acc ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
  }
  for (; i < n16; i += stride) {
    const uint4 v = __ldcs(p + i);
    acc ^= v.x ^ v.y ^ v.z ^ v.w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xFFFFFFFFu, acc, o);
  if ((threadIdx.x & 31) == 0) wx[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t c = 0;
#pragma unroll
    for (int w = 0; w < kStreamThreads / 32; ++w) c ^= wx[w];
    atomicXor(checksum, c);
  }
}

}  // namespace

cudaError_t launch_stream_read(const void* buf, long long bytes, uint32_t* checksum,
                               cudaStream_t stream) {
  stream_read_kernel<<<2 * num_sms(), kStreamThreads, 0, stream>>>(
      static_cast<const uint4*>(buf), bytes / 16, checksum);
  return cudaGetLastError();
}

cudaError_t launch_row_gather(const void* mat, int rows, int d, long long n, unsigned seed,
                              uint32_t* checksum, cudaStream_t stream) {
  row_gather_kernel<<<num_sms(), 32 * kWarpsG, 0, stream>>>(
      static_cast<const uint4*>(mat), rows, d / 8, n, seed, checksum);
  return cudaGetLastError();
}

}  // namespace tw
