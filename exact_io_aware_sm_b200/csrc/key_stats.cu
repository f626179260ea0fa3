// key_stats.cu -- per-(b, KV head) key statistics for the bound-based
// softmax ("TPU attention optimisation guide", step 4): the mean key kbar
// and the radius max_j ||k_j - kbar|| of the centred keys.  With them every
// score of row i satisfies  q_i . (k_j - kbar) <= ||q_i|| radius  (Cauchy-
// Schwarz), which the prefill kernel uses as the row's exponent base.
//
// Three launches over 128-key chunks, each thread moving 16 bytes (eight
// keys' columns) per load with several loads in flight:
//   key_sum_kernel     per-chunk column sums into scratch;
//   key_mean_kernel    kbar = (sum of the chunk sums) / Nkv, eight runs of
//                      consecutive chunks summed in parallel and then added in
//                      run order, so the result does not depend on scheduling;
//   key_radius_kernel  the largest centred norm of each chunk, folded into
//                      `radius` (zeroed by the mean kernel) with an integer
//                      atomicMax on the float's bits (non-negative floats
//                      order like their bit patterns).
// The second and third are programmatic dependents of the one before them:
// they start while it drains, and the radius kernel loads its keys (an input
// of the call) before it waits for the mean.
#include <cuda_bf16.h>

#include "kernels.h"
#include "pdl.cuh"

namespace eio {
namespace {

constexpr int kChunkKeys = 128;
constexpr int kStatThreads = 256;
constexpr int kMeanRuns = 8;  // runs of chunks summed in parallel per column

__device__ __forceinline__ void add8(float* acc, const uint4& u) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    acc[2 * i] += f.x;
    acc[2 * i + 1] += f.y;
  }
}

template <int D>
__global__ void __launch_bounds__(kStatThreads) key_sum_kernel(const KeyStatsArgs a) {
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  constexpr int TPR = D / 8;                 // threads per key row, 16 bytes each
  constexpr int RPI = kStatThreads / TPR;    // rows per pass (32 at d = 64, 16 at d = 128)
  const int c8 = threadIdx.x % TPR, r = threadIdx.x / TPR;
  const int j0 = split * kChunkKeys, j1 = min(a.Nkv, j0 + kChunkKeys);
  const uint4* k = reinterpret_cast<const uint4*>(a.k);
  if (threadIdx.x == 0) pdl_launch_dependents();
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int p = 0; p < kChunkKeys / RPI; ++p) {
    const int j = j0 + r + p * RPI;
    if (j < j1) add8(acc, k[((static_cast<size_t>(b) * a.Nkv + j) * a.Hkv + h) * TPR + c8]);
  }
  __shared__ float red[RPI][D];
#pragma unroll
  for (int i = 0; i < 8; ++i) red[r][c8 * 8 + i] = acc[i];
  __syncthreads();
  if (threadIdx.x < D) {
    float s = 0.f;
#pragma unroll 8
    for (int i = 0; i < RPI; ++i) s += red[i][threadIdx.x];
    a.part[((static_cast<size_t>(b) * a.Hkv + h) * a.nsplit + split) * D + threadIdx.x] = s;
  }
}

template <int D>
__global__ void __launch_bounds__(kMeanRuns * D) key_mean_kernel(const KeyStatsArgs a) {
  const size_t bh = static_cast<size_t>(blockIdx.y) * a.Hkv + blockIdx.x;
  const int c = threadIdx.x % D, run = threadIdx.x / D;
  if (threadIdx.x == 0) pdl_launch_dependents();
  const int per = (a.nsplit + kMeanRuns - 1) / kMeanRuns;
  const int i0 = run * per, i1 = min(a.nsplit, i0 + per);
  pdl_wait();  // the chunk sums are complete
  const float* p = a.part + bh * a.nsplit * D + c;
  float s = 0.f;
#pragma unroll 8
  for (int i = i0; i < i1; ++i) s += p[static_cast<size_t>(i) * D];
  __shared__ float runs[kMeanRuns][D];
  runs[run][c] = s;
  __syncthreads();
  if (threadIdx.x == 0) a.radius[bh] = 0.f;  // folded into the maximum by the radius kernel
  if (run == 0) {
    float t = 0.f;
#pragma unroll
    for (int r = 0; r < kMeanRuns; ++r) t += runs[r][c];
    a.kbar[bh * D + c] = t / static_cast<float>(a.Nkv);
  }
}

template <int D>
__global__ void __launch_bounds__(kStatThreads) key_radius_kernel(const KeyStatsArgs a) {
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const size_t bh = static_cast<size_t>(b) * a.Hkv + h;
  constexpr int TPR = D / 8, RPI = kStatThreads / TPR;
  const int c8 = threadIdx.x % TPR, r = threadIdx.x / TPR;
  const int j0 = split * kChunkKeys, j1 = min(a.Nkv, j0 + kChunkKeys);
  const uint4* k = reinterpret_cast<const uint4*>(a.k);
  constexpr int NP = kChunkKeys / RPI;
  uint4 kv[NP];  // this thread's keys, loaded while the mean is still being formed
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const int j = j0 + r + p * RPI;
    kv[p] = j < j1 ? k[((static_cast<size_t>(b) * a.Nkv + j) * a.Hkv + h) * TPR + c8] : make_uint4(0, 0, 0, 0);
  }
  pdl_wait();  // kbar is complete
  float kb[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) kb[i] = a.kbar[bh * D + c8 * 8 + i];
  float mx = 0.f;
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const int j = j0 + r + p * RPI;
    float ss = 0.f;
    if (j < j1) {
      const uint4 u = kv[p];
      const __nv_bfloat162* hh = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(hh[i]);
        const float c0 = f.x - kb[2 * i], c1 = f.y - kb[2 * i + 1];
        ss = fmaf(c0, c0, fmaf(c1, c1, ss));
      }
    }
    // the TPR lanes of one row are consecutive lanes of a warp
#pragma unroll
    for (int o = TPR / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    mx = fmaxf(mx, ss);
  }
  __shared__ float wmax[kStatThreads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = mx;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = 0.f;
    for (int w = 0; w < kStatThreads / 32; ++w) m = fmaxf(m, wmax[w]);
    atomicMax(reinterpret_cast<unsigned int*>(a.radius + bh), __float_as_uint(sqrtf(m)));
  }
}

template <int D>
cudaError_t launch_d(const KeyStatsArgs& a, cudaStream_t s) {
  const dim3 grid(a.nsplit, a.Hkv, a.B);
  key_sum_kernel<D><<<grid, kStatThreads, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = launch_after_pdl(key_mean_kernel<D>, dim3(a.Hkv, a.B), dim3(kMeanRuns * D), 0, s, a);
  if (e != cudaSuccess) return e;
  return launch_after_pdl(key_radius_kernel<D>, grid, dim3(kStatThreads), 0, s, a);
}

}  // namespace

int key_stats_splits(int Nkv) { return (Nkv + kChunkKeys - 1) / kChunkKeys; }

cudaError_t launch_key_stats(int d, const KeyStatsArgs& a, cudaStream_t s) {
  return d == 64 ? launch_d<64>(a, s) : launch_d<128>(a, s);
}

}  // namespace eio
