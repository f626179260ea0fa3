// prefill_f32.cu -- exact attention forward for fp32 inputs (CUDA cores).
//
// fp32 inputs keep fp32 arithmetic end to end: rounding them to bf16 for the
// tensor cores would move the LSE by about 2e-3 at d = 64, above the 1e-3
// tolerance.  The algorithm is the same tiled online softmax as the tensor
// path (FlashAttention page, sections 2-3): one warp per query row, keys
// staged through shared memory 32 at a time, each lane scoring one key, the
// running (m, l) and the accumulator rescaled per key block.
#include <cuda_runtime.h>

#include "kernels.h"

namespace eio {
namespace {

constexpr int kRowsPerCta = 8;
constexpr int kKeys = 32;

__device__ __forceinline__ bool allowed(const PrefillF32Args& a, int i, int j) {
  if (j >= a.Nkv) return false;
  if (a.mask_kind == 1) return j <= i + (a.Nkv - a.Nq);
  if (a.mask_kind == 2) {
    const int nbc = (a.Nkv + 15) / 16;
    return a.block_map[static_cast<size_t>(i / 16) * nbc + j / 16] != 0;
  }
  return true;
}

template <int D>
__global__ void __launch_bounds__(kRowsPerCta * 32) prefill_f32_kernel(const PrefillF32Args a) {
  constexpr int VPL = D / 32;  // output dims per lane
  __shared__ float qs[kRowsPerCta][D];
  __shared__ float ks[kKeys][D + 1];
  __shared__ float vs[kKeys][D];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * kRowsPerCta + warp;
  const int hq = blockIdx.y, b = blockIdx.z;
  const int hkv = hq / (a.Hq / a.Hkv);
  const bool active = i < a.Nq;

  for (int t = lane; t < D; t += 32)
    qs[warp][t] = active ? a.q[((static_cast<size_t>(b) * a.Nq + i) * a.Hq + hq) * D + t] : 0.f;

  float m = -INFINITY, l = 0.f, acc[VPL];
#pragma unroll
  for (int u = 0; u < VPL; ++u) acc[u] = 0.f;

  for (int j0 = 0; j0 < a.Nkv; j0 += kKeys) {
    __syncthreads();
    for (int e = threadIdx.x; e < kKeys * D; e += blockDim.x) {
      const int jj = e / D, t = e % D;
      const int j = j0 + jj;
      const size_t off = ((static_cast<size_t>(b) * a.Nkv + j) * a.Hkv + hkv) * D + t;
      ks[jj][t] = j < a.Nkv ? a.k[off] : 0.f;
      vs[jj][t] = j < a.Nkv ? a.v[off] : 0.f;
    }
    __syncthreads();
    if (!active) continue;
    const int j = j0 + lane;
    float s = -INFINITY;
    if (allowed(a, i, j)) {
      float dot = 0.f;
#pragma unroll 8
      for (int t = 0; t < D; ++t) dot = fmaf(qs[warp][t], ks[lane][t], dot);
      s = dot * a.scale;
    }
    float mx = s;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float m_new = fmaxf(m, mx);
    if (m_new == -INFINITY) continue;  // nothing allowed yet
    const float alpha = (m == -INFINITY) ? 0.f : expf(m - m_new);
    const float p = (s == -INFINITY) ? 0.f : expf(s - m_new);
    float ps = p;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
    l = l * alpha + ps;
#pragma unroll
    for (int u = 0; u < VPL; ++u) acc[u] *= alpha;
    for (int jj = 0; jj < kKeys; ++jj) {
      const float pj = __shfl_sync(0xffffffffu, p, jj);
#pragma unroll
      for (int u = 0; u < VPL; ++u) acc[u] = fmaf(pj, vs[jj][lane + 32 * u], acc[u]);
    }
    m = m_new;
  }
  if (!active) return;
  const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
  for (int u = 0; u < VPL; ++u)
    a.o[((static_cast<size_t>(b) * a.Nq + i) * a.Hq + hq) * D + lane + 32 * u] = acc[u] * inv;
  if (lane == 0 && a.lse != nullptr)
    a.lse[(static_cast<size_t>(b) * a.Hq + hq) * a.Nq + i] = l > 0.f ? m + logf(l) : -INFINITY;
}

template <int D>
cudaError_t launch(const PrefillF32Args& a, cudaStream_t s) {
  dim3 grid((a.Nq + kRowsPerCta - 1) / kRowsPerCta, a.Hq, a.B);
  prefill_f32_kernel<D><<<grid, kRowsPerCta * 32, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_f32(int d, const PrefillF32Args& a, cudaStream_t s) {
  if (d == 32) return launch<32>(a, s);
  if (d == 64) return launch<64>(a, s);
  return launch<128>(a, s);
}

}  // namespace eio
