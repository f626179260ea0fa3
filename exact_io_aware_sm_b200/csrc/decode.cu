// decode.cu -- single-token GQA decode over a KV cache, split along the keys.
//
// Decode reads the whole cache once per step and does about 2 FLOPs per byte
// (inference page, "Why Decode is Memory-bound"), so this path is built for
// HBM streaming on the CUDA cores rather than for the tensor cores:
//
//   decode_split_kernel   one CTA per (split of 512 keys, KV head, sequence).
//     Each half-warp owns one key row at a time; each lane holds d/16
//     consecutive elements (16-byte loads for d = 128), so a warp-wide load
//     moves two full 256-byte rows.  The G query heads of the group share
//     every K/V row that is loaded.  Scores are reduced with xor-shuffles
//     inside the half-warp; each half-warp keeps its own online-softmax state
//     (m, l, acc) over its keys; the halves and the four warps are merged at
//     the end.  Output: a normalised partial O and its log2-sum-exp per
//     (sequence, query head, split).
//   decode_combine_kernel  one CTA per (sequence, query head): merges the
//     splits with the block rule of the FlashAttention page, section 2
//     (rescale each part by 2^(lse_s - lse)), writes O (bf16) and LSE
//     (natural log).
#include <cuda_bf16.h>

#include "kernels.h"

namespace eio {
namespace {

constexpr int kWarps = 4;
constexpr int kPairsPerIter = 4;  // key pairs in flight per lane per iteration
constexpr float kLn2 = 0.69314718055994530942f;

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int VEC>
struct Vec;  // VEC bf16 values in one load
template <>
struct Vec<8> {
  using T = uint4;
};
template <>
struct Vec<4> {
  using T = uint2;
};

__device__ __forceinline__ void unpack(const uint4& r, float* f) {
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void unpack(const uint2& r, float* f) {
  const uint32_t w[2] = {r.x, r.y};
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ int checked_len(const DecodeArgs& a, int b) {
  const int len = a.seqlens[b];
  if (len < 0 || len > a.Lmax) {
    atomicCAS(a.err, 0, kErrDeviceArg);
    return 0;
  }
  return len;
}

template <int D, int G>
__global__ void __launch_bounds__(kWarps * 32) decode_split_kernel(const DecodeArgs a) {
  constexpr int VEC = D / 16;  // elements per lane
  using LoadT = typename Vec<VEC>::T;
  const int split = blockIdx.x, hkv = blockIdx.y, b = blockIdx.z;
  const int len = checked_len(a, b);
  const int k0 = split * kDecodeChunk;
  if (k0 >= len) return;
  const int k1 = min(k0 + kDecodeChunk, len);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int half = lane >> 4, sl = lane & 15;

  // q for the G heads of this KV head, this lane's VEC dims, in fp32.
  float qf[G][VEC];
  const __nv_bfloat16* qb = reinterpret_cast<const __nv_bfloat16*>(a.q);
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const LoadT r = *reinterpret_cast<const LoadT*>(
        qb + (static_cast<size_t>(b) * a.Hq + hkv * G + g) * D + sl * VEC);
    unpack(r, qf[g]);
  }

  float m[G], l[G], acc[G][VEC];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[g][e] = 0.f;
  }

  const size_t row_stride = static_cast<size_t>(a.Hkv) * D;  // elements between cache rows
  const __nv_bfloat16* kb =
      reinterpret_cast<const __nv_bfloat16*>(a.kc) + (static_cast<size_t>(b) * a.Lmax * a.Hkv + hkv) * D + sl * VEC;
  const __nv_bfloat16* vb =
      reinterpret_cast<const __nv_bfloat16*>(a.vc) + (static_cast<size_t>(b) * a.Lmax * a.Hkv + hkv) * D + sl * VEC;

  // This warp's contiguous share of the split.
  const int per_warp = (kDecodeChunk / kWarps);
  const int w0 = k0 + warp * per_warp;
  const int w1 = min(w0 + per_warp, k1);

  for (int kb0 = w0; kb0 < w1; kb0 += 2 * kPairsPerIter) {
    LoadT kr[kPairsPerIter], vr[kPairsPerIter];
#pragma unroll
    for (int u = 0; u < kPairsPerIter; ++u) {
      const int key = kb0 + 2 * u + half;
      if (key < w1) {
        kr[u] = __ldcs(reinterpret_cast<const LoadT*>(kb + key * row_stride));
        vr[u] = __ldcs(reinterpret_cast<const LoadT*>(vb + key * row_stride));
      } else {
        kr[u] = LoadT{};
        vr[u] = LoadT{};
      }
    }
    float s[G][kPairsPerIter];
#pragma unroll
    for (int u = 0; u < kPairsPerIter; ++u) {
      float kf[VEC];
      unpack(kr[u], kf);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float dot = 0.f;
#pragma unroll
        for (int e = 0; e < VEC; ++e) dot = fmaf(qf[g][e], kf[e], dot);
        s[g][u] = dot;
      }
    }
#pragma unroll
    for (int off = 8; off > 0; off >>= 1)
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int u = 0; u < kPairsPerIter; ++u) s[g][u] += __shfl_xor_sync(0xffffffffu, s[g][u], off);

#pragma unroll
    for (int g = 0; g < G; ++g) {
      float mx = -INFINITY;
#pragma unroll
      for (int u = 0; u < kPairsPerIter; ++u) {
        const int key = kb0 + 2 * u + half;
        s[g][u] = key < w1 ? s[g][u] * a.scale_log2 : -INFINITY;
        mx = fmaxf(mx, s[g][u]);
      }
      const float m_new = fmaxf(m[g], mx);
      // alpha is 0 when m was -inf (and 1 while nothing has been seen yet)
      const float alpha = m_new == -INFINITY ? 1.f : ex2(m[g] - m_new);
      const float base = m_new == -INFINITY ? 0.f : m_new;
      l[g] *= alpha;
#pragma unroll
      for (int e = 0; e < VEC; ++e) acc[g][e] *= alpha;
      m[g] = m_new;
#pragma unroll
      for (int u = 0; u < kPairsPerIter; ++u) {
        const float p = ex2(s[g][u] - base);
        l[g] += p;
        float vf[VEC];
        unpack(vr[u], vf);
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[g][e] = fmaf(p, vf[e], acc[g][e]);
      }
    }
  }

  // Merge the two half-warps (same dims, different keys).
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float mo = __shfl_xor_sync(0xffffffffu, m[g], 16);
    const float lo = __shfl_xor_sync(0xffffffffu, l[g], 16);
    const float mn = fmaxf(m[g], mo);
    const float fa = mn == -INFINITY ? 0.f : ex2(m[g] - mn);
    const float fb = mn == -INFINITY ? 0.f : ex2(mo - mn);
    l[g] = l[g] * fa + lo * fb;
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      const float ao = __shfl_xor_sync(0xffffffffu, acc[g][e], 16);
      acc[g][e] = acc[g][e] * fa + ao * fb;
    }
    m[g] = mn;
  }

  // Merge the warps through shared memory.
  __shared__ float s_acc[kWarps][G][D];
  __shared__ float s_m[kWarps][G], s_l[kWarps][G];
  if (half == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
      for (int e = 0; e < VEC; ++e) s_acc[warp][g][sl * VEC + e] = acc[g][e];
      if (sl == 0) {
        s_m[warp][g] = m[g];
        s_l[warp][g] = l[g];
      }
    }
  }
  __syncthreads();
  const size_t part_base = static_cast<size_t>(b) * a.Hq + hkv * G;
  for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
    const int g = idx / D, t = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, s_m[w][g]);
    float L = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float f = s_m[w][g] == -INFINITY ? 0.f : ex2(s_m[w][g] - M);
      L += s_l[w][g] * f;
      O += s_acc[w][g][t] * f;
    }
    const size_t p = (part_base + g) * a.nsplit + split;
    a.opart[p * D + t] = O / L;
    if (t == 0) a.lpart[p] = M + __log2f(L);
  }
}

template <int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(const DecodeArgs a) {
  const int bh = blockIdx.x;
  const int b = bh / a.Hq;
  const int t = threadIdx.x;
  const int len = checked_len(a, b);
  const int ns = (len + kDecodeChunk - 1) / kDecodeChunk;
  __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(a.o) + static_cast<size_t>(bh) * D;
  if (ns == 0) {
    o[t] = __float2bfloat16_rn(0.f);
    if (t == 0 && a.lse != nullptr) a.lse[bh] = -INFINITY;
    return;
  }
  const float* lp = a.lpart + static_cast<size_t>(bh) * a.nsplit;
  const float* op = a.opart + static_cast<size_t>(bh) * a.nsplit * D;
  float M = -INFINITY;
  for (int s = 0; s < ns; ++s) M = fmaxf(M, lp[s]);
  float W = 0.f, O = 0.f;
  for (int s = 0; s < ns; ++s) {
    const float w = ex2(lp[s] - M);
    W += w;
    O = fmaf(w, op[static_cast<size_t>(s) * D + t], O);
  }
  o[t] = __float2bfloat16_rn(O / W);
  if (t == 0 && a.lse != nullptr) a.lse[bh] = (M + __log2f(W)) * kLn2;
}

template <int D, int G>
cudaError_t launch_dg(const DecodeArgs& a, cudaStream_t s) {
  dim3 grid(a.nsplit, a.Hkv, a.B);
  decode_split_kernel<D, G><<<grid, kWarps * 32, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_combine_kernel<D><<<a.B * a.Hq, D, 0, s>>>(a);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(int G, const DecodeArgs& a, cudaStream_t s) {
  switch (G) {
    case 1: return launch_dg<D, 1>(a, s);
    case 2: return launch_dg<D, 2>(a, s);
    case 4: return launch_dg<D, 4>(a, s);
    case 8: return launch_dg<D, 8>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

size_t decode_partial_floats(int B, int Hq, int Lmax, int d) {
  const size_t ns = (static_cast<size_t>(Lmax) + kDecodeChunk - 1) / kDecodeChunk;
  return static_cast<size_t>(B) * Hq * ns * (d + 1);
}

cudaError_t launch_decode(int d, int G, const DecodeArgs& a, cudaStream_t s) {
  if (d == 64) return launch_d<64>(G, a, s);
  return launch_d<128>(G, a, s);
}

}  // namespace eio
