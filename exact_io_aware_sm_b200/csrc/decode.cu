// decode.cu -- GQA decode of the newest token (or the Sq newest tokens) of
// each sequence over a KV cache, split along the keys.
//
// Decode reads the whole cache once per step and does little arithmetic per
// byte (inference page, "Why Decode is Memory-bound"): 4d FLOPs per query
// head per cached key against 4d bytes of K and V, i.e. G FLOPs per byte for
// G query heads per KV head (times Sq for Sq tokens).  So this path is built
// to keep HBM streaming and to spend as few instructions per byte as possible:
//
//   decode_split_kernel   persistent, one CTA per SM, four warps.  A work
//     item is (sequence b, KV head, split of 512 keys), for the Sq newest
//     query tokens of the sequence (Sq = 1: plain decode; Sq > 1: several
//     tokens at once, each seeing the keys up to its own position); only splits below the
//     sequence's length exist.  Every CTA counts the live splits from seqlens
//     (prefix sums in shared memory); warps draw items one at a time from a
//     global counter, so the work evens out to within one item per warp
//     (the combine kernel zeroes the counter for the next call).
//     Each warp is its own pipeline: a ring of 32-key stages (K and V tiles
//     brought in by TMA, 128-byte swizzle) that it refills as it consumes, so
//     every warp keeps up to 48 KB of loads in flight.  The G query heads x Sq
//     tokens of the item (at most 16) share every K/V tile; they fill one or
//     two groups of 8 MMA columns (NCG):
//       S^T (16 keys x 8 columns) = K (16 x d) q^T     mma.m16n8k16, K by ldmatrix
//       online softmax on the fragment (max over the 16 keys by 3 shuffles)
//       O^T (d x 8 columns) += V^T (d x 16) P^T       V by ldmatrix.trans, P^T by movmatrix
//     per column group, the K and V fragments loaded once for both groups.
//     Columns past G * Sq are zero.  The output is a normalised partial O
//     and its log2-sum-exp per (sequence, query head, split).
//   decode_combine_kernel  one CTA per (sequence, token, query head): merges the
//     splits with the block rule of the FlashAttention page, section 2
//     (rescale each part by 2^(lse_s - lse)), writes O (bf16) and LSE
//     (natural log).
#include <cuda_bf16.h>

#include "kernels.h"
#include "pdl.cuh"
#include "ptx_sm100.cuh"
#include "warp_mma.cuh"

namespace eio {
namespace {

constexpr int kWarps = 4;            // independent pipelines per CTA
constexpr int kStageKeys = 32;       // keys per pipeline stage
constexpr int kBoxRows = 16;         // rows per TMA box
constexpr int kWarpRingBytes = 48 * 1024;
constexpr int kMaxB = 2048;          // sequences per launch (prefix sums in shared memory)
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kRebase = 8.f;       // move the exponent base only when the max grows by more

template <int D>
struct DCfg {
  static constexpr int KB = D / 64;                        // 128-byte column blocks per row
  static constexpr int kBlockBytes = kStageKeys * 128;     // one column block of a tile
  static constexpr int kTileBytes = KB * kBlockBytes;      // K (or V) of one stage
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int R = kWarpRingBytes / kStageBytes;   // stages per warp: 3 (d=128), 6 (d=64)
  static constexpr int kOffBars = kWarps * R * kStageBytes;
  static constexpr int kOffMeta = kOffBars + kWarps * R * 8;
  static constexpr int kOffPre = kOffMeta + kWarps * R * 16;  // int[kMaxB + 1] prefix, int[kMaxB] lengths
  static constexpr int kSmem = kOffPre + (2 * kMaxB + 1) * 4 + 1024;  // + slack to align the base to 1 KB
};

__device__ __forceinline__ int checked_len(const DecodeArgs& a, int b) {
  const int len = a.seqlens[b];
  if (len < 0 || len > a.Lmax) {
    atomicCAS(a.err, 0, kErrDeviceArg);
    return 0;
  }
  return len;
}

// Producer cursor of one warp (warp-uniform).
struct Cursor {
  int b, hkv, split, k, kend;
};

template <int D, int G, int NCG>
__global__ void __launch_bounds__(kWarps * 32, 1)
    decode_split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const DecodeArgs a) {
  using C = DCfg<D>;
  constexpr int R = C::R, KB = C::KB;
  constexpr int NK = D / 16;  // k-steps of S, m-tiles of O
  const int NC = G * a.Sq;    // live columns of the 8 * NCG: (head, token) pairs of the group
  extern __shared__ uint8_t dsmem[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBars) + warp * R;
  int4* meta = reinterpret_cast<int4*>(smem + C::kOffMeta) + warp * R;
  int* pre = reinterpret_cast<int*>(smem + C::kOffPre);  // [B + 1] live splits before sequence b
  int* lens = pre + kMaxB + 1;                             // [B]
  uint8_t* ring = smem + warp * R * C::kStageBytes;
  const uint32_t ring_u32 = smem_u32(ring);

  if (lane == 0) {
    for (int r = 0; r < R; ++r) mbar_init(&bars[r], 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  // The combine kernel may be scheduled as this kernel's CTAs finish; it
  // waits for this grid before it reads the partials.
  if (threadIdx.x == 0) pdl_launch_dependents();
  if (warp == 0) {
    int carry = 0;
    if (lane == 0) pre[0] = 0;
    for (int b0 = 0; b0 < a.B; b0 += 32) {
      const int b = b0 + lane;
      int n = 0;
      if (b < a.B) {
        const int len = checked_len(a, b);
        lens[b] = len;
        n = (len + kDecodeChunk - 1) / kDecodeChunk;
      }
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, n, off);
        if (lane >= off) n += v;
      }
      if (b < a.B) pre[b + 1] = carry + n;
      carry += __shfl_sync(0xffffffffu, n, 31);
    }
  }
  __syncthreads();

  const long long total = static_cast<long long>(pre[a.B]) * a.Hkv;

  // Next item into the cursor; false when none is left.
  auto fetch = [&](Cursor& c) -> bool {
    int it = 0;
    if (lane == 0) it = atomicAdd(a.counter, 1);
    it = __shfl_sync(0xffffffffu, it, 0);
    const long long i = it;
    if (i >= total) return false;
    const int j = static_cast<int>(i / a.Hkv);
    c.hkv = static_cast<int>(i % a.Hkv);
    int lo = 0, hi = a.B;  // largest b with pre[b] <= j
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (pre[mid] <= j) lo = mid;
      else hi = mid;
    }
    c.b = lo;
    c.split = j - pre[lo];
    c.k = c.split * kDecodeChunk;
    c.kend = min(c.k + kDecodeChunk, lens[lo]);
    return true;
  };

  Cursor cur{0, 0, 0, 0, 0};
  bool more = true;
  // Issue the next stage of this warp's stream into ring slot `slot`.
  auto produce = [&](int slot) -> bool {
    if (cur.k >= cur.kend && !fetch(cur)) return false;
    const int nvalid = min(kStageKeys, cur.kend - cur.k);
    const int flags = (cur.k == cur.split * kDecodeChunk ? 1 : 0) | (cur.k + kStageKeys >= cur.kend ? 2 : 0);
    const int stage = (cur.k - cur.split * kDecodeChunk) / kStageKeys;  // stage of the split, < 16
    if (lane == 0) meta[slot] = make_int4(cur.b, cur.hkv, cur.split, nvalid | (flags << 16) | (stage << 20));
    const int nbox = nvalid > kBoxRows ? 2 : 1;
    uint8_t* st = ring + slot * C::kStageBytes;
    fence_proxy_async_smem();  // earlier generic writes to this slot come first
    mbar_arrive_expect_tx_elect(&bars[slot], static_cast<uint32_t>(nbox * 2 * KB * kBoxRows * 128));
    for (int rh = 0; rh < nbox; ++rh) {
#pragma unroll
      for (int h = 0; h < KB; ++h) {
        const int off = h * C::kBlockBytes + rh * kBoxRows * 128;
        tma_load_4d_elect(st + off, &tmK, &bars[slot], 64 * h, cur.hkv, cur.k + rh * kBoxRows, cur.b);
        tma_load_4d_elect(st + C::kTileBytes + off, &tmV, &bars[slot], 64 * h, cur.hkv, cur.k + rh * kBoxRows,
                          cur.b);
      }
    }
    cur.k += kStageKeys;
    return true;
  };

  uint32_t produced = 0, consumed = 0;
  for (int r = 0; r < R && more; ++r) {
    more = produce(r);
    if (more) ++produced;
  }
  __syncwarp();

  const float sl2 = a.scale_log2;
  uint32_t qf[NCG][NK][2];
  float acc[NCG][NK][4];
  float m[NCG][2], l[NCG][2];
  bool ok = true;

  while (consumed < produced) {
    const int slot = static_cast<int>(consumed % R);
    const bool mine = mbar_wait(&bars[slot], (consumed / R) & 1);
    if (!__all_sync(0xffffffffu, mine)) {
      ok = false;
      break;
    }
    const int4 md = meta[slot];
    const int b = md.x, hkv = md.y, split = md.z;
    const int nvalid = md.w & 0xffff, flags = (md.w >> 16) & 3;
    const int k0 = split * kDecodeChunk + (md.w >> 20) * kStageKeys;  // first key of the stage
    const uint32_t kt = ring_u32 + slot * C::kStageBytes;
    const uint32_t vt = kt + C::kTileBytes;

    if (flags & 1) {  // first stage of an item: this item's queries, fresh state
#pragma unroll
      for (int cg = 0; cg < NCG; ++cg) {
        // Column cg*8 + g of q^T is (head c / Sq, token c % Sq) of this KV group.
        const int c = cg * 8 + g;
        const bool live = c < NC;
        const int gc = live ? c : 0;
        const __nv_bfloat16* qrow = reinterpret_cast<const __nv_bfloat16*>(a.q) +
                                    ((static_cast<size_t>(b) * a.Sq + gc % a.Sq) * a.Hq + hkv * G + gc / a.Sq) * D +
                                    2 * t;
#pragma unroll
        for (int ks = 0; ks < NK; ++ks) {
          qf[cg][ks][0] = live ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks) : 0u;
          qf[cg][ks][1] = live ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 8) : 0u;
        }
#pragma unroll
        for (int mt = 0; mt < NK; ++mt)
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[cg][mt][i] = 0.f;
        m[cg][0] = m[cg][1] = -INFINITY;
        l[cg][0] = l[cg][1] = 0.f;
      }
    }
    if (nvalid < kStageKeys) {
      // V rows past the sequence (read by the last box, or stale) must be
      // finite: zero them so that P = 0 there gives exactly 0.
      uint8_t* vrow = ring + slot * C::kStageBytes + C::kTileBytes;
      for (int idx = lane; idx < (kStageKeys - nvalid) * KB * 8; idx += 32) {
        const int r = nvalid + idx / (KB * 8), h = (idx / 8) % KB, c = idx % 8;
        *reinterpret_cast<uint4*>(vrow + h * C::kBlockBytes + r * 128 + c * 16) = make_uint4(0u, 0u, 0u, 0u);
      }
      __syncwarp();
    }

    const int nch = nvalid > 16 ? 2 : 1;
    // Keys of this stage visible to the lane's columns cg*8 + 2t + j: token s
    // (of Sq, the last at position len - 1) sees keys 0 .. len - Sq + s.
    int lim[NCG][2];
#pragma unroll
    for (int cg = 0; cg < NCG; ++cg)
#pragma unroll
      for (int j = 0; j < 2; ++j)
        lim[cg][j] = a.Sq > 1 ? min(nvalid, lens[b] - a.Sq + (cg * 8 + 2 * t + j) % a.Sq + 1 - k0) : nvalid;
    float s[2][NCG][4];
#pragma unroll
    for (int ch = 0; ch < 2; ++ch) {
#pragma unroll
      for (int cg = 0; cg < NCG; ++cg)
#pragma unroll
        for (int i = 0; i < 4; ++i) s[ch][cg][i] = 0.f;
      if (ch < nch) {
        const int r = ch * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
#pragma unroll
        for (int ks = 0; ks < NK; ++ks) {
          const int cc = (ks & 3) * 2 + (lane >> 4);
          uint32_t af[4];
          ldsm_x4(kt + (ks >> 2) * C::kBlockBytes + r * 128 + ((cc ^ (r & 7)) << 4), af);
#pragma unroll
          for (int cg = 0; cg < NCG; ++cg) mma_16816(s[ch][cg], af, qf[cg][ks][0], qf[cg][ks][1]);
        }
      }
      // keys past the valid ones, and past each token's own position, carry no weight
#pragma unroll
      for (int cg = 0; cg < NCG; ++cg)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int key = ch * 16 + g + (i >> 1) * 8;
          if (key >= lim[cg][i & 1]) s[ch][cg][i] = -INFINITY;
        }
    }

    // Running max per column (cg*8 + 2t and + 1), over the 32 keys of the stage.
#pragma unroll
    for (int cg = 0; cg < NCG; ++cg)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float v = fmaxf(fmaxf(s[0][cg][j], s[0][cg][j + 2]), fmaxf(s[1][cg][j], s[1][cg][j + 2]));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
        v *= sl2;
        if (v > m[cg][j] + kRebase) {  // move the base (always on the first stage)
          const float alpha = wm_ex2(m[cg][j] - v);
          l[cg][j] *= alpha;
#pragma unroll
          for (int mt = 0; mt < NK; ++mt) {
            acc[cg][mt][j] *= alpha;
            acc[cg][mt][j + 2] *= alpha;
          }
          m[cg][j] = v;
        }
      }

#pragma unroll
    for (int ch = 0; ch < 2; ++ch) {
      if (ch < nch) {
        uint32_t pb[NCG][2];
#pragma unroll
        for (int cg = 0; cg < NCG; ++cg) {
          float p[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            // a column that has seen no key yet keeps m = -inf: its p are 0
            const float mb = m[cg][i & 1];
            p[i] = wm_ex2(fmaf(s[ch][cg][i], sl2, mb == -INFINITY ? 0.f : -mb));
            l[cg][i & 1] += p[i];
          }
          pb[cg][0] = movmatrix_trans(wm_pack_bf16x2(p[0], p[1]));
          pb[cg][1] = movmatrix_trans(wm_pack_bf16x2(p[2], p[3]));
        }
        const int r = ch * 16 + (lane >> 4) * 8 + (lane & 7);
#pragma unroll
        for (int mt = 0; mt < NK; ++mt) {
          const int cc = (mt & 3) * 2 + ((lane >> 3) & 1);
          uint32_t af[4];
          ldsm_x4_trans(vt + (mt >> 2) * C::kBlockBytes + r * 128 + ((cc ^ (r & 7)) << 4), af);
#pragma unroll
          for (int cg = 0; cg < NCG; ++cg) mma_16816(acc[cg][mt], af, pb[cg][0], pb[cg][1]);
        }
      }
    }

    if (flags & 2) {  // last stage of the item: normalise and write the partial
#pragma unroll
      for (int cg = 0; cg < NCG; ++cg) {
        float lt[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          float v = l[cg][j];
          v += __shfl_xor_sync(0xffffffffu, v, 4);
          v += __shfl_xor_sync(0xffffffffu, v, 8);
          v += __shfl_xor_sync(0xffffffffu, v, 16);
          lt[j] = v;
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int col = cg * 8 + 2 * t + j;
          if (col < NC) {
            const size_t row = (static_cast<size_t>(b) * a.Sq + col % a.Sq) * a.Hq + hkv * G + col / a.Sq;
            const size_t p = row * a.nsplit + split;
            // a token may see no key of this split (its position precedes it)
            const float inv = lt[j] > 0.f ? 1.f / lt[j] : 0.f;
            float* op = a.opart + p * D;
#pragma unroll
            for (int mt = 0; mt < NK; ++mt) {
              op[16 * mt + g] = acc[cg][mt][j] * inv;
              op[16 * mt + g + 8] = acc[cg][mt][j + 2] * inv;
            }
            if (g == 0) a.lpart[p] = lt[j] > 0.f ? m[cg][j] + __log2f(lt[j]) : -INFINITY;
          }
        }
      }
    }

    __syncwarp();
    ++consumed;
    if (more) {
      more = produce(static_cast<int>(produced % R));
      if (more) ++produced;
    }
  }

  if (!ok) {
    if (lane == 0) atomicCAS(a.err, 0, kErrDeviceTimeout);
    // Let every copy this warp started land before the CTA retires.
    for (uint32_t c = consumed; c < produced; ++c) mbar_wait(&bars[c % R], (c / R) & 1);
  }
}

template <int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(const DecodeArgs a) {
  const int bh = blockIdx.x;  // query row (b, token, head) of [B, Sq, Hq]
  const int b = bh / (a.Sq * a.Hq);
  const int lse_at = (b * a.Hq + bh % a.Hq) * a.Sq + (bh / a.Hq) % a.Sq;  // LSE is [B, Hq, Sq]
  const int t = threadIdx.x;
  pdl_wait();  // the split kernels of this call have finished and their partials are visible
  // Zero their item counters for the next call.
  if (bh == 0 && t < (a.B + kMaxB - 1) / kMaxB) a.counter[t] = 0;
  const int len = checked_len(a, b);
  const int ns = (len + kDecodeChunk - 1) / kDecodeChunk;
  __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(a.o) + static_cast<size_t>(bh) * D;
  const float* lp = a.lpart + static_cast<size_t>(bh) * a.nsplit;
  const float* op = a.opart + static_cast<size_t>(bh) * a.nsplit * D;
  float M = -INFINITY;
  for (int s = 0; s < ns; ++s) M = fmaxf(M, lp[s]);
  if (M == -INFINITY) {  // no key visible to this query row
    o[t] = __float2bfloat16_rn(0.f);
    if (t == 0 && a.lse != nullptr) a.lse[lse_at] = -INFINITY;
    return;
  }
  float W = 0.f, O = 0.f;
  for (int s = 0; s < ns; ++s) {
    const float w = wm_ex2(lp[s] - M);
    W += w;
    O = fmaf(w, op[static_cast<size_t>(s) * D + t], O);
  }
  o[t] = __float2bfloat16_rn(O / W);
  if (t == 0 && a.lse != nullptr) a.lse[lse_at] = (M + __log2f(W)) * kLn2;
}



template <int D, int G, int NCG>
cudaError_t launch_dg(const DecodeArgs& a, cudaStream_t s) {
  static DeviceOnce attr_set;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!attr_set.test(dev)) {
    cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<D, G, NCG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         DCfg<D>::kSmem);
    if (e != cudaSuccess) return e;
    attr_set.set(dev);
  }
  int sms = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // Sequences go in groups of at most kMaxB per launch (the prefix sums live
  // in shared memory); every array is sequence-major, so a group is a pointer
  // offset.
  for (int b0 = 0; b0 < a.B; b0 += kMaxB) {
    DecodeArgs c = a;
    c.B = min(kMaxB, a.B - b0);
    const size_t cache_off = static_cast<size_t>(b0) * a.Lmax * a.Hkv * D * 2;
    c.q = static_cast<const uint8_t*>(a.q) + static_cast<size_t>(b0) * a.Sq * a.Hq * D * 2;
    c.kc = static_cast<const uint8_t*>(a.kc) + cache_off;
    c.vc = static_cast<const uint8_t*>(a.vc) + cache_off;
    c.seqlens = a.seqlens + b0;
    c.counter = a.counter + b0 / kMaxB;
    c.opart = a.opart + static_cast<size_t>(b0) * a.Sq * a.Hq * a.nsplit * D;
    c.lpart = a.lpart + static_cast<size_t>(b0) * a.Sq * a.Hq * a.nsplit;
    CUtensorMap tk, tv;
    if (!encode_bf16_map(&tk, c.kc, c.B, a.Lmax, a.Hkv, D, kBoxRows) ||
        !encode_bf16_map(&tv, c.vc, c.B, a.Lmax, a.Hkv, D, kBoxRows))
      return cudaErrorInvalidValue;
    const long long items = static_cast<long long>(c.B) * a.nsplit * a.Hkv;
    const long long want = (items + kWarps - 1) / kWarps;
    const int grid = static_cast<int>(want < sms ? want : sms);
    decode_split_kernel<D, G, NCG><<<grid, kWarps * 32, DCfg<D>::kSmem, s>>>(tk, tv, c);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return launch_after_pdl(decode_combine_kernel<D>, dim3(a.B * a.Sq * a.Hq), dim3(D), 0, s, a);
}

template <int D>
cudaError_t launch_d(int G, const DecodeArgs& a, cudaStream_t s) {
  // One group of 8 MMA columns holds up to 8 (head, token) pairs, two up to 16.
  const bool two = G * a.Sq > 8;
  switch (G) {
    case 1: return two ? launch_dg<D, 1, 2>(a, s) : launch_dg<D, 1, 1>(a, s);
    case 2: return two ? launch_dg<D, 2, 2>(a, s) : launch_dg<D, 2, 1>(a, s);
    case 4: return two ? launch_dg<D, 4, 2>(a, s) : launch_dg<D, 4, 1>(a, s);
    case 8: return two ? launch_dg<D, 8, 2>(a, s) : launch_dg<D, 8, 1>(a, s);
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
