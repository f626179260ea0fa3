// backward.cu -- gradients of exact attention for an upstream gradient dO.
//
// The forward keeps only O and the row statistics (as the natural-log LSE);
// the backward recomputes S and P tile by tile from Q, K and the LSE instead
// of storing them ("FlashAttention: memory-saving exact attention",
// section 4).  With D_i = rowsum(dO_i * O_i) = sum_j P_ij dP_ij:
//
//   P = exp(S - LSE),  dV = P^T dO,  dP = dO V^T,  dS = P * (dP - D),
//   dQ = scale dS K,   dK = scale dS^T Q
//
// Three kernels:
//   bwd_prep_kernel   D and LSE * log2(e) per (b, head, row), into scratch.
//   bwd_dkdv_kernel   one CTA per (128-key tile, KV head, b): K and V stay in
//                     shared memory while the Q / dO tiles of every query
//                     head of the group stream through a TMA ring, so dK and
//                     dV of a KV head sum over its G query heads without
//                     atomics.  Per Q tile, on the tensor core:
//                       S^T  = K Q^T,   dP^T = V dO^T       (shared x shared)
//                       dV  += P^T dO,  dK  += dS^T Q       (TMEM x shared)
//   bwd_dq_kernel     one CTA per (128-row Q tile, query head, b): Q and dO
//                     stay while the K / V tiles stream through; per K/V tile
//                       S = Q K^T,  dP = dO V^T,  dQ += dS K.
// S and dP are recomputed by both stream kernels (seven products instead of
// five) so that neither needs atomics or a second pass over an fp32 dQ.
//
// Roles (192 threads): warp 0 issues the TMA copies, warp 1 owns TMEM and
// issues the tcgen05 MMAs from an elect.sync-chosen lane, warps 2..5 are the
// element-wise warps (thread <-> TMEM lane <-> key row in the dK/dV kernel,
// query row in the dQ kernel).  An element-wise thread loads its S row from
// TMEM, writes P (bf16 pairs) over the first 64 columns of that row, then
// turns each 32-column chunk of its dP row into dS and writes it (bf16
// pairs) over the front of the dP row: the TMEM-operand MMAs read P and dS
// from there.
//
// TMEM columns: S [0,128), dP [128,256), accumulators from 256 (dV then dK,
// or dQ), d columns each.
#include <cuda_bf16.h>

#include "kernels.h"
#include "ptx_sm100.cuh"
#include "warp_mma.cuh"

namespace eio {
namespace {

constexpr int kT = 128;  // rows of a Q tile, keys of a KV tile: the MMA's M
constexpr int kBThreads = 192;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct BCfg {
  static constexpr int NCH = D / 64;                 // 128-byte column chunks per row
  static constexpr int kChunk = kT * 128;            // one chunk of a 128-row tile
  static constexpr int kTile = NCH * kChunk;         // a 128 x D bf16 tile
  static constexpr int R = D == 64 ? 4 : 2;          // ring stages (two tiles each)
  static constexpr int kOffRing = 2 * kTile;         // after the two resident tiles
  static constexpr int kOffVec = kOffRing + R * 2 * kTile;  // per stage: lse2[128], D[128]
  static constexpr int kOffBar = kOffVec + R * 2 * kT * 4;
  // fixed_full, full[R], empty[R], s_full, dp_full, p_full, ds_full, mma_done, mma_idle
  static constexpr int kNumBars = 1 + 2 * R + 6;
  static constexpr int kSmem = kOffBar + 8 * kNumBars + 16 + 1024;
  static_assert(kSmem <= 227 * 1024, "shared memory per CTA");
};

__device__ __forceinline__ uint8_t* align1k(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// D and lse2 for every (b, head, row), one warp per row.
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const BwdArgs a) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const long long rows = static_cast<long long>(a.B) * a.Hq * a.Nq;
  if (row >= rows) return;
  const int i = static_cast<int>(row % a.Nq);
  const int hq = static_cast<int>((row / a.Nq) % a.Hq);
  const int b = static_cast<int>(row / (static_cast<long long>(a.Nq) * a.Hq));
  const size_t off = ((static_cast<size_t>(b) * a.Nq + i) * a.Hq + hq) * D;
  constexpr int E = D / 32;  // elements per lane
  const __nv_bfloat16* o = reinterpret_cast<const __nv_bfloat16*>(a.o) + off + lane * E;
  const __nv_bfloat16* g = reinterpret_cast<const __nv_bfloat16*>(a.dout) + off + lane * E;
  float acc = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) acc = fmaf(__bfloat162float(o[e]), __bfloat162float(g[e]), acc);
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
  if (lane == 0) {
    a.dvec[row] = acc;
    a.lse2[row] = a.lse[row] * kLog2e;
  }
}

// acc (+)= A B^T over d for two 128-row K-major tiles in shared memory
// (A the M side, B the N side; both 128-byte swizzled, 64-column chunks).
template <int D>
__device__ __forceinline__ void issue_ss(uint32_t d_tmem, uint32_t a_base, uint32_t b_base) {
  constexpr uint32_t id = idesc_bf16_f32(128, 128, 0, 0);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t koff = (kk >> 2) * BCfg<D>::kChunk + (kk & 3) * 32;
    mma_bf16_ss_elect(d_tmem, sdesc_sw128(a_base + koff, 16, 1024), sdesc_sw128(b_base + koff, 16, 1024), id,
                      kk > 0 ? 1u : 0u);
  }
}

// acc (+)= A B over 128 rows: A (128 x 128 bf16) from TMEM, B the 128 x D
// tile in shared memory read with its rows as the reduction (MN-major).
template <int D>
__device__ __forceinline__ void issue_ts(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_base, bool accumulate) {
  constexpr uint32_t id = idesc_bf16_f32(128, D, 0, 1);
#pragma unroll
  for (int kk = 0; kk < kT / 16; ++kk)
    mma_bf16_ts_elect(d_tmem, a_tmem + kk * 8, sdesc_sw128(b_base + kk * 2048, BCfg<D>::kChunk, 1024), id,
                      (accumulate || kk > 0) ? 1u : 0u);
}

// One thread's TMEM row of D fp32 values (times mul) to a bf16 row in HBM;
// dst == nullptr skips the store, have == false stores zeros.  Warp-uniform
// `have`: the TMEM loads are warp-collective.
template <int D>
__device__ __forceinline__ void store_row(uint32_t t, __nv_bfloat16* dst, float mul, bool have) {
#pragma unroll
  for (int c = 0; c < D; c += 32) {
    uint32_t r[32];
    if (have) {
      tmem_ld32(t + c, r);
      tmem_wait_ld();
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) r[i] = 0u;
    }
    if (dst != nullptr) {
#pragma unroll
      for (int u = 0; u < 4; ++u)
        *reinterpret_cast<uint4*>(dst + c + 8 * u) =
            make_uint4(wm_pack_bf16x2(__uint_as_float(r[8 * u + 0]) * mul, __uint_as_float(r[8 * u + 1]) * mul),
                       wm_pack_bf16x2(__uint_as_float(r[8 * u + 2]) * mul, __uint_as_float(r[8 * u + 3]) * mul),
                       wm_pack_bf16x2(__uint_as_float(r[8 * u + 4]) * mul, __uint_as_float(r[8 * u + 5]) * mul),
                       wm_pack_bf16x2(__uint_as_float(r[8 * u + 6]) * mul, __uint_as_float(r[8 * u + 7]) * mul));
    }
  }
}

// dS = P * (dP - D) for one thread's row, 32 columns at a time: dP is read
// from TMEM at t_dp and dS written back (bf16 pairs) over the front of the
// same row, behind the columns still to be read.  dvals(c) gives D for
// column c.
template <typename DFn>
__device__ __forceinline__ void write_ds(uint32_t t_dp, const float* p, DFn dvals) {
#pragma unroll
  for (int c4 = 0; c4 < 4; ++c4) {
    uint32_t dr[32], pk[16];
    tmem_ld32(t_dp + 32 * c4, dr);
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int c = 32 * c4 + 2 * j;
      const float2 dd = dvals(c);
      pk[j] = wm_pack_bf16x2(p[c] * (__uint_as_float(dr[2 * j]) - dd.x),
                             p[c + 1] * (__uint_as_float(dr[2 * j + 1]) - dd.y));
    }
    tmem_st16(t_dp + 16 * c4, pk);
  }
}

// ----------------------------------------------------------------- dK, dV
template <int D>
__global__ void __launch_bounds__(kBThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const BwdArgs a) {
  using C = BCfg<D>;
  constexpr int R = C::R;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1k(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* fixed_full = bars;
  uint64_t* full = bars + 1;
  uint64_t* empty = full + R;
  uint64_t* s_full = empty + R;
  uint64_t* dp_full = s_full + 1;
  uint64_t* p_full = dp_full + 1;
  uint64_t* ds_full = p_full + 1;
  uint64_t* mma_done = ds_full + 1;
  uint64_t* mma_idle = mma_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* vec = reinterpret_cast<float*>(smem + C::kOffVec);  // [R][2][128]: lse2, D

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Linear grid, KV tile slowest: under a causal mask the first tiles have
  // the most Q tiles to visit, so the longest CTAs start first.
  const int per_kt = a.Hkv * a.B;
  const int kt = static_cast<int>(blockIdx.x) / per_kt;
  const int hkv = (static_cast<int>(blockIdx.x) % per_kt) / a.B, b = static_cast<int>(blockIdx.x) % a.B;
  const int G = a.Hq / a.Hkv;
  const int k0 = kt * kT;
  const int off = a.Nkv - a.Nq;  // bottom-right causal alignment
  const int n_qt = (a.Nq + kT - 1) / kT;
  // causal: row i sees key k0 iff i >= k0 - off; earlier Q tiles see none of these keys
  const int first_qt = a.causal ? min(n_qt, max(0, k0 - off) / kT) : 0;
  const int per_head = n_qt - first_qt;
  const int steps = G * per_head;

  if (threadIdx.x == 0) {
    mbar_init(fixed_full, 1);
    for (int s = 0; s < R; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + 4);  // the MMA commit, and each element-wise warp after reading the vectors
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_full, 4);
    mbar_init(ds_full, 4);
    mbar_init(mma_done, 1);
    mbar_init(mma_idle, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto fail = [&](int code) {
    *abort_flag = 1;
    atomicCAS(a.err, 0, code);
  };
  auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
    const bool mine = !*abort_flag && mbar_wait(bar, parity);
    return __all_sync(0xffffffffu, mine);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmDO);
    }
    mbar_arrive_expect_tx_elect(fixed_full, 2 * C::kTile);
#pragma unroll
    for (int ch = 0; ch < C::NCH; ++ch) {
      tma_load_4d_elect(smem + ch * C::kChunk, &tmK, fixed_full, 64 * ch, hkv, k0, b);
      tma_load_4d_elect(smem + C::kTile + ch * C::kChunk, &tmV, fixed_full, 64 * ch, hkv, k0, b);
    }
    bool ok = true;
    int u = 0;
    for (; u < steps; ++u) {
      const int s = u % R;
      if (u >= R && !wwait(&empty[s], ((u / R) - 1) & 1)) {
        ok = false;
        break;
      }
      const int hq = hkv * G + u / per_head, qt = first_qt + u % per_head;
      // This stage's 128 lse2 and D values; rows past Nq get lse2 = +inf,
      // which makes their P exactly 0.
      const size_t vrow = (static_cast<size_t>(b) * a.Hq + hq) * a.Nq;
      float* vs = vec + s * 2 * kT;
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const int i = qt * kT + lane + 32 * h;
        vs[lane + 32 * h] = i < a.Nq ? a.lse2[vrow + i] : INFINITY;
        vs[kT + lane + 32 * h] = i < a.Nq ? a.dvec[vrow + i] : 0.f;
      }
      __syncwarp();
      uint8_t* st = smem + C::kOffRing + s * 2 * C::kTile;
      mbar_arrive_expect_tx_elect(&full[s], 2 * C::kTile);
#pragma unroll
      for (int ch = 0; ch < C::NCH; ++ch) {
        tma_load_4d_elect(st + ch * C::kChunk, &tmQ, &full[s], 64 * ch, hq, qt * kT, b);
        tma_load_4d_elect(st + C::kTile + ch * C::kChunk, &tmDO, &full[s], 64 * ch, hq, qt * kT, b);
      }
    }
    if (!ok && lane == 0) fail(kErrDeviceTimeout);
    // Every copy lands before the CTA retires.
    mbar_wait(fixed_full, 0);
    for (int w = u > R ? u - R : 0; w < u; ++w) mbar_wait(&full[w % R], (w / R) & 1);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t sK = smem_u32(smem), sV = sK + C::kTile;
    bool ok = wwait(fixed_full, 0);
    for (int u = 0; ok && u < steps; ++u) {
      const int s = u % R;
      const uint32_t sQ = smem_u32(smem + C::kOffRing + s * 2 * C::kTile), sdO = sQ + C::kTile;
      // S and dP are rewritten once the previous step's dV / dK MMAs have
      // read P and dS out of their columns.
      if (!wwait(&full[s], (u / R) & 1) || (u > 0 && !wwait(mma_done, (u - 1) & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      issue_ss<D>(tmem, sK, sQ);  // S^T = K Q^T
      mma_commit_elect(s_full);
      issue_ss<D>(tmem + 128, sV, sdO);  // dP^T = V dO^T
      mma_commit_elect(dp_full);
      if (!wwait(p_full, u & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      issue_ts<D>(tmem + 256, tmem, sdO, u > 0);  // dV += P^T dO
      if (!wwait(ds_full, u & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      issue_ts<D>(tmem + 256 + D, tmem + 128, sQ, u > 0);  // dK += dS^T Q
      mma_commit_elect(&empty[s]);
      mma_commit_elect(mma_done);
    }
    if (!ok && lane == 0) fail(kErrDeviceTimeout);
    // Every MMA issued above has finished before TMEM is released.
    mma_commit_elect(mma_idle);
    mbar_wait(mma_idle, 0);
  } else {
    // ------------------------------------------------------------ element-wise
    const int quarter = warp & 3;
    const int key = k0 + quarter * 32 + lane;  // this thread's key (TMEM lane)
    const uint32_t lo = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t t_s = tmem + lo, t_dp = t_s + 128, t_dv = t_s + 256, t_dk = t_s + 256 + D;
    const float sl2 = a.scale * kLog2e;
    bool ok = true;
    for (int u = 0; u < steps; ++u) {
      const int s = u % R;
      const int q0 = (first_qt + u % per_head) * kT;
      if (!wwait(&full[s], (u / R) & 1) || !wwait(s_full, u & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float* vs = vec + s * 2 * kT;
      float p[kT];
      {
        uint32_t sr[kT];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(t_s + 32 * c, sr + 32 * c);
        tmem_wait_ld();
        // causal: query q0 + c sees this key iff c >= key - off - q0
        const bool masked_tile = a.causal && k0 + kT - 1 > q0 + off;
        const int lim = masked_tile ? key - off - q0 : -1;
#pragma unroll
        for (int c = 0; c < kT; c += 4) {
          const float4 l4 = *reinterpret_cast<const float4*>(vs + c);
          const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e)
            p[c + e] = c + e < lim ? 0.f : wm_ex2(fmaf(__uint_as_float(sr[c + e]), sl2, -lv[e]));
        }
      }
      {
        uint32_t pk[32];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int j = 0; j < 32; ++j) pk[j] = wm_pack_bf16x2(p[64 * h + 2 * j], p[64 * h + 2 * j + 1]);
          tmem_st32(t_s + 32 * h, pk);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
      if (!wwait(dp_full, u & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      write_ds(t_dp, p, [&](int c) { return *reinterpret_cast<const float2*>(vs + kT + c); });
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(ds_full);
        mbar_arrive(&empty[s]);
      }
    }
    if (ok && steps > 0) {
      ok = wwait(mma_done, (steps - 1) & 1);
      tc_fence_after();
    }
    if (ok) {
      const size_t o = ((static_cast<size_t>(b) * a.Nkv + key) * a.Hkv + hkv) * D;
      const bool valid = key < a.Nkv;
      store_row<D>(t_dv, valid ? reinterpret_cast<__nv_bfloat16*>(a.dv) + o : nullptr, 1.f, steps > 0);
      store_row<D>(t_dk, valid ? reinterpret_cast<__nv_bfloat16*>(a.dk) + o : nullptr, a.scale, steps > 0);
    } else if (lane == 0) {
      fail(kErrDeviceTimeout);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// -------------------------------------------------------------------- dQ
template <int D>
__global__ void __launch_bounds__(kBThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const BwdArgs a) {
  using C = BCfg<D>;
  constexpr int R = C::R;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1k(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* fixed_full = bars;
  uint64_t* full = bars + 1;
  uint64_t* empty = full + R;
  uint64_t* s_full = empty + R;
  uint64_t* dp_full = s_full + 1;
  uint64_t* ds_full = dp_full + 2;  // p_full is unused here
  uint64_t* mma_done = ds_full + 1;
  uint64_t* mma_idle = mma_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Linear grid, Q tile slowest and last tile first: under a causal mask the
  // last tiles visit the most K/V tiles.
  const int per_qt = a.Hq * a.B;
  const int n_qt = (a.Nq + kT - 1) / kT;
  const int qt = n_qt - 1 - static_cast<int>(blockIdx.x) / per_qt;
  const int hq = (static_cast<int>(blockIdx.x) % per_qt) / a.B, b = static_cast<int>(blockIdx.x) % a.B;
  const int hkv = hq / (a.Hq / a.Hkv);
  const int q0 = qt * kT;
  const int off = a.Nkv - a.Nq;
  int n_kv = (a.Nkv + kT - 1) / kT;
  if (a.causal) {
    const int last = min(q0 + kT - 1, a.Nq - 1) + off;  // largest key any row may see
    n_kv = last < 0 ? 0 : min(n_kv, last / kT + 1);
  }

  if (threadIdx.x == 0) {
    mbar_init(fixed_full, 1);
    for (int s = 0; s < R; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(ds_full, 4);
    mbar_init(mma_done, 1);
    mbar_init(mma_idle, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto fail = [&](int code) {
    *abort_flag = 1;
    atomicCAS(a.err, 0, code);
  };
  auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
    const bool mine = !*abort_flag && mbar_wait(bar, parity);
    return __all_sync(0xffffffffu, mine);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
    mbar_arrive_expect_tx_elect(fixed_full, 2 * C::kTile);
#pragma unroll
    for (int ch = 0; ch < C::NCH; ++ch) {
      tma_load_4d_elect(smem + ch * C::kChunk, &tmQ, fixed_full, 64 * ch, hq, q0, b);
      tma_load_4d_elect(smem + C::kTile + ch * C::kChunk, &tmDO, fixed_full, 64 * ch, hq, q0, b);
    }
    bool ok = true;
    int j = 0;
    for (; j < n_kv; ++j) {
      const int s = j % R;
      if (j >= R && !wwait(&empty[s], ((j / R) - 1) & 1)) {
        ok = false;
        break;
      }
      uint8_t* st = smem + C::kOffRing + s * 2 * C::kTile;
      mbar_arrive_expect_tx_elect(&full[s], 2 * C::kTile);
#pragma unroll
      for (int ch = 0; ch < C::NCH; ++ch) {
        tma_load_4d_elect(st + ch * C::kChunk, &tmK, &full[s], 64 * ch, hkv, j * kT, b);
        tma_load_4d_elect(st + C::kTile + ch * C::kChunk, &tmV, &full[s], 64 * ch, hkv, j * kT, b);
      }
    }
    if (!ok && lane == 0) fail(kErrDeviceTimeout);
    mbar_wait(fixed_full, 0);
    for (int w = j > R ? j - R : 0; w < j; ++w) mbar_wait(&full[w % R], (w / R) & 1);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t sQ = smem_u32(smem), sdO = sQ + C::kTile;
    bool ok = wwait(fixed_full, 0);
    for (int j = 0; ok && j < n_kv; ++j) {
      const int s = j % R;
      const uint32_t sK = smem_u32(smem + C::kOffRing + s * 2 * C::kTile), sV = sK + C::kTile;
      // S is rewritten once the previous dQ MMA has read dS out of its columns.
      if (!wwait(&full[s], (j / R) & 1) || (j > 0 && !wwait(mma_done, (j - 1) & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      issue_ss<D>(tmem, sQ, sK);  // S = Q K^T
      mma_commit_elect(s_full);
      issue_ss<D>(tmem + 128, sdO, sV);  // dP = dO V^T
      mma_commit_elect(dp_full);
      if (!wwait(ds_full, j & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      issue_ts<D>(tmem + 256, tmem + 128, sK, j > 0);  // dQ += dS K
      mma_commit_elect(&empty[s]);
      mma_commit_elect(mma_done);
    }
    if (!ok && lane == 0) fail(kErrDeviceTimeout);
    mma_commit_elect(mma_idle);
    mbar_wait(mma_idle, 0);
  } else {
    // ------------------------------------------------------------ element-wise
    const int quarter = warp & 3;
    const int row = q0 + quarter * 32 + lane;  // this thread's query row (TMEM lane)
    const uint32_t lo = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t t_s = tmem + lo, t_dp = t_s + 128, t_dq = t_s + 256;
    const float sl2 = a.scale * kLog2e;
    const size_t vrow = (static_cast<size_t>(b) * a.Hq + hq) * a.Nq;
    // rows past Nq: lse2 = +inf makes their P exactly 0
    const float l2 = row < a.Nq ? a.lse2[vrow + row] : INFINITY;
    const float dd = row < a.Nq ? a.dvec[vrow + row] : 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      if (!wwait(s_full, j & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // keys at or past column lim are masked: past Nkv, and past the
      // causal diagonal (rows with no visible key get lim <= 0)
      int lim = min(kT, a.Nkv - j * kT);
      if (a.causal) lim = min(lim, row + off + 1 - j * kT);
      float p[kT];
      {
        uint32_t sr[kT];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(t_s + 32 * c, sr + 32 * c);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < kT; ++c) p[c] = c < lim ? wm_ex2(fmaf(__uint_as_float(sr[c]), sl2, -l2)) : 0.f;
      }
      if (!wwait(dp_full, j & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      write_ds(t_dp, p, [&](int) { return make_float2(dd, dd); });
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(ds_full);
    }
    if (ok && n_kv > 0) {
      ok = wwait(mma_done, (n_kv - 1) & 1);
      tc_fence_after();
    }
    if (ok) {
      __nv_bfloat16* dst = row < a.Nq ? reinterpret_cast<__nv_bfloat16*>(a.dq) +
                                            ((static_cast<size_t>(b) * a.Nq + row) * a.Hq + hq) * D
                                      : nullptr;
      store_row<D>(t_dq, dst, a.scale, n_kv > 0);
    } else if (lane == 0) {
      fail(kErrDeviceTimeout);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int D>
cudaError_t launch_bwd_d(const BwdArgs& a, cudaStream_t s) {
  using C = BCfg<D>;
  static int attr_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (attr_dev != dev) {
    cudaError_t e = cudaFuncSetAttribute(bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    attr_dev = dev;
  }
  CUtensorMap tq, tdo, tk, tv;
  if (!encode_bf16_map(&tq, a.q, a.B, a.Nq, a.Hq, D, kT) || !encode_bf16_map(&tdo, a.dout, a.B, a.Nq, a.Hq, D, kT) ||
      !encode_bf16_map(&tk, a.k, a.B, a.Nkv, a.Hkv, D, kT) || !encode_bf16_map(&tv, a.v, a.B, a.Nkv, a.Hkv, D, kT))
    return cudaErrorInvalidValue;
  const long long rows = static_cast<long long>(a.B) * a.Hq * a.Nq;
  bwd_prep_kernel<D><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long n_qt = (a.Nq + kT - 1) / kT, n_kt = (a.Nkv + kT - 1) / kT;
  bwd_dq_kernel<D><<<static_cast<unsigned>(n_qt * a.Hq * a.B), kBThreads, C::kSmem, s>>>(tq, tdo, tk, tv, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  bwd_dkdv_kernel<D><<<static_cast<unsigned>(n_kt * a.Hkv * a.B), kBThreads, C::kSmem, s>>>(tq, tdo, tk, tv, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd(int d, const BwdArgs& a, cudaStream_t s) {
  if (d == 64) return launch_bwd_d<64>(a, s);
  return launch_bwd_d<128>(a, s);
}

}  // namespace eio
