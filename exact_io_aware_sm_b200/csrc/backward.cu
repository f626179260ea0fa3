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
// Two kernels, launched in this order:
//   bwd_dq_kernel     one CTA per (128-row Q tile, query head, b): Q, dO and
//                     O stay in shared memory while the K / V tiles stream
//                     through a TMA ring; per K/V tile, on the tensor core,
//                       S = Q K^T,  dP = dO V^T       (shared x shared)
//                       dQ += dS K                    (TMEM x shared)
//                     Its element-wise threads compute D from the O and dO
//                     tiles (while dP of the first tile is on the tensor
//                     core) and leave D and LSE*log2(e) in a scratch whose
//                     rows are padded to whole tiles (lse2 = +inf, D = 0).
//                     The dK/dV kernel fetches 128-row runs of both with bulk
//                     copies on the same barrier as its Q / dO tiles.
//   bwd_dkdv_kernel   one CTA per (128-key tile, KV head, b): K and V stay
//                     while the Q / dO tiles of every query head of the group
//                     stream through, so dK and dV of a KV head sum over its
//                     G query heads without atomics; per Q tile
//                       S^T = K Q^T,  dP^T = V dO^T
//                       dV += P^T dO,  dK += dS^T Q
// S and dP are recomputed by both kernels (seven products instead of five)
// so that neither needs atomics or a second pass over an fp32 dQ.
//
// Roles (320 threads): warp 0 issues the TMA copies, warp 1 owns TMEM and
// issues the tcgen05 MMAs from an elect.sync-chosen lane, warps 2..9 are two
// element-wise warpgroups: warpgroup h takes columns [64h, 64h+64) of every
// S and dP row (thread <-> TMEM lane <-> key row in the dK/dV kernel, query
// row in the dQ kernel).  A thread loads its 64 S values, writes P (bf16
// pairs, 32 columns) over the front of that same column range, then turns
// its dP values into dS and writes them (32 columns) behind P: dK/dV reads P
// from columns [64h, 64h+32) and dS from [64h+32, 64h+64); the dQ kernel
// keeps only dS, at [64h, 64h+32).  No warpgroup writes a column that the
// other still has to read, and dP is never written, so dP(t+1) may start as
// soon as both warpgroups have read dP(t).
//
// S is double-buffered in TMEM where the columns allow (dQ kernel; dK/dV
// kernel at d = 64): S(t+1) then runs on the tensor core while the
// element-wise warps still work on tile t.
//   dQ:         S0 [0,128) S1 [128,256) dP [256,384) dQ [384, 384+d)
//   dK/dV d=64: S0 [0,128) S1 [128,256) dP [256,384) dV [384,448) dK [448,512)
//   dK/dV d=128: S [0,128) dP [128,256) dV [256,384) dK [384,512)
#include <cuda_bf16.h>

#include "kernels.h"
#include "ptx_sm100.cuh"
#include "warp_mma.cuh"

namespace eio {
namespace {

constexpr int kT = 128;  // rows of a Q tile, keys of a KV tile: the MMA's M
constexpr int kBThreads = 320;
constexpr int kEW = 8;   // element-wise warps
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct BCfg {
  static constexpr int NCH = D / 64;                 // 128-byte column chunks per row
  static constexpr int kChunk = kT * 128;            // one chunk of a 128-row tile
  static constexpr int kTile = NCH * kChunk;         // a 128 x D bf16 tile
  static constexpr int R = D == 64 ? 4 : 2;          // ring stages (two tiles each)
  static constexpr int kOffRing = 2 * kTile;         // after the two resident tiles
  // dK/dV kernel: per stage lse2[128], D[128]; dQ kernel: the O tile
  static constexpr int kOffX = kOffRing + R * 2 * kTile;
  static constexpr int kOffBarKV = kOffX + R * 2 * kT * 4;
  static constexpr int kOffBarQ = kOffX + kTile;
  // fixed_full, full[R], empty[R], s_full[2], dp_full, p_full, ds_full, mma_done, mma_idle
  static constexpr int kNumBars = 1 + 2 * R + 7;
  static constexpr int kSmemKV = kOffBarKV + 8 * kNumBars + 16 + 1024;
  static constexpr int kSmemQ = kOffBarQ + 8 * kNumBars + 16 + 1024;
  static_assert(kSmemKV <= 227 * 1024 && kSmemQ <= 227 * 1024, "shared memory per CTA");
  static constexpr int kVecBytes = 2 * kT * 4;
  // S buffers in TMEM (dK/dV kernel; the dQ kernel always has two)
  static constexpr int kSBufKV = D == 64 ? 2 : 1;
};

__device__ __forceinline__ uint8_t* align1k(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// acc = A B^T over d for two 128-row K-major tiles in shared memory (A the M
// side, B the N side; both 128-byte swizzled, 64-column chunks).
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
// tile in shared memory read with its rows as the reduction (MN-major).  A's
// 64 packed columns sit in two runs of 32: [a, a+32) for reduction rows
// 0..63 and [a+64, a+96) for rows 64..127.
template <int D>
__device__ __forceinline__ void issue_ts(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_base, bool accumulate) {
  constexpr uint32_t id = idesc_bf16_f32(128, D, 0, 1);
#pragma unroll
  for (int kk = 0; kk < kT / 16; ++kk)
    mma_bf16_ts_elect(d_tmem, a_tmem + kk * 8 + (kk >= 4 ? 32 : 0),
                      sdesc_sw128(b_base + kk * 2048, BCfg<D>::kChunk, 1024), id, (accumulate || kk > 0) ? 1u : 0u);
}

// NC columns of one thread's TMEM row (times mul) to bf16 in HBM; dst ==
// nullptr skips the store, have == false stores zeros.  `have` is
// warp-uniform: the TMEM loads are warp-collective.
template <int NC>
__device__ __forceinline__ void store_cols(uint32_t t, __nv_bfloat16* dst, float mul, bool have) {
#pragma unroll
  for (int c = 0; c < NC; c += 32) {
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

// dS = P * (dP - D) for one thread's 64 columns: dP read from TMEM at t_dp,
// dS written (bf16 pairs, 32 columns) at t_ds.  dvals(c) gives D for the
// columns c, c + 1.
template <typename DFn>
__device__ __forceinline__ void write_ds(uint32_t t_dp, uint32_t t_ds, const float* p, DFn dvals) {
  uint32_t dr[64], pk[32];
  tmem_ld32(t_dp, dr);
  tmem_ld32(t_dp + 32, dr + 32);
  tmem_wait_ld();
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float2 dd = dvals(2 * j);
    pk[j] = wm_pack_bf16x2(p[2 * j] * (__uint_as_float(dr[2 * j]) - dd.x),
                           p[2 * j + 1] * (__uint_as_float(dr[2 * j + 1]) - dd.y));
  }
  tmem_st32(t_ds, pk);
}

// ----------------------------------------------------------------- dK, dV
template <int D>
__global__ void __launch_bounds__(kBThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const BwdArgs a) {
  using C = BCfg<D>;
  constexpr int R = C::R, NB = C::kSBufKV;
  constexpr uint32_t kColDP = 128 * NB, kColDV = kColDP + 128, kColDK = kColDV + D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1k(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBarKV);
  uint64_t* fixed_full = bars;
  uint64_t* full = bars + 1;
  uint64_t* empty = full + R;
  uint64_t* s_full = empty + R;  // [2]
  uint64_t* dp_full = s_full + 2;
  uint64_t* p_full = dp_full + 1;
  uint64_t* ds_full = p_full + 1;
  uint64_t* mma_done = ds_full + 1;
  uint64_t* mma_idle = mma_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* vec = reinterpret_cast<float*>(smem + C::kOffX);  // [R][2][128]: lse2, D

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
  const int nq_pad = n_qt * kT;  // rows per (b, head) of the lse2 / D scratch
  // causal: row i sees key k0 iff i >= k0 - off; earlier Q tiles see none of these keys
  const int first_qt = a.causal ? min(n_qt, max(0, k0 - off) / kT) : 0;
  const int per_head = n_qt - first_qt;
  const int steps = G * per_head;

  if (threadIdx.x == 0) {
    mbar_init(fixed_full, 1);
    for (int s = 0; s < R; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + kEW);  // the MMA commit, and each element-wise warp after reading the vectors
    }
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(dp_full, 1);
    mbar_init(p_full, kEW);
    mbar_init(ds_full, kEW);
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
      uint8_t* st = smem + C::kOffRing + s * 2 * C::kTile;
      mbar_arrive_expect_tx_elect(&full[s], 2 * C::kTile + C::kVecBytes);
#pragma unroll
      for (int ch = 0; ch < C::NCH; ++ch) {
        tma_load_4d_elect(st + ch * C::kChunk, &tmQ, &full[s], 64 * ch, hq, qt * kT, b);
        tma_load_4d_elect(st + C::kTile + ch * C::kChunk, &tmDO, &full[s], 64 * ch, hq, qt * kT, b);
      }
      // the tile's 128 lse2 and D values (padded rows: lse2 = +inf, D = 0)
      const size_t vrow = (static_cast<size_t>(b) * a.Hq + hq) * nq_pad + static_cast<size_t>(qt) * kT;
      bulk_load_elect(vec + s * 2 * kT, a.lse2 + vrow, kT * 4, &full[s]);
      bulk_load_elect(vec + s * 2 * kT + kT, a.dvec + vrow, kT * 4, &full[s]);
    }
    if (!ok && lane == 0) fail(kErrDeviceTimeout);
    // Every copy lands before the CTA retires.
    mbar_wait(fixed_full, 0);
    for (int w = u > R ? u - R : 0; w < u; ++w) mbar_wait(&full[w % R], (w / R) & 1);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Issue order per step t: S(t+1) (two S buffers), dV(t), dK(t), then
    // dP(t+1) -- the element-wise warps have read dP(t) by then.
    const uint32_t sK = smem_u32(smem), sV = sK + C::kTile;
    auto stage = [&](int t) { return smem_u32(smem + C::kOffRing + (t % R) * 2 * C::kTile); };
    bool ok = wwait(fixed_full, 0) && (steps == 0 || wwait(&full[0], 0));
    if (ok && steps > 0) {
      tc_fence_after();
      issue_ss<D>(tmem, sK, stage(0));  // S^T = K Q^T
      mma_commit_elect(&s_full[0]);
      issue_ss<D>(tmem + kColDP, sV, stage(0) + C::kTile);  // dP^T = V dO^T
      mma_commit_elect(dp_full);
    }
    for (int u = 0; ok && u < steps; ++u) {
      const int s = u % R, x = u % NB;
      const uint32_t sQ = stage(u), sdO = sQ + C::kTile;
      const bool next = u + 1 < steps;
      if (NB == 2 && next) {
        // S buffer (u+1)%2 was last read by dV(u-1) / dK(u-1)
        if (!wwait(&full[(u + 1) % R], ((u + 1) / R) & 1) || (u >= 1 && !wwait(mma_done, (u - 1) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_ss<D>(tmem + 128 * ((u + 1) % NB), sK, stage(u + 1));
        mma_commit_elect(&s_full[(u + 1) % NB]);
      }
      if (!wwait(p_full, u & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      issue_ts<D>(tmem + kColDV, tmem + 128 * x, sdO, u > 0);  // dV += P^T dO
      if (!wwait(ds_full, u & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      issue_ts<D>(tmem + kColDK, tmem + 128 * x + 32, sQ, u > 0);  // dK += dS^T Q
      mma_commit_elect(&empty[s]);
      mma_commit_elect(mma_done);
      if (next) {
        if (NB == 1) {
          // one S buffer: S(u+1) after dV(u) / dK(u) have read it
          if (!wwait(&full[(u + 1) % R], ((u + 1) / R) & 1) || !wwait(mma_done, u & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_ss<D>(tmem, sK, stage(u + 1));
          mma_commit_elect(&s_full[0]);
        }
        issue_ss<D>(tmem + kColDP, sV, stage(u + 1) + C::kTile);
        mma_commit_elect(dp_full);
      }
    }
    if (!ok && lane == 0) fail(kErrDeviceTimeout);
    // Every MMA issued above has finished before TMEM is released.
    mma_commit_elect(mma_idle);
    mbar_wait(mma_idle, 0);
  } else {
    // ------------------------------------------------------------ element-wise
    const int h = (warp - 2) >> 2;  // column half
    const int quarter = warp & 3;
    const int key = k0 + quarter * 32 + lane;  // this thread's key (TMEM lane)
    const uint32_t lo = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t t_row = tmem + lo;
    const float sl2 = a.scale * kLog2e;
    bool ok = true;
    for (int u = 0; u < steps; ++u) {
      const int s = u % R, x = u % NB;
      const int q0 = (first_qt + u % per_head) * kT + 64 * h;  // query of this thread's first column
      if (!wwait(&full[s], (u / R) & 1) || !wwait(&s_full[x], (u / NB) & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float* vs = vec + s * 2 * kT + 64 * h;
      const uint32_t t_s = t_row + 128 * x + 64 * h;
      float p[64];
      {
        uint32_t sr[64];
        tmem_ld32(t_s, sr);
        tmem_ld32(t_s + 32, sr + 32);
        tmem_wait_ld();
        // causal: query q0 + c sees this key iff c >= key - off - q0
        const bool masked_tile = a.causal && k0 + kT - 1 > q0 + off;
        const int lim = masked_tile ? key - off - q0 : -1;
#pragma unroll
        for (int c = 0; c < 64; c += 4) {
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
        for (int j = 0; j < 32; ++j) pk[j] = wm_pack_bf16x2(p[2 * j], p[2 * j + 1]);
        tmem_st32(t_s, pk);
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
      write_ds(t_row + kColDP + 64 * h, t_s + 32, p,
               [&](int c) { return *reinterpret_cast<const float2*>(vs + kT + c); });
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
      // each warpgroup stores half of the columns of dV and dK
      constexpr int HC = D / 2;
      const size_t o = ((static_cast<size_t>(b) * a.Nkv + key) * a.Hkv + hkv) * D + HC * h;
      const bool valid = key < a.Nkv;
      store_cols<HC>(t_row + kColDV + HC * h, valid ? reinterpret_cast<__nv_bfloat16*>(a.dv) + o : nullptr, 1.f,
                     steps > 0);
      store_cols<HC>(t_row + kColDK + HC * h, valid ? reinterpret_cast<__nv_bfloat16*>(a.dk) + o : nullptr,
                     a.scale, steps > 0);
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
                  const __grid_constant__ CUtensorMap tmO, const BwdArgs a) {
  using C = BCfg<D>;
  constexpr int R = C::R;
  constexpr uint32_t kColDP = 256, kColDQ = 384;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1k(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBarQ);
  uint64_t* fixed_full = bars;
  uint64_t* full = bars + 1;
  uint64_t* empty = full + R;
  uint64_t* s_full = empty + R;  // [2]
  uint64_t* dp_full = s_full + 2;
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
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(dp_full, 1);
    mbar_init(ds_full, kEW);
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
    mbar_arrive_expect_tx_elect(fixed_full, 3 * C::kTile);
#pragma unroll
    for (int ch = 0; ch < C::NCH; ++ch) {
      tma_load_4d_elect(smem + ch * C::kChunk, &tmQ, fixed_full, 64 * ch, hq, q0, b);
      tma_load_4d_elect(smem + C::kTile + ch * C::kChunk, &tmDO, fixed_full, 64 * ch, hq, q0, b);
      tma_load_4d_elect(smem + C::kOffX + ch * C::kChunk, &tmO, fixed_full, 64 * ch, hq, q0, b);
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
    // Issue order per step t: S(t+1) into the other S buffer, dQ(t), then
    // dP(t+1) -- the element-wise warps have read dP(t) by then.
    const uint32_t sQ = smem_u32(smem), sdO = sQ + C::kTile;
    auto stage = [&](int t) { return smem_u32(smem + C::kOffRing + (t % R) * 2 * C::kTile); };
    bool ok = wwait(fixed_full, 0) && (n_kv == 0 || wwait(&full[0], 0));
    if (ok && n_kv > 0) {
      tc_fence_after();
      issue_ss<D>(tmem, sQ, stage(0));  // S = Q K^T
      mma_commit_elect(&s_full[0]);
      issue_ss<D>(tmem + kColDP, sdO, stage(0) + C::kTile);  // dP = dO V^T
      mma_commit_elect(dp_full);
    }
    for (int j = 0; ok && j < n_kv; ++j) {
      const int s = j % R, x = j & 1;
      const bool next = j + 1 < n_kv;
      if (next) {
        // S buffer (j+1)%2 was last read by dQ(j-1)
        if (!wwait(&full[(j + 1) % R], ((j + 1) / R) & 1) || (j >= 1 && !wwait(mma_done, (j - 1) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_ss<D>(tmem + 128 * (x ^ 1), sQ, stage(j + 1));
        mma_commit_elect(&s_full[x ^ 1]);
      }
      if (!wwait(ds_full, j & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      issue_ts<D>(tmem + kColDQ, tmem + 128 * x, stage(j), j > 0);  // dQ += dS K
      mma_commit_elect(&empty[s]);
      mma_commit_elect(mma_done);
      if (next) {
        issue_ss<D>(tmem + kColDP, sdO, stage(j + 1) + C::kTile);
        mma_commit_elect(dp_full);
      }
    }
    if (!ok && lane == 0) fail(kErrDeviceTimeout);
    mma_commit_elect(mma_idle);
    mbar_wait(mma_idle, 0);
  } else {
    // ------------------------------------------------------------ element-wise
    const int h = (warp - 2) >> 2;  // column half
    const int quarter = warp & 3;
    const int row = q0 + quarter * 32 + lane;  // this thread's query row (TMEM lane)
    const uint32_t lo = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t t_row = tmem + lo;
    const float sl2 = a.scale * kLog2e;
    // rows past Nq: lse2 = +inf makes their P exactly 0
    const float l2 = row < a.Nq ? a.lse[(static_cast<size_t>(b) * a.Hq + hq) * a.Nq + row] * kLog2e : INFINITY;
    // D = rowsum(dO * O) from the resident O and dO tiles (zero rows past
    // Nq); with lse2 it goes to the padded scratch for the dK/dV kernel.
    float dd = 0.f;
    auto compute_d = [&]() -> bool {
      if (!wwait(fixed_full, 0)) return false;
      const int r = quarter * 32 + lane;
#pragma unroll
      for (int ch = 0; ch < C::NCH; ++ch)
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int o = ch * C::kChunk + r * 128 + ((u ^ (r & 7)) << 4);
          const uint4 ov = *reinterpret_cast<const uint4*>(smem + C::kOffX + o);
          const uint4 gv = *reinterpret_cast<const uint4*>(smem + C::kTile + o);
          const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
          const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gv);
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const float2 of = __bfloat1622float2(o2[w]), gf = __bfloat1622float2(g2[w]);
            dd = fmaf(of.x, gf.x, dd);
            dd = fmaf(of.y, gf.y, dd);
          }
        }
      if (h == 0) {
        const size_t vrow = (static_cast<size_t>(b) * a.Hq + hq) * (n_qt * kT) + row;
        a.dvec[vrow] = dd;
        a.lse2[vrow] = l2;
      }
      return true;
    };
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int x = j & 1;
      if (!wwait(&s_full[x], (j >> 1) & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // keys at or past column lim are masked: past Nkv, and past the
      // causal diagonal (rows with no visible key get lim <= 0)
      const int c0 = j * kT + 64 * h;  // key of this thread's first column
      int lim = min(64, a.Nkv - c0);
      if (a.causal) lim = min(lim, row + off + 1 - c0);
      const uint32_t t_s = t_row + 128 * x + 64 * h;
      float p[64];
      {
        uint32_t sr[64];
        tmem_ld32(t_s, sr);
        tmem_ld32(t_s + 32, sr + 32);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 64; ++c) p[c] = c < lim ? wm_ex2(fmaf(__uint_as_float(sr[c]), sl2, -l2)) : 0.f;
      }
      // D while dP(0) is on the tensor core
      if (j == 0 && !compute_d()) {
        ok = false;
        break;
      }
      if (!wwait(dp_full, j & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      write_ds(t_row + kColDP + 64 * h, t_s, p, [&](int) { return make_float2(dd, dd); });
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(ds_full);
    }
    if (ok && n_kv == 0) ok = compute_d();
    if (ok && n_kv > 0) {
      ok = wwait(mma_done, (n_kv - 1) & 1);
      tc_fence_after();
    }
    if (ok) {
      constexpr int HC = D / 2;
      __nv_bfloat16* dst = row < a.Nq ? reinterpret_cast<__nv_bfloat16*>(a.dq) +
                                            ((static_cast<size_t>(b) * a.Nq + row) * a.Hq + hq) * D + HC * h
                                      : nullptr;
      store_cols<HC>(t_row + kColDQ + HC * h, dst, a.scale, n_kv > 0);
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
    cudaError_t e = cudaFuncSetAttribute(bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemQ);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemKV);
    if (e != cudaSuccess) return e;
    attr_dev = dev;
  }
  CUtensorMap tq, tdo, tk, tv, to;
  if (!encode_bf16_map(&tq, a.q, a.B, a.Nq, a.Hq, D, kT) || !encode_bf16_map(&tdo, a.dout, a.B, a.Nq, a.Hq, D, kT) ||
      !encode_bf16_map(&tk, a.k, a.B, a.Nkv, a.Hkv, D, kT) || !encode_bf16_map(&tv, a.v, a.B, a.Nkv, a.Hkv, D, kT) ||
      !encode_bf16_map(&to, a.o, a.B, a.Nq, a.Hq, D, kT))
    return cudaErrorInvalidValue;
  const long long n_qt = (a.Nq + kT - 1) / kT, n_kt = (a.Nkv + kT - 1) / kT;
  // The dQ kernel also writes D and lse2, which the dK/dV kernel reads.
  bwd_dq_kernel<D><<<static_cast<unsigned>(n_qt * a.Hq * a.B), kBThreads, C::kSmemQ, s>>>(tq, tdo, tk, tv, to, a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  bwd_dkdv_kernel<D><<<static_cast<unsigned>(n_kt * a.Hkv * a.B), kBThreads, C::kSmemKV, s>>>(tq, tdo, tk, tv, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd(int d, const BwdArgs& a, cudaStream_t s) {
  if (d == 64) return launch_bwd_d<64>(a, s);
  return launch_bwd_d<128>(a, s);
}

}  // namespace eio
