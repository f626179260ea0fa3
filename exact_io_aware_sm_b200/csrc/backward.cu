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
//   bwd_dq_kernel     one CTA per (64-row Q tile, query head, b): the Q and
//                     dO tiles stay in shared memory while 64-key K/V tiles
//                     stream through a TMA ring; dQ accumulates in registers.
//   bwd_dkdv_kernel   one CTA per (64-key tile, KV head, b): the K and V tiles
//                     stay while the Q/dO tiles of every query head of the
//                     group stream through, so dK and dV of a KV head sum over
//                     its G query heads without atomics.
// Both stream kernels have four compute warps (16 rows or keys each) and one
// TMA producer warp; the products run as m16n8k16 warp MMAs on register
// fragments read with ldmatrix from 128-byte-swizzled tiles.
#include <cuda_bf16.h>

#include "kernels.h"
#include "ptx_sm100.cuh"
#include "warp_mma.cuh"

namespace eio {
namespace {

constexpr int kBT = 64;      // rows of a Q tile and keys of a KV tile
constexpr int kCW = 4;       // compute warps (16 rows or keys each); warp 4 produces
constexpr int kBThreads = (kCW + 1) * 32;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct BCfg {
  static constexpr int KB = D / 64;                  // 128-byte column blocks per row
  static constexpr int kBlock = kBT * 128;           // one column block of a 64-row tile
  static constexpr int kTile = KB * kBlock;          // a 64 x D bf16 tile
  static constexpr int kCtas = D == 64 ? 2 : 1;       // CTAs per SM (d = 128: registers for the accumulators)
  static constexpr int R = D == 64 ? 3 : 4;          // ring stages (two tiles each)
  static constexpr int kOffRing = 2 * kTile;         // after the two resident tiles
  static constexpr int kOffVec = kOffRing + R * 2 * kTile;  // per stage: lse2[64], D[64]
  static constexpr int kOffBars = kOffVec + R * 2 * kBT * 4;
  static constexpr int kSmem = kOffBars + 8 * (2 * R + 1) + 16 + 1024;
  static_assert(kSmem <= (kCtas == 2 ? 113 : 227) * 1024, "shared memory per CTA");
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

template <int D>
__global__ void __launch_bounds__(kBThreads, BCfg<D>::kCtas)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const BwdArgs a) {
  using C = BCfg<D>;
  constexpr int R = C::R, NK = D / 16;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1k(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBars);
  uint64_t* fixed_full = bars;
  uint64_t* full = bars + 1;
  uint64_t* empty = full + R;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int n_qt = gridDim.x;
  const int qt = n_qt - 1 - static_cast<int>(blockIdx.x);  // causal: longest tiles first
  const int hq = blockIdx.y, b = blockIdx.z;
  const int G = a.Hq / a.Hkv, hkv = hq / G;
  const int q0 = qt * kBT;
  const int off = a.Nkv - a.Nq;  // bottom-right causal alignment
  int n_kv = (a.Nkv + kBT - 1) / kBT;
  if (a.causal) {
    const int last = min(q0 + kBT - 1, a.Nq - 1) + off;  // largest key any row may see
    n_kv = last < 0 ? 0 : min(n_kv, last / kBT + 1);
  }

  if (threadIdx.x == 0) {
    mbar_init(fixed_full, 1);
    for (int s = 0; s < R; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCW);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kCW) {
    // ------------------------------------------------------------ producer
    mbar_arrive_expect_tx_elect(fixed_full, 2 * C::kTile);
#pragma unroll
    for (int h = 0; h < C::KB; ++h) {
      tma_load_4d_elect(smem + h * C::kBlock, &tmQ, fixed_full, 64 * h, hq, q0, b);
      tma_load_4d_elect(smem + C::kTile + h * C::kBlock, &tmDO, fixed_full, 64 * h, hq, q0, b);
    }
    bool ok = true;
    int j = 0;
    for (; j < n_kv; ++j) {
      const int s = j % R;
      if (j >= R && !__all_sync(0xffffffffu, mbar_wait(&empty[s], ((j / R) + 1) & 1))) {
        ok = false;
        break;
      }
      uint8_t* st = smem + C::kOffRing + s * 2 * C::kTile;
      mbar_arrive_expect_tx_elect(&full[s], 2 * C::kTile);
#pragma unroll
      for (int h = 0; h < C::KB; ++h) {
        tma_load_4d_elect(st + h * C::kBlock, &tmK, &full[s], 64 * h, hkv, j * kBT, b);
        tma_load_4d_elect(st + C::kTile + h * C::kBlock, &tmV, &full[s], 64 * h, hkv, j * kBT, b);
      }
    }
    if (!ok && lane == 0) atomicCAS(a.err, 0, kErrDeviceTimeout);
    // Every copy lands before the CTA retires.
    mbar_wait(fixed_full, 0);
    for (int u = j > R ? j - R : 0; u < j; ++u) mbar_wait(&full[u % R], (u / R) & 1);
    return;
  }

  // ------------------------------------------------------------ compute warps
  const float sl2 = a.scale * kLog2e;
  const int rA = q0 + 16 * warp + g, rB = rA + 8;  // this lane's two rows
  const size_t vrow = (static_cast<size_t>(b) * a.Hq + hq) * a.Nq;
  // rows past Nq: lse2 = +inf makes their P exactly 0
  const float lseA = rA < a.Nq ? a.lse2[vrow + rA] : INFINITY, lseB = rB < a.Nq ? a.lse2[vrow + rB] : INFINITY;
  const float dA = rA < a.Nq ? a.dvec[vrow + rA] : 0.f, dB = rB < a.Nq ? a.dvec[vrow + rB] : 0.f;

  float dq[NK * 2][4];
#pragma unroll
  for (int n = 0; n < NK * 2; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) dq[n][e] = 0.f;

  bool ok = __all_sync(0xffffffffu, mbar_wait(fixed_full, 0));
  const uint32_t sq = smem_u32(smem), sdo = sq + C::kTile;
  uint32_t qa[NK][4], da[NK][4];
  {
    const int r = 16 * warp + ((lane >> 3) & 1) * 8 + (lane & 7);
#pragma unroll
    for (int ks = 0; ks < NK; ++ks) {
      const uint32_t o = (ks >> 2) * C::kBlock + sw128(r, (ks & 3) * 2 + (lane >> 4));
      ldsm_x4(sq + o, qa[ks]);
      ldsm_x4(sdo + o, da[ks]);
    }
  }

  for (int j = 0; ok && j < n_kv; ++j) {
    const int s = j % R;
    if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (j / R) & 1))) {
      ok = false;
      break;
    }
    const uint32_t sk = smem_u32(smem + C::kOffRing + s * 2 * C::kTile), sv = sk + C::kTile;
#pragma unroll
    for (int kc = 0; kc < kBT / 16; ++kc) {
      float S[2][4] = {}, dP[2][4] = {};
      {
        const int m = lane >> 3;
        const int kr = kc * 16 + (m >> 1) * 8 + (lane & 7);
#pragma unroll
        for (int ks = 0; ks < NK; ++ks) {
          const uint32_t o = (ks >> 2) * C::kBlock + sw128(kr, (ks & 3) * 2 + (m & 1));
          uint32_t kb[4], vb[4];
          ldsm_x4(sk + o, kb);
          ldsm_x4(sv + o, vb);
          mma_16816(S[0], qa[ks], kb[0], kb[1]);
          mma_16816(S[1], qa[ks], kb[2], kb[3]);
          mma_16816(dP[0], da[ks], vb[0], vb[1]);
          mma_16816(dP[1], da[ks], vb[2], vb[3]);
        }
      }
      float ds[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = j * kBT + kc * 16 + nt * 8 + 2 * t + (e & 1);
          const int row = e < 2 ? rA : rB;
          const bool allowed = key < a.Nkv && (!a.causal || key <= row + off);
          const float p = allowed ? wm_ex2(fmaf(S[nt][e], sl2, -(e < 2 ? lseA : lseB))) : 0.f;
          ds[nt][e] = p * (dP[nt][e] - (e < 2 ? dA : dB));
        }
      const uint32_t dsa[4] = {wm_pack_bf16x2(ds[0][0], ds[0][1]), wm_pack_bf16x2(ds[0][2], ds[0][3]),
                               wm_pack_bf16x2(ds[1][0], ds[1][1]), wm_pack_bf16x2(ds[1][2], ds[1][3])};
      // dQ += dS K: K as the (keys x dims) operand, read transposed
      const int m = lane >> 3;
      const int kr = kc * 16 + (m & 1) * 8 + (lane & 7);
#pragma unroll
      for (int nd = 0; nd < NK; ++nd) {
        uint32_t kb[4];
        ldsm_x4_trans(sk + (nd >> 2) * C::kBlock + sw128(kr, (nd & 3) * 2 + (m >> 1)), kb);
        mma_16816(dq[2 * nd], dsa, kb[0], kb[1]);
        mma_16816(dq[2 * nd + 1], dsa, kb[2], kb[3]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
  if (!ok) {
    if (lane == 0) atomicCAS(a.err, 0, kErrDeviceTimeout);
    return;
  }
  __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.dq);
#pragma unroll
  for (int n = 0; n < NK * 2; ++n) {
    const int col = n * 8 + 2 * t;
    if (rA < a.Nq)
      *reinterpret_cast<uint32_t*>(out + ((static_cast<size_t>(b) * a.Nq + rA) * a.Hq + hq) * D + col) =
          wm_pack_bf16x2(dq[n][0] * a.scale, dq[n][1] * a.scale);
    if (rB < a.Nq)
      *reinterpret_cast<uint32_t*>(out + ((static_cast<size_t>(b) * a.Nq + rB) * a.Hq + hq) * D + col) =
          wm_pack_bf16x2(dq[n][2] * a.scale, dq[n][3] * a.scale);
  }
}

template <int D>
__global__ void __launch_bounds__(kBThreads, BCfg<D>::kCtas)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const BwdArgs a) {
  using C = BCfg<D>;
  constexpr int R = C::R, NK = D / 16;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1k(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBars);
  uint64_t* fixed_full = bars;
  uint64_t* full = bars + 1;
  uint64_t* empty = full + R;
  float* vec = reinterpret_cast<float*>(smem + C::kOffVec);  // [R][2][64]: lse2, D

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int hkv = blockIdx.y, b = blockIdx.z;
  const int G = a.Hq / a.Hkv;
  const int k0 = static_cast<int>(blockIdx.x) * kBT;
  const int off = a.Nkv - a.Nq;
  const int n_qt = (a.Nq + kBT - 1) / kBT;
  // causal: row i sees key k0 iff i >= k0 - off; earlier Q tiles see none of these keys
  const int first_qt = a.causal ? min(n_qt, max(0, k0 - off) / kBT) : 0;
  const int per_head = n_qt - first_qt;
  const int steps = G * per_head;

  if (threadIdx.x == 0) {
    mbar_init(fixed_full, 1);
    for (int s = 0; s < R; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCW);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kCW) {
    // ------------------------------------------------------------ producer
    mbar_arrive_expect_tx_elect(fixed_full, 2 * C::kTile);
#pragma unroll
    for (int h = 0; h < C::KB; ++h) {
      tma_load_4d_elect(smem + h * C::kBlock, &tmK, fixed_full, 64 * h, hkv, k0, b);
      tma_load_4d_elect(smem + C::kTile + h * C::kBlock, &tmV, fixed_full, 64 * h, hkv, k0, b);
    }
    bool ok = true;
    int u = 0;
    for (; u < steps; ++u) {
      const int s = u % R;
      if (u >= R && !__all_sync(0xffffffffu, mbar_wait(&empty[s], ((u / R) + 1) & 1))) {
        ok = false;
        break;
      }
      const int hq = hkv * G + u / per_head, qt = first_qt + u % per_head;
      // this stage's 64 lse2 and D values (0 past Nq; those rows are masked)
      const size_t vrow = (static_cast<size_t>(b) * a.Hq + hq) * a.Nq;
      float* vs = vec + s * 2 * kBT;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int i = qt * kBT + lane + 32 * h;
        vs[lane + 32 * h] = i < a.Nq ? a.lse2[vrow + i] : 0.f;
        vs[kBT + lane + 32 * h] = i < a.Nq ? a.dvec[vrow + i] : 0.f;
      }
      __syncwarp();
      uint8_t* st = smem + C::kOffRing + s * 2 * C::kTile;
      mbar_arrive_expect_tx_elect(&full[s], 2 * C::kTile);
#pragma unroll
      for (int h = 0; h < C::KB; ++h) {
        tma_load_4d_elect(st + h * C::kBlock, &tmQ, &full[s], 64 * h, hq, qt * kBT, b);
        tma_load_4d_elect(st + C::kTile + h * C::kBlock, &tmDO, &full[s], 64 * h, hq, qt * kBT, b);
      }
    }
    if (!ok && lane == 0) atomicCAS(a.err, 0, kErrDeviceTimeout);
    mbar_wait(fixed_full, 0);
    for (int w = u > R ? u - R : 0; w < u; ++w) mbar_wait(&full[w % R], (w / R) & 1);
    return;
  }

  // ------------------------------------------------------------ compute warps
  const float sl2 = a.scale * kLog2e;
  const int kA = k0 + 16 * warp + g, kB = kA + 8;  // this lane's two keys
  float dk[NK * 2][4], dv[NK * 2][4];
#pragma unroll
  for (int n = 0; n < NK * 2; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[n][e] = dv[n][e] = 0.f;

  bool ok = __all_sync(0xffffffffu, mbar_wait(fixed_full, 0));
  const uint32_t skt = smem_u32(smem), svt = skt + C::kTile;
  const int ar = 16 * warp + ((lane >> 3) & 1) * 8 + (lane & 7);  // A-fragment row of this warp's keys

  for (int u = 0; ok && u < steps; ++u) {
    const int s = u % R;
    if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (u / R) & 1))) {
      ok = false;
      break;
    }
    const int qt = first_qt + u % per_head;
    const uint32_t sq = smem_u32(smem + C::kOffRing + s * 2 * C::kTile), sdo = sq + C::kTile;
    const float* vs = vec + s * 2 * kBT;
#pragma unroll
    for (int qc = 0; qc < kBT / 16; ++qc) {
      float St[2][4] = {}, dPt[2][4] = {};
      {
        const int m = lane >> 3;
        const int qr = qc * 16 + (m >> 1) * 8 + (lane & 7);
#pragma unroll
        for (int ks = 0; ks < NK; ++ks) {
          const uint32_t ao = (ks >> 2) * C::kBlock + sw128(ar, (ks & 3) * 2 + (lane >> 4));
          const uint32_t bo = (ks >> 2) * C::kBlock + sw128(qr, (ks & 3) * 2 + (m & 1));
          uint32_t ka[4], va[4], qb[4], db[4];
          ldsm_x4(skt + ao, ka);
          ldsm_x4(svt + ao, va);
          ldsm_x4(sq + bo, qb);
          ldsm_x4(sdo + bo, db);
          mma_16816(St[0], ka, qb[0], qb[1]);
          mma_16816(St[1], ka, qb[2], qb[3]);
          mma_16816(dPt[0], va, db[0], db[1]);
          mma_16816(dPt[1], va, db[2], db[3]);
        }
      }
      float p[2][4], ds[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int c = qc * 16 + nt * 8 + 2 * t;  // this lane's query columns c, c + 1 of the tile
        const float2 l2 = *reinterpret_cast<const float2*>(vs + c);
        const float2 dd = *reinterpret_cast<const float2*>(vs + kBT + c);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int query = qt * kBT + c + (e & 1);
          const int key = e < 2 ? kA : kB;
          const bool allowed = query < a.Nq && (!a.causal || key <= query + off);
          p[nt][e] = allowed ? wm_ex2(fmaf(St[nt][e], sl2, -((e & 1) ? l2.y : l2.x))) : 0.f;
          ds[nt][e] = p[nt][e] * (dPt[nt][e] - ((e & 1) ? dd.y : dd.x));
        }
      }
      const uint32_t pa[4] = {wm_pack_bf16x2(p[0][0], p[0][1]), wm_pack_bf16x2(p[0][2], p[0][3]),
                              wm_pack_bf16x2(p[1][0], p[1][1]), wm_pack_bf16x2(p[1][2], p[1][3])};
      const uint32_t dsa[4] = {wm_pack_bf16x2(ds[0][0], ds[0][1]), wm_pack_bf16x2(ds[0][2], ds[0][3]),
                               wm_pack_bf16x2(ds[1][0], ds[1][1]), wm_pack_bf16x2(ds[1][2], ds[1][3])};
      // dV += P^T dO and dK += dS^T Q, with dO and Q as (queries x dims) operands read transposed
      const int m = lane >> 3;
      const int qr = qc * 16 + (m & 1) * 8 + (lane & 7);
#pragma unroll
      for (int nd = 0; nd < NK; ++nd) {
        const uint32_t o = (nd >> 2) * C::kBlock + sw128(qr, (nd & 3) * 2 + (m >> 1));
        uint32_t db[4], qb[4];
        ldsm_x4_trans(sdo + o, db);
        ldsm_x4_trans(sq + o, qb);
        mma_16816(dv[2 * nd], pa, db[0], db[1]);
        mma_16816(dv[2 * nd + 1], pa, db[2], db[3]);
        mma_16816(dk[2 * nd], dsa, qb[0], qb[1]);
        mma_16816(dk[2 * nd + 1], dsa, qb[2], qb[3]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
  if (!ok) {
    if (lane == 0) atomicCAS(a.err, 0, kErrDeviceTimeout);
    return;
  }
  __nv_bfloat16* odk = reinterpret_cast<__nv_bfloat16*>(a.dk);
  __nv_bfloat16* odv = reinterpret_cast<__nv_bfloat16*>(a.dv);
#pragma unroll
  for (int n = 0; n < NK * 2; ++n) {
    const int col = n * 8 + 2 * t;
    if (kA < a.Nkv) {
      const size_t o = ((static_cast<size_t>(b) * a.Nkv + kA) * a.Hkv + hkv) * D + col;
      *reinterpret_cast<uint32_t*>(odk + o) = wm_pack_bf16x2(dk[n][0] * a.scale, dk[n][1] * a.scale);
      *reinterpret_cast<uint32_t*>(odv + o) = wm_pack_bf16x2(dv[n][0], dv[n][1]);
    }
    if (kB < a.Nkv) {
      const size_t o = ((static_cast<size_t>(b) * a.Nkv + kB) * a.Hkv + hkv) * D + col;
      *reinterpret_cast<uint32_t*>(odk + o) = wm_pack_bf16x2(dk[n][2] * a.scale, dk[n][3] * a.scale);
      *reinterpret_cast<uint32_t*>(odv + o) = wm_pack_bf16x2(dv[n][2], dv[n][3]);
    }
  }
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
  if (!encode_bf16_map(&tq, a.q, a.B, a.Nq, a.Hq, D, kBT) || !encode_bf16_map(&tdo, a.dout, a.B, a.Nq, a.Hq, D, kBT) ||
      !encode_bf16_map(&tk, a.k, a.B, a.Nkv, a.Hkv, D, kBT) || !encode_bf16_map(&tv, a.v, a.B, a.Nkv, a.Hkv, D, kBT))
    return cudaErrorInvalidValue;
  const long long rows = static_cast<long long>(a.B) * a.Hq * a.Nq;
  bwd_prep_kernel<D><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  bwd_dq_kernel<D><<<dim3((a.Nq + kBT - 1) / kBT, a.Hq, a.B), kBThreads, C::kSmem, s>>>(tq, tdo, tk, tv, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  bwd_dkdv_kernel<D><<<dim3((a.Nkv + kBT - 1) / kBT, a.Hkv, a.B), kBThreads, C::kSmem, s>>>(tq, tdo, tk, tv, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd(int d, const BwdArgs& a, cudaStream_t s) {
  if (d == 64) return launch_bwd_d<64>(a, s);
  return launch_bwd_d<128>(a, s);
}

}  // namespace eio
