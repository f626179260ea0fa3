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
// Two persistent kernels (one CTA per SM, each walking a longest-first list
// of work items dealt in rounds of alternating direction), in this order:
//   bwd_dq_kernel     an item is a (128-row Q tile, query head, b): Q, dO and
//                     O stay in shared memory while the K / V tiles stream
//                     through a TMA ring; per K/V tile, on the tensor core,
//                       S = Q K^T,  dP = dO V^T       (shared x shared)
//                       dQ += dS K                    (TMEM x shared)
//                     Its element-wise threads compute D from the O and dO
//                     tiles (while dP of the first tile is on the tensor
//                     core) and leave -D and -LSE*log2(e) in a scratch whose
//                     rows are padded to whole tiles (-inf and 0 there).
//                     The dK/dV kernel fetches 128-row runs of both with bulk
//                     copies on the same barrier as its Q / dO tiles.
//   bwd_dkdv_kernel   an item is a (128-key tile, KV head, b): K and V stay
//                     while the Q / dO tiles of every query head of the group
//                     stream through, so dK and dV of a KV head sum over its
//                     G query heads without atomics; per Q tile
//                       S^T = K Q^T,  dP^T = V dO^T
//                       dV += P^T dO,  dK += dS^T Q
// S and dP are recomputed by both kernels (seven products instead of five)
// so that neither needs atomics or a second pass over an fp32 dQ.
//
// Masks: none; causal (bottom-right aligned, diagonal tiles masked by index);
// and 16 x 16 block maps, for which the host lists, per Q tile and per key
// tile, the tiles of the other kind that hold an allowed block, each with the
// 64-bit bitmap of its 8 x 8 allowed blocks: tiles without one are never
// visited, and the bitmap masks the blocks of a visited tile that are not
// allowed.
//
// Across items: the producer loads the next item's resident tiles as soon as
// the current item's last S / dP MMAs have read them, its first stream tiles
// queue in the ring behind the current ones, and the next item's first S and
// dP run on the tensor core while the element-wise warps write the current
// item's gradients out of TMEM.
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
//               (d = 64: a second dQ at [448,512), alternating by item)
//   dK/dV d=64: S0 [0,128) S1 [128,256) dP [256,384) dV [384,448) dK [448,512)
//   dK/dV d=128: S [0,128) dP [128,256) dV [256,384) dK [384,512)
#include <cuda_bf16.h>

#include "fastmath.cuh"
#include "kernels.h"
#include "pdl.cuh"
#include "ptx_sm100.cuh"
#include "warp_mma.cuh"

namespace eio {
namespace {

constexpr int kT = 128;  // rows of a Q tile, keys of a KV tile: the MMA's M
constexpr int kBThreads = 320;  // dQ: warp 0 producer, warp 1 MMA, warps 2-9 element-wise
constexpr int kEW = 8;   // element-wise warps
// dK/dV at d = 64: 384 threads.  Warpgroup 0: warp 0 the producer, warp 1
// the MMA issuer (and TMEM owner), warps 2 and 3 idle; warps 4-11
// (warpgroups 1 and 2) element-wise.  setmaxnreg moves registers from
// warpgroup 0 to the element-wise warps, which spilled at the 168 every
// thread gets otherwise.  The split is only safe when the kernel starts with
// exactly kKVLaunchRegs registers per thread; the host checks this before the
// first launch.  At d = 128 the dK/dV kernel keeps the dQ kernel's layout (it
// measured slower with the split).
template <int D>
constexpr bool kKVSplit = D == 64;
template <int D>
constexpr int kKVThreads = kKVSplit<D> ? 384 : kBThreads;
template <int D>
constexpr int kKVFirstEW = kKVSplit<D> ? 4 : 2;
constexpr int kKVLaunchRegs = 168;
constexpr int kKVRegsControl = 80;
constexpr int kKVRegsEW = 208;
static_assert(128 * kKVRegsControl + 256 * kKVRegsEW <= kKVThreads<64> * kKVLaunchRegs,
              "register split must fit in the launch allocation");
constexpr float kLog2e = 1.4426950408889634f;
// Of every 8 column pairs, this many take the polynomial 2^x on the FMA pipe
// instead of the MUFU unit (measured: 1 at d = 64 and 2 at d = 128 were
// best, by about 1 %; 0 to 3 all lie within 2 %).
template <int D>
constexpr int kPolyPairsB = D == 64 ? 1 : 2;

template <int D>
struct BCfg {
  static constexpr int NCH = D / 64;                 // 128-byte column chunks per row
  static constexpr int kChunk = kT * 128;            // one chunk of a 128-row tile
  static constexpr int kTile = NCH * kChunk;         // a 128 x D bf16 tile
  static constexpr int R = D == 64 ? 4 : 2;          // ring stages (two tiles each)
  static constexpr int kOffRing = 2 * kTile;         // after the two resident tiles
  // dK/dV kernel: per stage -lse2[128], -D[128]; dQ kernel: the O tile
  static constexpr int kOffX = kOffRing + R * 2 * kTile;
  // d = 64: the gradients leave through 128-byte-swizzled staging tiles in
  // shared memory and one TMA store per tile (dV and dK, or dQ), instead of
  // one 16-byte store per row and thread.
  static constexpr bool kStage = D == 64;
  static constexpr int kOffStgKV = kOffX + R * 2 * kT * 4;
  static constexpr int kOffBarKV = kOffStgKV + (kStage ? 2 * kTile : 0);
  static constexpr int kOffStgQ = kOffX + kTile;
  static constexpr int kOffBarQ = kOffStgQ + (kStage ? kTile : 0);
  // fixed_full, fixed_empty, full[R], empty[R], s_full[2], dp_full, p_full, ds_full,
  // mma_done, acc_free[2], mma_idle, stg_full, stg_free, p_full1
  static constexpr int kNumBars = 2 * R + 14;
  static constexpr int kSmemKV = kOffBarKV + 8 * kNumBars + 16 + 1024;
  static constexpr int kSmemQ = kOffBarQ + 8 * kNumBars + 16 + 1024;
  static_assert(kSmemKV <= 227 * 1024 && kSmemQ <= 227 * 1024, "shared memory per CTA");
  static constexpr int kVecBytes = 2 * kT * 4;
  // S buffers in TMEM (dK/dV kernel; the dQ kernel always has two)
  static constexpr int kSBufKV = D == 64 ? 2 : 1;
  static constexpr int kAccQ = D == 64 ? 2 : 1;  // dQ accumulators in TMEM
};

// Barriers shared by both kernels' layouts (p_full0/1 are unused by the dQ
// kernel).  With two S buffers (dK/dV kernel at d = 64) P of step t is
// signalled on p_full(t), alternating between two barriers: the issuer puts
// S(t+1) on the tensor core before it waits for P(t), so the element-wise
// warps may finish P(t) and P(t+1) before that wait, and a parity wait must
// never fall two phases behind its barrier.  With one S buffer, S(t+1)
// follows dK(t), which follows the wait for P(t), and p_full0 serves every
// step.
struct BBars {
  uint64_t *fixed_full, *fixed_empty, *full, *empty, *s_full, *dp_full, *p_full0, *ds_full, *mma_done, *acc_free,
      *mma_idle, *stg_full, *stg_free, *p_full1;
  __device__ BBars(uint64_t* b, int R)
      : fixed_full(b), fixed_empty(b + 1), full(b + 2), empty(b + 2 + R), s_full(b + 2 + 2 * R),
        dp_full(b + 4 + 2 * R), p_full0(b + 5 + 2 * R), ds_full(b + 6 + 2 * R), mma_done(b + 7 + 2 * R),
        acc_free(b + 8 + 2 * R), mma_idle(b + 10 + 2 * R), stg_full(b + 11 + 2 * R), stg_free(b + 12 + 2 * R),
        p_full1(b + 13 + 2 * R) {}
  template <int NB>
  __device__ uint64_t* p_full(uint32_t t) const { return (NB == 2 && (t & 1)) ? p_full1 : p_full0; }
  template <int NB>
  __device__ static uint32_t p_parity(uint32_t t) { return NB == 2 ? (t >> 1) & 1 : t & 1; }
};

// One element-wise thread's NC TMEM columns (times mul) as bf16 into a
// 128-byte-swizzled staging row, at 16-byte unit u0 onwards.
template <int NC>
__device__ __forceinline__ void stage_row(uint8_t* stg, int r, int u0, const uint32_t* v, float mul) {
#pragma unroll
  for (int u = 0; u < NC / 8; ++u)
    *reinterpret_cast<uint4*>(stg + r * 128 + (((u0 + u) ^ (r & 7)) << 4)) =
        make_uint4(wm_pack_bf16x2(__uint_as_float(v[8 * u + 0]) * mul, __uint_as_float(v[8 * u + 1]) * mul),
                   wm_pack_bf16x2(__uint_as_float(v[8 * u + 2]) * mul, __uint_as_float(v[8 * u + 3]) * mul),
                   wm_pack_bf16x2(__uint_as_float(v[8 * u + 4]) * mul, __uint_as_float(v[8 * u + 5]) * mul),
                   wm_pack_bf16x2(__uint_as_float(v[8 * u + 6]) * mul, __uint_as_float(v[8 * u + 7]) * mul));
}

// The k-th item of this CTA, or -1: items are numbered longest first and
// dealt in rounds of gridDim.x, alternating direction.
__device__ __forceinline__ long long bwd_item(long long k, long long n_items) {
  const long long g = gridDim.x, base = k * g;
  if (base >= n_items) return -1;
  const long long idx = (k & 1) ? base + (g - 1 - blockIdx.x) : base + blockIdx.x;
  return idx < n_items ? idx : -1;
}

// dK/dV item: KV tile slowest (under a causal mask the first tiles visit the
// most Q tiles).
struct KvItem {
  int b, hkv, k0, first_qt, per_head, steps;
  const int4* list;  // BLOCK masks: the key tile's live Q tiles; else null
};
template <bool BLK>
__device__ __forceinline__ KvItem kv_item(const BwdArgs& a, long long w) {
  KvItem it;
  const int per_kt = a.Hkv * a.B;
  const int r = static_cast<int>(w % per_kt);
  int kt = static_cast<int>(w / per_kt);
  it.hkv = r / a.B;
  it.b = r % a.B;
  const int n_qt = (a.Nq + kT - 1) / kT;
  it.list = nullptr;
  if (BLK) {
    kt = a.kord[kt];
    it.list = a.klist + a.koff[kt];
    it.first_qt = 0;
    it.per_head = a.koff[kt + 1] - a.koff[kt];
  } else {
    // causal: row i sees key k0 iff i >= k0 - off; earlier Q tiles see none of these keys
    it.first_qt = a.causal ? min(n_qt, max(0, kt * kT - (a.Nkv - a.Nq)) / kT) : 0;
    it.per_head = n_qt - it.first_qt;
  }
  it.k0 = kt * kT;
  it.steps = (a.Hq / a.Hkv) * it.per_head;
  return it;
}

// The Q tile and live-block bitmap of step u of a dK/dV item.
template <bool BLK>
__device__ __forceinline__ int kv_step_qt(const KvItem& it, int u, unsigned long long* bits) {
  const int idx = u % it.per_head;
  if (!BLK) {
    *bits = ~0ull;
    return it.first_qt + idx;
  }
  const int4 e = it.list[idx];
  *bits = static_cast<unsigned>(e.y) | (static_cast<unsigned long long>(static_cast<unsigned>(e.z)) << 32);
  return e.x;
}

// dQ item: Q tile slowest, last tile first (under a causal mask the last
// tiles visit the most K/V tiles).
struct QItem {
  int b, hq, q0, n_kv;
  const int4* list;  // BLOCK masks: the Q tile's live key tiles; else null
};
template <bool BLK>
__device__ __forceinline__ QItem q_item(const BwdArgs& a, long long w) {
  QItem it;
  const int per_qt = a.Hq * a.B;
  const int n_qt = (a.Nq + kT - 1) / kT;
  const int r = static_cast<int>(w % per_qt);
  it.hq = r / a.B;
  it.b = r % a.B;
  it.list = nullptr;
  if (BLK) {
    const int qt = a.qord[w / per_qt];
    it.q0 = qt * kT;
    it.list = a.qlist + a.qoff[qt];
    it.n_kv = a.qoff[qt + 1] - a.qoff[qt];
    return it;
  }
  it.q0 = (n_qt - 1 - static_cast<int>(w / per_qt)) * kT;
  int n_kv = (a.Nkv + kT - 1) / kT;
  if (a.causal) {
    const int last = min(it.q0 + kT - 1, a.Nq - 1) + (a.Nkv - a.Nq);  // largest key any row may see
    n_kv = last < 0 ? 0 : min(n_kv, last / kT + 1);
  }
  it.n_kv = n_kv;
  return it;
}

// The key tile and live-block bitmap of step j of a dQ item.
template <bool BLK>
__device__ __forceinline__ int q_step_kt(const QItem& it, int j, unsigned long long* bits) {
  if (!BLK) {
    *bits = ~0ull;
    return j;
  }
  const int4 e = it.list[j];
  *bits = static_cast<unsigned>(e.y) | (static_cast<unsigned long long>(static_cast<unsigned>(e.z)) << 32);
  return e.x;
}

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

// p = 2^(s * sl2 - lse2) for one thread's 64 columns (sr: the S values as
// loaded from TMEM); nl(c) gives -lse2 for the columns c, c + 1.  MASK:
// columns outside [lo, hi), and columns of a 16-column group whose bit in
// `groups` is clear, are 0.
template <int NP, bool MASK, typename NLFn>
__device__ __forceinline__ void p_row(float* p, const uint32_t* sr, float sl2, NLFn nl, int lo, int hi,
                                      unsigned groups = 0xFu) {
  const float2 sl = make_float2(sl2, sl2);
#pragma unroll
  for (int c = 0; c < 64; c += 2) {
    float2 e = ffma2(make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sl, nl(c));
    if (MASK) {
      const bool live = (groups >> (c >> 4)) & 1u;  // c and c + 1 share their group
      if (!live || c < lo || c >= hi) e.x = -INFINITY;
      if (!live || c + 1 < lo || c + 1 >= hi) e.y = -INFINITY;
    }
    const float2 v = ((c >> 1) & 7) < NP ? exp2_poly2(e) : make_float2(wm_ex2(e.x), wm_ex2(e.y));
    p[c] = v.x;
    p[c + 1] = v.y;
  }
}

// dS = P * (dP - D) for one thread's 64 columns: dP read from TMEM at t_dp,
// dS written (bf16 pairs, 32 columns) at t_ds.  nd(c) gives -D for the
// columns c, c + 1.
template <typename DFn>
__device__ __forceinline__ void write_ds(uint32_t t_dp, uint32_t t_ds, const float* p, DFn nd) {
  uint32_t dr[64], pk[32];
  tmem_ld32(t_dp, dr);
  tmem_ld32(t_dp + 32, dr + 32);
  tmem_wait_ld();
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float2 d = fadd2(make_float2(__uint_as_float(dr[2 * j]), __uint_as_float(dr[2 * j + 1])), nd(2 * j));
    const float2 ds = fmul2(make_float2(p[2 * j], p[2 * j + 1]), d);
    pk[j] = wm_pack_bf16x2(ds.x, ds.y);
  }
  tmem_st32(t_ds, pk);
}

// ----------------------------------------------------------------- dK, dV
// BLK: block-sparse mask (tile lists with block bitmaps); otherwise no mask
// or causal.
template <int D, bool BLK>
__global__ void __launch_bounds__(kKVThreads<D>, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmDK, const __grid_constant__ CUtensorMap tmDV,
                    const BwdArgs a) {
  using C = BCfg<D>;
  constexpr int R = C::R, NB = C::kSBufKV;
  constexpr uint32_t kColDP = 128 * NB, kColDV = kColDP + 128, kColDK = kColDV + D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1k(smem_raw);
  uint64_t* bar_base = reinterpret_cast<uint64_t*>(smem + C::kOffBarKV);
  const BBars br(bar_base, R);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_base + C::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* vec = reinterpret_cast<float*>(smem + C::kOffX);  // [R][2][128]: -lse2, -D

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.Hq / a.Hkv;
  const int off = a.Nkv - a.Nq;  // bottom-right causal alignment
  const int nq_pad = (a.Nq + kT - 1) / kT * kT;  // rows per (b, head) of the lse2 / D scratch
  const long long n_items = static_cast<long long>((a.Nkv + kT - 1) / kT) * a.Hkv * a.B;

  if (threadIdx.x == 0) {
    mbar_init(br.fixed_full, 1);
    mbar_init(br.fixed_empty, 1);
    for (int s = 0; s < R; ++s) {
      mbar_init(&br.full[s], 1);
      mbar_init(&br.empty[s], 1 + kEW);  // the MMA commit, and each element-wise warp after reading the vectors
    }
    mbar_init(&br.s_full[0], 1);
    mbar_init(&br.s_full[1], 1);
    mbar_init(br.dp_full, 1);
    mbar_init(br.p_full0, kEW);
    mbar_init(br.p_full1, kEW);
    mbar_init(br.ds_full, kEW);
    mbar_init(br.mma_done, 1);
    mbar_init(&br.acc_free[0], kEW);
    mbar_init(&br.acc_free[1], kEW);
    mbar_init(br.mma_idle, 1);
    mbar_init(br.stg_full, kEW);
    mbar_init(br.stg_free, 1);
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
  auto stage = [&](uint32_t t) { return smem + C::kOffRing + (t % R) * 2 * C::kTile; };

  constexpr int kFirstEW = kKVFirstEW<D>;
  if (warp < kFirstEW) {
  if constexpr (kKVSplit<D>) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kKVRegsControl));
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmDO);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
    uint32_t g = 0, nfix = 0;
    bool ok = true, vec_ready = false;
    for (long long k = 0; ok; ++k) {
      const long long w = bwd_item(k, n_items);
      if (w < 0) break;
      const KvItem it = kv_item<BLK>(a, w);
      // K and V of the previous item are free once its last S and dP have run
      if (k > 0 && !wwait(br.fixed_empty, (k - 1) & 1)) {
        ok = false;
        break;
      }
      mbar_arrive_expect_tx_elect(br.fixed_full, 2 * C::kTile);
#pragma unroll
      for (int ch = 0; ch < C::NCH; ++ch) {
        tma_load_4d_elect(smem + ch * C::kChunk, &tmK, br.fixed_full, 64 * ch, it.hkv, it.k0, it.b);
        tma_load_4d_elect(smem + C::kTile + ch * C::kChunk, &tmV, br.fixed_full, 64 * ch, it.hkv, it.k0, it.b);
      }
      ++nfix;
      for (int u = 0; u < it.steps; ++u, ++g) {
        const int s = g % R;
        if (g >= R && !wwait(&br.empty[s], ((g / R) - 1) & 1)) {
          ok = false;
          break;
        }
        unsigned long long bits;
        const int hq = it.hkv * G + u / it.per_head, qt = kv_step_qt<BLK>(it, u, &bits);
        uint8_t* st = stage(g);
        mbar_arrive_expect_tx_elect(&br.full[s], 2 * C::kTile + C::kVecBytes);
#pragma unroll
        for (int ch = 0; ch < C::NCH; ++ch) {
          tma_load_4d_elect(st + ch * C::kChunk, &tmQ, &br.full[s], 64 * ch, hq, qt * kT, it.b);
          tma_load_4d_elect(st + C::kTile + ch * C::kChunk, &tmDO, &br.full[s], 64 * ch, hq, qt * kT, it.b);
        }
        // the tile's 128 -lse2 and -D values (padded rows: -lse2 = -inf, D = 0)
        const size_t vrow = (static_cast<size_t>(it.b) * a.Hq + hq) * nq_pad + static_cast<size_t>(qt) * kT;
        // -lse2 and -D are written by the dQ kernel, which may still be
        // running (programmatic dependent launch): wait for it before the
        // first copy of them.
        if (!vec_ready) {
          pdl_wait();
          vec_ready = true;
        }
        bulk_load_elect(vec + s * 2 * kT, a.neg_lse2 + vrow, kT * 4, &br.full[s]);
        bulk_load_elect(vec + s * 2 * kT + kT, a.neg_d + vrow, kT * 4, &br.full[s]);
      }
    }
    if (!ok && lane == 0) fail(kErrDeviceTimeout);
    // Every copy lands before the CTA retires.
    if (nfix > 0) mbar_wait(br.fixed_full, (nfix - 1) & 1);
    for (uint32_t t = g > R ? g - R : 0; t < g; ++t) mbar_wait(&br.full[t % R], (t / R) & 1);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Issue order per step t: S(t+1) (two S buffers), dV(t), dK(t), then
    // dP(t+1) -- the element-wise warps have read dP(t) by then.
    const uint32_t sK = smem_u32(smem), sV = sK + C::kTile;
    uint32_t g = 0;
    bool ok = true;
    for (long long k = 0; ok; ++k) {
      const long long w = bwd_item(k, n_items);
      if (w < 0) break;
      const KvItem it = kv_item<BLK>(a, w);
      if (!wwait(br.fixed_full, k & 1)) {
        ok = false;
        break;
      }
      if (it.steps == 0) {
        mma_commit_elect(br.fixed_empty);
        continue;
      }
      // every earlier MMA has completed: both S buffers and dP are free
      if (!wwait(&br.full[g % R], (g / R) & 1) || (g > 0 && !wwait(br.mma_done, (g - 1) & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      issue_ss<D>(tmem + 128 * (g % NB), sK, smem_u32(stage(g)));  // S^T = K Q^T
      mma_commit_elect(&br.s_full[g % NB]);
      issue_ss<D>(tmem + kColDP, sV, smem_u32(stage(g)) + C::kTile);  // dP^T = V dO^T
      mma_commit_elect(br.dp_full);
      if (it.steps == 1) mma_commit_elect(br.fixed_empty);
      for (int u = 0; u < it.steps; ++u, ++g) {
        const int s = g % R, x = g % NB;
        const uint32_t sQ = smem_u32(stage(g)), sdO = sQ + C::kTile;
        const bool next = u + 1 < it.steps;
        if (NB == 2 && next) {
          // S buffer (g+1)%2 was last read by dV(g-1) / dK(g-1)
          if (!wwait(&br.full[(g + 1) % R], ((g + 1) / R) & 1) || (u >= 1 && !wwait(br.mma_done, (g - 1) & 1))) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_ss<D>(tmem + 128 * ((g + 1) % NB), sK, smem_u32(stage(g + 1)));
          mma_commit_elect(&br.s_full[(g + 1) % NB]);
        }
        // dV / dK of the previous item have been read out of TMEM
        if (!wwait(br.p_full<NB>(g), BBars::p_parity<NB>(g)) ||
            (u == 0 && k > 0 && !wwait(&br.acc_free[0], (k - 1) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_ts<D>(tmem + kColDV, tmem + 128 * x, sdO, u > 0);  // dV += P^T dO
        if (!wwait(br.ds_full, g & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_ts<D>(tmem + kColDK, tmem + 128 * x + 32, sQ, u > 0);  // dK += dS^T Q
        mma_commit_elect(&br.empty[s]);
        mma_commit_elect(br.mma_done);
        if (next) {
          if (NB == 1) {
            // one S buffer: S(g+1) after dV(g) / dK(g) have read it
            if (!wwait(&br.full[(g + 1) % R], ((g + 1) / R) & 1) || !wwait(br.mma_done, g & 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_ss<D>(tmem, sK, smem_u32(stage(g + 1)));
            mma_commit_elect(&br.s_full[0]);
          }
          issue_ss<D>(tmem + kColDP, sV, smem_u32(stage(g + 1)) + C::kTile);
          mma_commit_elect(br.dp_full);
          if (u + 2 == it.steps) mma_commit_elect(br.fixed_empty);  // the item's last S and dP
        }
      }
    }
    if (!ok && lane == 0) fail(kErrDeviceTimeout);
    // Every MMA issued above has finished before TMEM is released.
    mma_commit_elect(br.mma_idle);
    mbar_wait(br.mma_idle, 0);
  }  // d = 64: warps 2 and 3 have no role
  } else {
    if constexpr (kKVSplit<D>) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kKVRegsEW));
    // ------------------------------------------------------------ element-wise
    const int h = (warp - kFirstEW) >> 2;  // column half
    const int quarter = warp & 3;
    const uint32_t lo = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t t_row = tmem + lo;
    const float sl2 = a.scale * kLog2e;
    constexpr int STG = C::kOffStgKV;
    // Staged output of the k-th item: wait until the previous item's TMA
    // stores have read the staging tiles, write this thread's rows (fill),
    // and have the first element-wise warp store the tiles (issue) once every element-wise warp
    // has written.  All waits are bounded.
    auto stage_out = [&](long long k, auto fill, auto issue) -> bool {
      uint8_t* stg = smem + STG;
      if (k > 0) {
        if (warp == kFirstEW) {
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
          if (lane == 0) mbar_arrive(br.stg_free);
        }
        if (!wwait(br.stg_free, (k - 1) & 1)) return false;
      }
      fill(stg);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(br.stg_full);
      if (warp == kFirstEW) {
        if (!wwait(br.stg_full, k & 1)) return false;
        if (lane == 0) {
          issue(stg);
          bulk_commit();
        }
      }
      return true;
    };
    uint32_t g = 0;
    bool ok = true;
    for (long long k = 0; ok; ++k) {
      const long long w = bwd_item(k, n_items);
      if (w < 0) break;
      const KvItem it = kv_item<BLK>(a, w);
      const int key = it.k0 + quarter * 32 + lane;  // this thread's key (TMEM lane)
      for (int u = 0; u < it.steps; ++u, ++g) {
        const int s = g % R, x = g % NB;
        unsigned long long bits;
        const int q0 = kv_step_qt<BLK>(it, u, &bits) * kT + 64 * h;  // query of this thread's first column
        if (!wwait(&br.full[s], (g / R) & 1) || !wwait(&br.s_full[x], (g / NB) & 1)) {
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
          auto nl = [&](int c) { return *reinterpret_cast<const float2*>(vs + c); };
          // block masks: this key's 16-key block j against the four 16-query
          // groups of the thread's columns
          const int kb = (quarter * 32 + lane) >> 4;
          unsigned groups = 0xFu;
          if (BLK) {
            groups = 0u;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) groups |= static_cast<unsigned>((bits >> ((4 * h + q4) * 8 + kb)) & 1ull) << q4;
          }
          if (a.causal && it.k0 + kT - 1 > q0 + off)
            p_row<kPolyPairsB<D>, true>(p, sr, sl2, nl, key - off - q0, 64);
          else if (BLK && __any_sync(0xffffffffu, groups != 0xFu))
            p_row<kPolyPairsB<D>, true>(p, sr, sl2, nl, 0, 64, groups);
          else
            p_row<kPolyPairsB<D>, false>(p, sr, sl2, nl, 0, 64);
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
        if (lane == 0) mbar_arrive(br.p_full<NB>(g));
        if (!wwait(br.dp_full, g & 1)) {
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
          mbar_arrive(br.ds_full);
          mbar_arrive(&br.empty[s]);
        }
      }
      if (!ok) break;
      if (it.steps > 0) {
        if (!wwait(br.mma_done, (g - 1) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      // each warpgroup writes half of the columns of dV and dK
      constexpr int HC = D / 2;
      if constexpr (C::kStage) {
        uint32_t rv[HC], rk[HC];
        if (it.steps > 0) {
          tmem_ld32(t_row + kColDV + HC * h, rv);
          tmem_ld32(t_row + kColDK + HC * h, rk);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < HC; ++i) rv[i] = rk[i] = 0u;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&br.acc_free[0]);
        if (!stage_out(k, [&](uint8_t* stg) {
              stage_row<HC>(stg, quarter * 32 + lane, 4 * h, rv, 1.f);
              stage_row<HC>(stg + C::kTile, quarter * 32 + lane, 4 * h, rk, a.scale);
            }, [&](uint8_t* stg) {
              tma_store_4d(&tmDV, stg, 0, it.hkv, it.k0, it.b);
              tma_store_4d(&tmDK, stg + C::kTile, 0, it.hkv, it.k0, it.b);
            })) {
          ok = false;
          break;
        }
      } else {
        const size_t o = ((static_cast<size_t>(it.b) * a.Nkv + key) * a.Hkv + it.hkv) * D + HC * h;
        const bool valid = key < a.Nkv;
        store_cols<HC>(t_row + kColDV + HC * h, valid ? reinterpret_cast<__nv_bfloat16*>(a.dv) + o : nullptr, 1.f,
                       it.steps > 0);
        store_cols<HC>(t_row + kColDK + HC * h, valid ? reinterpret_cast<__nv_bfloat16*>(a.dk) + o : nullptr,
                       a.scale, it.steps > 0);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&br.acc_free[0]);
      }
    }
    if (!ok && lane == 0) fail(kErrDeviceTimeout);
    if (C::kStage && warp == kFirstEW && lane == 0) bulk_wait_all();  // stores done before the CTA retires
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// -------------------------------------------------------------------- dQ
template <int D, bool BLK>
__global__ void __launch_bounds__(kBThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmDQ,
                  const BwdArgs a) {
  using C = BCfg<D>;
  constexpr int R = C::R, NA = C::kAccQ;
  constexpr uint32_t kColDP = 256, kColDQ = 384;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1k(smem_raw);
  uint64_t* bar_base = reinterpret_cast<uint64_t*>(smem + C::kOffBarQ);
  const BBars br(bar_base, R);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_base + C::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.Hq / a.Hkv;
  const int off = a.Nkv - a.Nq;
  const int nq_pad = (a.Nq + kT - 1) / kT * kT;
  const long long n_items = static_cast<long long>((a.Nq + kT - 1) / kT) * a.Hq * a.B;
  // The dK/dV kernel may be scheduled as this kernel's CTAs finish; it
  // waits for this grid before it reads -lse2 and -D.
  if (threadIdx.x == 0) pdl_launch_dependents();

  if (threadIdx.x == 0) {
    mbar_init(br.fixed_full, 1);
    mbar_init(br.fixed_empty, 1 + kEW);  // the MMA commit, and each element-wise warp after reading O and dO
    for (int s = 0; s < R; ++s) {
      mbar_init(&br.full[s], 1);
      mbar_init(&br.empty[s], 1);
    }
    mbar_init(&br.s_full[0], 1);
    mbar_init(&br.s_full[1], 1);
    mbar_init(br.dp_full, 1);
    mbar_init(br.ds_full, kEW);
    mbar_init(br.mma_done, 1);
    mbar_init(&br.acc_free[0], kEW);
    mbar_init(&br.acc_free[1], kEW);
    mbar_init(br.mma_idle, 1);
    mbar_init(br.stg_full, kEW);
    mbar_init(br.stg_free, 1);
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
  auto stage = [&](uint32_t t) { return smem + C::kOffRing + (t % R) * 2 * C::kTile; };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmDO);
      tma_prefetch_desc(&tmO);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
    uint32_t g = 0, nfix = 0;
    bool ok = true;
    for (long long k = 0; ok; ++k) {
      const long long w = bwd_item(k, n_items);
      if (w < 0) break;
      const QItem it = q_item<BLK>(a, w);
      // Q, dO and O of the previous item are free once its last S and dP
      // have run and D has been computed
      if (k > 0 && !wwait(br.fixed_empty, (k - 1) & 1)) {
        ok = false;
        break;
      }
      mbar_arrive_expect_tx_elect(br.fixed_full, 3 * C::kTile);
#pragma unroll
      for (int ch = 0; ch < C::NCH; ++ch) {
        tma_load_4d_elect(smem + ch * C::kChunk, &tmQ, br.fixed_full, 64 * ch, it.hq, it.q0, it.b);
        tma_load_4d_elect(smem + C::kTile + ch * C::kChunk, &tmDO, br.fixed_full, 64 * ch, it.hq, it.q0, it.b);
        tma_load_4d_elect(smem + C::kOffX + ch * C::kChunk, &tmO, br.fixed_full, 64 * ch, it.hq, it.q0, it.b);
      }
      ++nfix;
      const int hkv = it.hq / G;
      for (int j = 0; j < it.n_kv; ++j, ++g) {
        const int s = g % R;
        if (g >= R && !wwait(&br.empty[s], ((g / R) - 1) & 1)) {
          ok = false;
          break;
        }
        uint8_t* st = stage(g);
        unsigned long long bits;
        const int kt = q_step_kt<BLK>(it, j, &bits);
        mbar_arrive_expect_tx_elect(&br.full[s], 2 * C::kTile);
#pragma unroll
        for (int ch = 0; ch < C::NCH; ++ch) {
          tma_load_4d_elect(st + ch * C::kChunk, &tmK, &br.full[s], 64 * ch, hkv, kt * kT, it.b);
          tma_load_4d_elect(st + C::kTile + ch * C::kChunk, &tmV, &br.full[s], 64 * ch, hkv, kt * kT, it.b);
        }
      }
    }
    if (!ok && lane == 0) fail(kErrDeviceTimeout);
    if (nfix > 0) mbar_wait(br.fixed_full, (nfix - 1) & 1);
    for (uint32_t t = g > R ? g - R : 0; t < g; ++t) mbar_wait(&br.full[t % R], (t / R) & 1);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Issue order per step t: S(t+1) into the other S buffer, dQ(t), then
    // dP(t+1) -- the element-wise warps have read dP(t) by then.
    const uint32_t sQ = smem_u32(smem), sdO = sQ + C::kTile;
    uint32_t g = 0;
    bool ok = true;
    for (long long k = 0; ok; ++k) {
      const long long w = bwd_item(k, n_items);
      if (w < 0) break;
      const QItem it = q_item<BLK>(a, w);
      const int acc = static_cast<int>(k % NA);
      if (!wwait(br.fixed_full, k & 1)) {
        ok = false;
        break;
      }
      if (it.n_kv == 0) {
        mma_commit_elect(br.fixed_empty);
        continue;
      }
      // every earlier MMA has completed: both S buffers and dP are free
      if (!wwait(&br.full[g % R], (g / R) & 1) || (g > 0 && !wwait(br.mma_done, (g - 1) & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      issue_ss<D>(tmem + 128 * (g & 1), sQ, smem_u32(stage(g)));  // S = Q K^T
      mma_commit_elect(&br.s_full[g & 1]);
      issue_ss<D>(tmem + kColDP, sdO, smem_u32(stage(g)) + C::kTile);  // dP = dO V^T
      mma_commit_elect(br.dp_full);
      if (it.n_kv == 1) mma_commit_elect(br.fixed_empty);
      for (int j = 0; j < it.n_kv; ++j, ++g) {
        const int s = g % R, x = g & 1;
        const bool next = j + 1 < it.n_kv;
        if (next) {
          // S buffer (g+1)%2 was last read by dQ(g-1)
          if (!wwait(&br.full[(g + 1) % R], ((g + 1) / R) & 1) || (j >= 1 && !wwait(br.mma_done, (g - 1) & 1))) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_ss<D>(tmem + 128 * (x ^ 1), sQ, smem_u32(stage(g + 1)));
          mma_commit_elect(&br.s_full[x ^ 1]);
        }
        // this dQ buffer was read out by the epilogue of item k - NA
        if (!wwait(br.ds_full, g & 1) || (j == 0 && k >= NA && !wwait(&br.acc_free[acc], ((k / NA) - 1) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_ts<D>(tmem + kColDQ + D * acc, tmem + 128 * x, smem_u32(stage(g)), j > 0);  // dQ += dS K
        mma_commit_elect(&br.empty[s]);
        mma_commit_elect(br.mma_done);
        if (next) {
          issue_ss<D>(tmem + kColDP, sdO, smem_u32(stage(g + 1)) + C::kTile);
          mma_commit_elect(br.dp_full);
          if (j + 2 == it.n_kv) mma_commit_elect(br.fixed_empty);  // the item's last S and dP
        }
      }
    }
    if (!ok && lane == 0) fail(kErrDeviceTimeout);
    mma_commit_elect(br.mma_idle);
    mbar_wait(br.mma_idle, 0);
  } else {
    // ------------------------------------------------------------ element-wise
    const int h = (warp - 2) >> 2;  // column half
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // this thread's row of the tile (TMEM lane)
    const uint32_t lo = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t t_row = tmem + lo;
    const float sl2 = a.scale * kLog2e;
    constexpr int STG = C::kOffStgQ;
    // Staged output of the k-th item: wait until the previous item's TMA
    // stores have read the staging tiles, write this thread's rows (fill),
    // and have warp 2 store the tiles (issue) once every element-wise warp
    // has written.  All waits are bounded.
    auto stage_out = [&](long long k, auto fill, auto issue) -> bool {
      uint8_t* stg = smem + STG;
      if (k > 0) {
        if (warp == 2) {
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
          if (lane == 0) mbar_arrive(br.stg_free);
        }
        if (!wwait(br.stg_free, (k - 1) & 1)) return false;
      }
      fill(stg);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(br.stg_full);
      if (warp == 2) {
        if (!wwait(br.stg_full, k & 1)) return false;
        if (lane == 0) {
          issue(stg);
          bulk_commit();
        }
      }
      return true;
    };
    uint32_t g = 0;
    bool ok = true;
    for (long long k = 0; ok; ++k) {
      const long long w = bwd_item(k, n_items);
      if (w < 0) break;
      const QItem it = q_item<BLK>(a, w);
      const int acc = static_cast<int>(k % NA);
      const int row = it.q0 + r;
      // rows past Nq: lse2 = +inf makes their P exactly 0
      const float l2 =
          row < a.Nq ? a.lse[(static_cast<size_t>(it.b) * a.Hq + it.hq) * a.Nq + row] * kLog2e : INFINITY;
      // D = rowsum(dO * O) from the resident O and dO tiles (zero rows past
      // Nq); with lse2 it goes to the padded scratch for the dK/dV kernel.
      float dd = 0.f;
      auto compute_d = [&]() -> bool {
        if (!wwait(br.fixed_full, k & 1)) return false;
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
            for (int e = 0; e < 4; ++e) {
              const float2 of = __bfloat1622float2(o2[e]), gf = __bfloat1622float2(g2[e]);
              dd = fmaf(of.x, gf.x, dd);
              dd = fmaf(of.y, gf.y, dd);
            }
          }
        __syncwarp();
        if (lane == 0) mbar_arrive(br.fixed_empty);  // O and dO read
        if (h == 0) {
          const size_t vrow = (static_cast<size_t>(it.b) * a.Hq + it.hq) * nq_pad + row;
          a.neg_d[vrow] = -dd;
          a.neg_lse2[vrow] = -l2;
        }
        return true;
      };
      for (int j = 0; j < it.n_kv; ++j, ++g) {
        const int x = g & 1;
        if (!wwait(&br.s_full[x], (g >> 1) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // keys at or past column lim are masked: past Nkv, and past the
        // causal diagonal (rows with no visible key get lim <= 0); block
        // masks: the four 16-key groups of the thread's columns against its
        // 16-row block
        unsigned long long bits;
        const int c0 = q_step_kt<BLK>(it, j, &bits) * kT + 64 * h;  // key of this thread's first column
        int lim = min(64, a.Nkv - c0);
        if (a.causal) lim = min(lim, row + off + 1 - c0);
        const unsigned groups = BLK ? static_cast<unsigned>((bits >> ((r >> 4) * 8 + 4 * h)) & 0xFull) : 0xFu;
        const uint32_t t_s = t_row + 128 * x + 64 * h;
        float p[64];
        {
          uint32_t sr[64];
          tmem_ld32(t_s, sr);
          tmem_ld32(t_s + 32, sr + 32);
          tmem_wait_ld();
          auto nl = [&](int) { return make_float2(-l2, -l2); };
          if (__any_sync(0xffffffffu, lim < 64 || groups != 0xFu))
            p_row<kPolyPairsB<D>, true>(p, sr, sl2, nl, 0, lim, groups);
          else
            p_row<kPolyPairsB<D>, false>(p, sr, sl2, nl, 0, 64);
        }
        // D while dP of the first tile is on the tensor core
        if (j == 0 && !compute_d()) {
          ok = false;
          break;
        }
        if (!wwait(br.dp_full, g & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        write_ds(t_row + kColDP + 64 * h, t_s, p, [&](int) { return make_float2(-dd, -dd); });
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(br.ds_full);
      }
      if (!ok) break;
      if (it.n_kv == 0 && !compute_d()) {
        ok = false;
        break;
      }
      if (it.n_kv > 0) {
        if (!wwait(br.mma_done, (g - 1) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      constexpr int HC = D / 2;
      if constexpr (C::kStage) {
        uint32_t rq[HC];
        if (it.n_kv > 0) {
          tmem_ld32(t_row + kColDQ + D * acc + HC * h, rq);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < HC; ++i) rq[i] = 0u;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&br.acc_free[acc]);
        if (!stage_out(k, [&](uint8_t* stg) { stage_row<HC>(stg, r, 4 * h, rq, a.scale); },
                       [&](uint8_t* stg) { tma_store_4d(&tmDQ, stg, 0, it.hq, it.q0, it.b); })) {
          ok = false;
          break;
        }
      } else {
        __nv_bfloat16* dst = row < a.Nq ? reinterpret_cast<__nv_bfloat16*>(a.dq) +
                                              ((static_cast<size_t>(it.b) * a.Nq + row) * a.Hq + it.hq) * D + HC * h
                                        : nullptr;
        store_cols<HC>(t_row + kColDQ + D * acc + HC * h, dst, a.scale, it.n_kv > 0);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&br.acc_free[acc]);
      }
    }
    if (!ok && lane == 0) fail(kErrDeviceTimeout);
    if (C::kStage && warp == 2 && lane == 0) bulk_wait_all();  // stores done before the CTA retires
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int D, bool BLK>
cudaError_t launch_bwd_d(const BwdArgs& a, cudaStream_t s) {
  using C = BCfg<D>;
  static DeviceOnce attr_set;
  int dev = 0, n_sm = 0;
  cudaGetDevice(&dev);
  if (!attr_set.test(dev)) {
    // The dK/dV kernel's warpgroup register split needs every thread to start
    // with exactly kKVLaunchRegs registers.
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, bwd_dkdv_kernel<D, BLK>);
    if (e != cudaSuccess) return e;
    if (kKVSplit<D> && (fa.numRegs != kKVLaunchRegs || fa.maxThreadsPerBlock < kKVThreads<D>))
      return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(bwd_dq_kernel<D, BLK>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemQ);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(bwd_dkdv_kernel<D, BLK>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemKV);
    if (e != cudaSuccess) return e;
    attr_set.set(dev);
  }
  {
    const cudaError_t e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
  }
  CUtensorMap tq, tdo, tk, tv, to, tdq, tdk, tdv;
  if (!encode_bf16_map(&tq, a.q, a.B, a.Nq, a.Hq, D, kT) || !encode_bf16_map(&tdo, a.dout, a.B, a.Nq, a.Hq, D, kT) ||
      !encode_bf16_map(&tk, a.k, a.B, a.Nkv, a.Hkv, D, kT) || !encode_bf16_map(&tv, a.v, a.B, a.Nkv, a.Hkv, D, kT) ||
      !encode_bf16_map(&to, a.o, a.B, a.Nq, a.Hq, D, kT) || !encode_bf16_map(&tdq, a.dq, a.B, a.Nq, a.Hq, D, kT) ||
      !encode_bf16_map(&tdk, a.dk, a.B, a.Nkv, a.Hkv, D, kT) || !encode_bf16_map(&tdv, a.dv, a.B, a.Nkv, a.Hkv, D, kT))
    return cudaErrorInvalidValue;
  const long long n_q = static_cast<long long>((a.Nq + kT - 1) / kT) * a.Hq * a.B;
  const long long n_kv = static_cast<long long>((a.Nkv + kT - 1) / kT) * a.Hkv * a.B;
  // The dQ kernel also writes D and lse2, which the dK/dV kernel reads.
  bwd_dq_kernel<D, BLK><<<static_cast<unsigned>(n_q < n_sm ? n_q : n_sm), kBThreads, C::kSmemQ, s>>>(tq, tdo, tk, tv, to,
                                                                                                 tdq, a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_after_pdl(bwd_dkdv_kernel<D, BLK>, dim3(static_cast<unsigned>(n_kv < n_sm ? n_kv : n_sm)),
                          dim3(kKVThreads<D>), C::kSmemKV, s, tq, tdo, tk, tv, tdk, tdv, a);
}

}  // namespace

cudaError_t launch_bwd(int d, const BwdArgs& a, cudaStream_t s) {
  const bool blk = a.qlist != nullptr;
  if (d == 64) return blk ? launch_bwd_d<64, true>(a, s) : launch_bwd_d<64, false>(a, s);
  return blk ? launch_bwd_d<128, true>(a, s) : launch_bwd_d<128, false>(a, s);
}

}  // namespace eio
