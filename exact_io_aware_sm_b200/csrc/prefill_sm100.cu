// prefill_sm100.cu -- exact attention forward on sm_100a tensor cores.
//
// The fused, tiled forward pass of "FlashAttention: memory-saving exact
// attention" (section 3) in the Q-outer loop order, with block-sparse
// skipping (section 6): the host plan lists only the live KV tiles of each Q
// tile, and marks the few that need an element predicate.
//
// Persistent CTAs (one per SM) walk a list of work items.  An item is two
// 128-row Q tiles ("slots" A and B) that share every K/V tile loaded into
// shared memory: two query heads of one GQA group on the same rows, or two Q
// tiles of one head whose KV lists nest (slot A visits a prefix of slot B's
// list).  While the softmax warps of one slot work, the tensor core runs the
// other slot's GEMMs.
//
// Roles (384 threads, three warpgroups; the first gives registers to the
// two softmax warpgroups with setmaxnreg: 128 x 72 + 256 x 216 <= 384 x 168, or 80 and 208):
//   warp 0        TMA producer: Q_A, Q_B once per item (double-buffered for
//                 d = 64, whose items are short), then K_j, V_j into a ring of
//                 shared-memory stages.
//   warps 1, 2    MMA issuers for slot A and slot B (warp 1 also owns TMEM):
//                   S_X = Q_X K_j^T      (A and B from shared memory)
//                   O_X += P_X V_j       (P_X from TMEM, V_j from shared memory)
//                 issued from the converged warp by an elect.sync-chosen lane.
//   warp 3        idle.
//   warps 4..7    softmax for slot A, one thread per query row.
//   warps 8..11   softmax for slot B.
// Each softmax thread loads its whole S row from TMEM (one wait), takes the
// row max, keeps the running max m and sum l (online softmax: FlashAttention
// page section 2, inference page "Online-Softmax"), packs P to bf16 in
// registers and writes it to TMEM (64 columns of bf16 pairs), where the PV
// MMA reads it.  At the end of an item it writes O / l (bf16) and LSE.
//
// The exponent base moves only when a tile's row max exceeds it by more than
// 8 (log2 units); P may then reach 2^8, with O and l scaled against the same
// base, so the result is exactly softmax(S) V while most rescales vanish.
//
// TMEM columns: S_A [0,128), S_B [128,256), O_A [256, 256+d), O_B after O_A.
// d = 128: P_X overwrites the first 64 columns of S_X; the MMA issuer issues
// S_X(j+1) right after PV_X(j), and the tensor core's in-order execution of
// one thread's MMAs keeps the overwrite behind that PV's read of P.  d = 64 leaves 128 columns
// free: P_A [384,448) and P_B [448,512) have their own, and S_X(j+1) is
// issued as soon as the softmax threads have loaded S_X(j) into registers,
// so it overlaps their exponentials.
#include <cuda_bf16.h>

#include "fastmath.cuh"
#include "kernels.h"
#include "ptx_sm100.cuh"

namespace eio {
namespace {

constexpr int kThreads = 384;
// Register split between the warpgroups.  The kernel must be compiled to
// exactly kLaunchRegs registers per thread: the host refuses to launch it
// otherwise, since an increase that the pool cannot cover never returns.
constexpr int kLaunchRegs = 168;
// Warpgroup 0 (producer, MMA issuers) and warpgroups 1 and 2 (softmax).  The
// d = 128 running-max softmax (128 scores per thread) needs 216 to run without
// spills; the d = 64 forms and the bound-based half-tile forms fit their
// softmax in 208, and their issuers (more per-item state) spill at 72.
template <int D, bool BOUND>
struct RegSplit {
  static constexpr int kControl = (D == 64 || BOUND) ? 80 : 72;
  static constexpr int kSoftmax = (D == 64 || BOUND) ? 208 : 216;
  static_assert(128 * kControl + 256 * kSoftmax <= kThreads * kLaunchRegs,
                "register split must fit in the launch allocation");
};
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// Bound-based softmax: a row keeps the bound as its base only if no P can fall
// below 2^-kBoundLimit2 (every centred score lies within +-bound).
constexpr float kBoundLimit2 = 100.0f;
constexpr float kLn2 = 0.69314718055994530942f;

template <int D, bool BOUND = false>
struct Cfg {
  // Of every 8 column pairs of a tile, this many take the polynomial exp2
  // on the FMA pipe instead of the MUFU unit.  At d = 64, where the MUFU is
  // the bound, one in eight measured about 1 % faster; two in eight, and any
  // share at d = 128, measured slower.
  static constexpr int kPolyPairs = D == 64 ? 1 : 0;
  static constexpr int kQBuf = (D == 64) ? 2 : 1;         // Q buffers per slot
  // d = 64 leaves 128 TMEM columns free: P gets its own columns, so the next
  // S of a slot can be computed while the softmax of the current tile runs.
  static constexpr bool kSepP = D == 64;
  // Half-tile pipeline (d = 128, bound-based softmax): d = 128 has no free
  // TMEM columns for a separate P, so S is computed in halves of 64 keys into
  // two alternating 64-column buffers per slot, and the S of the next
  // half-tile runs on the tensor core while the softmax works on the current
  // one (P overwrites its own S half).  It pays where the softmax is short
  // (no row max: +16 % on the long-context workload); with the running max
  // the fixed per-step costs of twice as many steps cancel the overlap, so
  // that softmax keeps whole 128-key tiles.
  static constexpr bool kHalf = D == 128 && BOUND;
  static constexpr int kRing = (D == 64) ? 8 : 4;         // K/V tiles in flight
  static constexpr int kChunkBytes = 128 * 128;           // 128 rows x 64 bf16 (one swizzle span)
  static constexpr int kTileBytes = 128 * D * 2;          // Q, K or V tile (128 rows)
  static constexpr int kOffQ = 0;                         // Q[slot][buffer]
  static constexpr int kOffRing = 2 * kQBuf * kTileBytes;
  // d = 64: the epilogue stages each slot's bf16 O tile (128 rows x 128 B) in
  // shared memory so that rows are stored to HBM as whole 128-byte lines.
  static constexpr bool kStageO = D == 64;
  static constexpr int kOffStage = kOffRing + kRing * kTileBytes;
  static constexpr int kOffBar = kOffStage + (kStageO ? 2 * 128 * D * 2 : 0);
  // q_full[2*QB] q_empty[2*QB] ring_full[R] ring_empty[R] s_full[2] p_full[2]
  // pv_done[2] o_free[2] mma_idle[2] s_free[2] b_first[kQBuf] o_ready[2] p_fullb[2]
  static constexpr int kNumBars = 4 * kQBuf + 2 * kRing + 8 + 2 + 2 + kQBuf + 2 + 2;
  static constexpr int kSmem = kOffBar + 8 * kNumBars + 16 + 1024;  // + alignment slack
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Bound-based softmax ("TPU attention optimisation guide", step 4): the
// exponent base of a row, in log2 units, from the Cauchy-Schwarz bound on its
// centred scores, q . (k_j - kbar) <= ||q|| radius:
//   base = scale*log2(e) * (q . kbar + ||q|| radius).
// The centring only shifts all scores of the row by q . kbar, so P, O and the
// LSE are those of the plain definition.  Returns false (base untouched) when
// 2 * scale*log2(e) * ||q|| radius exceeds kBoundLimit2, where the row keeps
// the running max.  Rows past the tile's valid rows take base 0: their
// results are discarded.
template <int D>
__device__ __forceinline__ bool bound_base(const PrefillArgs& a, int b, int head, int hkv, int grow, bool valid,
                                           float sl2, float* base) {
  if (!valid) {
    *base = 0.f;
    return true;
  }
  const uint4* qr = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(a.q) +
                                                   ((static_cast<size_t>(b) * a.Nq + grow) * a.Hq + head) * D);
  const float4* kb = reinterpret_cast<const float4*>(a.kbar + (static_cast<size_t>(b) * a.Hkv + hkv) * D);
  float qk = 0.f, qq = 0.f;
#pragma unroll 4
  for (int e = 0; e < D / 8; ++e) {
    const uint4 u = qr[e];
    const float4 k0 = kb[2 * e], k1 = kb[2 * e + 1];
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
    const float2 f0 = __bfloat1622float2(h2[0]), f1 = __bfloat1622float2(h2[1]);
    const float2 f2 = __bfloat1622float2(h2[2]), f3 = __bfloat1622float2(h2[3]);
    qk = fmaf(f0.x, k0.x, fmaf(f0.y, k0.y, fmaf(f1.x, k0.z, fmaf(f1.y, k0.w, qk))));
    qk = fmaf(f2.x, k1.x, fmaf(f2.y, k1.y, fmaf(f3.x, k1.z, fmaf(f3.y, k1.w, qk))));
    qq = fmaf(f0.x, f0.x, fmaf(f0.y, f0.y, fmaf(f1.x, f1.x, fmaf(f1.y, f1.y, qq))));
    qq = fmaf(f2.x, f2.x, fmaf(f2.y, f2.y, fmaf(f3.x, f3.x, fmaf(f3.y, f3.y, qq))));
  }
  const float m = sl2 * sqrtf(qq) * a.radius[static_cast<size_t>(b) * a.Hkv + hkv];
  if (!(2.f * m <= kBoundLimit2)) return false;
  *base = fmaf(sl2, qk, m);
  return true;
}

// One work item, decoded identically by every role.
struct Item {
  int b, hkv, headA, headB;
  int rowA, nrowsA, rowB, nrowsB;
  int kv_first, nA, nB;
};

__device__ __forceinline__ Item decode_item(const PrefillArgs& a, long long w) {
  const long long per_rank = static_cast<long long>(a.B) * a.Hkv * a.HP;
  const int rank = static_cast<int>(w / per_rank);
  long long rem = w - rank * per_rank;
  Item it;
  it.b = static_cast<int>(rem / (static_cast<long long>(a.Hkv) * a.HP));
  rem -= static_cast<long long>(it.b) * a.Hkv * a.HP;
  it.hkv = static_cast<int>(rem / a.HP);
  const int hp = static_cast<int>(rem - static_cast<long long>(it.hkv) * a.HP);
  const int4 x0 = a.pairs[2 * rank];
  const int4 x1 = a.pairs[2 * rank + 1];
  it.rowA = x0.x;
  it.nrowsA = x0.y;
  it.rowB = x0.z;
  it.nrowsB = x0.w;
  it.kv_first = x1.x;
  it.nA = x1.y;
  it.nB = x1.z;
  if (a.rows_mode) {
    it.headA = it.headB = it.hkv;  // one query head per KV head
  } else {
    it.headA = it.hkv * a.G + 2 * hp;
    if (2 * hp + 1 < a.G) {
      it.headB = it.headA + 1;
    } else {  // odd group: its last head runs alone in slot B
      it.headB = it.headA;
      it.nrowsA = 0;
      it.nA = 0;
    }
  }
  return it;
}

// The k-th work item of this CTA, or -1 when there is none.  Items are sorted
// by size (largest first); rounds of gridDim.x items are dealt to the CTAs in
// alternating directions, which evens out the total work per CTA.
__device__ __forceinline__ long long item_index(long long k, long long n_items) {
  const long long g = gridDim.x, base = k * g;
  if (base >= n_items) return -1;
  const long long idx = (k & 1) ? base + (g - 1 - blockIdx.x) : base + blockIdx.x;
  return idx < n_items ? idx : -1;
}

constexpr bool kFirstLoadsFirst = true;
// Q tiles and O rows are each touched once: load and store them as
// evict_first in L2, so that they do not push out K/V tiles that the items
// of later rounds read again.
constexpr bool kStreamHintQ = true;
constexpr bool kStreamHintO = true;

// STAGGER: both slots of every pair visit the same number of KV tiles, and
// slot A starts each item after slot B's first exponentials (see below).
// BOUND: the bound-based softmax (see bound_base).
template <int D, bool STAGGER, bool BOUND>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_bf16_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ CUtensorMap tmO,
                        const __grid_constant__ CUtensorMap tmK16,
                        const __grid_constant__ CUtensorMap tmV16, const PrefillArgs a) {
  using C = Cfg<D, BOUND>;
  constexpr int R = C::kRing;
  constexpr int NCH = D / 64;  // 64-element swizzle chunks per row

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  constexpr int QB = C::kQBuf;
  uint64_t* q_full = bars;            // [2][QB]
  uint64_t* q_empty = bars + 2 * QB;  // [2][QB]
  uint64_t* ring_full = bars + 4 * QB;  // [R]
  uint64_t* ring_empty = ring_full + R;
  uint64_t* s_full = ring_empty + R;  // [2]
  uint64_t* p_full = s_full + 2;      // [2]
  uint64_t* pv_done = p_full + 2;     // [2]
  uint64_t* o_free = pv_done + 2;     // [2]
  uint64_t* mma_idle = o_free + 2;    // [2]
  uint64_t* s_free = mma_idle + 2;    // [2] (separate-P layout): S loaded by the softmax
  // b_first[i]: slot B has finished the exponentials of the first tile of an
  // offset item, item n on b_first[n % QB].  Slot B can start an item only
  // once the in-order producer has loaded slot A's Q for it, which needs slot
  // A's Q buffer of QB offset items earlier, freed only after slot A's wait
  // for that item; so slot B is at most QB - 1 items ahead of that wait, and
  // with QB barriers in turn no parity wait falls two phases behind.
  uint64_t* b_first = s_free + 2;     // [QB]
  // Half-tile layout (d = 128): s_full[x] and s_free[x] signal S in buffer 0
  // and 1 of slot x, p_full[x] and p_fullb[x] the P of buffer 0 and 1 (one
  // barrier per buffer: the softmax can finish the step after the next
  // before the issuer waits, and a parity wait must never be two phases
  // behind), and o_ready[x] the last PV of an item.
  uint64_t* o_ready = b_first + QB;   // [2]
  uint64_t* p_fullb = o_ready + 2;    // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2 * QB; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&s_full[x], 1);
      mbar_init(&p_full[x], 4);
      mbar_init(&pv_done[x], 1);
      mbar_init(&o_free[x], 4);
      mbar_init(&s_free[x], C::kHalf ? 1 : 4);
      mbar_init(&o_ready[x], 1);
      mbar_init(&p_fullb[x], 4);
    }
    for (int i = 0; i < R; ++i) {
      mbar_init(&ring_full[i], 1);
      mbar_init(&ring_empty[i], 2);  // released by both slot issuers
    }
    mbar_init(&mma_idle[0], 1);
    mbar_init(&mma_idle[1], 1);
    for (int i = 0; i < QB; ++i) mbar_init(&b_first[i], 4);
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

  const uint32_t sQ = smem_u32(smem + C::kOffQ);
  const uint32_t sRing = smem_u32(smem + C::kOffRing);
  const long long n_items = a.n_items;

  if (warp < 4) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(RegSplit<D, BOUND>::kControl));
  // The producer and MMA warps run converged; elect.sync picks the lane that
  // issues each TMA copy, MMA and commit.
  auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
    const bool mine = !*abort_flag && mbar_wait(bar, parity);
    return __all_sync(0xffffffffu, mine);
  };
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
    uint32_t seq = 0;
    uint32_t qcnt[2] = {0, 0};
    bool ok = true;
    long long wk = 0, w = item_index(0, n_items);
    Item it_next = w >= 0 ? decode_item(a, w) : Item{};
    for (; ok && w >= 0;) {
      const Item it = it_next;  // decoded one item ahead
      w = item_index(++wk, n_items);
      if (w >= 0) it_next = decode_item(a, w);
      const int nX[2] = {it.nA, it.nB};
      const int rowX[2] = {it.rowA, it.rowB};
      const int headX[2] = {it.headA, it.headB};
      for (int x = 0; x < 2 && ok; ++x) {
        if (nX[x] == 0) continue;
        const uint32_t qb = qcnt[x] % QB, use = qcnt[x] / QB;
        if (use > 0 && !wwait(&q_empty[x * QB + qb], (use - 1) & 1)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx_elect(&q_full[x * QB + qb], C::kTileBytes);
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch) {
          uint8_t* qdst = smem + C::kOffQ + (x * QB + qb) * C::kTileBytes + ch * C::kChunkBytes;
          if constexpr (kStreamHintQ)
            tma_load_4d_elect_hint(qdst, &tmQ, &q_full[x * QB + qb], ch * 64, headX[x], rowX[x], it.b,
                                   l2_policy_evict_first());
          else
            tma_load_4d_elect(qdst, &tmQ, &q_full[x * QB + qb], ch * 64, headX[x], rowX[x], it.b);
        }
        qcnt[x]++;
      }
      int4 kt_next = it.nB > 0 ? a.kvtiles[it.kv_first] : make_int4(0, 0, 0, 0);
      for (int j = 0; ok && j < it.nB; ++j) {
        const int4 kt = kt_next;  // read one tile ahead of its use
        if (j + 1 < it.nB) kt_next = a.kvtiles[it.kv_first + j + 1];
        for (int t = 0; t < 2; ++t) {
          const uint32_t slot = seq % R;
          if (seq >= R && !wwait(&ring_empty[slot], ((seq / R) + 1) & 1)) {
            ok = false;
            break;
          }
          if (a.fault == 1 && blockIdx.x == 0 && seq == 0) {  // test hook: never filled
            ++seq;
            continue;
          }
          const int n0 = (kt.z >> 8) & 0xFF;  // two-segment tile: keys in the first segment
          uint8_t* dst = smem + C::kOffRing + slot * C::kTileBytes;
          if (n0 == 0) {
            mbar_arrive_expect_tx_elect(&ring_full[slot], C::kTileBytes);
            const CUtensorMap* map = t == 0 ? &tmK : &tmV;
#pragma unroll
            for (int ch = 0; ch < NCH; ++ch)
              tma_load_4d_elect(dst + ch * C::kChunkBytes, map, &ring_full[slot], ch * 64, it.hkv, kt.x, it.b);
          } else {
            // [kt.x, kt.x + n0) then [kt.w, ...) into consecutive rows, 16 rows per copy
            mbar_arrive_expect_tx_elect(&ring_full[slot], static_cast<uint32_t>(kt.y) * 128 * NCH);
            const CUtensorMap* map = t == 0 ? &tmK16 : &tmV16;
            for (int r = 0; r < kt.y; r += 16) {
              const int src = r < n0 ? kt.x + r : kt.w + (r - n0);
#pragma unroll
              for (int ch = 0; ch < NCH; ++ch)
                tma_load_4d_elect(dst + ch * C::kChunkBytes + r * 128, map, &ring_full[slot], ch * 64, it.hkv, src,
                                  it.b);
            }
          }
          ++seq;
          // At start-up every CTA fills its whole ring at once; let the first
          // K tile (and the Q tiles issued before it) land before queueing the
          // rest, so that the first S does not wait behind the whole burst.
          if (kFirstLoadsFirst && seq == 2 && !wwait(&ring_full[0], 0)) {
            ok = false;
            break;
          }
        }
      }
    }
    if (!ok) {
      if (lane == 0) fail(kErrDeviceTimeout);
      // Let every copy this warp started land before the CTA retires.
      for (int x = 0; x < 2; ++x)
        for (uint32_t c = qcnt[x] > QB ? qcnt[x] - QB : 0; c < qcnt[x]; ++c)
          mbar_wait(&q_full[x * QB + c % QB], (c / QB) & 1);
      for (uint32_t s = seq > R ? seq - R : 0; s < seq; ++s)
        mbar_wait(&ring_full[s % R], (s / R) & 1);
    }
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------------ MMA issuers
    // Warp 1 issues slot A's GEMMs, warp 2 slot B's, so each slot's chain
    // (S -> softmax -> PV) advances on its own.
    const int x = warp - 1;
    const uint32_t idO = idesc_bf16_f32(128, D, 0, 1);  // A = P (TMEM), B = V (MN-major)
    const uint32_t s_col = tmem + static_cast<uint32_t>(x * 128);
    const uint32_t o_col = tmem + static_cast<uint32_t>(256 + x * D);
    const uint32_t p_col = C::kSepP ? tmem + static_cast<uint32_t>(256 + 2 * D + x * 64) : s_col;
    uint32_t seq = 0, qcnt = 0, scnt = 0, pcnt = 0, ocnt = 0;
    bool ok = true;
    auto wait_bar = [&](uint64_t* bar, uint32_t parity) -> bool {
      if (!ok) return false;
      ok = wwait(bar, parity);
      return ok;
    };
    // S_X = Q_X K^T for the K tile in ring slot kslot; releases the stage.
    auto issue_s = [&](uint32_t qbase, int ncols, uint32_t kslot) {
      // S_X is rewritten.  Separate P: the softmax must have loaded S_X.  P in
      // S's columns: the PV that reads P was issued just before by this
      // thread, and the tensor core executes one thread's MMAs in issue
      // order, so this S overwrites P only after that PV has read it.
      if (C::kSepP && scnt > 0 && !wait_bar(&s_free[x], (scnt - 1) & 1)) return;
      tc_fence_after();
      const uint32_t id = idesc_bf16_f32(128, static_cast<uint32_t>(ncols), 0, 0);
      const uint32_t kbase = sRing + kslot * C::kTileBytes;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t koff = (kk >> 2) * C::kChunkBytes + (kk & 3) * 32;
        mma_bf16_ss_elect(s_col, sdesc_sw128(qbase + koff, 16, 1024), sdesc_sw128(kbase + koff, 16, 1024),
                          id, kk > 0 ? 1u : 0u);
      }
      mma_commit_elect(&s_full[x]);
      mma_commit_elect(&ring_empty[kslot]);
      scnt++;
    };
    // O_X (+)= P_X V for the V tile in ring slot vslot; releases the stage.
    auto issue_pv = [&](int j, int ncols, uint32_t vslot) {
      if (!wait_bar(&p_full[x], pcnt & 1)) return;
      if (j == 0 && ocnt > 0 && !wait_bar(&o_free[x], (ocnt - 1) & 1)) return;
      tc_fence_after();
      const uint32_t vbase = sRing + vslot * C::kTileBytes;
      for (int kk = 0; kk < (ncols >> 4); ++kk)
        mma_bf16_ts_elect(o_col, p_col + kk * 8, sdesc_sw128(vbase + kk * 2048, C::kChunkBytes, 1024),
                          idO, (j > 0 || kk > 0) ? 1u : 0u);
      mma_commit_elect(&pv_done[x]);
      mma_commit_elect(&ring_empty[vslot]);
      pcnt++;
    };

    long long wk = 0, w = item_index(0, n_items);
    Item it_next = w >= 0 ? decode_item(a, w) : Item{};
    for (; ok && w >= 0;) {
      const Item it = it_next;  // decoded one item ahead
      w = item_index(++wk, n_items);
      if (w >= 0) it_next = decode_item(a, w);
      if constexpr (C::kHalf) {
        // Half-tile steps: each KV tile of up to 128 keys is one or two steps
        // of up to 64 keys (h = 0, 1).  Step s writes S into buffer s & 1 of
        // this slot; the issue order S(0), S(1), then per step PV(s), S(s + 2)
        // lets S(s + 2) overwrite the buffer of P(s) only after PV(s) has read
        // it (one thread's MMAs execute in order).
        const int nX = x == 0 ? it.nA : it.nB;
        const int nB = it.nB;
        const int4* kv = a.kvtiles + it.kv_first;
        uint32_t qbuf = 0;
        if (nX > 0) {
          qbuf = qcnt % QB;
          if (!wait_bar(&q_full[x * QB + qbuf], (qcnt / QB) & 1)) break;
          qcnt++;
          const uint32_t qbase = sQ + (x * QB + qbuf) * C::kTileBytes;
          int sj = 0, sh = 0, snc = kv[0].y;  // next S step: tile, half, tile width
          int pj = 0, ph = 0, pnc = snc;      // next PV step
          auto issue_sh = [&]() {
            const uint32_t kpos = seq + 2 * sj;
            if (sh == 0 && !wait_bar(&ring_full[kpos % R], (kpos / R) & 1)) return;
            tc_fence_after();
            const uint32_t ncols = static_cast<uint32_t>(min(64, snc - 64 * sh));
            const uint32_t b = scnt & 1;
            const uint32_t id = idesc_bf16_f32(128, ncols, 0, 0);
            const uint32_t kbase = sRing + (kpos % R) * C::kTileBytes + sh * 64 * 128;  // rows 64h.. of K
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t koff = (kk >> 2) * C::kChunkBytes + (kk & 3) * 32;
              mma_bf16_ss_elect(s_col + b * 64, sdesc_sw128(qbase + koff, 16, 1024),
                                sdesc_sw128(kbase + koff, 16, 1024), id, kk > 0 ? 1u : 0u);
            }
            mma_commit_elect(b == 0 ? &s_full[x] : &s_free[x]);
            const bool last = sh == 1 || snc <= 64;
            if (last) mma_commit_elect(&ring_empty[kpos % R]);  // K tile read by both halves
            scnt++;
            if (last) {
              ++sj;
              sh = 0;
              snc = sj < nX ? kv[sj].y : 0;
            } else {
              sh = 1;
            }
          };
          auto issue_pvh = [&]() {
            const uint32_t vpos = seq + 2 * pj + 1;
            if (!wait_bar((pcnt & 1) == 0 ? &p_full[x] : &p_fullb[x], (pcnt >> 1) & 1)) return;
            if (pj == 0 && ph == 0 && ocnt > 0 && !wait_bar(&o_free[x], (ocnt - 1) & 1)) return;
            if (ph == 0 && !wait_bar(&ring_full[vpos % R], (vpos / R) & 1)) return;
            tc_fence_after();
            const int nk = min(64, pnc - 64 * ph);
            const uint32_t b = pcnt & 1;
            const uint32_t vbase = sRing + (vpos % R) * C::kTileBytes;
            for (int i = 0; i < (nk >> 4); ++i)
              mma_bf16_ts_elect(o_col, s_col + b * 64 + i * 8,
                                sdesc_sw128(vbase + (4 * ph + i) * 2048, C::kChunkBytes, 1024), idO,
                                (pj > 0 || ph > 0 || i > 0) ? 1u : 0u);
            mma_commit_elect(&pv_done[x]);
            const bool last = ph == 1 || pnc <= 64;
            if (last) mma_commit_elect(&ring_empty[vpos % R]);
            pcnt++;
            if (last) {
              ++pj;
              ph = 0;
              pnc = pj < nX ? kv[pj].y : 0;
            } else {
              ph = 1;
            }
          };
          issue_sh();
          if (ok && sj < nX) issue_sh();
          while (ok && pj < nX) {
            issue_pvh();
            if (ok && sj < nX) issue_sh();
          }
          if (ok) mma_commit_elect(&o_ready[x]);  // the item's last PV
          ocnt++;
        }
        // Stages of tiles this slot does not visit: release once filled.
        for (int j = nX; ok && j < nB; ++j) {
          const uint32_t kseq = seq + 2 * j, vseq = kseq + 1;
          if (!wait_bar(&ring_full[kseq % R], (kseq / R) & 1)) break;
          mbar_arrive_elect(&ring_empty[kseq % R]);
          if (!wait_bar(&ring_full[vseq % R], (vseq / R) & 1)) break;
          mbar_arrive_elect(&ring_empty[vseq % R]);
        }
        seq += 2 * nB;
        if (!ok) break;
        if (nX > 0) mma_commit_elect(&q_empty[x * QB + qbuf]);
        continue;
      }
      const int nX = x == 0 ? it.nA : it.nB;
      const int nB = it.nB;
      const int4* kv = a.kvtiles + it.kv_first;
      // Tile widths are read one tile ahead of their use.
      int nc_cur = nX > 0 ? kv[0].y : 0, nc_next = nX > 1 ? kv[1].y : 0;
      uint32_t qbuf = 0;
      if (nX > 0) {
        qbuf = qcnt % QB;
        if (!wait_bar(&q_full[x * QB + qbuf], (qcnt / QB) & 1)) break;
        qcnt++;
        const uint32_t qbase = sQ + (x * QB + qbuf) * C::kTileBytes;
        if (!wait_bar(&ring_full[seq % R], (seq / R) & 1)) break;
        issue_s(qbase, nc_cur, seq % R);
        for (int j = 0; ok && j < nX; ++j) {
          const uint32_t vseq = seq + 2 * j + 1, kseq = vseq + 1;
          const bool next = j + 1 < nX;
          const int nc_after = j + 2 < nX ? kv[j + 2].y : 0;
          if (C::kSepP && next) {  // next S as soon as the softmax has loaded this one
            if (!wait_bar(&ring_full[kseq % R], (kseq / R) & 1)) break;
            issue_s(qbase, nc_next, kseq % R);
          }
          if (!wait_bar(&ring_full[vseq % R], (vseq / R) & 1)) break;
          issue_pv(j, nc_cur, vseq % R);
          if (!C::kSepP && next) {  // P shares S's columns: right after this PV
            if (!wait_bar(&ring_full[kseq % R], (kseq / R) & 1)) break;
            issue_s(qbase, nc_next, kseq % R);
          }
          nc_cur = nc_next;
          nc_next = nc_after;
        }
        ocnt++;
      }
      // Stages of tiles this slot does not visit: release once filled.
      for (int j = nX; ok && j < nB; ++j) {
        const uint32_t kseq = seq + 2 * j, vseq = kseq + 1;
        if (!wait_bar(&ring_full[kseq % R], (kseq / R) & 1)) break;
        mbar_arrive_elect(&ring_empty[kseq % R]);
        if (!wait_bar(&ring_full[vseq % R], (vseq / R) & 1)) break;
        mbar_arrive_elect(&ring_empty[vseq % R]);
      }
      seq += 2 * nB;
      if (!ok) break;
      if (nX > 0) mma_commit_elect(&q_empty[x * QB + qbuf]);
    }
    if (!ok && lane == 0) fail(kErrDeviceTimeout);
    // Every MMA issued above has finished before TMEM is released.
    mma_commit_elect(&mma_idle[x]);
    mbar_wait(&mma_idle[x], 0);
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(RegSplit<D, BOUND>::kSoftmax));
    // ------------------------------------------------------------ softmax
    const int x = (warp - 4) >> 2;  // slot
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t s_tmem = tmem + lane_off + static_cast<uint32_t>(x * 128);
    const uint32_t o_tmem = tmem + lane_off + static_cast<uint32_t>(256 + x * D);
    const uint32_t p_tmem = C::kSepP ? tmem + lane_off + static_cast<uint32_t>(256 + 2 * D + x * 64) : s_tmem;
    const float sl2 = a.scale_log2;
    uint32_t tcnt = 0, bcnt = 0, icnt = 0;
    bool ok = true;
    // Waits and the abort decision are made warp-uniform, because the warp
    // then executes .sync.aligned tcgen05 instructions together.
    auto warp_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
      const bool mine = !*abort_flag && mbar_wait(bar, parity);
      return __all_sync(0xffffffffu, mine);
    };

    long long wk = 0, w = item_index(0, n_items);
    Item it_next = w >= 0 ? decode_item(a, w) : Item{};
    for (; ok && w >= 0;) {
      const Item it = it_next;  // decoded one item ahead
      w = item_index(++wk, n_items);
      if (w >= 0) it_next = decode_item(a, w);
      const int nX = x == 0 ? it.nA : it.nB;
      const int nrows = x == 0 ? it.nrowsA : it.nrowsB;
      const int row0 = x == 0 ? it.rowA : it.rowB;
      const int head = x == 0 ? it.headA : it.headB;
      if (nrows == 0) continue;  // slot unused in this item
      // Offset the two slots, so that one slot's exponentials overlap the
      // other's loads, stores and waits instead of both contending for the
      // MUFU at once: slot A starts an item when slot B has finished the
      // exponentials of its first tile.  Done when both slots of every pair
      // visit the same number of KV tiles (GQA head pairs, Q tiles inside one
      // frame); the offset then persists through the item.
      const int grow = row0 + row;
      float m_b = -INFINITY;  // exponent base, log2 units
      // Bound-based softmax: rows with a fixed base skip the max; a warp whose
      // rows all have one skips the row-max reduction entirely.  (Computed
      // before the slot offset below, so that its loads overlap that wait.)
      bool fixed = false;
      if constexpr (BOUND) {
        fixed = bound_base<D>(a, it.b, head, it.hkv, grow, row < nrows, sl2, &m_b);
        const unsigned fb = __ballot_sync(0xffffffffu, !fixed);
        if (lane == 0 && fb != 0u && a.n_fallback != nullptr) atomicAdd(a.n_fallback, __popc(fb));
      }
      const bool skip_max = BOUND && __all_sync(0xffffffffu, fixed);
      const bool stagger = STAGGER && it.nA > 0;
      if (stagger && x == 0) {
        if (!warp_wait(&b_first[bcnt % QB], (bcnt / QB) & 1)) {
          ok = false;
          break;
        }
      }
      if (stagger) bcnt++;
      const int4* kv = a.kvtiles + it.kv_first;
      float l = 0.f;
      int4 kt_next = nX > 0 ? kv[0] : make_int4(0, 0, 0, 0);

      if constexpr (C::kHalf) {
      // Half-tile steps (see the MMA issuer): step t of this slot reads S from
      // buffer t & 1 (64 columns), writes its P over the first 32 of them.
      const uint32_t tcnt0 = tcnt;
      for (int j = 0; j < nX && ok; ++j) {
        const int4 kt = kt_next;
        if (j + 1 < nX) kt_next = kv[j + 1];
        const int nh = kt.y > 64 ? 2 : 1;
        for (int h = 0; h < nh; ++h) {
          const uint32_t b = tcnt & 1;
          if (!warp_wait(b == 0 ? &s_full[x] : &s_free[x], (tcnt >> 1) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // Columns at or past `lim` are masked: past the half's width always,
          // and on partial tiles past Nkv and past the causal diagonal.
          int lim = min(64, kt.y - 64 * h);
          if ((kt.z >> x) & 1) {
            lim = min(lim, a.Nkv - kt.x - 64 * h);
            if (a.causal) lim = min(lim, grow + a.causal_off + 1 - kt.x - 64 * h);
          }
          uint32_t sr[64];
          tmem_ld32(s_tmem + b * 64, sr);
          tmem_ld32(s_tmem + b * 64 + 32, sr + 32);
          tmem_wait_ld();
          if (__any_sync(0xffffffffu, lim < 64)) {
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (c >= lim) sr[c] = __float_as_uint(-INFINITY);
          }
          float mx_s = -INFINITY;
          if (!BOUND || !skip_max) {
            float mx4[4];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              float m = __uint_as_float(sr[q4 * 16]);
#pragma unroll
              for (int c = 1; c < 15; c += 2)
                m = max3f(m, __uint_as_float(sr[q4 * 16 + c]), __uint_as_float(sr[q4 * 16 + c + 1]));
              mx4[q4] = fmaxf(m, __uint_as_float(sr[q4 * 16 + 15]));
            }
            mx_s = max3f(fmaxf(mx4[0], mx4[1]), mx4[2], mx4[3]) * sl2;
          }
          const bool upd = (!BOUND || !fixed) && mx_s > m_b + kRescaleThreshold;
          const float alpha = upd ? ex2(m_b - mx_s) : 1.f;  // 0 when m_b was -inf
          if (upd) m_b = mx_s;
          const float base = m_b == -INFINITY ? 0.f : m_b;
          float2 acc[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
          const float2 sl = make_float2(sl2, sl2), nb = make_float2(-base, -base);
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            const float2 e = ffma2(make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sl, nb);
            const float2 p = make_float2(ex2(e.x), ex2(e.y));
            acc[(c >> 1) & 3] = fadd2(acc[(c >> 1) & 3], p);
            sr[c >> 1] = pack_bf16x2(p.x, p.y);
          }
          if (stagger && x == 1 && tcnt == tcnt0) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&b_first[(bcnt - 1) % QB]);  // bcnt counts this item already
          }
          if (tcnt > tcnt0 && __any_sync(0xffffffffu, upd)) {
            // O holds the earlier steps: the previous step's PV must have
            // completed before O is rescaled.
            if (!warp_wait(&pv_done[x], (tcnt - 1) & 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < D; c += 32) {
              uint32_t orr[32];
              tmem_ld32(o_tmem + c, orr);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) orr[i] = __float_as_uint(__uint_as_float(orr[i]) * alpha);
              tmem_st32(o_tmem + c, orr);
            }
          }
          const float2 s01 = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
          l = l * alpha + (s01.x + s01.y);
          tmem_st32(s_tmem + b * 64, sr);  // P: 64 keys as 32 columns of bf16 pairs
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(b == 0 ? &p_full[x] : &p_fullb[x]);
          tcnt++;
        }
      }
      } else {
      for (int t = 0; t < nX; ++t) {
        const int4 kt = kt_next;
        if (t + 1 < nX) kt_next = kv[t + 1];
        const int nc = kt.y;
        if (!warp_wait(&s_full[x], tcnt & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // Columns at or past `lim` are masked: past the tile width always,
        // and on partial tiles past Nkv and past the causal diagonal.
        int lim = nc;
        if ((kt.z >> x) & 1) {
          lim = min(lim, a.Nkv - kt.x);
          if (a.causal) lim = min(lim, grow + a.causal_off + 1 - kt.x);
        }
        uint32_t sr[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(s_tmem + c * 32, sr + c * 32);
        tmem_wait_ld();
        if constexpr (C::kSepP) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&s_free[x]);
        }
        if (__any_sync(0xffffffffu, lim < 128)) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= lim) sr[c] = __float_as_uint(-INFINITY);
        }
        // Row max: four independent chains of 3-input max.
        float mx_s = -INFINITY;
        if (!BOUND || !skip_max) {
          float mx4[4];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            float m = __uint_as_float(sr[q4 * 32]);
#pragma unroll
            for (int c = 1; c < 31; c += 2)
              m = max3f(m, __uint_as_float(sr[q4 * 32 + c]), __uint_as_float(sr[q4 * 32 + c + 1]));
            mx4[q4] = fmaxf(m, __uint_as_float(sr[q4 * 32 + 31]));
          }
          mx_s = max3f(fmaxf(mx4[0], mx4[1]), mx4[2], mx4[3]) * sl2;
        }
        const bool upd = (!BOUND || !fixed) && mx_s > m_b + kRescaleThreshold;
        const float alpha = upd ? ex2(m_b - mx_s) : 1.f;  // 0 when m_b was -inf
        if (upd) m_b = mx_s;
        const float base = m_b == -INFINITY ? 0.f : m_b;
        // p = 2^(s * scale*log2e - base); packed bf16 pairs overwrite sr[0..63].
        float2 acc[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
        const float2 sl = make_float2(sl2, sl2), nb = make_float2(-base, -base);
#pragma unroll
        for (int c = 0; c < 128; c += 2) {
          const float2 e = ffma2(make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sl, nb);
          const float2 p = ((c >> 1) & 7) < C::kPolyPairs ? exp2_poly2(e) : make_float2(ex2(e.x), ex2(e.y));
          acc[(c >> 1) & 3] = fadd2(acc[(c >> 1) & 3], p);
          sr[c >> 1] = pack_bf16x2(p.x, p.y);
        }
        if (stagger && x == 1 && t == 0) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&b_first[(bcnt - 1) % QB]);  // bcnt counts this item already
        }
        if (C::kSepP && t > 0) {
          // P_X and O_X are free once PV_{t-1} has completed.
          if (!warp_wait(&pv_done[x], (tcnt - 1) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        if (t > 0 && __any_sync(0xffffffffu, upd)) {
          // O holds earlier tiles (PV_{t-1} has completed): rescale it.
#pragma unroll
          for (int c = 0; c < D; c += 32) {
            uint32_t orr[32];
            tmem_ld32(o_tmem + c, orr);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) orr[i] = __float_as_uint(__uint_as_float(orr[i]) * alpha);
            tmem_st32(o_tmem + c, orr);
          }
        }
        const float2 s01 = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
        l = l * alpha + (s01.x + s01.y);
        // P over the first 64 columns of this S row.
        tmem_st32(p_tmem, sr);
        tmem_st32(p_tmem + 32, sr + 32);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[x]);
        tcnt++;
      }
      }
      if (!ok) break;

      // ---------------------------------------------------------- epilogue
      if (nX > 0) {
        // the item's last PV has completed
        if (!warp_wait(C::kHalf ? &o_ready[x] : &pv_done[x], C::kHalf ? (icnt & 1) : ((tcnt - 1) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        icnt++;
      }
      const float inv_l = l > 0.f ? 1.0f / l : 0.f;
      const bool valid = row < nrows;
      if constexpr (C::kStageO) {
        // Row -> shared staging (16-byte units XOR-swizzled by row), then
        // each warp stores its 32 rows as whole lines.
        uint8_t* stg = smem + C::kOffStage + x * (128 * D * 2);
        // The previous item's stores from this buffer must have read it.
        if (lane == 0) bulk_wait_read_all();
        __syncwarp();
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t orr[32];
          if (nX > 0) {
            tmem_ld32(o_tmem + c, orr);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) orr[i] = 0u;
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int unit = c / 8 + u;
            *reinterpret_cast<uint4*>(stg + row * (D * 2) + ((unit ^ (row & 7)) << 4)) = make_uint4(
                pack_bf16x2(__uint_as_float(orr[u * 8 + 0]) * inv_l, __uint_as_float(orr[u * 8 + 1]) * inv_l),
                pack_bf16x2(__uint_as_float(orr[u * 8 + 2]) * inv_l, __uint_as_float(orr[u * 8 + 3]) * inv_l),
                pack_bf16x2(__uint_as_float(orr[u * 8 + 4]) * inv_l, __uint_as_float(orr[u * 8 + 5]) * inv_l),
                pack_bf16x2(__uint_as_float(orr[u * 8 + 6]) * inv_l, __uint_as_float(orr[u * 8 + 7]) * inv_l));
          }
        }
        // The staging rows are in the 128-byte-swizzled layout of the O map:
        // one TMA store per 16 rows of the tile (a tile's row count is a
        // multiple of 16 unless it ends at Nq, where the map clips).
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
#pragma unroll
          for (int h = 0; h < 2; ++h)
            if (quarter * 32 + 16 * h < nrows) {
              if constexpr (kStreamHintO)
                tma_store_4d_hint(&tmO, stg + (quarter * 32 + 16 * h) * (D * 2), 0, head,
                                  row0 + quarter * 32 + 16 * h, it.b, l2_policy_evict_first());
              else
                tma_store_4d(&tmO, stg + (quarter * 32 + 16 * h) * (D * 2), 0, head, row0 + quarter * 32 + 16 * h,
                             it.b);
            }
          bulk_commit();
        }
      } else {
      uint8_t* orow = reinterpret_cast<uint8_t*>(a.o) +
                      2 * (((static_cast<size_t>(it.b) * a.Nq + grow) * a.Hq + head) * D);
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t orr[32];
        if (nX > 0) {
          tmem_ld32(o_tmem + c, orr);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) orr[i] = 0u;
        }
        if (valid) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const uint4 v = make_uint4(
                pack_bf16x2(__uint_as_float(orr[u * 8 + 0]) * inv_l, __uint_as_float(orr[u * 8 + 1]) * inv_l),
                pack_bf16x2(__uint_as_float(orr[u * 8 + 2]) * inv_l, __uint_as_float(orr[u * 8 + 3]) * inv_l),
                pack_bf16x2(__uint_as_float(orr[u * 8 + 4]) * inv_l, __uint_as_float(orr[u * 8 + 5]) * inv_l),
                pack_bf16x2(__uint_as_float(orr[u * 8 + 6]) * inv_l, __uint_as_float(orr[u * 8 + 7]) * inv_l));
            if constexpr (kStreamHintO)
              st_global_v4_hint(orow + 2 * (c + u * 8), v, l2_policy_evict_first());
            else
              *reinterpret_cast<uint4*>(orow + 2 * (c + u * 8)) = v;
          }
        }
      }
      }
      if (nX > 0) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&o_free[x]);
      }
      if (a.lse != nullptr && valid)
        a.lse[(static_cast<size_t>(it.b) * a.Hq + head) * a.Nq + grow] =
            l > 0.f ? (m_b + __log2f(l)) * kLn2 : -INFINITY;
    }
    if (!ok) fail(kErrDeviceTimeout);
    if constexpr (C::kStageO) {
      if (lane == 0) bulk_wait_all();  // O stores complete before the CTA retires
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int D, bool STAGGER, bool BOUND>
cudaError_t launch_ds(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                      const CUtensorMap& to, const CUtensorMap& tk16, const CUtensorMap& tv16,
                      const PrefillArgs& a, cudaStream_t s) {
  static DeviceOnce attr_set;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!attr_set.test(dev)) {
    // The warpgroup register split is only safe when every thread starts with
    // exactly kLaunchRegs registers.
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, prefill_bf16_kernel<D, STAGGER, BOUND>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != kLaunchRegs || fa.maxThreadsPerBlock < kThreads) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(prefill_bf16_kernel<D, STAGGER, BOUND>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg<D, BOUND>::kSmem);
    if (e != cudaSuccess) return e;
    attr_set.set(dev);
  }
  if (a.n_items == 0) return cudaSuccess;
  const long long grid = a.n_items < a.num_ctas ? a.n_items : a.num_ctas;
  prefill_bf16_kernel<D, STAGGER, BOUND>
      <<<static_cast<unsigned>(grid), kThreads, Cfg<D, BOUND>::kSmem, s>>>(tq, tk, tv, to, tk16, tv16, a);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                     const CUtensorMap& to, const CUtensorMap& tk16, const CUtensorMap& tv16,
                     const PrefillArgs& a, cudaStream_t s) {
  if (a.bound)
    return a.stagger ? launch_ds<D, true, true>(tq, tk, tv, to, tk16, tv16, a, s)
                     : launch_ds<D, false, true>(tq, tk, tv, to, tk16, tv16, a, s);
  return a.stagger ? launch_ds<D, true, false>(tq, tk, tv, to, tk16, tv16, a, s)
                   : launch_ds<D, false, false>(tq, tk, tv, to, tk16, tv16, a, s);
}

}  // namespace

int prefill_bf16_smem_bytes(int d) { return d == 64 ? Cfg<64>::kSmem : Cfg<128>::kSmem; }

cudaError_t launch_prefill_bf16(int d, const CUtensorMap& tq, const CUtensorMap& tk,
                                const CUtensorMap& tv, const CUtensorMap& to, const CUtensorMap& tk16,
                                const CUtensorMap& tv16, const PrefillArgs& a, cudaStream_t s) {
  if (d == 64) return launch_d<64>(tq, tk, tv, to, tk16, tv16, a, s);
  return launch_d<128>(tq, tk, tv, to, tk16, tv16, a, s);
}

}  // namespace eio
