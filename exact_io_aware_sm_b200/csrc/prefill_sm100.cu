// prefill_sm100.cu -- exact attention forward on sm_100a tensor cores.
//
// One CTA computes one 128-row Q tile of one (batch, query head): the fused,
// tiled forward pass of "FlashAttention: memory-saving exact attention"
// (section 3), in the Q-outer loop order, with block-sparse skipping
// (section 6): the host plan lists only the live KV tiles of each Q tile.
//
// Roles (192 threads):
//   warp 0      TMA producer: Q once, then K_j / V_j into a ring of stages.
//   warp 1      MMA issuer (one thread): S_j = Q K_j^T into one of two TMEM
//               score buffers, and O += P_j V_j into a TMEM accumulator.
//               Also owns the TMEM allocation.
//   warps 2..5  softmax: one thread per query row.  Reads S_j from TMEM,
//               applies the predicate on partial tiles only, updates the
//               running max m and sum l (online softmax, FlashAttention page
//               section 2; inference page "Online-Softmax"), writes P_j
//               (bf16) to shared memory, rescales O in TMEM when m moved,
//               and finally writes O / l and LSE.
//
// The running max is only moved when the new row max exceeds it by more than
// 2^8 in the exponent; otherwise the old base is kept and P may reach 256.
// O and l are always scaled against the same base, so the result is exactly
// softmax(S) V; the threshold only skips accumulator rescales.
//
// TMEM columns: [0,128) S buffer 0, [128,256) S buffer 1, [256, 256+d) O.
#include <cuda_bf16.h>

#include "kernels.h"
#include "ptx_sm100.cuh"

namespace eio {
namespace {

constexpr int kThreads = 192;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr float kLn2 = 0.69314718055994530942f;

template <int D>
struct Cfg {
  static constexpr int kStages = (D == 64) ? 4 : 2;
  static constexpr int kChunkBytes = 128 * 128;        // 128 rows x 64 bf16 (one swizzle span)
  static constexpr int kTileBytes = 128 * D * 2;       // Q, K or V tile (128 rows)
  static constexpr int kPBytes = 128 * 128 * 2;        // P tile (128 x 128 bf16)
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kTileBytes;
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  static constexpr int kOffP = kOffV + kStages * kTileBytes;
  static constexpr int kOffBar = kOffP + kPBytes;
  static constexpr int kNumBars = 1 + 4 * kStages + 2 + 2 + 1 + 1 + 1;
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

// Packed fp32 pair arithmetic (sm_100): one instruction for two lanes of work.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_bf16_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const PrefillArgs a) {
  using C = Cfg<D>;
  constexpr int S = C::kStages;
  constexpr int NCH = D / 64;  // 64-element swizzle chunks per row

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = k_full + S;
  uint64_t* k_empty = v_full + S;
  uint64_t* v_empty = k_empty + S;
  uint64_t* s_full = v_empty + S;   // [2]
  uint64_t* s_free = s_full + 2;    // [2]
  uint64_t* p_full = s_free + 2;
  uint64_t* pv_done = p_full + 1;
  uint64_t* mma_idle = pv_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int bh = a.B * a.Hq;
  const int rank = blockIdx.x / bh;
  const int rem = blockIdx.x - rank * bh;
  const int b = rem / a.Hq;
  const int hq = rem - b * a.Hq;
  const int hkv = hq / (a.Hq / a.Hkv);
  const int4 qt = a.qtiles[a.order[rank]];
  const int q_row0 = qt.x, q_rows = qt.y, kv_first = qt.z, n_kv = qt.w;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < S; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
    }
    mbar_init(p_full, 4);
    mbar_init(pv_done, 1);
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

  const uint32_t sQ = smem_u32(smem + C::kOffQ);
  const uint32_t sK = smem_u32(smem + C::kOffK);
  const uint32_t sV = smem_u32(smem + C::kOffV);
  const uint32_t sP = smem_u32(smem + C::kOffP);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n_kv > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(q_full, C::kTileBytes);
#pragma unroll
      for (int ch = 0; ch < NCH; ++ch)
        tma_load_4d(smem + C::kOffQ + ch * C::kChunkBytes, &tmQ, q_full, ch * 64, hq, q_row0, b);
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < n_kv; ++j) {
        if (*abort_flag) break;
        const int4 kt = a.kvtiles[kv_first + j];
        const int st = j % S;
        const uint32_t ph_empty = ((j / S) + 1) & 1;
        if (j >= S && !mbar_wait(&k_empty[st], ph_empty)) {
          fail(kErrDeviceTimeout);
          break;
        }
        mbar_arrive_expect_tx(&k_full[st], C::kTileBytes);
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch)
          tma_load_4d(smem + C::kOffK + st * C::kTileBytes + ch * C::kChunkBytes, &tmK, &k_full[st],
                      ch * 64, hkv, kt.x, b);
        k_issued = j + 1;
        if (j >= S && !mbar_wait(&v_empty[st], ph_empty)) {
          fail(kErrDeviceTimeout);
          break;
        }
        mbar_arrive_expect_tx(&v_full[st], C::kTileBytes);
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch)
          tma_load_4d(smem + C::kOffV + st * C::kTileBytes + ch * C::kChunkBytes, &tmV, &v_full[st],
                      ch * 64, hkv, kt.x, b);
        v_issued = j + 1;
      }
      if (*abort_flag) {
        // Let every copy this thread started land before the CTA retires.
        mbar_wait(q_full, 0);
        for (int j = k_issued - S < 0 ? 0 : k_issued - S; j < k_issued; ++j)
          mbar_wait(&k_full[j % S], (j / S) & 1);
        for (int j = v_issued - S < 0 ? 0 : v_issued - S; j < v_issued; ++j)
          mbar_wait(&v_full[j % S], (j / S) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_kv > 0) {
      const uint32_t idO = idesc_bf16_f32(128, D, 0, 1);  // A = P (K-major), B = V (MN-major)
      bool ok = mbar_wait(q_full, 0);
      if (!ok) fail(kErrDeviceTimeout);
      tc_fence_after();

      auto issue_s = [&](int j) -> bool {
        const int4 kt = a.kvtiles[kv_first + j];
        const int st = j % S;
        if (*abort_flag) return false;
        if (!mbar_wait(&k_full[st], (j / S) & 1)) return false;
        if (j >= 2 && !mbar_wait(&s_free[j & 1], ((j >> 1) - 1) & 1)) return false;
        tc_fence_after();
        const uint32_t d_tmem = tmem + static_cast<uint32_t>((j & 1) * 128);
        const uint32_t id = idesc_bf16_f32(128, static_cast<uint32_t>(kt.y), 0, 0);
        const uint32_t kbase = sK + st * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * C::kChunkBytes + (kk & 3) * 32;
          mma_bf16_ss(d_tmem, sdesc_sw128(sQ + koff, 16, 1024), sdesc_sw128(kbase + koff, 16, 1024),
                      id, kk > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[j & 1]);
        mma_commit(&k_empty[st]);
        return true;
      };
      auto issue_pv = [&](int j) -> bool {
        const int4 kt = a.kvtiles[kv_first + j];
        const int st = j % S;
        if (*abort_flag) return false;
        if (!mbar_wait(p_full, j & 1)) return false;
        if (!mbar_wait(&v_full[st], (j / S) & 1)) return false;
        tc_fence_after();
        const uint32_t vbase = sV + st * C::kTileBytes;
        const int ksteps = kt.y >> 4;
        for (int kk = 0; kk < ksteps; ++kk) {
          const uint32_t poff = (kk >> 2) * C::kChunkBytes + (kk & 3) * 32;
          // V: 16 kv rows per step (2 groups of 8 rows at 1024 B); the two
          // 64-wide d chunks are C::kChunkBytes apart (leading byte offset).
          mma_bf16_ss(tmem + 256, sdesc_sw128(sP + poff, 16, 1024),
                      sdesc_sw128(vbase + kk * 2048, C::kChunkBytes, 1024), idO,
                      (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(pv_done);
        mma_commit(&v_empty[st]);
        return true;
      };

      if (ok) ok = issue_s(0);
      for (int j = 1; ok && j < n_kv; ++j) {
        ok = issue_s(j);
        if (ok) ok = issue_pv(j - 1);
      }
      if (ok) ok = issue_pv(n_kv - 1);
      if (!ok) fail(kErrDeviceTimeout);
      // Every MMA issued above has finished before TMEM is released.
      mma_commit(mma_idle);
      mbar_wait(mma_idle, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int grow = q_row0 + row;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float sl2 = a.scale_log2;
    float m_b = -INFINITY;  // exponent base, log2 units (scaled)
    float l = 0.f;
    bool ok = true;
    // Waits and the abort decision are made warp-uniform, because the warp
    // then executes .sync.aligned tcgen05 instructions together.
    auto warp_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
      const bool mine = !*abort_flag && mbar_wait(bar, parity);
      return __all_sync(0xffffffffu, mine);
    };

    for (int j = 0; j < n_kv; ++j) {
      const int4 kt = a.kvtiles[kv_first + j];
      const int nc = kt.y;
      if (!warp_wait(&s_full[j & 1], (j >> 1) & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[128];
      const uint32_t sbase = tmem + lane_off + static_cast<uint32_t>((j & 1) * 128);
      const bool full = nc == 128 && !kt.z;
      if (full) {
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(sbase + c * 32, sr + c * 32);
      } else {
#pragma unroll
        for (int c = 0; c < 8; ++c)
          if (c * 16 < nc) tmem_ld16(sbase + c * 16, sr + c * 16);
      }
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[j & 1]);

      // Predicate: only on partial tiles and on columns past a narrow tile.
      if (!full) {
        int lim = nc;  // allowed iff c < lim
        if (kt.z) {
          const int c0 = kt.x;
          lim = min(lim, a.Nkv - c0);
          if (a.causal) lim = min(lim, grow + a.causal_off + 1 - c0);
        }
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= lim) sr[c] = __float_as_uint(-INFINITY);
      }
      // Row max: four independent chains of 3-input max.
      float mx4[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        float m = __uint_as_float(sr[t * 32]);
#pragma unroll
        for (int c = 1; c < 31; c += 2)
          m = max3f(m, __uint_as_float(sr[t * 32 + c]), __uint_as_float(sr[t * 32 + c + 1]));
        mx4[t] = fmaxf(m, __uint_as_float(sr[t * 32 + 31]));
      }
      const float mx = max3f(fmaxf(mx4[0], mx4[1]), mx4[2], mx4[3]);
      const float mx_s = mx * sl2;
      const bool upd = mx_s > m_b + kRescaleThreshold;
      const float m_new = upd ? mx_s : m_b;
      const float alpha = upd ? ex2(m_b - m_new) : 1.0f;
      const float base = (m_new == -INFINITY) ? 0.f : m_new;

      // p = 2^(s * scale*log2e - base), packed two at a time; row sum in
      // four independent pairs of accumulators.
      float2 acc[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
      uint32_t pk[64];
#pragma unroll
      for (int c = 0; c < 128; c += 2) {
        const float2 t = ffma2(make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])),
                               make_float2(sl2, sl2), make_float2(-base, -base));
        const float2 p = make_float2(ex2(t.x), ex2(t.y));
        acc[(c >> 1) & 3] = fadd2(acc[(c >> 1) & 3], p);
        pk[c >> 1] = pack_bf16x2(p.x, p.y);
      }
      const float2 s01 = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
      const float sum = s01.x + s01.y;

      // P buffer and O are free once PV_{j-1} has completed.
      if (j > 0) {
        if (!warp_wait(pv_done, (j - 1) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      uint8_t* prow = smem + C::kOffP + row * 128;
#pragma unroll
      for (int ch = 0; ch < 2; ++ch)
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (ch * 64 + u * 8 < nc)
            *reinterpret_cast<uint4*>(prow + ch * C::kChunkBytes + ((u ^ (row & 7)) << 4)) =
                make_uint4(pk[ch * 32 + u * 4 + 0], pk[ch * 32 + u * 4 + 1],
                           pk[ch * 32 + u * 4 + 2], pk[ch * 32 + u * 4 + 3]);
      fence_proxy_async_smem();

      if (j > 0 && __any_sync(0xffffffffu, upd)) {
        const uint32_t obase = tmem + lane_off + 256;
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t orr[32];
          tmem_ld32(obase + c, orr);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) orr[i] = __float_as_uint(__uint_as_float(orr[i]) * alpha);
          tmem_st32(obase + c, orr);
        }
        tmem_wait_st();
      }
      l = l * alpha + sum;
      m_b = m_new;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }

    if (!ok) {
      fail(kErrDeviceTimeout);
    } else {
      if (n_kv > 0) {
        if (!warp_wait(pv_done, (n_kv - 1) & 1)) {
          fail(kErrDeviceTimeout);
          ok = false;
        }
        tc_fence_after();
      }
    }
    if (ok) {
      const float inv_l = l > 0.f ? 1.0f / l : 0.f;
      const float lse_val = l > 0.f ? (m_b + __log2f(l)) * kLn2 : -INFINITY;
      // Stage the bf16 O row in the (now idle) P buffer, 16-byte units
      // XOR-swizzled by row to keep the shared-memory banks apart.
      constexpr int UPR = D / 8;  // 16-byte units per row
      uint8_t* stg = smem + C::kOffP;
      const uint32_t obase = tmem + lane_off + 256;
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t orr[32];
        if (n_kv > 0) {
          tmem_ld32(obase + c, orr);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) orr[i] = 0u;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int unit = c / 8 + u;
          const int sw = (unit & ~7) | ((unit & 7) ^ (row & 7));
          *reinterpret_cast<uint4*>(stg + row * (D * 2) + sw * 16) = make_uint4(
              pack_bf16x2(__uint_as_float(orr[u * 8 + 0]) * inv_l,
                          __uint_as_float(orr[u * 8 + 1]) * inv_l),
              pack_bf16x2(__uint_as_float(orr[u * 8 + 2]) * inv_l,
                          __uint_as_float(orr[u * 8 + 3]) * inv_l),
              pack_bf16x2(__uint_as_float(orr[u * 8 + 4]) * inv_l,
                          __uint_as_float(orr[u * 8 + 5]) * inv_l),
              pack_bf16x2(__uint_as_float(orr[u * 8 + 6]) * inv_l,
                          __uint_as_float(orr[u * 8 + 7]) * inv_l));
        }
      }
      __syncwarp();
      constexpr int RPI = 32 / UPR;  // rows per warp-wide store
      uint8_t* obytes = reinterpret_cast<uint8_t*>(a.o);
#pragma unroll 4
      for (int it = 0; it < 32 / RPI; ++it) {
        const int r = quarter * 32 + it * RPI + lane / UPR;
        const int unit = lane % UPR;
        if (r < q_rows) {
          const int sw = (unit & ~7) | ((unit & 7) ^ (r & 7));
          const uint4 val = *reinterpret_cast<const uint4*>(stg + r * (D * 2) + sw * 16);
          const size_t off = ((static_cast<size_t>(b) * a.Nq + q_row0 + r) * a.Hq + hq) * D + unit * 8;
          *reinterpret_cast<uint4*>(obytes + off * 2) = val;
        }
      }
      if (a.lse != nullptr && row < q_rows)
        a.lse[(static_cast<size_t>(b) * a.Hq + hq) * a.Nq + grow] = lse_val;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int D>
cudaError_t launch_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                     const PrefillArgs& a, cudaStream_t s) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(prefill_bf16_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<D>::kSmem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const long long grid = static_cast<long long>(a.n_qtiles) * a.B * a.Hq;
  if (grid == 0) return cudaSuccess;
  prefill_bf16_kernel<D><<<static_cast<unsigned>(grid), kThreads, Cfg<D>::kSmem, s>>>(tq, tk, tv, a);
  return cudaGetLastError();
}

}  // namespace

int prefill_bf16_smem_bytes(int d) { return d == 64 ? Cfg<64>::kSmem : Cfg<128>::kSmem; }

cudaError_t launch_prefill_bf16(int d, const CUtensorMap& tq, const CUtensorMap& tk,
                                const CUtensorMap& tv, const PrefillArgs& a, cudaStream_t s) {
  if (d == 64) return launch_d<64>(tq, tk, tv, a, s);
  return launch_d<128>(tq, tk, tv, a, s);
}

}  // namespace eio
