// api.cu -- the C ABI of libattn_b200.so (declared in include/attn.h).
//
// Host work only: argument validation, the tile plan (built once per mask and
// cached on the device), TMA tensor-map encoding, the per-device workspace,
// and kernel launches on the caller's stream.  No attention arithmetic runs
// on the host.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <list>
#include <map>
#include <memory>
#include <mutex>
#include <vector>

#include "../../include/attn.h"
#include "kernels.h"
#include "plan.h"

namespace {

using namespace eio;

thread_local char g_err[512] = "";
thread_local int g_fault_next = 0;  // test hook for the next attn_fwd on this thread

int set_err(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return code;
}

int cuda_err(cudaError_t e, const char* what) {
  return set_err(ATTN_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ------------------------------------------------------------------ workspace
struct DevPlan {
  int mask_kind, Nq, Nkv, rows_mode;
  std::vector<uint8_t> map;  // copy of the host block map (BLOCK only)
  int n_q = 0, n_kv = 0;
  int4* d_q = nullptr;
  int4* d_kv = nullptr;
  int* d_order = nullptr;
  uint8_t* d_map = nullptr;  // device copy of the block map (fp32 path)
  int n_pairs = 0;
  int equal_pairs = 0;  // every used slot A visits as many KV tiles as its slot B
  int4* d_pairs = nullptr;   // tensor-core path: Q-tile pairs in visit order, their KV lists
  int4* d_pkv = nullptr;
};

// Backward tile lists under a BLOCK mask: for every 128-row Q tile the live
// 128-key tiles, and for every key tile the live Q tiles, each entry with the
// 8 x 8 bitmap of its 16 x 16 blocks; visit orders longest list first.
struct BwdPlan {
  std::vector<uint8_t> map;
  int Nq = 0, Nkv = 0;
  int* d_qoff = nullptr;
  int4* d_qlist = nullptr;
  int* d_qord = nullptr;
  int* d_koff = nullptr;
  int4* d_klist = nullptr;
  int* d_kord = nullptr;
};

void free_bwd_plan(BwdPlan& p) {
  cudaFree(p.d_qoff);
  cudaFree(p.d_qlist);
  cudaFree(p.d_qord);
  cudaFree(p.d_koff);
  cudaFree(p.d_klist);
  cudaFree(p.d_kord);
  p.d_qoff = p.d_koff = p.d_qord = p.d_kord = nullptr;
  p.d_qlist = p.d_klist = nullptr;
}

struct DevWs {
  int* d_err = nullptr;
  float* d_part = nullptr;
  size_t part_floats = 0;
  float* d_stats = nullptr;  // key-statistics partial sums
  size_t stats_floats = 0;
  std::list<DevPlan> plans;  // most recent first
  std::list<BwdPlan> bplans;  // most recent first
};

std::mutex g_mu;
std::map<int, DevWs> g_ws;
constexpr size_t kMaxPlans = 8;

void free_plan(DevPlan& p) {
  cudaFree(p.d_q);
  cudaFree(p.d_kv);
  cudaFree(p.d_order);
  cudaFree(p.d_map);
  cudaFree(p.d_pairs);
  cudaFree(p.d_pkv);
  p.d_pairs = nullptr;
  p.d_pkv = nullptr;
  p.d_q = nullptr;
  p.d_kv = nullptr;
  p.d_order = nullptr;
  p.d_map = nullptr;
}

int get_ws(DevWs** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_err(e, "cudaGetDevice");
  DevWs& ws = g_ws[dev];
  if (!ws.d_err) {
    // [0] the error word, [1..] decode work-item counters
    e = cudaMalloc(&ws.d_err, (1 + kDecodeMaxCounters) * sizeof(int));
    if (e != cudaSuccess) return set_err(ATTN_ERR_WORKSPACE, "error word: %s", cudaGetErrorString(e));
    e = cudaMemset(ws.d_err, 0, (1 + kDecodeMaxCounters) * sizeof(int));
    if (e != cudaSuccess) return cuda_err(e, "cudaMemset");
  }
  *out = &ws;
  return ATTN_OK;
}

int check_device_sm100() {
  int dev = 0, major = 0, minor = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_err(e, "cudaGetDevice");
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0)
    return set_err(ATTN_ERR_UNSUPPORTED, "device is sm_%d%d; this library is built for sm_100a",
                   major, minor);
  return ATTN_OK;
}

template <class T>
int upload(T** dst, const T* src, size_t n, cudaStream_t s) {
  cudaError_t e = cudaMalloc(dst, sizeof(T) * (n ? n : 1));
  if (e != cudaSuccess) return set_err(ATTN_ERR_WORKSPACE, "plan buffer: %s", cudaGetErrorString(e));
  if (n) {
    e = cudaMemcpyAsync(*dst, src, sizeof(T) * n, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return cuda_err(e, "plan upload");
  }
  return ATTN_OK;
}

// Find or build the device-resident plan for a mask.
int get_plan(DevWs& ws, int mask_kind, const uint8_t* block_map, int Nq, int Nkv, bool need_map,
             int rows_mode, cudaStream_t s, DevPlan** out) {
  const size_t map_bytes =
      mask_kind == ATTN_MASK_BLOCK
          ? static_cast<size_t>((Nq + kGrain - 1) / kGrain) * ((Nkv + kGrain - 1) / kGrain)
          : 0;
  for (auto it = ws.plans.begin(); it != ws.plans.end(); ++it) {
    if (it->mask_kind != mask_kind || it->Nq != Nq || it->Nkv != Nkv || it->rows_mode != rows_mode)
      continue;
    if (map_bytes && (it->map.size() != map_bytes ||
                      std::memcmp(it->map.data(), block_map, map_bytes) != 0))
      continue;
    if (need_map && map_bytes && !it->d_map) continue;
    ws.plans.splice(ws.plans.begin(), ws.plans, it);
    *out = &ws.plans.front();
    return ATTN_OK;
  }
  Plan p;
  build_plan(mask_kind, block_map, Nq, Nkv, &p);
  DevPlan dp;
  dp.mask_kind = mask_kind;
  dp.Nq = Nq;
  dp.Nkv = Nkv;
  dp.rows_mode = rows_mode;
  if (map_bytes) dp.map.assign(block_map, block_map + map_bytes);
  dp.n_q = static_cast<int>(p.q.size());
  dp.n_kv = static_cast<int>(p.kv.size());
  PairPlan pp;
  build_pairs(p, rows_mode != 0, &pp);
  dp.n_pairs = static_cast<int>(pp.pairs.size());
  dp.equal_pairs = 1;
  for (const PairTile& t : pp.pairs)
    if (t.nrowsA > 0 && t.nA != t.nB) dp.equal_pairs = 0;
  static_assert(sizeof(PairTile) == 2 * sizeof(int4) && sizeof(PairKV) == sizeof(int4), "layout");
  // The kernel visits pairs in this order (most KV tiles first).
  std::vector<PairTile> sorted(pp.pairs.size());
  for (size_t i = 0; i < sorted.size(); ++i) sorted[i] = pp.pairs[pp.order[i]];
  int rc;
  if ((rc = upload(&dp.d_q, reinterpret_cast<const int4*>(p.q.data()), p.q.size(), s)) ||
      (rc = upload(&dp.d_kv, reinterpret_cast<const int4*>(p.kv.data()), p.kv.size(), s)) ||
      (rc = upload(&dp.d_order, p.order.data(), p.order.size(), s)) ||
      (rc = upload(&dp.d_pairs, reinterpret_cast<const int4*>(sorted.data()), 2 * sorted.size(), s)) ||
      (rc = upload(&dp.d_pkv, reinterpret_cast<const int4*>(pp.kv.data()), pp.kv.size(), s)) ||
      (map_bytes && need_map && (rc = upload(&dp.d_map, block_map, map_bytes, s)))) {
    free_plan(dp);
    return rc;
  }
  // The host vectors die with this scope: finish the copies first.
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    free_plan(dp);
    return cuda_err(e, "plan upload");
  }
  ws.plans.push_front(std::move(dp));
  while (ws.plans.size() > kMaxPlans) {
    cudaDeviceSynchronize();
    free_plan(ws.plans.back());
    ws.plans.pop_back();
  }
  *out = &ws.plans.front();
  return ATTN_OK;
}

int get_bwd_plan(DevWs& ws, const uint8_t* block_map, int Nq, int Nkv, cudaStream_t s, BwdPlan** out) {
  const int nbq = (Nq + kGrain - 1) / kGrain, nbk = (Nkv + kGrain - 1) / kGrain;
  const size_t map_bytes = static_cast<size_t>(nbq) * nbk;
  for (auto it = ws.bplans.begin(); it != ws.bplans.end(); ++it) {
    if (it->Nq != Nq || it->Nkv != Nkv || it->map.size() != map_bytes ||
        std::memcmp(it->map.data(), block_map, map_bytes) != 0)
      continue;
    ws.bplans.splice(ws.bplans.begin(), ws.bplans, it);
    *out = &ws.bplans.front();
    return ATTN_OK;
  }
  const int n_qt = (Nq + 127) / 128, n_kt = (Nkv + 127) / 128;
  std::vector<std::vector<int4>> ql(n_qt), kl(n_kt);
  for (int qt = 0; qt < n_qt; ++qt)
    for (int kt = 0; kt < n_kt; ++kt) {
      unsigned long long m = 0;
      for (int i = 0; i < 8 && qt * 8 + i < nbq; ++i)
        for (int j = 0; j < 8 && kt * 8 + j < nbk; ++j)
          if (block_map[static_cast<size_t>(qt * 8 + i) * nbk + kt * 8 + j]) m |= 1ull << (i * 8 + j);
      if (!m) continue;
      const int lo = static_cast<int>(m & 0xffffffffull), hi = static_cast<int>(m >> 32);
      ql[qt].push_back(make_int4(kt, lo, hi, 0));
      kl[kt].push_back(make_int4(qt, lo, hi, 0));
    }
  auto flatten = [](const std::vector<std::vector<int4>>& l, std::vector<int>* off, std::vector<int4>* flat,
                    std::vector<int>* ord) {
    off->assign(1, 0);
    for (const auto& v : l) {
      flat->insert(flat->end(), v.begin(), v.end());
      off->push_back(static_cast<int>(flat->size()));
    }
    ord->resize(l.size());
    for (size_t i = 0; i < l.size(); ++i) (*ord)[i] = static_cast<int>(i);
    std::stable_sort(ord->begin(), ord->end(), [&](int a, int b) { return l[a].size() > l[b].size(); });
    if (flat->empty()) flat->push_back(make_int4(0, 0, 0, 0));  // never read: every list is empty
  };
  std::vector<int> qoff, qord, koff, kord;
  std::vector<int4> qflat, kflat;
  flatten(ql, &qoff, &qflat, &qord);
  flatten(kl, &koff, &kflat, &kord);
  BwdPlan bp;
  bp.map.assign(block_map, block_map + map_bytes);
  bp.Nq = Nq;
  bp.Nkv = Nkv;
  int rc;
  if ((rc = upload(&bp.d_qoff, qoff.data(), qoff.size(), s)) || (rc = upload(&bp.d_qlist, qflat.data(), qflat.size(), s)) ||
      (rc = upload(&bp.d_qord, qord.data(), qord.size(), s)) || (rc = upload(&bp.d_koff, koff.data(), koff.size(), s)) ||
      (rc = upload(&bp.d_klist, kflat.data(), kflat.size(), s)) || (rc = upload(&bp.d_kord, kord.data(), kord.size(), s))) {
    free_bwd_plan(bp);
    return rc;
  }
  cudaError_t e = cudaStreamSynchronize(s);  // the host vectors die with this scope
  if (e != cudaSuccess) {
    free_bwd_plan(bp);
    return cuda_err(e, "backward plan upload");
  }
  ws.bplans.push_front(std::move(bp));
  while (ws.bplans.size() > kMaxPlans) {
    cudaDeviceSynchronize();
    free_bwd_plan(ws.bplans.back());
    ws.bplans.pop_back();
  }
  *out = &ws.bplans.front();
  return ATTN_OK;
}

// ------------------------------------------------------------------ TMA maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

int get_encoder(EncodeTiledFn* fn) {
  static EncodeTiledFn cached = nullptr;
  if (!cached) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !p)
      return set_err(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    cached = reinterpret_cast<EncodeTiledFn>(p);
  }
  *fn = cached;
  return ATTN_OK;
}

// [B, N, H, d] bf16 viewed as 4-D {d, H, N, B}; box {64, 1, box_rows, 1}, 128-byte swizzle;
// rows past N read as zeros.
CUresult encode_map(CUtensorMap* m, const void* base, int B, int N, int H, int d, int box_rows) {
  EncodeTiledFn enc;
  if (get_encoder(&enc)) return CUDA_ERROR_NOT_SUPPORTED;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(d) * 2,
                                 static_cast<cuuint64_t>(H) * d * 2,
                                 static_cast<cuuint64_t>(N) * H * d * 2};
  const cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

int make_map(CUtensorMap* m, const void* base, int B, int N, int H, int d) {
  EncodeTiledFn enc;
  if (int rc = get_encoder(&enc)) return rc;
  CUresult r = encode_map(m, base, B, N, H, d, 128);
  if (r != CUDA_SUCCESS) return set_err(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return ATTN_OK;
}

int check_mask_args(int mask_kind, const uint8_t* block_map) {
  if (mask_kind < ATTN_MASK_NONE || mask_kind > ATTN_MASK_BLOCK)
    return set_err(ATTN_ERR_MASK, "mask_kind %d is not NONE, CAUSAL or BLOCK", mask_kind);
  if (mask_kind == ATTN_MASK_BLOCK && !block_map)
    return set_err(ATTN_ERR_MASK, "ATTN_MASK_BLOCK needs a block map");
  return ATTN_OK;
}

}  // namespace

void eio::set_error_detail(const char* msg) { std::snprintf(g_err, sizeof g_err, "%s", msg); }

int eio::require_sm100() { return check_device_sm100(); }

bool eio::encode_bf16_map(CUtensorMap* m, const void* base, int B, int N, int H, int d, int box_rows) {
  const CUresult r = encode_map(m, base, B, N, H, d, box_rows);
  if (r != CUDA_SUCCESS) {
    set_err(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return false;
  }
  return true;
}

// The bf16 tensor-core forward; kbar != nullptr selects the bound-based
// softmax.  Called with g_mu held and the arguments validated.
static int fwd_bf16(DevWs& wsr, const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
             int Nq, int Nkv, int d, float scale, int mask_kind, const uint8_t* block_map, const float* kbar,
             const float* radius, int* n_fallback, cudaStream_t s) {
  DevWs* ws = &wsr;
  const int G = Hq / Hkv;
  const int rows_mode = G == 1 ? 1 : 0;
  DevPlan* pl = nullptr;
  if (int rc = get_plan(*ws, mask_kind, block_map, Nq, Nkv, false, rows_mode, s, &pl)) return rc;
  CUtensorMap tq, tk, tv;
  if (int rc = make_map(&tq, q, B, Nq, Hq, d)) return rc;
  if (int rc = make_map(&tk, k, B, Nkv, Hkv, d)) return rc;
  if (int rc = make_map(&tv, v, B, Nkv, Hkv, d)) return rc;
  CUtensorMap to, tk16, tv16;
  if (!encode_bf16_map(&to, o, B, Nq, Hq, d, 16) || !encode_bf16_map(&tk16, k, B, Nkv, Hkv, d, 16) ||
      !encode_bf16_map(&tv16, v, B, Nkv, Hkv, d, 16))
    return ATTN_ERR_CUDA;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  PrefillArgs a{};
  a.pairs = pl->d_pairs;
  a.kvtiles = pl->d_pkv;
  a.o = o;
  a.lse = lse;
  a.err = ws->d_err;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.Nq = Nq;
  a.Nkv = Nkv;
  a.G = G;
  a.HP = rows_mode ? 1 : (G + 1) / 2;
  a.rows_mode = rows_mode;
  a.n_items = static_cast<long long>(pl->n_pairs) * B * Hkv * a.HP;
  a.num_ctas = sms > 0 ? sms : 148;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.causal = mask_kind == ATTN_MASK_CAUSAL;
  a.causal_off = Nkv - Nq;
  a.stagger = pl->equal_pairs;
  a.fault = g_fault_next;
  g_fault_next = 0;
  a.bound = kbar != nullptr;
  a.q = q;
  a.kbar = kbar;
  a.radius = radius;
  a.n_fallback = n_fallback;
  cudaError_t e = launch_prefill_bf16(d, tq, tk, tv, to, tk16, tv16, a, s);
  return e == cudaSuccess ? ATTN_OK : cuda_err(e, "prefill launch");
}

extern "C" {

int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
             int Hkv, int Nq, int Nkv, int d, float scale, int mask_kind, const uint8_t* block_map,
             int dtype, void* stream) {
  if (!q || !k || !v || !o) return set_err(ATTN_ERR_NULL, "q, k, v and o must be non-NULL");
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nkv < 1)
    return set_err(ATTN_ERR_SHAPE, "B, Hq, Hkv, Nq, Nkv must be >= 1");
  if (Hq % Hkv != 0) return set_err(ATTN_ERR_SHAPE, "Hq (%d) is not a multiple of Hkv (%d)", Hq, Hkv);
  if (!(scale > 0.f) || !std::isfinite(scale))
    return set_err(ATTN_ERR_SHAPE, "scale must be positive and finite");
  if (int rc = check_mask_args(mask_kind, block_map)) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (lse && !aligned16(lse)))
    return set_err(ATTN_ERR_ALIGN, "device pointers must be 16-byte aligned");
  if (dtype == ATTN_BF16) {
    if (d != 64 && d != 128) return set_err(ATTN_ERR_UNSUPPORTED, "bf16 path needs d in {64, 128}");
  } else if (dtype == ATTN_F32) {
    if (d != 32 && d != 64 && d != 128)
      return set_err(ATTN_ERR_UNSUPPORTED, "fp32 path needs d in {32, 64, 128}");
    if (Hq > 65535 || B > 65535) return set_err(ATTN_ERR_SHAPE, "fp32 path: Hq and B must be <= 65535");
  } else {
    return set_err(ATTN_ERR_UNSUPPORTED, "dtype %d is not ATTN_BF16 or ATTN_F32", dtype);
  }
  if (int rc = check_device_sm100()) return rc;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lk(g_mu);
  DevWs* ws;
  if (int rc = get_ws(&ws)) return rc;

  if (dtype == ATTN_F32) {
    DevPlan* pl = nullptr;
    if (mask_kind == ATTN_MASK_BLOCK) {
      if (int rc = get_plan(*ws, mask_kind, block_map, Nq, Nkv, true, 0, s, &pl)) return rc;
    }
    PrefillF32Args a{};
    a.q = static_cast<const float*>(q);
    a.k = static_cast<const float*>(k);
    a.v = static_cast<const float*>(v);
    a.o = static_cast<float*>(o);
    a.lse = lse;
    a.block_map = pl ? pl->d_map : nullptr;
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.Nq = Nq;
    a.Nkv = Nkv;
    a.mask_kind = mask_kind;
    a.scale = scale;
    cudaError_t e = launch_prefill_f32(d, a, s);
    return e == cudaSuccess ? ATTN_OK : cuda_err(e, "fp32 prefill launch");
  }

  return fwd_bf16(*ws, q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, d, scale, mask_kind, block_map, nullptr, nullptr, nullptr,
                  s);
}

int attn_key_stats(const void* k, float* kbar, float* radius, int B, int Nkv, int Hkv, int d, void* stream) {
  if (!k || !kbar || !radius) return set_err(ATTN_ERR_NULL, "k, kbar and radius must be non-NULL");
  if (B < 1 || Nkv < 1 || Hkv < 1) return set_err(ATTN_ERR_SHAPE, "B, Nkv, Hkv must be >= 1");
  if (d != 64 && d != 128) return set_err(ATTN_ERR_UNSUPPORTED, "attn_key_stats needs d in {64, 128}");
  if (B > 65535 || Hkv > 65535 || static_cast<long long>(B) * Nkv * Hkv >= (1ll << 31))
    return set_err(ATTN_ERR_SHAPE, "too many keys");
  if (!aligned16(k) || !aligned16(kbar) || (reinterpret_cast<uintptr_t>(radius) & 3u))
    return set_err(ATTN_ERR_ALIGN, "k and kbar must be 16-byte aligned, radius 4-byte aligned");
  if (int rc = check_device_sm100()) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lk(g_mu);
  DevWs* ws;
  if (int rc = get_ws(&ws)) return rc;
  const int nsplit = key_stats_splits(Nkv);
  const size_t need = static_cast<size_t>(B) * Hkv * nsplit * d;
  if (ws->stats_floats < need) {
    cudaDeviceSynchronize();
    cudaFree(ws->d_stats);
    ws->d_stats = nullptr;
    ws->stats_floats = 0;
    cudaError_t e = cudaMalloc(&ws->d_stats, need * sizeof(float));
    if (e != cudaSuccess) return set_err(ATTN_ERR_WORKSPACE, "key statistics scratch: %s", cudaGetErrorString(e));
    ws->stats_floats = need;
  }
  KeyStatsArgs a{};
  a.k = k;
  a.part = ws->d_stats;
  a.kbar = kbar;
  a.radius = radius;
  a.B = B;
  a.Nkv = Nkv;
  a.Hkv = Hkv;
  a.nsplit = nsplit;
  cudaError_t e = launch_key_stats(d, a, s);
  return e == cudaSuccess ? ATTN_OK : cuda_err(e, "key statistics launch");
}

int attn_fwd_bound(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Nq,
                   int Nkv, int d, float scale, int mask_kind, const uint8_t* block_map, const float* kbar,
                   const float* radius, int* n_fallback, void* stream) {
  if (!q || !k || !v || !o || !kbar || !radius)
    return set_err(ATTN_ERR_NULL, "q, k, v, o, kbar and radius must be non-NULL");
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nkv < 1)
    return set_err(ATTN_ERR_SHAPE, "B, Hq, Hkv, Nq, Nkv must be >= 1");
  if (Hq % Hkv != 0) return set_err(ATTN_ERR_SHAPE, "Hq (%d) is not a multiple of Hkv (%d)", Hq, Hkv);
  if (!(scale > 0.f) || !std::isfinite(scale))
    return set_err(ATTN_ERR_SHAPE, "scale must be positive and finite");
  if (int rc = check_mask_args(mask_kind, block_map)) return rc;
  if (d != 64 && d != 128) return set_err(ATTN_ERR_UNSUPPORTED, "attn_fwd_bound needs d in {64, 128}");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (lse && !aligned16(lse)) ||
      !aligned16(kbar) || (reinterpret_cast<uintptr_t>(radius) & 3u) ||
      (reinterpret_cast<uintptr_t>(n_fallback) & 3u))
    return set_err(ATTN_ERR_ALIGN, "device pointers must be 16-byte aligned (radius, n_fallback: 4-byte)");
  if (int rc = check_device_sm100()) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lk(g_mu);
  DevWs* ws;
  if (int rc = get_ws(&ws)) return rc;
  return fwd_bf16(*ws, q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, d, scale, mask_kind, block_map, kbar, radius,
                  n_fallback, s);
}

int attn_decode_multi(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens,
                      void* o, float* lse, int B, int Sq, int Hq, int Hkv, int Lmax, int d, float scale,
                      void* stream) {
  if (!q || !k_cache || !v_cache || !seqlens || !o)
    return set_err(ATTN_ERR_NULL, "q, k_cache, v_cache, seqlens and o must be non-NULL");
  if (B < 1 || Sq < 1 || Hq < 1 || Hkv < 1 || Lmax < 1)
    return set_err(ATTN_ERR_SHAPE, "B, Sq, Hq, Hkv, Lmax must be >= 1");
  if (Hq % Hkv != 0) return set_err(ATTN_ERR_SHAPE, "Hq (%d) is not a multiple of Hkv (%d)", Hq, Hkv);
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8)
    return set_err(ATTN_ERR_UNSUPPORTED, "decode supports Hq/Hkv in {1, 2, 4, 8}, got %d", G);
  if (G * Sq > 16)
    return set_err(ATTN_ERR_UNSUPPORTED, "decode needs (Hq/Hkv) * Sq <= 16, got %d * %d", G, Sq);
  if (static_cast<long long>(B) * Sq * Hq > (1ll << 30)) return set_err(ATTN_ERR_SHAPE, "too many query rows");
  if (d != 64 && d != 128) return set_err(ATTN_ERR_UNSUPPORTED, "decode needs d in {64, 128}");
  if (!(scale > 0.f) || !std::isfinite(scale))
    return set_err(ATTN_ERR_SHAPE, "scale must be positive and finite");
  if (B > 65535 || Hkv > 65535) return set_err(ATTN_ERR_SHAPE, "B and Hkv must be <= 65535");
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
      (lse && !aligned16(lse)) || (reinterpret_cast<uintptr_t>(seqlens) & 3u))
    return set_err(ATTN_ERR_ALIGN, "device pointers must be 16-byte aligned");
  if (int rc = check_device_sm100()) return rc;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lk(g_mu);
  DevWs* ws;
  if (int rc = get_ws(&ws)) return rc;
  const size_t need = decode_partial_floats(B * Sq, Hq, Lmax, d);
  if (ws->part_floats < need) {
    cudaDeviceSynchronize();
    cudaFree(ws->d_part);
    ws->d_part = nullptr;
    ws->part_floats = 0;
    cudaError_t e = cudaMalloc(&ws->d_part, need * sizeof(float));
    if (e != cudaSuccess) return set_err(ATTN_ERR_WORKSPACE, "decode partials: %s", cudaGetErrorString(e));
    ws->part_floats = need;
  }
  DecodeArgs a{};
  a.q = q;
  a.kc = k_cache;
  a.vc = v_cache;
  a.seqlens = seqlens;
  a.o = o;
  a.lse = lse;
  a.nsplit = (Lmax + kDecodeChunk - 1) / kDecodeChunk;
  a.opart = ws->d_part;
  a.lpart = ws->d_part + static_cast<size_t>(B) * Sq * Hq * a.nsplit * d;
  a.err = ws->d_err;
  a.counter = ws->d_err + 1;
  a.Sq = Sq;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.Lmax = Lmax;
  a.scale_log2 = scale * 1.4426950408889634f;
  cudaError_t e = launch_decode(d, G, a, s);
  return e == cudaSuccess ? ATTN_OK : cuda_err(e, "decode launch");
}

int attn_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens,
                void* o, float* lse, int B, int Hq, int Hkv, int Lmax, int d, float scale,
                void* stream) {
  return attn_decode_multi(q, k_cache, v_cache, seqlens, o, lse, B, 1, Hq, Hkv, Lmax, d, scale, stream);
}

int attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
             void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq, int Nkv, int d, float scale,
             int mask_kind, const uint8_t* block_map, void* stream) {
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv)
    return set_err(ATTN_ERR_NULL, "every tensor of attn_bwd must be non-NULL");
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nkv < 1) return set_err(ATTN_ERR_SHAPE, "sizes must be >= 1");
  if (Hq % Hkv != 0) return set_err(ATTN_ERR_SHAPE, "Hq (%d) is not a multiple of Hkv (%d)", Hq, Hkv);
  if (d != 64 && d != 128) return set_err(ATTN_ERR_UNSUPPORTED, "attn_bwd needs d in {64, 128}");
  if (int rc = check_mask_args(mask_kind, block_map)) return rc;
  if (!(scale > 0.f) || !std::isfinite(scale)) return set_err(ATTN_ERR_SHAPE, "scale must be positive and finite");
  if (B > 65535 || Hq > 65535 || static_cast<long long>(B) * Hq * Nq >= (1ll << 31) ||
      static_cast<long long>(B) * Hkv * Nkv >= (1ll << 31))
    return set_err(ATTN_ERR_SHAPE, "too many rows");
  for (const void* p : {q, k, v, o, dout, static_cast<const void*>(lse), static_cast<const void*>(dq),
                        static_cast<const void*>(dk), static_cast<const void*>(dv)})
    if (!aligned16(p)) return set_err(ATTN_ERR_ALIGN, "device pointers must be 16-byte aligned");
  if (int rc = check_device_sm100()) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lk(g_mu);
  DevWs* ws;
  if (int rc = get_ws(&ws)) return rc;
  // D and LSE * log2(e), rows padded to whole 128-row tiles
  const size_t need = 2 * static_cast<size_t>(B) * Hq * ((static_cast<size_t>(Nq) + 127) / 128 * 128);
  if (ws->part_floats < need) {
    cudaDeviceSynchronize();
    cudaFree(ws->d_part);
    ws->d_part = nullptr;
    ws->part_floats = 0;
    cudaError_t e = cudaMalloc(&ws->d_part, need * sizeof(float));
    if (e != cudaSuccess) return set_err(ATTN_ERR_WORKSPACE, "backward scratch: %s", cudaGetErrorString(e));
    ws->part_floats = need;
  }
  BwdArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.dout = dout;
  a.lse = lse;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.neg_d = ws->d_part;
  a.neg_lse2 = ws->d_part + need / 2;
  a.err = ws->d_err;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.Nq = Nq;
  a.Nkv = Nkv;
  a.causal = mask_kind == ATTN_MASK_CAUSAL;
  a.scale = scale;
  if (mask_kind == ATTN_MASK_BLOCK) {
    BwdPlan* bp = nullptr;
    if (int rc = get_bwd_plan(*ws, block_map, Nq, Nkv, s, &bp)) return rc;
    a.qoff = bp->d_qoff;
    a.qlist = bp->d_qlist;
    a.qord = bp->d_qord;
    a.koff = bp->d_koff;
    a.klist = bp->d_klist;
    a.kord = bp->d_kord;
  }
  cudaError_t e = launch_bwd(d, a, s);
  return e == cudaSuccess ? ATTN_OK : cuda_err(e, "backward launch");
}

int attn_frame_block_map(int n_frames, int frame_len, uint8_t* out) {
  if (!out) return set_err(ATTN_ERR_NULL, "out must be non-NULL");
  if (n_frames < 1 || frame_len < 1) return set_err(ATTN_ERR_SHAPE, "n_frames and frame_len must be >= 1");
  if (frame_len % kGrain != 0)
    return set_err(ATTN_ERR_SHAPE, "frame_len (%d) must be a multiple of 16", frame_len);
  if (static_cast<long long>(n_frames) * frame_len >= (1ll << 31))
    return set_err(ATTN_ERR_SHAPE, "sequence too long");
  frame_block_map(n_frames, frame_len, out);
  return ATTN_OK;
}

int attn_classify(int mask_kind, const uint8_t* block_map, int Nq, int Nkv, int tq, int tk,
                  uint8_t* out) {
  if (!out) return set_err(ATTN_ERR_NULL, "out must be non-NULL");
  if (Nq < 1 || Nkv < 1 || tq < 1 || tk < 1) return set_err(ATTN_ERR_SHAPE, "sizes must be >= 1");
  if (int rc = check_mask_args(mask_kind, block_map)) return rc;
  classify_tiles(mask_kind, block_map, Nq, Nkv, tq, tk, out);
  return ATTN_OK;
}

int attn_plan(int mask_kind, const uint8_t* block_map, int Nq, int Nkv, int32_t* qtiles, int qcap,
              int32_t* kvtiles, int kvcap, int* n_q, int* n_kv) {
  if (!n_q || !n_kv) return set_err(ATTN_ERR_NULL, "n_q and n_kv must be non-NULL");
  if (Nq < 1 || Nkv < 1) return set_err(ATTN_ERR_SHAPE, "Nq and Nkv must be >= 1");
  if (int rc = check_mask_args(mask_kind, block_map)) return rc;
  Plan p;
  build_plan(mask_kind, block_map, Nq, Nkv, &p);
  *n_q = static_cast<int>(p.q.size());
  *n_kv = static_cast<int>(p.kv.size());
  if ((qtiles && qcap < *n_q) || (kvtiles && kvcap < *n_kv))
    return set_err(ATTN_ERR_SHAPE, "capacity too small: need %d Q tiles and %d KV tiles", *n_q, *n_kv);
  if (qtiles)
    for (size_t i = 0; i < p.q.size(); ++i) {
      qtiles[4 * i + 0] = p.q[i].row0;
      qtiles[4 * i + 1] = p.q[i].nrows;
      qtiles[4 * i + 2] = p.q[i].first_kv;
      qtiles[4 * i + 3] = p.q[i].n_kv;
    }
  if (kvtiles)
    for (size_t i = 0; i < p.kv.size(); ++i) {
      kvtiles[3 * i + 0] = p.kv[i].col0;
      kvtiles[3 * i + 1] = p.kv[i].ncols;
      kvtiles[3 * i + 2] = p.kv[i].partial;
    }
  return ATTN_OK;
}

int attn_sync_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_err(e, "cudaStreamSynchronize");
  std::lock_guard<std::mutex> lk(g_mu);
  DevWs* ws;
  if (int rc = get_ws(&ws)) return rc;
  int h = 0;
  e = cudaMemcpy(&h, ws->d_err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_err(e, "reading the error word");
  if (h == 0) return ATTN_OK;
  cudaMemset(ws->d_err, 0, sizeof(int));
  if (h == ATTN_ERR_DEVICE_TIMEOUT) return set_err(h, "a kernel's bounded wait ran out");
  if (h == ATTN_ERR_DEVICE_ARG) return set_err(h, "a seqlens entry was outside [0, Lmax]");
  return set_err(h, "device error %d", h);
}

int attn_last_error_detail(char* buf, int len) {
  if (!buf || len < 1) return ATTN_ERR_NULL;
  std::snprintf(buf, static_cast<size_t>(len), "%s", g_err);
  return ATTN_OK;
}

int attn_shutdown(void) {
  noalloc_forget();
  std::lock_guard<std::mutex> lk(g_mu);
  int cur = 0;
  cudaGetDevice(&cur);
  for (auto& kv : g_ws) {
    if (cudaSetDevice(kv.first) != cudaSuccess) continue;
    cudaDeviceSynchronize();
    for (auto& p : kv.second.plans) free_plan(p);
    for (auto& p : kv.second.bplans) free_bwd_plan(p);
    cudaFree(kv.second.d_part);
    cudaFree(kv.second.d_stats);
    cudaFree(kv.second.d_err);
  }
  g_ws.clear();
  cudaSetDevice(cur);
  return ATTN_OK;
}

int attn_debug_fault(int kind) {
  if (kind < 0 || kind > 1) return set_err(ATTN_ERR_SHAPE, "unknown fault kind %d", kind);
  g_fault_next = kind;
  return ATTN_OK;
}

const char* attn_version(void) { return "exact_io_aware_sm_b200 0.1"; }

}  // extern "C"
