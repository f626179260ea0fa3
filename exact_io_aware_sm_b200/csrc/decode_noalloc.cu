// decode_noalloc.cu -- attn_decode_noalloc: split-KV decode whose scratch is a
// fixed, file-scope device array instead of memory the library allocates.
//
// Some callers cannot let a library call cudaMalloc: a host framework that
// owns all device memory through its own pool and forbids allocations behind
// its back, a serving process whose memory budget is fixed and reserved at
// start-up, or a caller that cannot afford the device-wide synchronisation
// that cudaMalloc / cudaFree may cause.  This entry point runs the same split
// and combine kernels as attn_decode, but keeps the fp32 partials and the
// error word in `g_noalloc_scratch` below, which the CUDA runtime creates when
// the library's module is loaded on a device and keeps until the process
// exits.  The entry point itself allocates nothing (no cudaMalloc, no
// cudaFree, no allocating library routine).
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <mutex>

#include "../../include/attn.h"
#include "kernels.h"

namespace {

constexpr size_t kScratchBytes = ATTN_NOALLOC_SCRATCH_BYTES;
constexpr size_t kErrSlotBytes = 256;  // error word and decode item counters, padded to keep the partials aligned
static_assert((1 + eio::kDecodeMaxCounters) * sizeof(int) <= kErrSlotBytes, "error slot layout");

// The scratch: [error word (256 B)] [O partials] [log2-sum-exp partials].
// Host code must not use this name as an address (it is a host-side stand-in);
// the device address comes from cudaGetSymbolAddress in scratch_on_device().
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

int fail(int code, const char* msg) {
  eio::set_error_detail(msg);
  return code;
}

// Device address of the scratch on the current device, looked up once per
// device (with that device current) and cached until attn_shutdown.
int scratch_on_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return fail(ATTN_ERR_CUDA, "attn_decode_noalloc: no usable current device");
  if (int rc = eio::require_sm100()) return rc;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return fail(ATTN_ERR_CUDA, "attn_decode_noalloc: cudaGetSymbolAddress failed");
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return ATTN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

void eio::noalloc_forget() {
  std::lock_guard<std::mutex> lk(g_mu);
  for (void*& p : g_addr) p = nullptr;
}

extern "C" int attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                   const int32_t* seqlens, void* o, float* lse, int B, int Hq,
                                   int Hkv, int Lmax, int d, float scale, void* stream) {
  if (!q || !k_cache || !v_cache || !seqlens || !o)
    return fail(ATTN_ERR_NULL, "q, k_cache, v_cache, seqlens and o must be non-NULL");
  if (B < 1 || Hq < 1 || Hkv < 1 || Lmax < 1 || Hq % Hkv != 0 || B > 65535 || Hkv > 65535)
    return fail(ATTN_ERR_SHAPE, "bad B / Hq / Hkv / Lmax");
  const int G = Hq / Hkv;
  if ((G != 1 && G != 2 && G != 4 && G != 8) || (d != 64 && d != 128))
    return fail(ATTN_ERR_UNSUPPORTED, "decode supports Hq/Hkv in {1,2,4,8} and d in {64,128}");
  if (!(scale > 0.f) || !std::isfinite(scale)) return fail(ATTN_ERR_SHAPE, "scale must be positive and finite");
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
      (lse && !aligned16(lse)) || (reinterpret_cast<uintptr_t>(seqlens) & 3u))
    return fail(ATTN_ERR_ALIGN, "device pointers must be 16-byte aligned");

  const size_t part_floats = eio::decode_partial_floats(B, Hq, Lmax, d);
  const size_t need = kErrSlotBytes + part_floats * sizeof(float);
  if (need > kScratchBytes) {
    char msg[256];
    std::snprintf(msg, sizeof msg,
                  "attn_decode_noalloc needs %zu bytes of scratch for this shape; its fixed array "
                  "holds %zu (use attn_decode)",
                  need, kScratchBytes);
    return fail(ATTN_ERR_WORKSPACE, msg);
  }

  void* base = nullptr;
  if (int rc = scratch_on_device(&base)) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The error word is zero when the module loads and stays latched until
  // attn_decode_noalloc_status reads and clears it; the partials are written
  // before they are read.
  int* err = static_cast<int*>(base);

  eio::DecodeArgs a{};
  a.q = q;
  a.kc = k_cache;
  a.vc = v_cache;
  a.seqlens = seqlens;
  a.o = o;
  a.lse = lse;
  a.nsplit = (Lmax + eio::kDecodeChunk - 1) / eio::kDecodeChunk;
  a.opart = reinterpret_cast<float*>(static_cast<unsigned char*>(base) + kErrSlotBytes);
  a.lpart = a.opart + static_cast<size_t>(B) * Hq * a.nsplit * d;
  a.err = err;
  a.counter = err + 1;  // zero at load, and zeroed again at the end of every call
  a.Sq = 1;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.Lmax = Lmax;
  a.scale_log2 = scale * 1.4426950408889634f;
  const cudaError_t e = eio::launch_decode(d, G, a, s);
  if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, cudaGetErrorString(e));
  return ATTN_OK;
}

extern "C" int attn_decode_noalloc_status(void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const cudaError_t es = cudaStreamSynchronize(s);
  if (es != cudaSuccess) return fail(ATTN_ERR_CUDA, cudaGetErrorString(es));
  void* base = nullptr;
  if (int rc = scratch_on_device(&base)) return rc;
  int h = 0;
  if (cudaMemcpy(&h, base, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return fail(ATTN_ERR_CUDA, "attn_decode_noalloc_status: reading the error word failed");
  if (h == 0) return ATTN_OK;
  const int zero = 0;
  if (cudaMemcpy(base, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
    return fail(ATTN_ERR_CUDA, "attn_decode_noalloc_status: clearing the error word failed");
  if (h == eio::kErrDeviceTimeout)
    return fail(h, "attn_decode_noalloc: a bounded wait ran out; O and LSE of that call are undefined");
  if (h == eio::kErrDeviceArg) return fail(h, "attn_decode_noalloc: a seqlens entry was outside [0, Lmax]");
  return fail(h, "attn_decode_noalloc: device error");
}
