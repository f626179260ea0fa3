// kernels.h -- launchers shared between the C ABI (api.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

namespace eio {

// Per-device record of one-time launch set-up (kernel attributes), safe to
// test and set from several host threads.  The set-up it guards is
// idempotent, so two threads that both find a device's bit clear both run it,
// which is harmless; a bit is set only after the set-up succeeded.
struct DeviceOnce {
  std::atomic<unsigned long long> done{0};
  bool test(int dev) const {
    return dev >= 0 && dev < 64 && ((done.load(std::memory_order_acquire) >> dev) & 1ull) != 0;
  }
  void set(int dev) {
    if (dev >= 0 && dev < 64) done.fetch_or(1ull << dev, std::memory_order_release);
  }
};

// Device error codes latched by kernels (same values as attn_status).
constexpr int kErrDeviceTimeout = 7;
constexpr int kErrDeviceArg = 9;

struct PrefillArgs {
  const int4* pairs;    // per pair, most KV tiles first: (rowA, nrowsA, rowB, nrowsB), (kv_first, nA, nB, 0)
  const int4* kvtiles;  // (col0, ncols, flags, 0); flags bit 0 partial for A, bit 1 for B
  void* o;              // [B, Nq, Hq, d] bf16
  float* lse;           // [B, Hq, Nq] or nullptr
  int* err;
  int B, Hq, Hkv, Nq, Nkv;
  int G;                // query heads per KV head
  int HP;               // head pairs per KV head (ceil(G/2)), 1 in rows mode
  int rows_mode;        // 1: slots are two Q tiles of one head (G == 1)
  long long n_items;    // pairs * B * Hkv * HP
  int num_ctas;         // persistent grid size (SM count)
  float scale_log2;     // scale * log2(e)
  int causal, causal_off;
  int stagger;          // 1: both slots of every pair visit the same number of KV tiles
  int fault;            // test hook: 1 = CTA 0 skips its first K load (a wait then runs out)
  // Bound-based softmax (bound = 1): each row's exponent base is
  // scale*log2(e)*(q.kbar + ||q|| radius) instead of the running max.
  int bound;
  const void* q;        // [B, Nq, Hq, d] bf16 (read for the row norms)
  const float* kbar;    // [B, Hkv, d]
  const float* radius;  // [B, Hkv]
  int* n_fallback;      // rows that kept the running max are added here (may be null)
};

// Key statistics for the bound-based softmax.
struct KeyStatsArgs {
  const void* k;  // [B, Nkv, Hkv, d] bf16
  float* part;    // scratch [B, Hkv, nsplit, d]
  float* kbar;    // [B, Hkv, d] (written)
  float* radius;  // [B, Hkv] (written)
  int B, Nkv, Hkv, nsplit;
};
int key_stats_splits(int Nkv);
cudaError_t launch_key_stats(int d, const KeyStatsArgs& a, cudaStream_t s);

// bf16 tensor-core prefill (tcgen05 / TMA).  d in {64, 128}.
// to: O as {d, Hq, Nq, B} with a {64, 1, 16, 1} box (used by the d = 64 epilogue);
// tk16, tv16: K and V with 16-row boxes (two-segment KV tiles).
cudaError_t launch_prefill_bf16(int d, const CUtensorMap& tq, const CUtensorMap& tk,
                                const CUtensorMap& tv, const CUtensorMap& to, const CUtensorMap& tk16,
                                const CUtensorMap& tv16, const PrefillArgs& a, cudaStream_t s);
int prefill_bf16_smem_bytes(int d);

struct PrefillF32Args {
  const float* q;
  const float* k;
  const float* v;
  float* o;
  float* lse;
  const uint8_t* block_map;  // device, or nullptr
  int B, Hq, Hkv, Nq, Nkv, mask_kind;
  float scale;
};
cudaError_t launch_prefill_f32(int d, const PrefillF32Args& a, cudaStream_t s);

// Split-KV decode.
constexpr int kDecodeChunk = 512;
struct DecodeArgs {
  const void* q;    // [B, Sq, Hq, d] bf16
  const void* kc;   // [B, Lmax, Hkv, d] bf16
  const void* vc;
  const int32_t* seqlens;
  void* o;          // [B, Sq, Hq, d] bf16
  float* lse;       // [B, Hq, Sq] or nullptr
  float* opart;     // [B, Sq, Hq, nsplit, d]
  float* lpart;     // [B, Sq, Hq, nsplit]  (log2 domain)
  int* err;
  int* counter;     // work-item counters, one per group of 2048 sequences; zero before the call, zeroed after
  int B, Hq, Hkv, Lmax, nsplit;
  int Sq;           // query tokens per sequence (the newest Sq positions); G * Sq <= 16
  float scale_log2;
};
constexpr int kDecodeMaxCounters = 63;  // sequence groups one call may need (B <= 65535)
cudaError_t launch_decode(int d, int G, const DecodeArgs& a, cudaStream_t s);
size_t decode_partial_floats(int B, int Hq, int Lmax, int d);

// Backward (dQ, dK, dV) for an upstream dO; bf16 tensors, d in {64, 128}.
struct BwdArgs {
  const void* q;      // [B, Nq, Hq, d]
  const void* k;      // [B, Nkv, Hkv, d]
  const void* v;
  const void* o;      // [B, Nq, Hq, d] forward output
  const void* dout;   // [B, Nq, Hq, d]
  const float* lse;   // [B, Hq, Nq] forward LSE (natural log)
  void* dq;           // [B, Nq, Hq, d] (written)
  void* dk;           // [B, Nkv, Hkv, d] (written)
  void* dv;
  float* neg_d;       // scratch [B, Hq, Nq rounded up to 128]: -rowsum(dO * O)
  float* neg_lse2;    // scratch, same layout: -LSE * log2(e)
  int* err;
  int B, Hq, Hkv, Nq, Nkv, causal;
  float scale;
  // BLOCK masks (all null otherwise): per 128-row Q tile qt, entries
  // qlist[qoff[qt] .. qoff[qt+1]) = (key tile, bitmap low, bitmap high, 0),
  // bit i*8+j set when the 16 x 16 block (query block i, key block j) of the
  // tile pair is live; klist / koff the same per key tile with (Q tile, ...).
  // qord / kord: the tiles in visit order (longest list first).
  const int* qoff;
  const int4* qlist;
  const int* qord;
  const int* koff;
  const int4* klist;
  const int* kord;
};
cudaError_t launch_bwd(int d, const BwdArgs& a, cudaStream_t s);

// TMA map of a [B, N, H, d] bf16 array as {d, H, N, B} with a {64, 1, box_rows, 1}
// box and 128-byte swizzle; rows past N read as zeros.  False (with the error
// detail set) if the driver refuses it.
bool encode_bf16_map(CUtensorMap* m, const void* base, int B, int N, int H, int d, int box_rows);

// Sets the text returned by attn_last_error_detail() on this thread.
void set_error_detail(const char* msg);

// ATTN_OK if the current device is sm_100, else ATTN_ERR_UNSUPPORTED (or
// ATTN_ERR_CUDA) with the error detail set.
int require_sm100();

// Forgets the cached device addresses of attn_decode_noalloc's scratch array
// (called by attn_shutdown, so that a device reset after it starts afresh).
void noalloc_forget();

}  // namespace eio
