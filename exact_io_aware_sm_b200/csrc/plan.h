// plan.h -- host-side tile planning for the prefill kernels.
//
// A plan lists, for every Q tile (<= 128 rows), the KV tiles (<= 128 columns,
// a multiple of 16) it must visit.  Empty tiles are never listed, so the
// kernel skips them without looking (block-sparse skipping, FlashAttention
// page section 6).  Tiles marked partial carry an element predicate in the
// kernel; all other tiles run without one (TPU attention guide, step 3).
#pragma once

#include <cstdint>
#include <vector>

namespace eio {

constexpr int kTileQ = 128;
constexpr int kTileKV = 128;
constexpr int kGrain = 16;

struct QTile {
  int32_t row0, nrows, first_kv, n_kv;
};
struct KVTile {
  int32_t col0, ncols, partial, pad;
};

struct Plan {
  std::vector<QTile> q;
  std::vector<KVTile> kv;
  std::vector<int32_t> order;  // Q tiles, most KV tiles first
  int64_t n_partial = 0;
};

// Build the plan.  mask_kind: 0 none, 1 causal, 2 block (block_map required).
void build_plan(int mask_kind, const uint8_t* block_map, int Nq, int Nkv, Plan* out);

// Tile classes over an arbitrary grid: 0 empty, 1 full, 2 partial.
void classify_tiles(int mask_kind, const uint8_t* block_map, int Nq, int Nkv, int tq, int tk,
                    uint8_t* out);

// Frame-aligned block map: query frame f sees key frames {0, f-1, f}.
// Requires frame_len % 16 == 0.
void frame_block_map(int n_frames, int frame_len, uint8_t* out);

}  // namespace eio
