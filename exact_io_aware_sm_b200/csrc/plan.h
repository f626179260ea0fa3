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

// Q tiles processed two at a time by one CTA ("slots" A and B) that share
// every K/V tile: slot B visits the whole KV list, slot A a prefix of it.
//   mode 'heads' (query heads per KV head G >= 2): A and B are the same Q tile
//     for two query heads of one KV group (identical KV lists);
//   mode 'rows' (G == 1): A and B are two Q tiles of one head whose KV lists
//     nest (A's list is a prefix of B's), e.g. consecutive causal tiles.
// A Q tile without a partner runs alone in slot B.
struct PairTile {
  int32_t rowA, nrowsA, rowB, nrowsB;  // nrowsA == 0: slot A unused
  int32_t kv_first, nA, nB, pad;       // KV tiles [kv_first, kv_first + nB); A uses the first nA
};
// A KV tile of up to 128 keys in one or two contiguous segments:
// [col0, col0 + n0) then [col1, col1 + ncols - n0), n0 = flags >> 8 (0: one
// segment of ncols keys from col0).  Two segments join the short tails of
// separate key spans of a block-sparse list (never on partial tiles).
struct PairKV {
  int32_t col0, ncols, flags, col1;  // flags bit 0: partial for A, bit 1: partial for B; bits 8..15: n0
};
struct PairPlan {
  bool rows_mode = false;
  std::vector<PairTile> pairs;
  std::vector<PairKV> kv;
  std::vector<int32_t> order;  // pairs, most KV tiles first
};
void build_pairs(const Plan& plan, bool rows_mode, PairPlan* out);

// Tile classes over an arbitrary grid: 0 empty, 1 full, 2 partial.
void classify_tiles(int mask_kind, const uint8_t* block_map, int Nq, int Nkv, int tq, int tk,
                    uint8_t* out);

// Frame-aligned block map: query frame f sees key frames {0, f-1, f}.
// Requires frame_len % 16 == 0.
void frame_block_map(int n_frames, int frame_len, uint8_t* out);

}  // namespace eio
