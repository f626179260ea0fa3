// Host check of the prefill pair builder: the two-segment re-cut of every pair's KV list covers
// exactly the keys of the original plan, each once, all allowed by the block map, in tiles of at
// most 128 keys.
#include "plan.h"
#include <cstdio>
#include <set>
#include <vector>
#include <random>
using namespace eio;
int main() {
  std::mt19937 rng(5);
  int bad = 0, two = 0, tiles = 0, orig = 0;
  for (int trial = 0; trial < 300; ++trial) {
    int Nq, Nkv; std::vector<uint8_t> map;
    if (trial == 0) { Nq = Nkv = 24 * 1040; map.resize((Nq / 16) * (Nkv / 16)); frame_block_map(24, 1040, map.data()); }
    else { Nq = 16 * (1 + rng() % 40); Nkv = 16 * (1 + rng() % 60); map.resize((Nq / 16) * (Nkv / 16)); for (auto& m : map) m = (rng() % 100) < 40; }
    Plan p; build_plan(2, map.data(), Nq, Nkv, &p);
    for (int rm = 0; rm < 2; ++rm) {
      PairPlan pp; build_pairs(p, rm == 1, &pp);
      for (const auto& t : pp.pairs) {
        std::set<int> got;
        long visits = 0;  // keys visited, counted with multiplicity: each must be visited once
        for (int k = 0; k < t.nB; ++k) {
          const PairKV& v = pp.kv[t.kv_first + k];
          int n0 = (v.flags >> 8) & 0xFF; tiles++;
          if (v.ncols > 128 || v.ncols % 16) bad++;
          visits += v.ncols;
          if (n0) { two++; for (int c = 0; c < n0; ++c) got.insert(v.col0 + c); for (int c = 0; c < v.ncols - n0; ++c) got.insert(v.col1 + c); }
          else for (int c = 0; c < v.ncols; ++c) got.insert(v.col0 + c);
        }
        if (visits != static_cast<long>(got.size())) bad++;  // a key visited twice
        // keys of slot B's Q tile from the original plan
        const QTile* qb = nullptr;
        for (const auto& q : p.q) if (q.row0 == t.rowB) qb = &q;
        std::set<int> want;
        for (int k = 0; k < qb->n_kv; ++k) { const KVTile& x = p.kv[qb->first_kv + k]; for (int c = 0; c < x.ncols; ++c) want.insert(x.col0 + c); }
        if (rm == 1 && trial == 0) orig += qb->n_kv;
        if (got != want) bad++;
        // allowed by the map for every row of the tile
        for (int c : got) for (int r = t.rowB; r < t.rowB + t.nrowsB; r += 16) if (!map[(r / 16) * (Nkv / 16) + c / 16]) bad++;
      }
    }
  }
  printf("bad %d  two-segment tiles %d of %d\n", bad, two, tiles);
  return bad != 0;
}
