// Host check of the prefill pair builder over every mask kind and both pairing modes.  For random
// shapes (ragged lengths included) and random block maps, every pair plan must satisfy what the
// kernel relies on:
//   - every Q tile of the plan runs exactly once, in slot A or slot B of one pair;
//   - 'heads' mode pairs a Q tile with itself (two query heads, one KV list);
//   - slot B's tiles cover exactly the keys of its Q tile in the plan, each once, slot A's keys are
//     exactly those of the first nA tiles of the same list, and no tile is wider than 128 keys;
//   - a tile of a pair kept without re-cutting carries, per slot, the partial flag of that slot's
//     own tile in the plan; a re-cut tile has no partial flag (re-cutting is for predicate-free lists);
//   - the visit order is a permutation of the pairs, most KV tiles first.
#include <algorithm>
#include <cstdio>
#include <random>
#include <set>
#include <vector>

#include "plan.h"
using namespace eio;

static std::set<int> tile_keys(const PairKV& v) {
  std::set<int> s;
  const int n0 = (v.flags >> 8) & 0xFF;
  if (n0) {
    for (int c = 0; c < n0; ++c) s.insert(v.col0 + c);
    for (int c = 0; c < v.ncols - n0; ++c) s.insert(v.col1 + c);
  } else {
    for (int c = 0; c < v.ncols; ++c) s.insert(v.col0 + c);
  }
  return s;
}

static std::set<int> plan_keys(const Plan& p, const QTile& q) {
  std::set<int> s;
  for (int k = 0; k < q.n_kv; ++k) {
    const KVTile& t = p.kv[q.first_kv + k];
    for (int c = 0; c < t.ncols; ++c) s.insert(t.col0 + c);
  }
  return s;
}

int main() {
  std::mt19937 rng(11);
  int bad = 0, pairs = 0, recut = 0, trials = 0;
  auto fail = [&](const char* what, int trial) {
    if (bad < 20) printf("trial %d: %s\n", trial, what);
    ++bad;
  };
  for (int trial = 0; trial < 600; ++trial) {
    const int kind = trial % 3;
    int Nq, Nkv;
    std::vector<uint8_t> map;
    if (kind == 2) {
      Nq = 1 + rng() % 700;
      Nkv = 1 + rng() % 900;
      const int nbq = (Nq + 15) / 16, nbk = (Nkv + 15) / 16;
      map.resize(static_cast<size_t>(nbq) * nbk);
      const int pct = 10 + rng() % 80;
      for (auto& m : map) m = static_cast<int>(rng() % 100) < pct;
      if (trial % 2) {  // runs of identical block rows, as under frame masks
        for (int r = 1; r < nbq; ++r)
          if (rng() % 4) std::copy(map.begin() + (r - 1) * nbk, map.begin() + r * nbk, map.begin() + r * nbk);
      }
    } else {
      Nq = 1 + rng() % 1500;
      Nkv = 1 + rng() % 1500;
    }
    Plan p;
    build_plan(kind, kind == 2 ? map.data() : nullptr, Nq, Nkv, &p);
    ++trials;
    for (int rm = 0; rm < 2; ++rm) {
      PairPlan pp;
      build_pairs(p, rm == 1, &pp);
      std::vector<int> uses(p.q.size(), 0);
      auto qtile = [&](int row0) -> int {
        for (size_t i = 0; i < p.q.size(); ++i)
          if (p.q[i].row0 == row0) return static_cast<int>(i);
        return -1;
      };
      for (const PairTile& t : pp.pairs) {
        ++pairs;
        const int ib = qtile(t.rowB);
        if (ib < 0 || p.q[ib].nrows != t.nrowsB) {
          fail("slot B is not a plan Q tile", trial);
          continue;
        }
        const QTile& qb = p.q[ib];
        uses[ib]++;
        int ia = -1;
        if (t.nrowsA > 0) {
          ia = qtile(t.rowA);
          if (ia < 0 || p.q[ia].nrows != t.nrowsA) {
            fail("slot A is not a plan Q tile", trial);
            continue;
          }
          if (rm == 1) uses[ia]++;
          else if (ia != ib) fail("heads mode pairs two different Q tiles", trial);
        }
        if (t.nA > t.nB || (t.nrowsA == 0 && t.nA != 0)) fail("slot A's tile count", trial);
        std::set<int> kb, ka;
        long vb = 0, va = 0;  // keys visited by each slot, with multiplicity
        bool is_recut = false;
        for (int k = 0; k < t.nB; ++k) {
          const PairKV& v = pp.kv[t.kv_first + k];
          if (v.ncols < 1 || v.ncols > 128) fail("tile width", trial);
          if ((v.flags >> 8) & 0xFF) is_recut = true;
          const std::set<int> s = tile_keys(v);
          kb.insert(s.begin(), s.end());
          vb += v.ncols;
          if (k < t.nA) {
            ka.insert(s.begin(), s.end());
            va += v.ncols;
          }
        }
        if (vb != static_cast<long>(kb.size()) || va != static_cast<long>(ka.size()))
          fail("a slot visits a key twice", trial);
        if (kb != plan_keys(p, qb)) fail("slot B's keys differ from the plan", trial);
        if (ia >= 0 && ka != plan_keys(p, p.q[ia])) fail("slot A's keys differ from the plan", trial);
        // per-slot partial flags
        const bool kept = t.nB == qb.n_kv && !is_recut &&
                          [&] {
                            for (int k = 0; k < t.nB; ++k) {
                              const PairKV& v = pp.kv[t.kv_first + k];
                              const KVTile& x = p.kv[qb.first_kv + k];
                              if (v.col0 != x.col0 || v.ncols != x.ncols) return false;
                            }
                            return true;
                          }();
        if (kept) {
          for (int k = 0; k < t.nB; ++k) {
            const PairKV& v = pp.kv[t.kv_first + k];
            if (((v.flags >> 1) & 1) != (p.kv[qb.first_kv + k].partial ? 1 : 0)) fail("slot B's partial flag", trial);
            if (k < t.nA && ((v.flags & 1) != (p.kv[p.q[ia].first_kv + k].partial ? 1 : 0)))
              fail("slot A's partial flag", trial);
          }
        } else {
          ++recut;
          for (int k = 0; k < t.nB; ++k)
            if (pp.kv[t.kv_first + k].flags & 3) fail("a re-cut tile carries a partial flag", trial);
          for (int k = 0; k < qb.n_kv; ++k)
            if (p.kv[qb.first_kv + k].partial) fail("a list with partial tiles was re-cut", trial);
        }
      }
      for (size_t i = 0; i < uses.size(); ++i)
        if (uses[i] != 1) fail("a Q tile does not run exactly once", trial);
      std::vector<int> ord(pp.order.begin(), pp.order.end());
      std::sort(ord.begin(), ord.end());
      for (size_t i = 0; i < ord.size(); ++i)
        if (ord[i] != static_cast<int>(i)) fail("order is not a permutation", trial);
      for (size_t i = 1; i < pp.order.size(); ++i)
        if (pp.pairs[pp.order[i - 1]].nB < pp.pairs[pp.order[i]].nB) fail("order is not longest first", trial);
    }
  }
  printf("bad %d  trials %d  pairs %d  re-cut pairs %d\n", bad, trials, pairs, recut);
  return bad != 0;
}
