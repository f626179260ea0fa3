// plan.cpp -- host tile planner and classifier (see plan.h).
#include "plan.h"

#include <algorithm>
#include <utility>
#include <cstring>

namespace eio {

static inline int ceil_div(int a, int b) { return (a + b - 1) / b; }
static inline int round_up16(int a) { return (a + 15) & ~15; }

void build_plan(int mask_kind, const uint8_t* block_map, int Nq, int Nkv, Plan* out) {
  out->q.clear();
  out->kv.clear();
  out->order.clear();
  out->n_partial = 0;
  if (mask_kind == 0 || mask_kind == 1) {
    // Dense grid of 128x128 tiles.  Causal (bottom-right aligned):
    // key j allowed for query i iff j <= i + off.
    const int off = Nkv - Nq;
    for (int r0 = 0; r0 < Nq; r0 += kTileQ) {
      const int nr = std::min(kTileQ, Nq - r0);
      QTile qt{r0, nr, static_cast<int32_t>(out->kv.size()), 0};
      for (int c0 = 0; c0 < Nkv; c0 += kTileKV) {
        const int nreal = std::min(kTileKV, Nkv - c0);
        bool full = true;
        if (mask_kind == 1) {
          const int last_row = r0 + nr - 1;
          if (c0 > last_row + off) break;  // this and every later tile is empty
          full = (c0 + nreal - 1) <= r0 + off;
        }
        const int nc = round_up16(nreal);
        const bool partial = !full || nc != nreal;
        out->kv.push_back(KVTile{c0, nc, partial ? 1 : 0, 0});
        out->n_partial += partial;
        qt.n_kv++;
      }
      out->q.push_back(qt);
    }
  } else {
    // Block map: group consecutive 16-row block rows whose map rows are
    // identical; within such a segment every 16-column block is either
    // allowed for all rows or for none, so the merged spans of allowed
    // blocks cut into <= 128-column tiles are all full (no predicate),
    // except where a tile runs past Nkv.
    const int nbr = ceil_div(Nq, kGrain), nbc = ceil_div(Nkv, kGrain);
    int br = 0;
    while (br < nbr) {
      int br1 = br + 1;
      const uint8_t* rowp = block_map + static_cast<size_t>(br) * nbc;
      while (br1 < nbr && std::memcmp(rowp, block_map + static_cast<size_t>(br1) * nbc, nbc) == 0)
        ++br1;
      const int first = static_cast<int>(out->kv.size());
      int cb = 0;
      while (cb < nbc) {
        if (!rowp[cb]) {
          ++cb;
          continue;
        }
        int cb1 = cb;
        while (cb1 < nbc && rowp[cb1]) ++cb1;
        for (int c0 = cb * kGrain; c0 < cb1 * kGrain; c0 += kTileKV) {
          const int nc = std::min(kTileKV, cb1 * kGrain - c0);
          const bool partial = c0 + nc > Nkv;
          out->kv.push_back(KVTile{c0, nc, partial ? 1 : 0, 0});
          out->n_partial += partial;
        }
        cb = cb1;
      }
      const int nkv = static_cast<int>(out->kv.size()) - first;
      const int r_end = std::min(br1 * kGrain, Nq);
      for (int r0 = br * kGrain; r0 < r_end; r0 += kTileQ)
        out->q.push_back(QTile{r0, std::min(kTileQ, r_end - r0), first, nkv});
      br = br1;
    }
  }
  out->order.resize(out->q.size());
  for (size_t i = 0; i < out->q.size(); ++i) out->order[i] = static_cast<int32_t>(i);
  std::stable_sort(out->order.begin(), out->order.end(), [&](int32_t a, int32_t b) {
    return out->q[a].n_kv > out->q[b].n_kv;
  });
}

// A Q tile's KV list re-cut into tiles of up to 128 keys made of at most two
// contiguous segments: the list's spans of consecutive keys are laid end to
// end and cut every 128 keys, a tile taking the head of the next span when its
// own span ends early.  Returns false (out untouched) for a list with a
// partial tile, which keeps its own tiles.
static bool recut(const Plan& plan, const QTile& q, std::vector<PairKV>* out) {
  std::vector<std::pair<int, int>> spans;  // (first key, keys)
  for (int k = 0; k < q.n_kv; ++k) {
    const KVTile& t = plan.kv[q.first_kv + k];
    if (t.partial) return false;
    if (!spans.empty() && spans.back().first + spans.back().second == t.col0)
      spans.back().second += t.ncols;
    else
      spans.push_back({t.col0, t.ncols});
  }
  size_t si = 0;
  int off = 0;  // keys of spans[si] already placed
  while (si < spans.size()) {
    PairKV v{};
    const int n0 = std::min(kTileKV, spans[si].second - off);
    v.col0 = spans[si].first + off;
    v.ncols = n0;
    off += n0;
    if (off == spans[si].second) {
      ++si;
      off = 0;
    }
    if (v.ncols < kTileKV && si < spans.size()) {
      const int n1 = std::min(kTileKV - v.ncols, spans[si].second);
      v.col1 = spans[si].first;
      v.ncols += n1;
      v.flags = n0 << 8;
      off = n1;
      if (off == spans[si].second) {
        ++si;
        off = 0;
      }
    }
    out->push_back(v);
  }
  return true;
}

void build_pairs(const Plan& plan, bool rows_mode, PairPlan* out) {
  out->rows_mode = rows_mode;
  out->pairs.clear();
  out->kv.clear();
  out->order.clear();
  auto same = [](const PairKV& x, const PairKV& y) {
    return x.col0 == y.col0 && x.ncols == y.ncols && x.flags == y.flags && x.col1 == y.col1;
  };
  auto push_pair = [&](const QTile* a, const QTile& b) {
    // Two-segment tiles where both lists allow them and A's stays a prefix of B's.
    std::vector<PairKV> vb, va;
    if (recut(plan, b, &vb) && (!a || recut(plan, *a, &va))) {
      bool ok = va.size() <= vb.size();
      for (size_t k = 0; ok && k < va.size(); ++k) ok = same(va[k], vb[k]);
      if (ok) {
        PairTile pt{};
        pt.rowB = b.row0;
        pt.nrowsB = b.nrows;
        pt.nB = static_cast<int32_t>(vb.size());
        pt.kv_first = static_cast<int32_t>(out->kv.size());
        if (a) {
          pt.rowA = a->row0;
          pt.nrowsA = a->nrows;
          pt.nA = static_cast<int32_t>(va.size());
        }
        out->kv.insert(out->kv.end(), vb.begin(), vb.end());
        out->pairs.push_back(pt);
        return;
      }
    }
    PairTile pt{};
    pt.rowB = b.row0;
    pt.nrowsB = b.nrows;
    pt.nB = b.n_kv;
    pt.kv_first = static_cast<int32_t>(out->kv.size());
    if (a) {
      pt.rowA = a->row0;
      pt.nrowsA = a->nrows;
      pt.nA = a->n_kv;
    }
    for (int k = 0; k < b.n_kv; ++k) {
      const KVTile& t = plan.kv[b.first_kv + k];
      int flags = t.partial ? 2 : 0;
      if (a && k < a->n_kv && plan.kv[a->first_kv + k].partial) flags |= 1;
      out->kv.push_back(PairKV{t.col0, t.ncols, flags, 0});
    }
    out->pairs.push_back(pt);
  };
  // A's KV list is a prefix of B's (same tiles, same order).
  auto nests = [&](const QTile& a, const QTile& b) {
    if (a.n_kv > b.n_kv) return false;
    for (int k = 0; k < a.n_kv; ++k) {
      const KVTile& x = plan.kv[a.first_kv + k];
      const KVTile& y = plan.kv[b.first_kv + k];
      if (x.col0 != y.col0 || x.ncols != y.ncols) return false;
    }
    return true;
  };
  const size_t nq = plan.q.size();
  if (!rows_mode) {
    for (size_t i = 0; i < nq; ++i) push_pair(&plan.q[i], plan.q[i]);
  } else {
    size_t i = 0;
    while (i < nq) {
      if (i + 1 < nq && nests(plan.q[i], plan.q[i + 1])) {
        push_pair(&plan.q[i], plan.q[i + 1]);
        i += 2;
      } else if (i + 1 < nq && nests(plan.q[i + 1], plan.q[i])) {
        push_pair(&plan.q[i + 1], plan.q[i]);
        i += 2;
      } else {
        push_pair(nullptr, plan.q[i]);
        i += 1;
      }
    }
  }
  out->order.resize(out->pairs.size());
  for (size_t i = 0; i < out->pairs.size(); ++i) out->order[i] = static_cast<int32_t>(i);
  std::stable_sort(out->order.begin(), out->order.end(), [&](int32_t x, int32_t y) {
    return out->pairs[x].nB > out->pairs[y].nB;
  });
}

void classify_tiles(int mask_kind, const uint8_t* block_map, int Nq, int Nkv, int tq, int tk,
                    uint8_t* out) {
  const int nti = ceil_div(Nq, tq), ntj = ceil_div(Nkv, tk);
  const int off = Nkv - Nq;
  const int nbc = ceil_div(Nkv, kGrain);
  for (int ti = 0; ti < nti; ++ti) {
    const int r0 = ti * tq, r1 = std::min(Nq, r0 + tq);
    for (int tj = 0; tj < ntj; ++tj) {
      const int c0 = tj * tk, c1 = std::min(Nkv, c0 + tk);
      uint8_t cls;
      if (mask_kind == 0) {
        cls = 1;
      } else if (mask_kind == 1) {
        if (c0 > (r1 - 1) + off)
          cls = 0;
        else if ((c1 - 1) <= r0 + off)
          cls = 1;
        else
          cls = 2;
      } else {
        // Every (block row, block column) overlap with the tile is uniform.
        bool any = false, all = true;
        for (int bi = r0 / kGrain; bi <= (r1 - 1) / kGrain; ++bi)
          for (int bj = c0 / kGrain; bj <= (c1 - 1) / kGrain; ++bj) {
            const bool a = block_map[static_cast<size_t>(bi) * nbc + bj] != 0;
            any |= a;
            all &= a;
          }
        cls = !any ? 0 : (all ? 1 : 2);
      }
      out[static_cast<size_t>(ti) * ntj + tj] = cls;
    }
  }
}

void frame_block_map(int n_frames, int frame_len, uint8_t* out) {
  const long N = static_cast<long>(n_frames) * frame_len;
  const int nb = static_cast<int>((N + kGrain - 1) / kGrain);
  for (int bi = 0; bi < nb; ++bi) {
    const int fq = static_cast<int>(static_cast<long>(bi) * kGrain / frame_len);
    for (int bj = 0; bj < nb; ++bj) {
      const int fk = static_cast<int>(static_cast<long>(bj) * kGrain / frame_len);
      out[static_cast<size_t>(bi) * nb + bj] = (fk == 0 || fk == fq || fk == fq - 1) ? 1 : 0;
    }
  }
}

}  // namespace eio
