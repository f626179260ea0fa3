// plan_shim.cpp -- test-only C entry point to the host tile planner (plan.cpp), so that a copy of the
// planner can be built with g++ alone and checked from Python against the oracle's schedule checker.
// Output format as attn_plan: qtiles [n][4] = (row0, nrows, first_kv, n_kv), kvtiles [m][3] =
// (col0, ncols, partial).
#include <cstdint>

#include "plan.h"

extern "C" int shim_plan(int mask_kind, const uint8_t* block_map, int Nq, int Nkv, int32_t* qtiles, int qcap,
                         int32_t* kvtiles, int kvcap, int* n_q, int* n_kv) {
  eio::Plan p;
  eio::build_plan(mask_kind, block_map, Nq, Nkv, &p);
  *n_q = static_cast<int>(p.q.size());
  *n_kv = static_cast<int>(p.kv.size());
  if ((qtiles && qcap < *n_q) || (kvtiles && kvcap < *n_kv)) return 2;
  for (size_t i = 0; qtiles && i < p.q.size(); ++i) {
    qtiles[4 * i + 0] = p.q[i].row0;
    qtiles[4 * i + 1] = p.q[i].nrows;
    qtiles[4 * i + 2] = p.q[i].first_kv;
    qtiles[4 * i + 3] = p.q[i].n_kv;
  }
  for (size_t i = 0; kvtiles && i < p.kv.size(); ++i) {
    kvtiles[3 * i + 0] = p.kv[i].col0;
    kvtiles[3 * i + 1] = p.kv[i].ncols;
    kvtiles[3 * i + 2] = p.kv[i].partial;
  }
  return 0;
}
