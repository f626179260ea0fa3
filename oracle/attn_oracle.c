/*
 * attn_oracle.c -- plain, slow, fp64 CPU oracle for exact attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA library under exact_io_aware_sm_b200/.
 *
 * What it computes is the plain definition, with S and P materialised:
 *
 *   Scaled dot-product attention, "Attention Mechanism Optimization for
 *   Efficient LLM Inference" (pyy0715.github.io), section "Background: Scaled
 *   Dot-Product Attention", equation Attention(Q,K,V) = softmax(QK^T/sqrt(d_k))V,
 *   and its "Kernel Fusion" table: S = QK^T * scale, P = softmax(S), O = PV,
 *   each a full pass.  FlashAttention returns exactly this result
 *   ("FlashAttention: memory-saving exact attention", base.kaita.kr, section 3,
 *   Theorem 1), so the oracle is the definition written out, not the tiled
 *   algorithm.
 *
 *   Safe softmax (max subtraction): same FlashAttention page, section 2 step 1;
 *   the inference page's softmax equation in section "Tiling".
 *
 *   GQA head mapping: query heads form contiguous groups that share one KV
 *   head (inference page, section "Grouped-Query Attention", mapping diagram),
 *   so hkv = hq / (Hq / Hkv).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - the mask is boolean, applied as -inf on the scaled logits;
 *   - causal alignment is bottom-right: key j allowed for query i iff
 *     j <= i + (Nkv - Nq);
 *   - a row with no allowed key has O = 0 and LSE = -inf;
 *   - LSE is the natural log-sum-exp of the scaled logits, m + ln(l);
 *   - BLOCK masks are 16x16-granular: allowed iff block_map[i/16][j/16] != 0;
 *   - the frame rule: query frame f sees key frames {0, f-1, f} (a set);
 *   - bound-based softmax ("TPU attention optimisation guide", step 4): keys
 *     are centred on the mean over all keys of their (b, KV head); a row uses
 *     the bound where it keeps every P at or above 2^-limit2 and falls back to
 *     its exact max otherwise (the guide checks eligibility per head; this is
 *     the same test per row, and a head is eligible iff all its rows are).
 *
 * Inputs are read element by element and converted to double from exactly the
 * stored value (bf16 bit patterns, fp32 or fp64).
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORA_MASK_NONE 0
#define ORA_MASK_CAUSAL 1
#define ORA_MASK_BLOCK 2

#define ORA_BF16 0
#define ORA_F32 1
#define ORA_F64 2

#define ORA_GRAIN 16 /* block-map granularity (rows and columns) */

static double ld(const void *p, int dtype, size_t idx) {
  if (dtype == ORA_BF16) {
    uint32_t u = (uint32_t)((const uint16_t *)p)[idx] << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
  }
  if (dtype == ORA_F32) return (double)((const float *)p)[idx];
  return ((const double *)p)[idx];
}

/* Element mask, from its definition (no tiles involved). */
int ora_allowed(int mask_kind, const uint8_t *block_map, int Nq, int Nkv, int i, int j) {
  if (i < 0 || i >= Nq || j < 0 || j >= Nkv) return 0;
  if (mask_kind == ORA_MASK_NONE) return 1;
  if (mask_kind == ORA_MASK_CAUSAL) return j <= i + (Nkv - Nq);
  if (mask_kind == ORA_MASK_BLOCK) {
    int nbc = (Nkv + ORA_GRAIN - 1) / ORA_GRAIN;
    return block_map[(size_t)(i / ORA_GRAIN) * nbc + (j / ORA_GRAIN)] != 0;
  }
  return 0;
}

/*
 * One query row against keys [0, nkeys) of one (b, hkv) slice.
 * q_at(t), k_at(j,t), v_at(j,t) are expressed through base offsets and strides
 * (in elements).  Writes o[0..d) (fp64) and *lse.
 */
static void one_row(const void *q, size_t q_off, const void *k, const void *v, size_t kv_off,
                    size_t kv_row_stride, int nkeys, int d, double scale, int dtype,
                    int mask_kind, const uint8_t *block_map, int Nq, int Nkv, int qi,
                    double *S, double *o, double *lse) {
  /* S = scale * q k^T for allowed keys, -inf otherwise (materialised row). */
  double m = -INFINITY;
  for (int j = 0; j < nkeys; ++j) {
    if (mask_kind >= 0 && !ora_allowed(mask_kind, block_map, Nq, Nkv, qi, j)) {
      S[j] = -INFINITY;
      continue;
    }
    double acc = 0.0;
    for (int t = 0; t < d; ++t)
      acc += ld(q, dtype, q_off + t) * ld(k, dtype, kv_off + (size_t)j * kv_row_stride + t);
    S[j] = scale * acc;
    if (S[j] > m) m = S[j];
  }
  for (int t = 0; t < d; ++t) o[t] = 0.0;
  if (m == -INFINITY) { /* no allowed key */
    *lse = -INFINITY;
    return;
  }
  /* P = exp(S - m) (materialised in place), l = sum P. */
  double l = 0.0;
  for (int j = 0; j < nkeys; ++j) {
    S[j] = (S[j] == -INFINITY) ? 0.0 : exp(S[j] - m);
    l += S[j];
  }
  /* O = P V / l. */
  for (int j = 0; j < nkeys; ++j) {
    if (S[j] == 0.0) continue;
    for (int t = 0; t < d; ++t)
      o[t] += S[j] * ld(v, dtype, kv_off + (size_t)j * kv_row_stride + t);
  }
  for (int t = 0; t < d; ++t) o[t] /= l;
  *lse = m + log(l);
}

/*
 * Prefill attention for a list of rows.
 * Layouts (contiguous): q [B,Nq,Hq,d], k/v [B,Nkv,Hkv,d].
 * rows: nrows triples (b, hq, i).  o: [nrows][d] fp64, lse: [nrows] fp64.
 * Returns 0, or -1 on bad arguments.
 */
int ora_attn_rows(const void *q, const void *k, const void *v, int dtype, int B, int Hq, int Hkv,
                  int Nq, int Nkv, int d, double scale, int mask_kind, const uint8_t *block_map,
                  const int32_t *rows, int nrows, double *o, double *lse) {
  if (Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || Nq < 0 || Nkv < 0) return -1;
  if (mask_kind == ORA_MASK_BLOCK && !block_map) return -1;
  int G = Hq / Hkv;
  int bad = 0;
#pragma omp parallel
  {
    double *S = (double *)malloc(sizeof(double) * (size_t)(Nkv > 0 ? Nkv : 1));
#pragma omp for schedule(dynamic, 4)
    for (int r = 0; r < nrows; ++r) {
      int b = rows[3 * r], hq = rows[3 * r + 1], i = rows[3 * r + 2];
      if (b < 0 || b >= B || hq < 0 || hq >= Hq || i < 0 || i >= Nq) {
        bad = 1;
        continue;
      }
      int hkv = hq / G;
      size_t q_off = (((size_t)b * Nq + i) * Hq + hq) * d;
      size_t kv_off = ((size_t)b * Nkv * Hkv + hkv) * d;
      one_row(q, q_off, k, v, kv_off, (size_t)Hkv * d, Nkv, d, scale, dtype, mask_kind, block_map,
              Nq, Nkv, i, S, o + (size_t)r * d, lse + r);
    }
    free(S);
  }
  return bad ? -1 : 0;
}

/* Every row: o [B,Nq,Hq,d] fp64, lse [B,Hq,Nq] fp64. */
int ora_attn_fwd(const void *q, const void *k, const void *v, int dtype, int B, int Hq, int Hkv,
                 int Nq, int Nkv, int d, double scale, int mask_kind, const uint8_t *block_map,
                 double *o, double *lse) {
  if (Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || Nq < 0 || Nkv < 0) return -1;
  if (mask_kind == ORA_MASK_BLOCK && !block_map) return -1;
  int G = Hq / Hkv;
  long total = (long)B * Hq * Nq;
#pragma omp parallel
  {
    double *S = (double *)malloc(sizeof(double) * (size_t)(Nkv > 0 ? Nkv : 1));
#pragma omp for schedule(dynamic, 16)
    for (long r = 0; r < total; ++r) {
      int i = (int)(r % Nq);
      int hq = (int)((r / Nq) % Hq);
      int b = (int)(r / ((long)Nq * Hq));
      int hkv = hq / G;
      size_t q_off = (((size_t)b * Nq + i) * Hq + hq) * d;
      size_t kv_off = ((size_t)b * Nkv * Hkv + hkv) * d;
      one_row(q, q_off, k, v, kv_off, (size_t)Hkv * d, Nkv, d, scale, dtype, mask_kind, block_map,
              Nq, Nkv, i, S, o + q_off, lse + ((size_t)b * Hq + hq) * Nq + i);
    }
    free(S);
  }
  return 0;
}

/*
 * Single-token decode over a KV cache (inference page, section "Decode":
 * the new query attends to every cached K_1..K_t, V_1..V_t).
 * q [B,Hq,d]; caches [B,Lmax,Hkv,d]; seqlens[B] (host) in [0, Lmax].
 * o [B,Hq,d] fp64, lse [B,Hq] fp64.  No mask beyond the cache length.
 */
int ora_decode(const void *q, const void *kc, const void *vc, int dtype, const int32_t *seqlens,
               int B, int Hq, int Hkv, int Lmax, int d, double scale, double *o, double *lse) {
  if (Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || Lmax < 0) return -1;
  for (int b = 0; b < B; ++b)
    if (seqlens[b] < 0 || seqlens[b] > Lmax) return -1;
  int G = Hq / Hkv;
#pragma omp parallel
  {
    double *S = (double *)malloc(sizeof(double) * (size_t)(Lmax > 0 ? Lmax : 1));
#pragma omp for schedule(dynamic, 1)
    for (int r = 0; r < B * Hq; ++r) {
      int b = r / Hq, hq = r % Hq, hkv = hq / G;
      size_t q_off = ((size_t)b * Hq + hq) * d;
      size_t kv_off = ((size_t)b * Lmax * Hkv + hkv) * d;
      one_row(q, q_off, kc, vc, kv_off, (size_t)Hkv * d, seqlens[b], d, scale, dtype,
              -1 /* no mask */, NULL, 1, seqlens[b], 0, S, o + q_off, lse + r);
    }
    free(S);
  }
  return 0;
}

/*
 * Online (block-wise) softmax statistics of one vector, for checking the
 * merge rule against the pages' worked examples ("FlashAttention" page,
 * section 2: per-block max m and sum l, merged with e^(m_block - m_all);
 * inference page, section "Online-Softmax": m_new = max(m_old, max B),
 * d_new = d_old * exp(m_old - m_new) + sum exp(B - m_new)).
 * bounds[0..nb]: block b covers x[bounds[b] .. bounds[b+1]).
 * Outputs per block: m_blk, l_blk (the block alone), m_run, l_run (merged
 * through block b), resc (the factor exp(m_run[b-1] - m_run[b]) applied to
 * the old sum; 1 for b = 0).
 */
int ora_online_softmax(const double *x, const int *bounds, int nb, double *m_blk, double *l_blk,
                       double *m_run, double *l_run, double *resc) {
  double m = -INFINITY, l = 0.0;
  for (int b = 0; b < nb; ++b) {
    int lo = bounds[b], hi = bounds[b + 1];
    if (hi < lo) return -1;
    double mb = -INFINITY;
    for (int j = lo; j < hi; ++j)
      if (x[j] > mb) mb = x[j];
    double lb = 0.0;
    for (int j = lo; j < hi; ++j) lb += exp(x[j] - mb);
    m_blk[b] = mb;
    l_blk[b] = lb;
    double mn = mb > m ? mb : m;
    double r = (b == 0 || m == -INFINITY) ? 1.0 : exp(m - mn);
    double lnew = (b == 0 ? 0.0 : l * r) + (mb == -INFINITY ? 0.0 : lb * exp(mb - mn));
    resc[b] = r;
    m = mn;
    l = lnew;
    m_run[b] = m;
    l_run[b] = l;
  }
  return 0;
}

/*
 * Merge of partial results over disjoint key sets (the same rule as above,
 * written for normalised partial outputs): given S partials (O_s [d], lse_s),
 * lse = log sum_s exp(lse_s) and O = sum_s exp(lse_s - lse) O_s.
 * A partial with lse_s = -inf contributes nothing.
 */
int ora_merge_partials(const double *o_parts, const double *lse_parts, int nparts, int d,
                       double *o, double *lse) {
  double m = -INFINITY;
  for (int s = 0; s < nparts; ++s)
    if (lse_parts[s] > m) m = lse_parts[s];
  for (int t = 0; t < d; ++t) o[t] = 0.0;
  if (m == -INFINITY) {
    *lse = -INFINITY;
    return 0;
  }
  double sum = 0.0;
  for (int s = 0; s < nparts; ++s) sum += exp(lse_parts[s] - m);
  double L = m + log(sum);
  for (int s = 0; s < nparts; ++s) {
    if (lse_parts[s] == -INFINITY) continue;
    double w = exp(lse_parts[s] - L);
    for (int t = 0; t < d; ++t) o[t] += w * o_parts[(size_t)s * d + t];
  }
  *lse = L;
  return 0;
}

/*
 * Frame-aligned element mask (TPU attention guide, aibase.it, step 3: the
 * live region follows frame boundaries; query frame f attends to its own
 * frame, the previous frame and the reference frame 0).
 */
int ora_frame_allowed(int frame_len, int i, int j) {
  int fi = i / frame_len, fj = j / frame_len;
  return fj == 0 || fj == fi || fj == fi - 1;
}

/*
 * 16x16 block map of the frame mask, by brute force over elements.  Fails
 * (-1) unless every 16x16 block is uniformly allowed or disallowed.
 * out: [ceil(N/16)][ceil(N/16)] with N = n_frames * frame_len.
 */
int ora_frame_block_map(int n_frames, int frame_len, uint8_t *out) {
  if (n_frames <= 0 || frame_len <= 0) return -1;
  long N = (long)n_frames * frame_len;
  int nb = (int)((N + ORA_GRAIN - 1) / ORA_GRAIN);
  for (int bi = 0; bi < nb; ++bi)
    for (int bj = 0; bj < nb; ++bj) {
      int any = 0, all = 1;
      for (int i = bi * ORA_GRAIN; i < (bi + 1) * ORA_GRAIN && i < N; ++i)
        for (int j = bj * ORA_GRAIN; j < (bj + 1) * ORA_GRAIN && j < N; ++j) {
          int a = ora_frame_allowed(frame_len, i, j);
          any |= a;
          all &= a;
        }
      if (any && !all) return -1;
      out[(size_t)bi * nb + bj] = (uint8_t)any;
    }
  return 0;
}

/*
 * Tile classification by brute force over elements: 0 empty (no element
 * allowed), 1 full (every element of the tile inside [0,Nq)x[0,Nkv) allowed),
 * 2 partial.  out: [ceil(Nq/tq)][ceil(Nkv/tk)].
 */
int ora_classify(int mask_kind, const uint8_t *block_map, int Nq, int Nkv, int tq, int tk,
                 uint8_t *out) {
  if (tq <= 0 || tk <= 0 || Nq < 0 || Nkv < 0) return -1;
  if (mask_kind == ORA_MASK_BLOCK && !block_map) return -1;
  int nti = (Nq + tq - 1) / tq, ntj = (Nkv + tk - 1) / tk;
#pragma omp parallel for schedule(dynamic, 1)
  for (int ti = 0; ti < nti; ++ti)
    for (int tj = 0; tj < ntj; ++tj) {
      long cnt = 0, tot = 0;
      for (int i = ti * tq; i < (ti + 1) * tq && i < Nq; ++i)
        for (int j = tj * tk; j < (tj + 1) * tk && j < Nkv; ++j) {
          cnt += ora_allowed(mask_kind, block_map, Nq, Nkv, i, j);
          ++tot;
        }
      out[(size_t)ti * ntj + tj] = (uint8_t)(cnt == 0 ? 0 : (cnt == tot ? 1 : 2));
    }
  return 0;
}

/* Number of allowed (query, key) pairs, by brute force. */
long long ora_count_allowed(int mask_kind, const uint8_t *block_map, int Nq, int Nkv) {
  long long c = 0;
#pragma omp parallel for reduction(+ : c) schedule(static)
  for (int i = 0; i < Nq; ++i)
    for (int j = 0; j < Nkv; ++j) c += ora_allowed(mask_kind, block_map, Nq, Nkv, i, j);
  return c;
}

/*
 * Check a tile schedule for one mask.  qtiles: nq x (row0, nrows, first, count),
 * kvtiles: nk x (col0, ncols, partial).  A tile's columns may run past Nkv
 * (padding), but every listed key must be < Nkv or the tile must be marked
 * partial.  Conditions checked:
 *   (1) the Q tiles partition [0, Nq) (in any order, no overlap, no gap);
 *   (2) within one Q tile the KV tiles are pairwise disjoint;
 *   (3) for every row of the Q tile, the union of its KV tiles, clipped to
 *       the allowed set, is exactly the row's allowed set (coverage);
 *   (4) every tile not marked partial is fully allowed for all its rows and
 *       columns (including columns < Nkv only).
 * Returns 0 when valid, or a positive code naming the first failed condition.
 */
int ora_check_schedule(int mask_kind, const uint8_t *block_map, int Nq, int Nkv,
                       const int32_t *qtiles, int nq, const int32_t *kvtiles, int nk) {
  uint8_t *rowseen = (uint8_t *)calloc((size_t)(Nq > 0 ? Nq : 1), 1);
  uint8_t *colseen = (uint8_t *)malloc((size_t)(Nkv > 0 ? Nkv : 1) + 4096);
  int rc = 0;
  for (int t = 0; t < nq && !rc; ++t) {
    int r0 = qtiles[4 * t], nr = qtiles[4 * t + 1], f = qtiles[4 * t + 2], c = qtiles[4 * t + 3];
    if (nr <= 0 || r0 < 0 || r0 + nr > Nq || f < 0 || c < 0 || f + c > nk) {
      rc = 1;
      break;
    }
    for (int i = r0; i < r0 + nr; ++i) {
      if (rowseen[i]) rc = 1;
      rowseen[i] = 1;
    }
    if (rc) break;
    memset(colseen, 0, (size_t)(Nkv > 0 ? Nkv : 1));
    for (int u = f; u < f + c && !rc; ++u) {
      int c0 = kvtiles[3 * u], nc = kvtiles[3 * u + 1], part = kvtiles[3 * u + 2];
      if (c0 < 0 || nc <= 0) {
        rc = 2;
        break;
      }
      for (int j = c0; j < c0 + nc && j < Nkv; ++j) {
        if (colseen[j]) rc = 2;
        colseen[j] = 1;
      }
      if (!part) {
        if (c0 + nc > Nkv) rc = 4;
        for (int i = r0; i < r0 + nr && !rc; ++i)
          for (int j = c0; j < c0 + nc && !rc; ++j)
            if (!ora_allowed(mask_kind, block_map, Nq, Nkv, i, j)) rc = 4;
      }
    }
    for (int i = r0; i < r0 + nr && !rc; ++i)
      for (int j = 0; j < Nkv && !rc; ++j)
        if (ora_allowed(mask_kind, block_map, Nq, Nkv, i, j) && !colseen[j]) rc = 3;
  }
  for (int i = 0; i < Nq && !rc; ++i)
    if (!rowseen[i]) rc = 1;
  free(rowseen);
  free(colseen);
  return rc;
}

/*
 * Gradients of attention for a given upstream gradient dO ("FlashAttention:
 * memory-saving exact attention", section 4: the backward needs S and P,
 * which the fast path recomputes from Q, K, V and the saved (m, l); the
 * oracle simply materialises them again from the definition).  For one
 * (b, hq) with hkv = hq / G and allowed pairs (i, j):
 *
 *   P[i][j]  = exp(S[i][j] - m_i) / l_i        (the forward's softmax)
 *   dV[j]   += P[i][j] * dO[i]                 (O = P V)
 *   dP[i][j] = dO[i] . V[j]
 *   D_i      = sum_j P[i][j] * dP[i][j]        (softmax Jacobian: dS = P (dP - D))
 *   dS[i][j] = P[i][j] * (dP[i][j] - D_i)
 *   dQ[i]    = scale * sum_j dS[i][j] * K[j]   (S = scale Q K^T)
 *   dK[j]   += scale * dS[i][j] * Q[i]
 *
 * dK and dV of a KV head sum over the G query heads that share it.  Masked
 * pairs carry no gradient; a row without allowed keys has dQ = 0.
 * Layouts: q, dO [B,Nq,Hq,d]; k, v [B,Nkv,Hkv,d] (dtype as ora_attn_fwd);
 * dq [B,Nq,Hq,d], dk and dv [B,Nkv,Hkv,d], all fp64.  Returns 0, or -1 on bad
 * arguments.
 */
int ora_attn_bwd(const void *q, const void *k, const void *v, const void *dout, int dtype, int B,
                 int Hq, int Hkv, int Nq, int Nkv, int d, double scale, int mask_kind,
                 const uint8_t *block_map, double *dq, double *dk, double *dv) {
  if (Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || Nq < 0 || Nkv < 0) return -1;
  if (mask_kind == ORA_MASK_BLOCK && !block_map) return -1;
  int G = Hq / Hkv;
  memset(dq, 0, sizeof(double) * (size_t)B * Nq * Hq * d);
  memset(dk, 0, sizeof(double) * (size_t)B * Nkv * Hkv * d);
  memset(dv, 0, sizeof(double) * (size_t)B * Nkv * Hkv * d);
  long slices = (long)B * Hkv;
#pragma omp parallel
  {
    size_t n = (size_t)(Nkv > 0 ? Nkv : 1);
    double *S = (double *)malloc(sizeof(double) * n);
    double *P = (double *)malloc(sizeof(double) * n);
    double *dP = (double *)malloc(sizeof(double) * n);
#pragma omp for schedule(dynamic, 1)
    for (long sl = 0; sl < slices; ++sl) {  /* one (b, hkv): its dK, dV are private to it */
      int b = (int)(sl / Hkv), hkv = (int)(sl % Hkv);
      size_t kv_base = ((size_t)b * Nkv * Hkv + hkv) * d, kv_stride = (size_t)Hkv * d;
      for (int g = 0; g < G; ++g) {
        int hq = hkv * G + g;
        for (int i = 0; i < Nq; ++i) {
          size_t q_off = (((size_t)b * Nq + i) * Hq + hq) * d;
          double m = -INFINITY;
          for (int j = 0; j < Nkv; ++j) {
            if (!ora_allowed(mask_kind, block_map, Nq, Nkv, i, j)) {
              S[j] = -INFINITY;
              continue;
            }
            double acc = 0.0;
            for (int t = 0; t < d; ++t)
              acc += ld(q, dtype, q_off + t) * ld(k, dtype, kv_base + (size_t)j * kv_stride + t);
            S[j] = acc * scale;
            if (S[j] > m) m = S[j];
          }
          if (m == -INFINITY) continue; /* no allowed key: no gradient */
          double l = 0.0;
          for (int j = 0; j < Nkv; ++j) {
            P[j] = S[j] == -INFINITY ? 0.0 : exp(S[j] - m);
            l += P[j];
          }
          double D = 0.0;
          for (int j = 0; j < Nkv; ++j) {
            P[j] /= l;
            dP[j] = 0.0;
            if (P[j] == 0.0 && S[j] == -INFINITY) continue;
            for (int t = 0; t < d; ++t)
              dP[j] += ld(dout, dtype, q_off + t) * ld(v, dtype, kv_base + (size_t)j * kv_stride + t);
            D += P[j] * dP[j];
          }
          for (int j = 0; j < Nkv; ++j) {
            if (S[j] == -INFINITY) continue;
            double ds = P[j] * (dP[j] - D);
            size_t kj = kv_base + (size_t)j * kv_stride;
            for (int t = 0; t < d; ++t) {
              dq[q_off + t] += scale * ds * ld(k, dtype, kj + t);
              dk[kj + t] += scale * ds * ld(q, dtype, q_off + t);
              dv[kj + t] += P[j] * ld(dout, dtype, q_off + t);
            }
          }
        }
      }
    }
    free(S);
    free(P);
    free(dP);
  }
  return 0;
}

/*
 * Bound-based softmax (TPU attention guide, step 4): the running max is
 * replaced by a per-row upper bound of the scores, found from Cauchy-Schwarz
 * after centring the keys on their mean.
 *
 * ora_key_stats: for every (b, hkv), kbar = (1/Nkv) sum_j k_j and
 * radius = max_j ||k_j - kbar|| over all Nkv keys.  kbar [B,Hkv,d] fp64,
 * radius [B,Hkv] fp64.
 */
int ora_key_stats(const void *k, int dtype, int B, int Nkv, int Hkv, int d, double *kbar,
                  double *radius) {
  if (B <= 0 || Nkv <= 0 || Hkv <= 0 || d <= 0) return -1;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < Hkv; ++h) {
      double *m = kbar + ((size_t)b * Hkv + h) * d;
      for (int t = 0; t < d; ++t) m[t] = 0.0;
      for (int j = 0; j < Nkv; ++j)
        for (int t = 0; t < d; ++t) m[t] += ld(k, dtype, (((size_t)b * Nkv + j) * Hkv + h) * d + t);
      for (int t = 0; t < d; ++t) m[t] /= Nkv;
      double r2 = 0.0;
      for (int j = 0; j < Nkv; ++j) {
        double s = 0.0;
        for (int t = 0; t < d; ++t) {
          double c = ld(k, dtype, (((size_t)b * Nkv + j) * Hkv + h) * d + t) - m[t];
          s += c * c;
        }
        if (s > r2) r2 = s;
      }
      radius[(size_t)b * Hkv + h] = sqrt(r2);
    }
  return 0;
}

/*
 * Prefill attention with the bound-based softmax.  For row i of query head
 * hq (KV head hkv = hq / G), with centred keys k'_j = k_j - kbar:
 *   S'_ij = scale * q_i . k'_j                (the centring shifts every score
 *                                              of the row by the same amount)
 *   M_i   = scale * ||q_i|| * radius          (>= S'_ij for every j)
 *   if 2 * M_i * log2(e) <= limit2 (no P can fall below 2^-limit2, since
 *   S'_ij >= -M_i as well): P_ij = exp(S'_ij - M_i), with no running max;
 *   otherwise the row falls back to the exact max of its scores.
 *   l_i = sum_j P_ij,  O_i = sum_j P_ij v_j / l_i,
 *   LSE_i = scale * q_i . kbar + M_i + ln l_i  (the scores' own LSE).
 * o [B,Nq,Hq,d] fp64, lse [B,Hq,Nq] fp64, bound_row [B,Hq,Nq] int32 (1 when
 * the row used the bound, 0 for the fallback).  kbar/radius as ora_key_stats.
 */
int ora_attn_fwd_bound(const void *q, const void *k, const void *v, int dtype, int B, int Hq, int Hkv,
                       int Nq, int Nkv, int d, double scale, int mask_kind, const uint8_t *block_map,
                       const double *kbar, const double *radius, double limit2, double *o, double *lse,
                       int32_t *bound_row) {
  if (Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || Nq < 0 || Nkv <= 0) return -1;
  if (mask_kind == ORA_MASK_BLOCK && !block_map) return -1;
  int G = Hq / Hkv;
  long total = (long)B * Hq * Nq;
#pragma omp parallel
  {
    double *P = (double *)malloc(sizeof(double) * (size_t)Nkv);
#pragma omp for schedule(dynamic, 16)
    for (long r = 0; r < total; ++r) {
      int i = (int)(r % Nq);
      int hq = (int)((r / Nq) % Hq);
      int b = (int)(r / ((long)Nq * Hq));
      int hkv = hq / G;
      const double *m = kbar + ((size_t)b * Hkv + hkv) * d;
      size_t q_off = (((size_t)b * Nq + i) * Hq + hq) * d;
      size_t li = ((size_t)b * Hq + hq) * Nq + i;
      double qn = 0.0, qm = 0.0;
      for (int t = 0; t < d; ++t) {
        double x = ld(q, dtype, q_off + t);
        qn += x * x;
        qm += x * m[t];
      }
      double M = scale * sqrt(qn) * radius[(size_t)b * Hkv + hkv];
      int use_bound = 2.0 * M * 1.4426950408889634 <= limit2;
      double base = M, smax = -INFINITY;
      for (int j = 0; j < Nkv; ++j) {
        if (!ora_allowed(mask_kind, block_map, Nq, Nkv, i, j)) {
          P[j] = -INFINITY;
          continue;
        }
        double acc = 0.0;
        for (int t = 0; t < d; ++t)
          acc += ld(q, dtype, q_off + t) * (ld(k, dtype, (((size_t)b * Nkv + j) * Hkv + hkv) * d + t) - m[t]);
        P[j] = scale * acc; /* S'_ij */
        if (P[j] > smax) smax = P[j];
      }
      if (!use_bound) base = smax; /* fallback: the exact max */
      double *orow = o + q_off;
      for (int t = 0; t < d; ++t) orow[t] = 0.0;
      bound_row[li] = use_bound;
      if (smax == -INFINITY) { /* no allowed key */
        lse[li] = -INFINITY;
        continue;
      }
      double l = 0.0;
      for (int j = 0; j < Nkv; ++j) {
        P[j] = P[j] == -INFINITY ? 0.0 : exp(P[j] - base);
        l += P[j];
      }
      for (int j = 0; j < Nkv; ++j) {
        if (P[j] == 0.0) continue;
        for (int t = 0; t < d; ++t) orow[t] += P[j] * ld(v, dtype, (((size_t)b * Nkv + j) * Hkv + hkv) * d + t);
      }
      for (int t = 0; t < d; ++t) orow[t] /= l;
      lse[li] = scale * qm + base + log(l);
    }
    free(P);
  }
  return 0;
}

/*
 * dQ for selected query rows only (the same definition as ora_attn_bwd,
 * restricted to one row: its whole S and P rows, dP_i = dO_i V^T,
 * D_i = sum_j P_ij dP_ij, dS_i = P_i * (dP_i - D_i), dQ_i = scale dS_i K).
 * rows: nrows triples (b, hq, i); dq: [nrows][d] fp64.
 */
int ora_attn_bwd_dq_rows(const void *q, const void *k, const void *v, const void *dout, int dtype, int B,
                         int Hq, int Hkv, int Nq, int Nkv, int d, double scale, int mask_kind,
                         const uint8_t *block_map, const int32_t *rows, int nrows, double *dq) {
  if (Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || Nq <= 0 || Nkv <= 0) return -1;
  if (mask_kind == ORA_MASK_BLOCK && !block_map) return -1;
  int G = Hq / Hkv, bad = 0;
#pragma omp parallel
  {
    double *S = (double *)malloc(sizeof(double) * (size_t)Nkv);
    double *dP = (double *)malloc(sizeof(double) * (size_t)Nkv);
#pragma omp for schedule(dynamic, 1)
    for (int r = 0; r < nrows; ++r) {
      int b = rows[3 * r], hq = rows[3 * r + 1], i = rows[3 * r + 2];
      double *out = dq + (size_t)r * d;
      for (int t = 0; t < d; ++t) out[t] = 0.0;
      if (b < 0 || b >= B || hq < 0 || hq >= Hq || i < 0 || i >= Nq) {
        bad = 1;
        continue;
      }
      int hkv = hq / G;
      size_t q_off = (((size_t)b * Nq + i) * Hq + hq) * d;
      size_t kv_base = ((size_t)b * Nkv * Hkv + hkv) * d, kv_stride = (size_t)Hkv * d;
      double m = -INFINITY;
      for (int j = 0; j < Nkv; ++j) {
        if (!ora_allowed(mask_kind, block_map, Nq, Nkv, i, j)) {
          S[j] = -INFINITY;
          continue;
        }
        double acc = 0.0;
        for (int t = 0; t < d; ++t) acc += ld(q, dtype, q_off + t) * ld(k, dtype, kv_base + (size_t)j * kv_stride + t);
        S[j] = acc * scale;
        if (S[j] > m) m = S[j];
      }
      if (m == -INFINITY) continue; /* no allowed key: zero gradient */
      double l = 0.0;
      for (int j = 0; j < Nkv; ++j) {
        S[j] = S[j] == -INFINITY ? 0.0 : exp(S[j] - m); /* P, unnormalised */
        l += S[j];
      }
      double D = 0.0;
      for (int j = 0; j < Nkv; ++j) {
        S[j] /= l;
        dP[j] = 0.0;
        if (S[j] == 0.0) continue;
        for (int t = 0; t < d; ++t)
          dP[j] += ld(dout, dtype, q_off + t) * ld(v, dtype, kv_base + (size_t)j * kv_stride + t);
        D += S[j] * dP[j];
      }
      for (int j = 0; j < Nkv; ++j) {
        if (S[j] == 0.0) continue;
        double ds = S[j] * (dP[j] - D);
        for (int t = 0; t < d; ++t) out[t] += scale * ds * ld(k, dtype, kv_base + (size_t)j * kv_stride + t);
      }
    }
    free(S);
    free(dP);
  }
  return bad ? -1 : 0;
}

/*
 * Threads for the parallel loops of this file: sets the count (for parallel
 * regions that the calling thread starts) when n > 0, and returns the count
 * the next such region will use.  Timing code reports this number.
 */
int ora_threads(int n) {
  if (n > 0) omp_set_num_threads(n);
  return omp_get_max_threads();
}
