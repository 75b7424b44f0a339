/*
 * NSA forward oracle: a plain, slow, fp64 CPU statement of what the
 * Native Sparse Attention forward pass computes.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the tests, the package smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header or constant with the
 * CUDA path.
 *
 * Sources (web pages on Native Sparse Attention):
 *  - "DeepSeek NSA ... config.toml" (qwbw.cn/news/106443), section 1: three
 *    parallel branches per query (compressed coarse attention, selected
 *    fine-grained blocks, sliding window) aggregated by a gate; section 3:
 *    the knobs compress_block_size, select_block_size, select_top_k,
 *    sliding_window, gate_type = learned, dtype = bfloat16.
 *  - "DeepSeek NSA in manufacturing" (chencunli.com), section "动态稀疏到底稀疏了什么":
 *    every block gets a learned compressed representation, the query attends
 *    coarsely to all compressed blocks and the highest-scoring blocks are
 *    selected; inside the selected blocks it attends token by token; the
 *    illustrative selector flattens each key block and applies one linear map.
 *  - "NSA vs MoBA" (gtnt.cn/news/122266), section 1: block compression,
 *    dynamic top-k selection, sliding-window local attention.
 *
 * Readings taken where the pages are silent (each one is listed in the design
 * notes of the repository):
 *  - compressor: one linear map per KV head, W[h] of shape [D, l*D], applied
 *    to the flattened block (element p*D + c is token p, channel c), no bias;
 *    separate maps for keys and values; the compressed tensor is stored in
 *    bf16 (round to nearest even), and steps 2-3 use that stored tensor;
 *  - a compressed block is visible to query t once its last token is <= t;
 *  - block score of selection block j (tokens j*l' .. j*l' + l' - 1) = sum
 *    over the query heads of the KV group of the compressed softmax
 *    probabilities of every visible compressed block (tokens i*d .. i*d + l - 1)
 *    that overlaps it; with l == d == l' that is the probability of block j
 *    itself, and the incomplete block holding t (which no visible compressed
 *    block overlaps) is a candidate with score 0; ties go to the lower block
 *    index; if there are at most n candidates, all are taken;
 *  - window = the w tokens ending at t (t included);
 *  - scale 1/sqrt(D) by default for all three branches;
 *  - an empty branch contributes 0;
 *  - gates are given per token, head and branch (order cmp, slc, win) and are
 *    applied as given.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
  int D;      /* head dim (d_k = d_v) */
  int Hq;     /* query heads */
  int Hkv;    /* key/value heads; G = Hq / Hkv query heads per group */
  int l;      /* compression block length */
  int d;      /* compression stride */
  int lsel;   /* selection block length l' */
  int n;      /* top-n selected blocks */
  int w;      /* sliding-window length */
  double scale;
} nsa_oracle_params;

/* ------------------------------------------------------------ bf16 <-> f64 */
double oracle_bf16_to_f64(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* Round an fp64 value to the nearest bf16 (ties to even), single rounding. */
uint16_t oracle_f64_to_bf16(double x) {
  if (x != x) return 0x7FC0;
  double ax = fabs(x);
  double r;
  if (ax == 0.0) {
    r = 0.0;
  } else if (ax < ldexp(1.0, -126)) {
    /* subnormal range: spacing 2^-133 */
    r = nearbyint(ax * ldexp(1.0, 133)) * ldexp(1.0, -133);
  } else {
    int e;
    double m = frexp(ax, &e);          /* ax = m * 2^e, m in [0.5, 1) */
    double q = nearbyint(m * 256.0);   /* 8 significant bits, ties to even */
    r = ldexp(q, e - 8);
    if (r >= ldexp(1.0, 128)) r = INFINITY;
  }
  float f = (float)r; /* exact: r is representable in bf16 */
  uint32_t u;
  memcpy(&u, &f, 4);
  uint16_t b = (uint16_t)(u >> 16);
  if (x < 0) b |= 0x8000;
  return b;
}

/* ------------------------------------------------------------ step 1 */
int oracle_num_cmp_blocks(const nsa_oracle_params* P, int T) {
  if (T < P->l) return 0;
  return (T - P->l) / P->d + 1;
}

/*
 * Compressed keys (or values) of one sequence.
 *   X   [T, Hkv, D] bf16 bits
 *   W   [Hkv, D, l*D] fp32
 *   out [C, Hkv, D] fp64 (unrounded) and bf16 (rounded), either may be NULL.
 */
void oracle_compress(const nsa_oracle_params* P, int T, const uint16_t* X, const float* W,
                     double* out_f64, uint16_t* out_bf16) {
  const int C = oracle_num_cmp_blocks(P, T);
  const int D = P->D, H = P->Hkv, L = P->l;
#pragma omp parallel for collapse(2) schedule(static)
  for (int i = 0; i < C; ++i) {
    for (int h = 0; h < H; ++h) {
      for (int c = 0; c < D; ++c) {
        const float* wrow = W + ((size_t)h * D + c) * (size_t)L * D;
        double acc = 0.0;
        for (int p = 0; p < L; ++p) {
          const uint16_t* x = X + ((size_t)(i * P->d + p) * H + h) * D;
          for (int cc = 0; cc < D; ++cc) acc += (double)wrow[p * D + cc] * oracle_bf16_to_f64(x[cc]);
        }
        size_t o = ((size_t)i * H + h) * D + c;
        if (out_f64) out_f64[o] = acc;
        if (out_bf16) out_bf16[o] = oracle_f64_to_bf16(acc);
      }
    }
  }
}

/* ------------------------------------------------------------ softmax attention */
/*
 * Softmax attention of one query head over an explicit list of key rows.
 *   q [D] fp64; keys/vals: bf16 rows of a [*, Hkv, D] tensor, head h.
 *   Writes o[D], the probabilities p[nk] (may be NULL) and returns the
 *   log-sum-exp of the scaled logits (-INFINITY when nk == 0, o = 0).
 */
static double attend(const nsa_oracle_params* P, const double* q, const uint16_t* keys,
                     const uint16_t* vals, int h, const int* rows, int nk, double* o, double* p,
                     double* scratch) {
  const int D = P->D, H = P->Hkv;
  for (int c = 0; c < D; ++c) o[c] = 0.0;
  if (nk == 0) return -INFINITY;
  double* z = scratch;
  double zmax = -INFINITY;
  for (int j = 0; j < nk; ++j) {
    const uint16_t* k = keys + ((size_t)rows[j] * H + h) * D;
    double s = 0.0;
    for (int c = 0; c < D; ++c) s += q[c] * oracle_bf16_to_f64(k[c]);
    z[j] = P->scale * s;
    if (z[j] > zmax) zmax = z[j];
  }
  double sum = 0.0;
  for (int j = 0; j < nk; ++j) sum += exp(z[j] - zmax);
  for (int j = 0; j < nk; ++j) {
    double pj = exp(z[j] - zmax) / sum;
    if (p) p[j] = pj;
    const uint16_t* v = vals + ((size_t)rows[j] * H + h) * D;
    for (int c = 0; c < D; ++c) o[c] += pj * oracle_bf16_to_f64(v[c]);
  }
  return zmax + log(sum);
}

/* ------------------------------------------------------------ step 4 */
/*
 * Top-n of S[0..ncand) under the order (score descending, index ascending).
 * Writes the chosen indices in ascending order to sel[0..n), -1 padded, and
 * returns the gap S_(n) - S_(n+1) between the n-th and (n+1)-th ranked
 * candidates (+INFINITY when every candidate is taken).
 */
double oracle_select(const double* S, int ncand, int n, int* sel) {
  int taken = 0;
  if (ncand <= n) {
    for (int j = 0; j < ncand; ++j) sel[taken++] = j;
    for (int j = taken; j < n; ++j) sel[j] = -1;
    return INFINITY;
  }
  /* selection by repeated maximum; ties keep the lower index */
  char* used = (char*)calloc((size_t)ncand, 1);
  double last = 0.0;
  for (int r = 0; r < n; ++r) {
    int best = -1;
    for (int j = 0; j < ncand; ++j) {
      if (used[j]) continue;
      if (best < 0 || S[j] > S[best]) best = j;
    }
    used[best] = 1;
    last = S[best];
  }
  int next = -1;
  for (int j = 0; j < ncand; ++j) {
    if (used[j]) continue;
    if (next < 0 || S[j] > S[next]) next = j;
  }
  for (int j = 0; j < ncand; ++j)
    if (used[j]) sel[taken++] = j;
  free(used);
  return last - S[next];
}

/* ------------------------------------------------------------ one query */
/*
 * The whole forward pass for one query token at (0-based) position t of a
 * sequence whose keys/values are k, v ([>= t+1, Hkv, D]) and whose stored
 * compressed keys/values are kc, vc ([>= C(t+1), Hkv, D], bf16).
 *   q      [Hq, D] bf16 bits, gates [Hq, 3] fp32 (cmp, slc, win)
 * Outputs (any may be NULL):
 *   o_cmp, o_slc, o_win, out  [Hq, D]
 *   lse    [Hq]               log-sum-exp of the compressed branch
 *   scores [Hkv, cmax]        selection-block scores (entries >= t / l' + 1 left 0)
 *   sel    [Hkv, n]           selected block indices (ascending, -1 pad)
 *   gap    [Hkv]              n-th minus (n+1)-th ranked score
 * Returns 0, or -1 on an invalid geometry (d > l, or a group size that does
 * not divide the heads).
 */
int oracle_nsa_query(const nsa_oracle_params* P, int t, const uint16_t* q, const uint16_t* k,
                     const uint16_t* v, const uint16_t* kc, const uint16_t* vc,
                     const float* gates, double* o_cmp, double* o_slc, double* o_win,
                     double* out, double* lse, double* scores, int cmax, int* sel,
                     double* gap) {
  const int D = P->D, Hq = P->Hq, Hkv = P->Hkv, G = Hq / Hkv;
  if (Hq % Hkv != 0 || P->d < 1 || P->l < P->d || P->lsel < 1) return -1;
  /* visible compressed blocks: i*d + l - 1 <= t */
  const int ncmp = (t + 1 >= P->l) ? (t + 1 - P->l) / P->d + 1 : 0;
  /* selection candidates: blocks j with j*l' <= t */
  const int ncand = t / P->lsel + 1;
  const int maxk = ncmp + P->n * P->lsel + P->w + 1;
  int* cmp_rows = (int*)malloc(sizeof(int) * (size_t)(ncmp + 1));
  int* sel_rows = (int*)malloc(sizeof(int) * (size_t)(P->n * P->lsel + 1));
  int* win_rows = (int*)malloc(sizeof(int) * (size_t)(P->w + 1));
  double* scratch = (double*)malloc(sizeof(double) * (size_t)maxk);
  double* prob = (double*)malloc(sizeof(double) * (size_t)(ncmp + 1));
  double* S = (double*)malloc(sizeof(double) * (size_t)ncand);
  int* chosen = (int*)malloc(sizeof(int) * (size_t)P->n);
  double* qh = (double*)malloc(sizeof(double) * (size_t)D);
  double* oc = (double*)malloc(sizeof(double) * (size_t)G * D);
  double* os = (double*)malloc(sizeof(double) * (size_t)D);
  double* ow = (double*)malloc(sizeof(double) * (size_t)D);
  for (int i = 0; i < ncmp; ++i) cmp_rows[i] = i;

  for (int g = 0; g < Hkv; ++g) {
    /* step 2 and 3: compressed branch of every head of the group, and the
       block scores summed over those heads */
    for (int j = 0; j < ncand; ++j) S[j] = 0.0;
    for (int hh = 0; hh < G; ++hh) {
      const int h = g * G + hh;
      for (int c = 0; c < D; ++c) qh[c] = oracle_bf16_to_f64(q[(size_t)h * D + c]);
      double L = attend(P, qh, kc, vc, g, cmp_rows, ncmp, oc + (size_t)hh * D, prob, scratch);
      if (lse) lse[h] = L;
      /* compressed block i covers tokens [i*d, i*d + l - 1]: its probability
         goes to every selection block [j*l', j*l' + l' - 1] it overlaps (all
         of them are candidates: i*d + l - 1 <= t) */
      for (int i = 0; i < ncmp; ++i) {
        const int j0 = (i * P->d) / P->lsel, j1 = (i * P->d + P->l - 1) / P->lsel;
        for (int j = j0; j <= j1; ++j) S[j] += prob[i];
      }
    }
    if (scores) {
      for (int j = 0; j < cmax; ++j) scores[(size_t)g * cmax + j] = (j < ncand) ? S[j] : 0.0;
    }
    /* step 4 */
    double gp = oracle_select(S, ncand, P->n, chosen);
    if (gap) gap[g] = gp;
    if (sel) memcpy(sel + (size_t)g * P->n, chosen, sizeof(int) * (size_t)P->n);
    /* step 5 keys: tokens u <= t inside the chosen blocks */
    int nsel = 0;
    for (int r = 0; r < P->n; ++r) {
      int j = chosen[r];
      if (j < 0) continue;
      for (int u = j * P->lsel; u < (j + 1) * P->lsel; ++u)
        if (u <= t) sel_rows[nsel++] = u;
    }
    /* step 6 keys: the w tokens ending at t */
    int nwin = 0;
    for (int u = (t - P->w + 1 > 0 ? t - P->w + 1 : 0); u <= t; ++u) win_rows[nwin++] = u;

    for (int hh = 0; hh < G; ++hh) {
      const int h = g * G + hh;
      for (int c = 0; c < D; ++c) qh[c] = oracle_bf16_to_f64(q[(size_t)h * D + c]);
      attend(P, qh, k, v, g, sel_rows, nsel, os, NULL, scratch);
      attend(P, qh, k, v, g, win_rows, nwin, ow, NULL, scratch);
      /* step 7 */
      const double g0 = gates[h * 3 + 0], g1 = gates[h * 3 + 1], g2 = gates[h * 3 + 2];
      for (int c = 0; c < D; ++c) {
        const size_t o = (size_t)h * D + c;
        const double ocv = oc[(size_t)hh * D + c];
        if (o_cmp) o_cmp[o] = ocv;
        if (o_slc) o_slc[o] = os[c];
        if (o_win) o_win[o] = ow[c];
        if (out) out[o] = g0 * ocv + g1 * os[c] + g2 * ow[c];
      }
    }
  }
  free(cmp_rows);
  free(sel_rows);
  free(win_rows);
  free(scratch);
  free(prob);
  free(S);
  free(chosen);
  free(qh);
  free(oc);
  free(os);
  free(ow);
  return 0;
}

/*
 * oracle_nsa_query for a list of rows of one packed sequence (prefill):
 *   q [T, Hq, D], k, v [T, Hkv, D], kc, vc [C, Hkv, D], gates [T, Hq, 3];
 *   output arrays are indexed by the position in `rows`.
 */
int oracle_nsa_rows(const nsa_oracle_params* P, int T, const uint16_t* q, const uint16_t* k,
                    const uint16_t* v, const uint16_t* kc, const uint16_t* vc,
                    const float* gates, const int* rows, int nrows, double* o_cmp,
                    double* o_slc, double* o_win, double* out, double* lse, double* scores,
                    int cmax, int* sel, double* gap) {
  const int D = P->D, Hq = P->Hq, Hkv = P->Hkv;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int r = 0; r < nrows; ++r) {
    const int t = rows[r];
    if (t < 0 || t >= T) {
      bad |= 1;
      continue;
    }
    const size_t hd = (size_t)Hq * D;
    int rc = oracle_nsa_query(
        P, t, q + (size_t)t * hd, k, v, kc, vc, gates + (size_t)t * Hq * 3,
        o_cmp ? o_cmp + r * hd : NULL, o_slc ? o_slc + r * hd : NULL,
        o_win ? o_win + r * hd : NULL, out ? out + r * hd : NULL,
        lse ? lse + (size_t)r * Hq : NULL, scores ? scores + (size_t)r * Hkv * cmax : NULL, cmax,
        sel ? sel + (size_t)r * Hkv * P->n : NULL, gap ? gap + (size_t)r * Hkv : NULL);
    bad |= (rc != 0);
  }
  return bad ? -1 : 0;
}

/*
 * Step 4 alone over a batch of score rows given in fp32 (used to replay the
 * selection on scores produced elsewhere): S [nrows, cstride], candidate
 * counts ncand [nrows]; entries at or beyond the complete-block count cmp_n
 * [nrows] are treated as 0 (the incomplete block).
 */
void oracle_select_f32(const float* S, int nrows, int cstride, const int* ncand,
                       const int* cmp_n, int n, int* sel, double* gap) {
#pragma omp parallel for schedule(static)
  for (int r = 0; r < nrows; ++r) {
    double* s = (double*)malloc(sizeof(double) * (size_t)(ncand[r] > 0 ? ncand[r] : 1));
    for (int j = 0; j < ncand[r]; ++j) s[j] = (j < cmp_n[r]) ? (double)S[(size_t)r * cstride + j] : 0.0;
    double gp = oracle_select(s, ncand[r], n, sel + (size_t)r * n);
    if (gap) gap[r] = gp;
    free(s);
  }
}

/* ------------------------------------------------------------ select-only block attention */
/*
 * Block attention with selection only, in the style of MoBA ("NSA vs MoBA"
 * page (gtnt.cn/news/122266), section 1: the sequence is cut into blocks and
 * a gate decides, per query, which key blocks it attends to, the way a
 * mixture of experts routes tokens).  The page gives no formula; the readings
 * (listed in the repository's design notes) are:
 *  - a block's routing key is the mean of its l' keys, stored in bf16 (round
 *    to nearest even);
 *  - the routing score of block j for query t and KV group g is the sum over
 *    the group's query heads of q . mean-key (the selection is shared by the
 *    group, as in the NSA branch);
 *  - the block holding t is always attended; the other n - 1 blocks are the
 *    best-scoring complete blocks before it (ties to the lower index; all of
 *    them when there are at most n - 1);
 *  - the output is one softmax attention of each head over the tokens u <= t
 *    of the chosen blocks (scale as in the NSA branches); no gate, no other
 *    branch.
 */

/* Mean keys of the complete blocks of one sequence: X [T, Hkv, D] bf16 bits,
 * out [T / l', Hkv, D] fp64 (unrounded) and bf16 (rounded); either may be NULL. */
void oracle_block_means(const nsa_oracle_params* P, int T, const uint16_t* X, double* out_f64,
                        uint16_t* out_bf16) {
  const int L = P->lsel, nb = T / L, D = P->D, H = P->Hkv;
  for (int j = 0; j < nb; ++j)
    for (int h = 0; h < H; ++h)
      for (int c = 0; c < D; ++c) {
        double acc = 0.0;
        for (int p = 0; p < L; ++p) acc += oracle_bf16_to_f64(X[((size_t)(j * L + p) * H + h) * D + c]);
        const double m = acc / L;
        const size_t o = ((size_t)j * H + h) * D + c;
        if (out_f64) out_f64[o] = m;
        if (out_bf16) out_bf16[o] = oracle_f64_to_bf16(m);
      }
}

/*
 * One query at position t of a sequence with keys/values k, v ([>= t+1, Hkv,
 * D] bf16) and stored mean keys kbar ([>= t / l', Hkv, D] bf16).
 *   q [Hq, D] bf16.  Outputs (any may be NULL):
 *   out    [Hq, D]      attention output
 *   scores [Hkv, cmax]  routing scores of the complete blocks before t's block
 *                       (entries >= t / l' left 0)
 *   sel    [Hkv, n]     attended blocks, ascending, -1 padded (t's block last)
 *   gap    [Hkv]        (n-1)-th minus n-th ranked routing score (+inf when
 *                       every candidate is taken)
 * Returns 0, or -1 on an invalid geometry.
 */
int oracle_block_select_query(const nsa_oracle_params* P, int t, const uint16_t* q,
                              const uint16_t* k, const uint16_t* v, const uint16_t* kbar,
                              double* out, double* scores, int cmax, int* sel, double* gap) {
  const int D = P->D, Hq = P->Hq, Hkv = P->Hkv, G = Hq / Hkv, L = P->lsel;
  if (Hq % Hkv != 0 || L < 1 || P->n < 1) return -1;
  const int cur = t / L;   /* the block holding t */
  const int npast = cur;   /* complete blocks before it: the candidates */
  const int m = P->n - 1;  /* blocks chosen by score */
  double* S = (double*)malloc(sizeof(double) * (size_t)(npast > 0 ? npast : 1));
  int* chosen = (int*)malloc(sizeof(int) * (size_t)(m > 0 ? m : 1));
  int* rows = (int*)malloc(sizeof(int) * (size_t)P->n * L);
  double* scratch = (double*)malloc(sizeof(double) * (size_t)P->n * L);
  double* qh = (double*)malloc(sizeof(double) * (size_t)D);
  double* o = (double*)malloc(sizeof(double) * (size_t)D);
  for (int g = 0; g < Hkv; ++g) {
    for (int j = 0; j < npast; ++j) {
      double s = 0.0;
      for (int hh = 0; hh < G; ++hh) {
        const int h = g * G + hh;
        for (int c = 0; c < D; ++c)
          s += oracle_bf16_to_f64(q[(size_t)h * D + c]) *
               oracle_bf16_to_f64(kbar[((size_t)j * Hkv + g) * D + c]);
      }
      S[j] = s;
    }
    if (scores)
      for (int j = 0; j < cmax; ++j) scores[(size_t)g * cmax + j] = (j < npast) ? S[j] : 0.0;
    double gp = INFINITY;
    int taken = 0;
    if (m > 0) {
      gp = oracle_select(S, npast, m, chosen);
      taken = npast < m ? npast : m;
    }
    if (gap) gap[g] = gp;
    if (sel) {
      for (int i = 0; i < P->n; ++i) sel[(size_t)g * P->n + i] = -1;
      for (int i = 0; i < taken; ++i) sel[(size_t)g * P->n + i] = chosen[i];
      sel[(size_t)g * P->n + taken] = cur;
    }
    int nk = 0;
    for (int i = 0; i < taken; ++i)
      for (int u = chosen[i] * L; u < (chosen[i] + 1) * L; ++u) rows[nk++] = u;
    for (int u = cur * L; u <= t; ++u) rows[nk++] = u;
    for (int hh = 0; hh < G; ++hh) {
      const int h = g * G + hh;
      for (int c = 0; c < D; ++c) qh[c] = oracle_bf16_to_f64(q[(size_t)h * D + c]);
      attend(P, qh, k, v, g, rows, nk, o, NULL, scratch);
      if (out)
        for (int c = 0; c < D; ++c) out[(size_t)h * D + c] = o[c];
    }
  }
  free(S);
  free(chosen);
  free(rows);
  free(scratch);
  free(qh);
  free(o);
  return 0;
}

/* oracle_block_select_query for a list of rows of one sequence:
 * q [T, Hq, D], k, v [T, Hkv, D], kbar [T / l', Hkv, D]; outputs are indexed
 * by the position in `rows`. */
int oracle_block_select_rows(const nsa_oracle_params* P, int T, const uint16_t* q,
                             const uint16_t* k, const uint16_t* v, const uint16_t* kbar,
                             const int* rows, int nrows, double* out, double* scores, int cmax,
                             int* sel, double* gap) {
  const int D = P->D, Hq = P->Hq, Hkv = P->Hkv;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int r = 0; r < nrows; ++r) {
    const int t = rows[r];
    if (t < 0 || t >= T) {
      bad |= 1;
      continue;
    }
    const size_t hd = (size_t)Hq * D;
    int rc = oracle_block_select_query(
        P, t, q + (size_t)t * hd, k, v, kbar, out ? out + r * hd : NULL,
        scores ? scores + (size_t)r * Hkv * cmax : NULL, cmax,
        sel ? sel + (size_t)r * Hkv * P->n : NULL, gap ? gap + (size_t)r * Hkv : NULL);
    bad |= (rc != 0);
  }
  return bad ? -1 : 0;
}

/* ------------------------------------------------------------ token-level selection (DSA style) */
/*
 * Sparse attention with a token-level top-k chosen by a light indexer, in the
 * style of DSA ("DeepSeek V3.2-Exp sparse attention" page
 * (bjdmk.com.cn/news/5181035), sections 1 and 3: an indexer with 8 or 16
 * heads and a ReLU activation scores every earlier token, the top_k = 2048
 * tokens per query take part in the main attention).  The page gives no
 * formula; the readings (listed in the repository's design notes) are:
 *  - index score I[t, s] = sum over indexer heads j of w[t, j] *
 *    ReLU(qi[t, j] . ki[s]) for s <= t (qi [T, Hi, Di], ki [T, Di] bf16, the
 *    per-token head weights w [T, Hi] fp32; the page's fp8 indexer is a
 *    precision choice this statement does not make);
 *  - the top_k tokens by I (ties to the lower index; all of them when there
 *    are at most top_k) are shared by every query head;
 *  - each head attends (one softmax, scale as in the NSA branches) to the
 *    keys and values of its KV group at the chosen tokens.
 */
typedef struct {
  int Hi;   /* indexer heads */
  int Di;   /* indexer head dim */
  int top_k;
} dsa_oracle_params;

/* One query at position t: q [Hq, D], k, v [>= t+1, Hkv, D] bf16 (main
 * attention), qi [Hi, Di] bf16 and w [Hi] fp32 of query t, ki [>= t+1, Di]
 * bf16.  Outputs (any may be NULL): out [Hq, D], index [t + 1] (I[t, s]),
 * sel [top_k] (ascending, -1 padded), gap (top_k-th minus (top_k+1)-th score). */
int oracle_dsa_query(const nsa_oracle_params* P, const dsa_oracle_params* X, int t,
                     const uint16_t* q, const uint16_t* k, const uint16_t* v,
                     const uint16_t* qi, const float* w, const uint16_t* ki, double* out,
                     double* index, int* sel, double* gap) {
  const int D = P->D, Hq = P->Hq, Hkv = P->Hkv, G = Hq / Hkv;
  if (Hq % Hkv != 0 || X->top_k < 1 || X->Hi < 1 || X->Di < 1) return -1;
  const int ncand = t + 1;
  double* I = (double*)malloc(sizeof(double) * (size_t)ncand);
  int* chosen = (int*)malloc(sizeof(int) * (size_t)X->top_k);
  int* rows = (int*)malloc(sizeof(int) * (size_t)X->top_k);
  double* scratch = (double*)malloc(sizeof(double) * (size_t)X->top_k);
  double* qh = (double*)malloc(sizeof(double) * (size_t)D);
  double* o = (double*)malloc(sizeof(double) * (size_t)D);
  for (int s = 0; s < ncand; ++s) {
    double acc = 0.0;
    for (int j = 0; j < X->Hi; ++j) {
      double dot = 0.0;
      for (int c = 0; c < X->Di; ++c)
        dot += oracle_bf16_to_f64(qi[(size_t)j * X->Di + c]) *
               oracle_bf16_to_f64(ki[(size_t)s * X->Di + c]);
      acc += (double)w[j] * (dot > 0.0 ? dot : 0.0);
    }
    I[s] = acc;
  }
  if (index)
    for (int s = 0; s < ncand; ++s) index[s] = I[s];
  const double gp = oracle_select(I, ncand, X->top_k, chosen);
  if (gap) *gap = gp;
  if (sel) memcpy(sel, chosen, sizeof(int) * (size_t)X->top_k);
  int nk = 0;
  for (int i = 0; i < X->top_k; ++i)
    if (chosen[i] >= 0) rows[nk++] = chosen[i];
  for (int g = 0; g < Hkv; ++g)
    for (int hh = 0; hh < G; ++hh) {
      const int h = g * G + hh;
      for (int c = 0; c < D; ++c) qh[c] = oracle_bf16_to_f64(q[(size_t)h * D + c]);
      attend(P, qh, k, v, g, rows, nk, o, NULL, scratch);
      if (out)
        for (int c = 0; c < D; ++c) out[(size_t)h * D + c] = o[c];
    }
  free(I);
  free(chosen);
  free(rows);
  free(scratch);
  free(qh);
  free(o);
  return 0;
}

/* oracle_dsa_query for a list of rows of one sequence: q [T, Hq, D], k, v
 * [T, Hkv, D], qi [T, Hi, Di], w [T, Hi], ki [T, Di]; outputs by position in
 * `rows` (index rows of length T). */
int oracle_dsa_rows(const nsa_oracle_params* P, const dsa_oracle_params* X, int T,
                    const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* qi,
                    const float* w, const uint16_t* ki, const int* rows, int nrows, double* out,
                    double* index, int* sel, double* gap) {
  const int D = P->D, Hq = P->Hq;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int r = 0; r < nrows; ++r) {
    const int t = rows[r];
    if (t < 0 || t >= T) {
      bad |= 1;
      continue;
    }
    const size_t hd = (size_t)Hq * D;
    int rc = oracle_dsa_query(P, X, t, q + (size_t)t * hd, k, v, qi + (size_t)t * X->Hi * X->Di,
                              w + (size_t)t * X->Hi, ki, out ? out + r * hd : NULL,
                              index ? index + (size_t)r * T : NULL,
                              sel ? sel + (size_t)r * X->top_k : NULL, gap ? gap + r : NULL);
    bad |= (rc != 0);
  }
  return bad ? -1 : 0;
}

/* ------------------------------------------------------------------------
 * Backward of the forward above with the block selection held fixed, in
 * fp64 on fp64 inputs: the same definition as oracle/backward.py, whose
 * header states the readings (fixed selection, the compressed tensor's
 * rounding taken as the identity, an empty branch passes no gradient).
 * OpenMP over query rows; the key-side gradients accumulate atomically.
 * ------------------------------------------------------------------------ */

/* One branch of query row q (D values) over `m` key rows keys[] of K and V
 * (row r at K + r * rs): forward softmax(scale q . k) and O = sum p v into
 * o_out; with upstream gradient dob: dq += scale sum dz k, dK[r] += scale dz
 * q, dV[r] += p dob, where dz = p (v . dob - sum p (v . dob)). */
static void bw_branch(int D, double scale, const double* qv, const double* K, const double* V,
                      size_t rs, const int* keys, int m, const double* dob, double* dq,
                      double* dK, double* dV, double* o_out, double* p, double* dp, int shared) {
  for (int c = 0; c < D; ++c) o_out[c] = 0.0;
  if (m == 0) return;
  double zmax = -INFINITY;
  for (int a = 0; a < m; ++a) {
    const double* kr = K + (size_t)keys[a] * rs;
    double z = 0.0;
    for (int c = 0; c < D; ++c) z += qv[c] * kr[c];
    p[a] = scale * z;
    if (p[a] > zmax) zmax = p[a];
  }
  double sum = 0.0;
  for (int a = 0; a < m; ++a) {
    p[a] = exp(p[a] - zmax);
    sum += p[a];
  }
  double dsum = 0.0;
  for (int a = 0; a < m; ++a) {
    p[a] /= sum;
    const double* vr = V + (size_t)keys[a] * rs;
    double x = 0.0;
    for (int c = 0; c < D; ++c) {
      o_out[c] += p[a] * vr[c];
      x += vr[c] * dob[c];
    }
    dp[a] = x;
    dsum += p[a] * x;
  }
  for (int a = 0; a < m; ++a) {
    const double dz = p[a] * (dp[a] - dsum);
    const double* kr = K + (size_t)keys[a] * rs;
    double* dkr = dK + (size_t)keys[a] * rs;
    double* dvr = dV + (size_t)keys[a] * rs;
    for (int c = 0; c < D; ++c) {
      dq[c] += scale * dz * kr[c];
      if (shared) {
#pragma omp atomic
        dkr[c] += scale * dz * qv[c];
#pragma omp atomic
        dvr[c] += p[a] * dob[c];
      } else {
        dkr[c] += scale * dz * qv[c];
        dvr[c] += p[a] * dob[c];
      }
    }
  }
}

static int cmp_int(const void* a, const void* b) {
  const int x = *(const int*)a, y = *(const int*)b;
  return (x > y) - (x < y);
}

/* Gradients of sum(dout * out) for one sequence of T tokens.  q [T,Hq,D],
 * k/v [T,Hkv,D], gates [T,Hq,3], w_k/w_v [Hkv,D,l*D], sel [T,Hkv,n] (-1
 * padded), dout [T,Hq,D]; kc_in/vc_in [C,Hkv,D] the compressed tensors to
 * attend to, or NULL for step 1 in fp64.  rows: the query rows whose terms
 * are summed (NULL: all T).  Outputs (overwritten): dq, dk, dv, dgates,
 * dw_k, dw_v, dkc, dvc.  Returns 0, or -1 for a geometry it cannot hold. */
int oracle_backward(const nsa_oracle_params* P, int T, const double* q, const double* k,
                    const double* v, const double* gates, const double* wk, const double* wv,
                    const int* sel, const double* dout, const double* kc_in,
                    const double* vc_in, const int* rows, int nrows, double* dq, double* dk,
                    double* dv, double* dgates, double* dwk, double* dwv, double* dkc,
                    double* dvc) {
  const int D = P->D, Hq = P->Hq, Hkv = P->Hkv, l = P->l, d = P->d, ls = P->lsel, n = P->n;
  if (Hkv <= 0 || Hq % Hkv != 0 || T < 0) return -1;
  const int G = Hq / Hkv, C = oracle_num_cmp_blocks(P, T), LD = l * D;
  const size_t rs = (size_t)Hkv * D;
  const double scale = P->scale;
  double* kc = (double*)malloc(sizeof(double) * ((size_t)C * rs + 1));
  double* vc = (double*)malloc(sizeof(double) * ((size_t)C * rs + 1));
  if (!kc || !vc) {
    free(kc);
    free(vc);
    return -1;
  }
  for (int i = 0; i < C; ++i)
    for (int g = 0; g < Hkv; ++g)
      for (int r = 0; r < D; ++r) {
        double sk = 0.0, sv = 0.0;
        for (int e = 0; e < LD; ++e) {
          const size_t x = ((size_t)(i * d + e / D) * Hkv + g) * D + e % D;
          sk += wk[((size_t)g * D + r) * LD + e] * k[x];
          sv += wv[((size_t)g * D + r) * LD + e] * v[x];
        }
        kc[((size_t)i * Hkv + g) * D + r] = kc_in ? kc_in[((size_t)i * Hkv + g) * D + r] : sk;
        vc[((size_t)i * Hkv + g) * D + r] = vc_in ? vc_in[((size_t)i * Hkv + g) * D + r] : sv;
      }
  memset(dq, 0, sizeof(double) * (size_t)T * Hq * D);
  memset(dk, 0, sizeof(double) * (size_t)T * rs);
  memset(dv, 0, sizeof(double) * (size_t)T * rs);
  memset(dgates, 0, sizeof(double) * (size_t)T * Hq * 3);
  memset(dwk, 0, sizeof(double) * (size_t)Hkv * D * LD);
  memset(dwv, 0, sizeof(double) * (size_t)Hkv * D * LD);
  memset(dkc, 0, sizeof(double) * (size_t)C * rs);
  memset(dvc, 0, sizeof(double) * (size_t)C * rs);
  const int R = rows ? nrows : T;
  int fail = 0;
  /* key-side gradients: each thread sums into its own copy, merged at the
   * end, when the copies fit in 2 GB; otherwise atomically into the result */
  const size_t kv_elems = ((size_t)T + C) * rs;
#pragma omp parallel
  {
    const int nthr = omp_get_num_threads();
    const int priv = (double)nthr * 2.0 * (double)kv_elems * sizeof(double) <= 2e9;
    double* pk = priv ? (double*)calloc(2 * kv_elems + 1, sizeof(double)) : NULL;
    const int use_priv = pk != NULL;
    double* tdk = use_priv ? pk : dk;
    double* tdv = use_priv ? pk + (size_t)T * rs : dv;
    double* tdkc = use_priv ? pk + 2 * (size_t)T * rs : dkc;
    double* tdvc = use_priv ? pk + 2 * (size_t)T * rs + (size_t)C * rs : dvc;
    const int cap = T + C + 1;
    int* ck = (int*)malloc(sizeof(int) * cap);
    int* sk = (int*)malloc(sizeof(int) * cap);
    int* wkeys = (int*)malloc(sizeof(int) * cap);
    double* p = (double*)malloc(sizeof(double) * cap);
    double* dp = (double*)malloc(sizeof(double) * cap);
    double* o = (double*)malloc(sizeof(double) * D);
    double* dob = (double*)malloc(sizeof(double) * D);
    const int ok = ck && sk && wkeys && p && dp && o && dob;
    if (!ok) {
#pragma omp atomic write
      fail = 1;
    }
    /* every thread takes part in the loop; one without scratch skips its rows */
#pragma omp for schedule(dynamic, 4)
    for (int rr = 0; rr < R; ++rr) {
      if (ok) {
        const int t = rows ? rows[rr] : rr;
        for (int h = 0; h < Hq; ++h) {
          const int g = h / G;
          int mc = 0, msl = 0, mw = 0;
          for (int i = 0; i < C; ++i)
            if (i * d + l - 1 <= t) ck[mc++] = i;
          for (int s = 0; s < n; ++s) {
            const int j = sel[((size_t)t * Hkv + g) * n + s];
            if (j < 0) continue;
            for (int u = j * ls; u < j * ls + ls && u <= t; ++u) sk[msl++] = u;
          }
          qsort(sk, msl, sizeof(int), cmp_int);
          for (int u = (t - P->w + 1 > 0 ? t - P->w + 1 : 0); u <= t; ++u) wkeys[mw++] = u;
          const double* qv = q + ((size_t)t * Hq + h) * D;
          const double* dov = dout + ((size_t)t * Hq + h) * D;
          double* dqv = dq + ((size_t)t * Hq + h) * D;
          const double* gt = gates + ((size_t)t * Hq + h) * 3;
          double* dg = dgates + ((size_t)t * Hq + h) * 3;
          for (int b = 0; b < 3; ++b) {
            for (int c = 0; c < D; ++c) dob[c] = gt[b] * dov[c];
            if (b == 0)
              bw_branch(D, scale, qv, kc + (size_t)g * D, vc + (size_t)g * D, rs, ck, mc, dob, dqv,
                        tdkc + (size_t)g * D, tdvc + (size_t)g * D, o, p, dp, !use_priv);
            else
              bw_branch(D, scale, qv, k + (size_t)g * D, v + (size_t)g * D, rs, b == 1 ? sk : wkeys,
                        b == 1 ? msl : mw, dob, dqv, tdk + (size_t)g * D, tdv + (size_t)g * D, o, p,
                        dp, !use_priv);
            double x = 0.0;
            for (int c = 0; c < D; ++c) x += dov[c] * o[c];
            dg[b] = x;
          }
        }
      }
    }
    if (use_priv) {
      /* atomic: a thread without a private copy may still be adding */
      for (size_t e = 0; e < (size_t)T * rs; ++e) {
#pragma omp atomic
        dk[e] += tdk[e];
#pragma omp atomic
        dv[e] += tdv[e];
      }
      for (size_t e = 0; e < (size_t)C * rs; ++e) {
#pragma omp atomic
        dkc[e] += tdkc[e];
#pragma omp atomic
        dvc[e] += tdvc[e];
      }
    }
    free(pk);
    free(ck);
    free(sk);
    free(wkeys);
    free(p);
    free(dp);
    free(o);
    free(dob);
  }
  /* step 1: K~[i, g] = W[g] vec(x[i d : i d + l, g]) */
  for (int i = 0; i < C && !fail; ++i)
    for (int g = 0; g < Hkv; ++g)
      for (int r = 0; r < D; ++r) {
        const double gk = dkc[((size_t)i * Hkv + g) * D + r];
        const double gv = dvc[((size_t)i * Hkv + g) * D + r];
        for (int e = 0; e < LD; ++e) {
          const size_t x = ((size_t)(i * d + e / D) * Hkv + g) * D + e % D;
          dwk[((size_t)g * D + r) * LD + e] += gk * k[x];
          dwv[((size_t)g * D + r) * LD + e] += gv * v[x];
          dk[x] += wk[((size_t)g * D + r) * LD + e] * gk;
          dv[x] += wv[((size_t)g * D + r) * LD + e] * gv;
        }
      }
  free(kc);
  free(vc);
  return fail ? -1 : 0;
}
