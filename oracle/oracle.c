/*
 * oracle.c -- plain fp64 CPU oracle for the NSA and MoBA forward pass.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark load this file. The CUDA library shares no code, header,
 * table or helper with it, and neither side includes the other.
 *
 * Sources (the pages print no equation; each step is the plainest reading of
 * their prose, with the constants of the workload statement):
 *   [EP94]     Zhang Xiaojun podcast EP94 notes (idealstate.vel.life), sections
 *              五 (NSA three-branch architecture), 六 (hardware-aligned design
 *              and GQA group sharing), 九/十 (MoBA), 十六 (parameter table).
 *   [LCH]      lchairun.cn article on DeepSeek NSA: the "three squads"
 *              paragraphs (compression, selection, window) and the gate.
 *   [LT103]    LateTalk ep.103 podcast transcript (latetalk.podhood.com): the
 *              512-token sliding window and MoBA's fixed own block.
 *
 * Everything is fp64. Inputs arrive as fp64 copies of the exact input values
 * (bf16 or fp32 converted without loss). Loops follow the steps in the order
 * the pages give them; there is no blocking, fusion or reordering.
 *
 * Parity status of each function is recorded next to it (what pins it).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Configuration                                                            */
/* ------------------------------------------------------------------------ */

typedef struct {
  int B, T, Hq, Hkv, d;        /* batch, tokens, query heads, kv heads, head dim */
  int cmp_block, cmp_stride;   /* l, s: compression block length and stride      */
  int sel_block, top_n;        /* selection block size and n (block 0 counted)   */
  int window;                  /* sliding window w                               */
  double scale;                /* softmax scale sigma                            */
  int gate_mode;               /* 0: g = sigmoid(q . Wg); 1: fixed gates         */
  double fixed_gates[3];       /* (cmp, slc, win) when gate_mode == 1            */
  int store;                   /* rounding of stored compressed K/V:
                                  0 none (keep fp64), 1 fp32, 2 bf16             */
  int score_mode;              /* block scores for the selection:
                                  0 compressed-branch mass, unweighted sum over
                                  overlapping compressed blocks; 1 the same
                                  weighted by overlap / l; 2 the Quest-style
                                  block bound (see step 3')                      */
  double top_p;                /* 0: top-n; in (0, 1]: adaptive selection that
                                  stops once the selected blocks hold top_p of
                                  the total score (at most n blocks)            */
} oracle_nsa_cfg;

typedef struct {
  int B, T, Hq, Hkv, d;
  int block;                   /* MoBA block size m                              */
  int top_k;                   /* k, the own block counted                       */
  double scale;                /* softmax scale sigma                            */
} oracle_moba_cfg;

/* ------------------------------------------------------------------------ */
/* Storage rounding                                                         */
/* ------------------------------------------------------------------------ */

/* Round x to the nearest value with p significant bits (ties to even), the
 * smallest quantum being 2^qexp (subnormal range), overflowing to infinity
 * above maxfinite. This is the IEEE-754 round-to-nearest-even definition for
 * a binary format, evaluated once from the exact fp64 value. */
static double round_to_format(double x, int p, int qexp, double maxfinite) {
  if (x == 0.0 || !isfinite(x)) return x;
  int e;
  frexp(x, &e);                    /* |x| = m 2^e, 0.5 <= m < 1 */
  int ulp_exp = e - p;             /* spacing of p-bit values in this binade */
  if (ulp_exp < qexp) ulp_exp = qexp;
  double r = ldexp(nearbyint(ldexp(x, -ulp_exp)), ulp_exp); /* ties-to-even */
  if (fabs(r) > maxfinite) return copysign(INFINITY, x);
  return r;
}

/* store: 0 none, 1 IEEE binary32, 2 bfloat16 (8 significant bits, binary32
 * exponent range). */
double oracle_round_store(int store, double x) {
  if (store == 1)
    return round_to_format(x, 24, -149, ldexp(2.0 - ldexp(1.0, -23), 127));
  if (store == 2)
    return round_to_format(x, 8, -133, ldexp(2.0 - ldexp(1.0, -7), 127));
  return x;
}

void oracle_round_store_array(int store, const double* x, double* y, long n) {
  for (long i = 0; i < n; ++i) y[i] = oracle_round_store(store, x[i]);
}

/* ------------------------------------------------------------------------ */
/* Step 1: token compression                                                */
/* [EP94 §五 branch one; LCH compression squad]: keys and values are cut    */
/* into consecutive blocks and each block becomes one representative. The  */
/* learnable map is a weight vector w of length l shared by K and V, applied */
/* to blocks of l tokens taken every s tokens.                               */
/* ------------------------------------------------------------------------ */

int oracle_num_cmp(int T, int l, int s) {
  if (T < l) return 0;
  return (T - l) / s + 1;
}

/* k, v: [B, T, Hkv, d]; w: [l]; kc, vc: [B, Nc, Hkv, d]. */
void oracle_compress(const oracle_nsa_cfg* c, const double* k, const double* v,
                     const double* w, double* kc, double* vc) {
  const int l = c->cmp_block, s = c->cmp_stride;
  const int Nc = oracle_num_cmp(c->T, l, s);
  const long tok = (long)c->Hkv * c->d;
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < c->B; ++b)
    for (int i = 0; i < Nc; ++i)
      for (int g = 0; g < c->Hkv; ++g)
        for (int e = 0; e < c->d; ++e) {
          double sk = 0.0, sv = 0.0;
          for (int j = 0; j < l; ++j) {
            long src = ((long)b * c->T + (long)i * s + j) * tok + (long)g * c->d + e;
            sk += w[j] * k[src];
            sv += w[j] * v[src];
          }
          long dst = ((long)b * Nc + i) * tok + (long)g * c->d + e;
          kc[dst] = oracle_round_store(c->store, sk);
          vc[dst] = oracle_round_store(c->store, sv);
        }
}

/* ------------------------------------------------------------------------ */
/* Softmax attention of one query over an explicit key list.                */
/* Scaled dot product, softmax normalisation, weighted sum of values        */
/* [EP94 §二 self-attention]. Returns the log-sum-exp of the scaled logits; */
/* with no keys the output is zero and the lse is -inf.                     */
/* ------------------------------------------------------------------------ */

static double attend(const double* q, const double* keys_base, const double* vals_base,
                     long row_stride, const int* key_rows, int nkeys, int d,
                     double scale, double* out, double* p /* [nkeys] scratch or NULL */) {
  for (int e = 0; e < d; ++e) out[e] = 0.0;
  if (nkeys == 0) return -INFINITY;
  double* z = p ? p : (double*)malloc(sizeof(double) * nkeys);
  double m = -INFINITY;
  for (int a = 0; a < nkeys; ++a) {
    const double* kr = keys_base + (long)key_rows[a] * row_stride;
    double dot = 0.0;
    for (int e = 0; e < d; ++e) dot += q[e] * kr[e];
    z[a] = scale * dot;
    if (z[a] > m) m = z[a];
  }
  double sum = 0.0;
  for (int a = 0; a < nkeys; ++a) {
    z[a] = exp(z[a] - m);
    sum += z[a];
  }
  for (int a = 0; a < nkeys; ++a) {
    z[a] /= sum;                      /* normalised probability */
    const double* vr = vals_base + (long)key_rows[a] * row_stride;
    for (int e = 0; e < d; ++e) out[e] += z[a] * vr[e];
  }
  if (!p) free(z);
  return m + log(sum);
}

/* Order for top selection: higher score first; equal scores go to the lower
 * block index (the tie rule of the workload statement). */
static int better(double sa, int ja, double sb, int jb) {
  if (sa > sb) return 1;
  if (sa < sb) return 0;
  return ja < jb;
}

static int cmp_int(const void* a, const void* b) {
  int x = *(const int*)a, y = *(const int*)b;
  return (x > y) - (x < y);
}

/* ------------------------------------------------------------------------ */
/* NSA forward for a list of query rows.                                     */
/*                                                                           */
/* rows_b/rows_t: batch index and position t of each row; q_rows: [nrows,Hq,d] */
/* k, v: [B, T, Hkv, d]; kc, vc: [B, Nc, Hkv, d] with Nc = oracle_num_cmp(T); */
/* wg: [d, 3] (gate weights, row-major; unused for fixed gates).             */
/* forced_sel: [nrows, Hkv, n] block list to use instead of the oracle's own */
/* selection (entries < 0 ignored), or NULL.                                 */
/* Outputs (each may be NULL): out/o_cmp/o_slc/o_win [nrows, Hq, d];         */
/* gates [nrows, Hq, 3]; lse_cmp [nrows, Hq]; scores [nrows, Hkv, nblk_max]  */
/* with nblk_max = ceil(T / sel_block) (-inf past the row's last candidate); */
/* sel [nrows, Hkv, n] ascending, -1 padded.                                 */
/* ------------------------------------------------------------------------ */

void oracle_nsa_rows(const oracle_nsa_cfg* c, int nrows, const int* rows_b, const int* rows_t,
                     const double* q_rows, const double* k, const double* v,
                     const double* kc, const double* vc, const double* wg,
                     const int* forced_sel, double* out, double* o_cmp, double* o_slc,
                     double* o_win, double* gates, double* lse_cmp, double* scores, int* sel) {
  const int d = c->d, Hq = c->Hq, Hkv = c->Hkv, G = Hq / Hkv;
  const int l = c->cmp_block, s = c->cmp_stride, bs = c->sel_block, n = c->top_n;
  const int Nc = oracle_num_cmp(c->T, l, s);
  const int nblk_max = (c->T + bs - 1) / bs;
  const long tok = (long)Hkv * d;

#pragma omp parallel for collapse(2) schedule(dynamic)
  for (int r = 0; r < nrows; ++r)
    for (int g = 0; g < Hkv; ++g) {
      const int b = rows_b[r], t = rows_t[r];
      const double* kb = k + (long)b * c->T * tok + (long)g * d;
      const double* vb = v + (long)b * c->T * tok + (long)g * d;
      const double* kcb = kc + (long)b * Nc * tok + (long)g * d;
      const double* vcb = vc + (long)b * Nc * tok + (long)g * d;

      /* Compressed block i covers tokens [i s, i s + l - 1]; it is visible to
       * the query at t when its last token is not in the future. */
      int nvis = 0;
      while (nvis < Nc && (long)nvis * s + l - 1 <= t) ++nvis;
      const int ncand = t / bs + 1;            /* selection blocks 0 .. t/bs */

      int* idx_all = (int*)malloc(sizeof(int) * (nvis > 0 ? nvis : 1));
      for (int i = 0; i < nvis; ++i) idx_all[i] = i;
      double* p = (double*)malloc(sizeof(double) * (nvis > 0 ? nvis : 1));
      double* blk = (double*)calloc(ncand, sizeof(double));
      double* oslc_h = (double*)malloc(sizeof(double) * d);
      double* owin_h = (double*)malloc(sizeof(double) * d);
      double** ocmp_g = (double**)malloc(sizeof(double*) * G);

      /* Step 2 [EP94 §五 branch one]: each query head attends to all visible
       * compressed representatives. Step 3 [EP94 §五 branch two, §六]: the
       * block importance of selection block j is the compressed-branch
       * probability mass on the compressed blocks overlapping j, summed over
       * the query heads of the GQA group so the group shares one choice. */
      for (int hh = 0; hh < G; ++hh) {
        const int h = g * G + hh;
        const double* qh = q_rows + ((long)r * Hq + h) * d;
        ocmp_g[hh] = (double*)malloc(sizeof(double) * d);
        double lse = attend(qh, kcb, vcb, tok, idx_all, nvis, d, c->scale, ocmp_g[hh], p);
        if (lse_cmp) lse_cmp[(long)r * Hq + h] = lse;
        for (int i = 0; i < nvis; ++i) {
          const long first = (long)i * s, last = (long)i * s + l - 1;
          for (long j = first / bs; j <= last / bs && j < ncand; ++j) {
            double wgt = 1.0;
            if (c->score_mode == 1) {
              long lo = first > j * bs ? first : j * bs;
              long hi = last < j * bs + bs - 1 ? last : j * bs + bs - 1;
              wgt = (double)(hi - lo + 1) / l;
            }
            blk[j] += wgt * p[i];
          }
        }
      }
      /* Step 3' (score_mode 2) [EP94 §八: the Quest-style heuristic block
       * score of the selection ablation; the pages print no formula, so the
       * one of the Quest paper they cite is used]: per selection block j the
       * element-wise minimum and maximum of its keys up to t, and the bound
       * sum_e max(q_e kmin_e, q_e kmax_e) >= max_u q . k_u over the block,
       * summed over the query heads of the GQA group. It replaces the
       * compressed-branch scores; the compressed branch itself is unchanged. */
      if (c->score_mode == 2) {
        double* kmin = (double*)malloc(sizeof(double) * d);
        double* kmax = (double*)malloc(sizeof(double) * d);
        for (int j = 0; j < ncand; ++j) {
          const int u1 = (j + 1) * bs - 1 < t ? (j + 1) * bs - 1 : t;
          for (int e = 0; e < d; ++e) {
            kmin[e] = INFINITY;
            kmax[e] = -INFINITY;
          }
          for (int u = j * bs; u <= u1; ++u)
            for (int e = 0; e < d; ++e) {
              const double x = kb[(long)u * tok + e];
              if (x < kmin[e]) kmin[e] = x;
              if (x > kmax[e]) kmax[e] = x;
            }
          double sc = 0.0;
          for (int hh = 0; hh < G; ++hh) {
            const double* qh = q_rows + ((long)r * Hq + g * G + hh) * d;
            for (int e = 0; e < d; ++e) {
              const double lo = qh[e] * kmin[e], hi = qh[e] * kmax[e];
              sc += lo > hi ? lo : hi;
            }
          }
          blk[j] = sc;
        }
        free(kmin);
        free(kmax);
      }
      if (scores) {
        double* srow = scores + ((long)r * Hkv + g) * nblk_max;
        for (int j = 0; j < nblk_max; ++j) srow[j] = j < ncand ? blk[j] : -INFINITY;
      }

      /* Step 4 [EP94 §五 branch two, §十六; LCH selection squad]: the top-n
       * blocks by score, block 0 always kept and counted in n. With n or fewer
       * candidates all of them are kept.
       * Adaptive variant (top_p > 0) [LCH, adaptive sparsification: choose
       * from the most important block on until the chosen scores add up to
       * p times the total]: block 0 first, then the others by score (higher
       * first, ties to the lower index), stopping at the first prefix whose
       * score sum reaches top_p times the sum over all candidates, or at n
       * blocks. */
      int* S = (int*)malloc(sizeof(int) * (n > 0 ? n : 1));
      int ns = 0;
      if (forced_sel) {
        const int* fr = forced_sel + ((long)r * Hkv + g) * n;
        for (int a = 0; a < n; ++a)
          if (fr[a] >= 0) S[ns++] = fr[a];
      } else if (c->top_p > 0.0) {
        double total = 0.0;
        for (int j = 0; j < ncand; ++j) total += blk[j];
        const double goal = c->top_p * total;
        char* taken = (char*)calloc(ncand > 0 ? ncand : 1, 1);
        S[ns++] = 0;
        taken[0] = 1;
        double cum = blk[0];
        while (ns < n && ns < ncand && cum < goal) {
          int best = -1;
          for (int j = 1; j < ncand; ++j)
            if (!taken[j] && (best < 0 || better(blk[j], j, blk[best], best))) best = j;
          taken[best] = 1;
          S[ns++] = best;
          cum += blk[best];
        }
        free(taken);
      } else if (ncand <= n) {
        for (int j = 0; j < ncand; ++j) S[ns++] = j;
      } else {
        char* taken = (char*)calloc(ncand, 1);
        S[ns++] = 0;
        taken[0] = 1;
        while (ns < n) {
          int best = -1;
          for (int j = 1; j < ncand; ++j)
            if (!taken[j] && (best < 0 || better(blk[j], j, blk[best], best))) best = j;
          taken[best] = 1;
          S[ns++] = best;
        }
        free(taken);
      }
      qsort(S, ns, sizeof(int), cmp_int);
      if (sel) {
        int* srow = sel + ((long)r * Hkv + g) * n;
        for (int a = 0; a < n; ++a) srow[a] = a < ns ? S[a] : -1;
      }

      /* Key lists of the selected branch (tokens of the chosen blocks up to t)
       * and of the sliding window (the last w tokens up to t). */
      int* keys_slc = (int*)malloc(sizeof(int) * ((long)ns * bs + 1));
      int nslc = 0;
      for (int a = 0; a < ns; ++a)
        for (int u = S[a] * bs; u < S[a] * bs + bs; ++u)
          if (u <= t) keys_slc[nslc++] = u;
      const int w0 = t - c->window + 1 > 0 ? t - c->window + 1 : 0;
      int* keys_win = (int*)malloc(sizeof(int) * (t - w0 + 1));
      int nwin = 0;
      for (int u = w0; u <= t; ++u) keys_win[nwin++] = u;
      double* pk = (double*)malloc(sizeof(double) * (nslc > nwin ? nslc : nwin) + 8);

      for (int hh = 0; hh < G; ++hh) {
        const int h = g * G + hh;
        const double* qh = q_rows + ((long)r * Hq + h) * d;
        /* Step 5 [EP94 §五 branch two]: fine-grained attention over every token
         * of the selected blocks. */
        attend(qh, kb, vb, tok, keys_slc, nslc, d, c->scale, oslc_h, pk);
        /* Step 6 [EP94 §五 branch three; LT103]: sliding-window attention. */
        attend(qh, kb, vb, tok, keys_win, nwin, d, c->scale, owin_h, pk);
        /* Step 7 [EP94 §五 gating; LCH gate]: per query and head, a sigmoid
         * gate per branch from the query, then the weighted sum. */
        double gt[3];
        for (int a = 0; a < 3; ++a) {
          if (c->gate_mode == 1) {
            gt[a] = c->fixed_gates[a];
          } else {
            double dot = 0.0;
            for (int e = 0; e < d; ++e) dot += qh[e] * wg[e * 3 + a];
            gt[a] = 1.0 / (1.0 + exp(-dot));
          }
        }
        const long o = ((long)r * Hq + h) * d;
        for (int e = 0; e < d; ++e) {
          if (o_cmp) o_cmp[o + e] = ocmp_g[hh][e];
          if (o_slc) o_slc[o + e] = oslc_h[e];
          if (o_win) o_win[o + e] = owin_h[e];
          if (out) out[o + e] = gt[0] * ocmp_g[hh][e] + gt[1] * oslc_h[e] + gt[2] * owin_h[e];
        }
        if (gates)
          for (int a = 0; a < 3; ++a) gates[((long)r * Hq + h) * 3 + a] = gt[a];
        free(ocmp_g[hh]);
      }
      free(pk);
      free(keys_win);
      free(keys_slc);
      free(S);
      free(ocmp_g);
      free(owin_h);
      free(oslc_h);
      free(blk);
      free(p);
      free(idx_all);
    }
}

/* ------------------------------------------------------------------------ */
/* MoBA                                                                      */
/* [EP94 §九, §十六; LCH MoBA paragraph]: one selected branch only; the block */
/* representative is the mean of the block's keys (no parameters); each head */
/* scores blocks by q . mean(K_block) and picks its own top-k (no sharing);  */
/* [LT103] the query's own block is always attended, causally masked.       */
/* ------------------------------------------------------------------------ */

/* kbar[b, j, g, :] = mean of K[b, j m .. j m + m - 1, g, :] over full blocks
 * j < T / m. kbar: [B, T / m, Hkv, d]. */
void oracle_moba_block_means(const oracle_moba_cfg* c, const double* k, double* kbar) {
  const int m = c->block, nfull = c->T / m;
  const long tok = (long)c->Hkv * c->d;
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < c->B; ++b)
    for (int j = 0; j < nfull; ++j)
      for (int g = 0; g < c->Hkv; ++g)
        for (int e = 0; e < c->d; ++e) {
          double acc = 0.0;
          for (int u = 0; u < m; ++u)
            acc += k[((long)b * c->T + (long)j * m + u) * tok + (long)g * c->d + e];
          kbar[((long)b * nfull + j) * tok + (long)g * c->d + e] = acc / m;
        }
}

/* q_rows: [nrows, Hq, d]; k, v: [B, T, Hkv, d]; kbar from
 * oracle_moba_block_means; forced_sel [nrows, Hq, k] or NULL.
 * Outputs (may be NULL): out [nrows, Hq, d]; sel [nrows, Hq, k] ascending,
 * -1 padded; scores [nrows, Hq, ceil(T/m)] (-inf for the own and later
 * blocks, which are not scored); lse [nrows, Hq]. */
void oracle_moba_rows(const oracle_moba_cfg* c, int nrows, const int* rows_b, const int* rows_t,
                      const double* q_rows, const double* k, const double* v,
                      const double* kbar, const int* forced_sel, double* out, int* sel,
                      double* scores, double* lse_out) {
  const int d = c->d, Hq = c->Hq, Hkv = c->Hkv, G = Hq / Hkv;
  const int m = c->block, K = c->top_k;
  const int nfull = c->T / m, nblk_max = (c->T + m - 1) / m;
  const long tok = (long)Hkv * d;

#pragma omp parallel for collapse(2) schedule(dynamic)
  for (int r = 0; r < nrows; ++r)
    for (int h = 0; h < Hq; ++h) {
      const int b = rows_b[r], t = rows_t[r], g = h / G;
      const int own = t / m;
      const double* qh = q_rows + ((long)r * Hq + h) * d;
      double* sc = (double*)malloc(sizeof(double) * (own > 0 ? own : 1));
      for (int j = 0; j < own; ++j) {
        const double* kb = kbar + ((long)b * nfull + j) * tok + (long)g * d;
        double dot = 0.0;
        for (int e = 0; e < d; ++e) dot += qh[e] * kb[e];
        sc[j] = dot;
      }
      if (scores) {
        double* srow = scores + ((long)r * Hq + h) * nblk_max;
        for (int j = 0; j < nblk_max; ++j) srow[j] = j < own ? sc[j] : -INFINITY;
      }
      int* S = (int*)malloc(sizeof(int) * (K > 0 ? K : 1));
      int ns = 0;
      if (forced_sel) {
        const int* fr = forced_sel + ((long)r * Hq + h) * K;
        for (int a = 0; a < K; ++a)
          if (fr[a] >= 0) S[ns++] = fr[a];
      } else {
        S[ns++] = own;
        if (own <= K - 1) {
          for (int j = 0; j < own; ++j) S[ns++] = j;
        } else {
          char* taken = (char*)calloc(own, 1);
          while (ns < K) {
            int best = -1;
            for (int j = 0; j < own; ++j)
              if (!taken[j] && (best < 0 || better(sc[j], j, sc[best], best))) best = j;
            taken[best] = 1;
            S[ns++] = best;
          }
          free(taken);
        }
      }
      qsort(S, ns, sizeof(int), cmp_int);
      if (sel) {
        int* srow = sel + ((long)r * Hq + h) * K;
        for (int a = 0; a < K; ++a) srow[a] = a < ns ? S[a] : -1;
      }
      /* One softmax over the tokens of the chosen blocks, causally masked. */
      int* keys = (int*)malloc(sizeof(int) * ((long)ns * m + 1));
      int nk = 0;
      for (int a = 0; a < ns; ++a)
        for (int u = S[a] * m; u < S[a] * m + m; ++u)
          if (u <= t) keys[nk++] = u;
      double* o = (double*)malloc(sizeof(double) * d);
      double lse = attend(qh, k + (long)b * c->T * tok + (long)g * d,
                          v + (long)b * c->T * tok + (long)g * d, tok, keys, nk, d, c->scale, o,
                          NULL);
      if (out)
        for (int e = 0; e < d; ++e) out[((long)r * Hq + h) * d + e] = o[e];
      if (lse_out) lse_out[(long)r * Hq + h] = lse;
      free(o);
      free(keys);
      free(S);
      free(sc);
    }
}
