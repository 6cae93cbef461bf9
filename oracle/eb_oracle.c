/*
 * eb_oracle.c -- CPU reference ("oracle") of one step of the entropy-bound
 * canvas sampler, float64, single-threaded.
 *
 * TEST INFRASTRUCTURE ONLY: used by tests/ and by the CPU-baseline leg of
 * bench.py.  The CUDA library never links or calls this file and shares no
 * source with it.  Source tags ([MC-BP], [DP-SCHED], ...) are defined in
 * eb_oracle.h.
 *
 * Every function follows the plain definition of the step it restates:
 * straight loops in vocabulary / position order, library exp/log, qsort.
 * There is no blocking, no fusion and no reordering beyond that.
 */
#include "eb_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------- */
/* Random draws                                                              */
/* ------------------------------------------------------------------------- */

/* Philox4x32 with 10 rounds [SALMON11]: each round multiplies words 0 and 2
   by the two Philox constants, crosses the high halves with words 1 and 3 and
   the round key, and keeps the low halves; the key is advanced by the two
   Weyl constants between rounds. */
void ebo_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  uint32_t x0 = ctr[0], x1 = ctr[1], x2 = ctr[2], x3 = ctr[3];
  uint32_t k0 = key[0], k1 = key[1];
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    uint64_t pa = (uint64_t)0xD2511F53u * (uint64_t)x0;
    uint64_t pb = (uint64_t)0xCD9E8D57u * (uint64_t)x2;
    uint32_t y0 = (uint32_t)(pb >> 32) ^ x1 ^ k0;
    uint32_t y1 = (uint32_t)pb;
    uint32_t y2 = (uint32_t)(pa >> 32) ^ x3 ^ k1;
    uint32_t y3 = (uint32_t)pa;
    x0 = y0; x1 = y1; x2 = y2; x3 = y3;
  }
  out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
}

uint32_t ebo_draw_word(uint64_t seed, uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3, int word) {
  uint32_t ctr[4] = {c0, c1, c2, c3};
  uint32_t key[2] = {(uint32_t)(seed & 0xffffffffu), (uint32_t)(seed >> 32)};
  uint32_t out[4];
  ebo_philox4x32_10(ctr, key, out);
  return out[word & 3];
}

/* Uniform in (0, 1) from the top 23 bits of a word: (2k + 1) 2^-24. */
double ebo_uniform(uint32_t x) { return (2.0 * (double)(x >> 9) + 1.0) * 0x1p-24; }

/* Standard Gumbel variate by inversion of its CDF exp(-exp(-g)). */
double ebo_gumbel(uint32_t x) { return -log(-log(ebo_uniform(x))); }

/* Uniform token in [0, V): high word of the 64-bit product x * V. */
uint32_t ebo_uniform_token(uint32_t x, uint32_t V) {
  return (uint32_t)(((uint64_t)x * (uint64_t)V) >> 32);
}

/* ------------------------------------------------------------------------- */
/* Temperature schedule [MC-BP], [DP-SCHED]                                  */
/* ------------------------------------------------------------------------- */

/* Linear from t_max at step 0 to t_min at step N-1 (a single step uses t_max).
   Greedy decoding (temperature 0.0, [DP-CALL]) shapes with T = 1. */
double ebo_temperature(const ebo_config_t* c, int s) {
  if (c->greedy) return 1.0;
  if (c->num_steps <= 1) return c->t_max;
  return c->t_max + (c->t_min - c->t_max) * (double)s / (double)(c->num_steps - 1);
}

/* ------------------------------------------------------------------------- */
/* Per-position statistics                                                   */
/* ------------------------------------------------------------------------- */

static double load_z(const void* row, int dtype, int v) {
  if (dtype == EBO_F32) return (double)((const float*)row)[v];
  uint32_t bits = (uint32_t)((const uint16_t*)row)[v] << 16; /* bf16 -> f32 is exact */
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

/* Softmax of the tempered logits y = z / T and its entropy in nats:
     m = max y,  S = sum exp(y - m),  W = sum exp(y - m) (y - m),
     H = log S - W / S  (= -sum p log p with p = exp(y - m) / S),
     pmax = 1 / S,  amax = lowest v with z_v = max z.
   The entropy is the quantity the pages sort by ("lowest-entropy tokens",
   [MC-BP]) and average for the stop test ([DP-STOP]).  H_direct is the same
   entropy computed the two-pass way, -sum p log p, for a self-check. */
void ebo_row_stats(const void* row, int dtype, int V, double inv_T,
                   double* H, double* pmax, int32_t* amax, double* H_direct) {
  double zmax = -INFINITY;
  int32_t am = 0;
  for (int v = 0; v < V; ++v) {
    double z = load_z(row, dtype, v);
    if (z > zmax) { zmax = z; am = v; }
  }
  double m = zmax * inv_T;
  double S = 0.0, W = 0.0;
  for (int v = 0; v < V; ++v) {
    double d = load_z(row, dtype, v) * inv_T - m;
    double e = exp(d);
    if (e > 0.0) { S += e; W += e * d; }
  }
  *H = log(S) - W / S;
  *pmax = 1.0 / S;
  *amax = am;
  if (H_direct) {
    double h = 0.0;
    for (int v = 0; v < V; ++v) {
      double p = exp(load_z(row, dtype, v) * inv_T - m) / S;
      if (p > 0.0) h -= p * log(p);
    }
    *H_direct = h;
  }
}

/* ------------------------------------------------------------------------- */
/* Categorical draw: Gumbel-max, taken in two levels                         */
/* ------------------------------------------------------------------------- */

static double rel_gap(double a, double b) {
  if (!(b > -INFINITY)) return INFINITY;
  double s = fabs(a);
  if (fabs(b) > s) s = fabs(b);
  if (s < 1.0) s = 1.0;
  return (a - b) / s;
}

/* Gumbel-max over the whole row with the element stream:
   x = argmax_v (y_v + g_v), lowest v on exact ties. */
int32_t ebo_sample_flat(const ebo_config_t* c, const void* row, int dtype, double inv_T,
                        int b, int l, int s, double* margin) {
  uint32_t bg = (uint32_t)(c->canvas_offset + b);
  double best = -INFINITY, second = -INFINITY;
  int32_t arg = -1;
  for (int v = 0; v < c->V; ++v) {
    uint32_t x = ebo_draw_word(c->seed, (uint32_t)v >> 2, (uint32_t)l, (uint32_t)s,
                               bg | ((uint32_t)EBO_STREAM_GUMBEL << 24), v & 3);
    double sc = load_z(row, dtype, v) * inv_T + ebo_gumbel(x);
    if (sc > best) { second = best; best = sc; arg = v; }
    else if (sc > second) { second = sc; }
  }
  if (margin) *margin = rel_gap(best, second);
  return arg;
}

/* The pages say the sampler "samples candidate tokens" each step ([DP-INTRO])
   without naming the method; the draw here is Gumbel-max over Philox4x32-10
   words, taken in two levels so that only one group of the row needs
   per-element noise:
     1. split the row into groups of group_size consecutive ids;
     2. for each group j: LSE_j = log sum_{v in j} exp(y_v), and
        M_j = LSE_j + g_j with g_j a Gumbel from the group stream;
     3. j* = argmax_j M_j (lowest j on exact ties);
     4. x = argmax_{v in j*} (y_v + g_v) with g_v from the element stream
        (lowest v on exact ties).
   The maximum of Gumbel-perturbed values over a group is itself Gumbel with
   location LSE_j, and is independent of which member attains it, so x has
   exactly the softmax(y) distribution.  With group_size >= V step 2 is
   trivial and the draw is the flat Gumbel-max of ebo_sample_flat. */
int32_t ebo_sample(const ebo_config_t* c, const void* row, int dtype, double inv_T,
                   int b, int l, int s, double* margin, int32_t* group) {
  const int V = c->V, G = c->group_size;
  const int ng = (V + G - 1) / G;
  uint32_t bg = (uint32_t)(c->canvas_offset + b);
  double best = -INFINITY, second = -INFINITY;
  int32_t jbest = -1;
  for (int j = 0; j < ng; ++j) {
    int lo = j * G, hi = lo + G < V ? lo + G : V;
    double mj = -INFINITY;
    for (int v = lo; v < hi; ++v) {
      double y = load_z(row, dtype, v) * inv_T;
      if (y > mj) mj = y;
    }
    if (!(mj > -INFINITY)) continue; /* a group of -inf logits never wins */
    double Sj = 0.0;
    for (int v = lo; v < hi; ++v) Sj += exp(load_z(row, dtype, v) * inv_T - mj);
    double lse = mj + log(Sj);
    uint32_t x = ebo_draw_word(c->seed, (uint32_t)j >> 2, (uint32_t)l, (uint32_t)s,
                               bg | ((uint32_t)EBO_STREAM_GROUP << 24), j & 3);
    double M = lse + ebo_gumbel(x);
    if (M > best) { second = best; best = M; jbest = j; }
    else if (M > second) { second = M; }
  }
  double m1 = rel_gap(best, second);
  if (group) *group = jbest;
  if (jbest < 0) { if (margin) *margin = INFINITY; return -1; }

  int lo = jbest * G, hi = lo + G < V ? lo + G : V;
  double eb = -INFINITY, es = -INFINITY;
  int32_t arg = -1;
  for (int v = lo; v < hi; ++v) {
    uint32_t x = ebo_draw_word(c->seed, (uint32_t)v >> 2, (uint32_t)l, (uint32_t)s,
                               bg | ((uint32_t)EBO_STREAM_GUMBEL << 24), v & 3);
    double sc = load_z(row, dtype, v) * inv_T + ebo_gumbel(x);
    if (sc > eb) { es = eb; eb = sc; arg = v; }
    else if (sc > es) { es = sc; }
  }
  double m2 = rel_gap(eb, es);
  if (margin) *margin = m1 < m2 ? m1 : m2;
  return arg;
}

/* ------------------------------------------------------------------------- */
/* Vocabulary-sharded logits                                                 */
/* ------------------------------------------------------------------------- */

/* One slice [v_off, v_off + V_slice) of a row (v_off a multiple of
   group_size, so that the draw's groups are whole), with global ids in every
   Philox counter: the quantities the full-row functions above build from it. */
void ebo_slice_record(const ebo_config_t* c, const void* row_slice, int dtype, int V_slice,
                      int v_off, double inv_T, int b, int l, int s, ebo_slice_t* out) {
  const int G = c->group_size;
  uint32_t bg = (uint32_t)(c->canvas_offset + b);
  double zmax = -INFINITY;
  int32_t am = -1;
  for (int v = 0; v < V_slice; ++v) {
    double z = load_z(row_slice, dtype, v);
    if (z > zmax) { zmax = z; am = v_off + v; }
  }
  double m = zmax * inv_T, S = 0.0, W = 0.0;
  for (int v = 0; v < V_slice; ++v) {
    double d = load_z(row_slice, dtype, v) * inv_T - m;
    double e = exp(d);
    if (e > 0.0) { S += e; W += e * d; }
  }
  out->S = S;
  out->W = W;
  out->zmax = zmax;
  out->amax = am;
  /* two-level draw restricted to the slice's groups (global group ids) */
  const int ng = (V_slice + G - 1) / G;
  double best = -INFINITY;
  int jbest = -1;
  for (int jl = 0; jl < ng; ++jl) {
    int lo = jl * G, hi = lo + G < V_slice ? lo + G : V_slice;
    double mj = -INFINITY;
    for (int v = lo; v < hi; ++v) {
      double y = load_z(row_slice, dtype, v) * inv_T;
      if (y > mj) mj = y;
    }
    if (!(mj > -INFINITY)) continue;
    double Sj = 0.0;
    for (int v = lo; v < hi; ++v) Sj += exp(load_z(row_slice, dtype, v) * inv_T - mj);
    int j = v_off / G + jl;
    uint32_t x = ebo_draw_word(c->seed, (uint32_t)j >> 2, (uint32_t)l, (uint32_t)s,
                               bg | ((uint32_t)EBO_STREAM_GROUP << 24), j & 3);
    double M = mj + log(Sj) + ebo_gumbel(x);
    if (M > best) { best = M; jbest = jl; }
  }
  out->gscore = best;
  out->sample = -1;
  if (jbest >= 0) {
    int lo = jbest * G, hi = lo + G < V_slice ? lo + G : V_slice;
    double eb = -INFINITY;
    for (int v = lo; v < hi; ++v) {
      int vg = v_off + v;
      uint32_t x = ebo_draw_word(c->seed, (uint32_t)vg >> 2, (uint32_t)l, (uint32_t)s,
                                 bg | ((uint32_t)EBO_STREAM_GUMBEL << 24), vg & 3);
      double sc = load_z(row_slice, dtype, v) * inv_T + ebo_gumbel(x);
      if (sc > eb) { eb = sc; out->sample = vg; }
    }
  }
}

/* The full row's quantities from its slices, given in increasing v_off:
   the maximum is the largest slice maximum; the sums rescale to it; the
   argmax is the first slice's argmax that attains it; the draw's winning
   group is the best slice's (the maximum over groups is the maximum over
   the slices' maxima; an earlier slice wins an exact tie, as the lower
   group does), and its element is that slice's. */
void ebo_combine_slices(const ebo_slice_t* sl, int n, double inv_T, double* H, double* pmax,
                        int32_t* amax, int32_t* sample) {
  double M = -INFINITY;
  int32_t am = -1;
  for (int i = 0; i < n; ++i)
    if (sl[i].zmax > M) { M = sl[i].zmax; am = sl[i].amax; }
  double S = 0.0, W = 0.0;
  for (int i = 0; i < n; ++i) {
    if (!(sl[i].zmax > -INFINITY)) continue;
    double dd = (sl[i].zmax - M) * inv_T;
    double f = exp(dd);
    S += f * sl[i].S;
    W += f * (sl[i].W + dd * sl[i].S);
  }
  *H = log(S) - W / S;
  *pmax = 1.0 / S;
  *amax = am;
  double best = -INFINITY;
  int32_t x = -1;
  for (int i = 0; i < n; ++i)
    if (sl[i].gscore > best) { best = sl[i].gscore; x = sl[i].sample; }
  *sample = x;
}

/* ------------------------------------------------------------------------- */
/* Canvas start [NEWS], [DP-INTRO]                                           */
/* ------------------------------------------------------------------------- */

/* A new canvas holds uniform-random tokens (uniform corruption, no mask
   token) and nothing is committed. */
void ebo_init_canvas(const ebo_config_t* c, int bl, int32_t* canvas, uint8_t* committed,
                     uint8_t* stop, int32_t* stable) {
  uint32_t bg = (uint32_t)(c->canvas_offset + bl);
  for (int l = 0; l < c->L; ++l) {
    uint32_t x = ebo_draw_word(c->seed, (uint32_t)l >> 2, 0u, 0u,
                               bg | ((uint32_t)EBO_STREAM_INIT << 24), l & 3);
    canvas[l] = (int32_t)ebo_uniform_token(x, (uint32_t)c->V);
    committed[l] = 0;
  }
  *stop = EBO_STOP_ACTIVE;
  *stable = 0;
}

/* ------------------------------------------------------------------------- */
/* Per-canvas decisions                                                      */
/* ------------------------------------------------------------------------- */

static const double* g_sort_key; /* qsort comparators see the key array here */

static int cmp_key_asc(const void* a, const void* b) { /* (key, l) ascending */
  int32_t la = *(const int32_t*)a, lb = *(const int32_t*)b;
  double ka = g_sort_key[la], kb = g_sort_key[lb];
  if (ka < kb) return -1;
  if (ka > kb) return 1;
  return (la > lb) - (la < lb);
}

static int cmp_key_desc(const void* a, const void* b) { /* (-key, l) ascending */
  int32_t la = *(const int32_t*)a, lb = *(const int32_t*)b;
  double ka = g_sort_key[la], kb = g_sort_key[lb];
  if (ka > kb) return -1;
  if (ka < kb) return 1;
  return (la > lb) - (la < lb);
}

/* Steps of one canvas after its per-position quantities are known:
   1. stability [DP-STOP]: the argmax of every position equals the previous
      step's; `stable` counts consecutive such steps (none at step 0);
   2. adaptive stop [MC-BP], [DP-STOP]: stable >= stability_steps and the mean
      entropy over all L positions below tau; then the canvas is frozen: open
      positions take the argmax, all are committed, stop = 1;
   3. otherwise the commit rule chooses open positions, which take their
      sampled token (greedy: the argmax):
      EB    [MC-BP], [DP-SCHED]: open positions sorted by (H, l); the longest
            prefix whose entropy sum stays <= gamma (the joint entropy of
            roughly independent tokens), at least one position;
      EB_MI the same with the prefix's sum minus its largest entropy <= gamma
            (the "mutual information bound" wording of the model cards);
      BR    [DP-SCHED]: open positions with pmax >= threshold, plus the next
            `quota` by (-pmax, l); with editing enabled, first, every position
            committed before this step whose argmax differs from its token
            takes the argmax when pmax >= editing_threshold ([DP-SCHED]:
            editing_threshold lets the scheduler re-edit committed tokens;
            the condition and the replacement token are this reading's);
   4. the last step (s = N-1) commits every remaining open position with its
      sampled token, stop = 3 (as the DDIM scheduler commits its predictions
      at the last step, [DP-SCHED]); if nothing is left open, stop = 2;
   5. renoise [MC-BP], [DP-INTRO]: every still-open position gets a fresh
      uniform-random token;
   6. prev_amax <- amax. */
void ebo_canvas_decide(const ebo_config_t* c, int bl, int s,
                       const double* H, const int32_t* amax, const double* pmax,
                       const int32_t* sample,
                       int32_t* canvas, uint8_t* committed, uint8_t* stop,
                       int32_t* prev_amax, int32_t* stable, ebo_margins_t* mg) {
  const int L = c->L;
  uint32_t bg = (uint32_t)(c->canvas_offset + bl);
  mg->cum_margin = INFINITY;
  mg->cut_gap = INFINITY;
  mg->stop_margin = INFINITY;
  mg->br_margin = INFINITY;
  mg->quota_gap = INFINITY;
  mg->n_commit = 0;
  mg->fired = 0;
  mg->edit_margin = INFINITY;
  mg->n_edit = 0;
  mg->pad = 0;

  /* 1. stability */
  int all_eq = s >= 1;
  for (int l = 0; l < L && all_eq; ++l)
    if (amax[l] != prev_amax[l]) all_eq = 0;
  *stable = all_eq ? *stable + 1 : 0;

  /* 2. adaptive stop */
  double sumH = 0.0;
  for (int l = 0; l < L; ++l) sumH += H[l];
  double meanH = sumH / (double)L;
  mg->mean_H = meanH;
  int fired = 0;
  if (c->stop_entropy >= 0.0 && *stable >= c->stability_steps) {
    mg->stop_margin = fabs(meanH - c->stop_entropy);
    fired = meanH < c->stop_entropy;
  }

  if (fired) {
    for (int l = 0; l < L; ++l) {
      if (!committed[l]) {
        canvas[l] = amax[l];
        committed[l] = 1;
        mg->n_commit++;
      }
    }
    *stop = EBO_STOP_ADAPTIVE;
    mg->fired = 1;
  } else {
    int32_t* open = (int32_t*)malloc(sizeof(int32_t) * (size_t)(L > 0 ? L : 1));
    int n = 0;
    for (int l = 0; l < L; ++l)
      if (!committed[l]) open[n++] = l;

    /* BR editing of positions committed before this step */
    if (c->rule == EBO_RULE_BR && c->editing_threshold >= 0.0) {
      for (int l = 0; l < L; ++l) {
        if (!committed[l] || amax[l] == canvas[l]) continue;
        double d = fabs(pmax[l] - c->editing_threshold);
        if (d < mg->edit_margin) mg->edit_margin = d;
        if (pmax[l] >= c->editing_threshold) {
          canvas[l] = amax[l];
          mg->n_edit++;
        }
      }
    }

    int32_t* pick = (int32_t*)malloc(sizeof(int32_t) * (size_t)(L > 0 ? L : 1));
    int np = 0;
    if (n > 0 && (c->rule == EBO_RULE_EB || c->rule == EBO_RULE_EB_MI)) {
      g_sort_key = H;
      qsort(open, (size_t)n, sizeof(int32_t), cmp_key_asc);
      double cum = 0.0;
      int k = 0;
      while (k < n && cum + H[open[k]] <= c->entropy_bound) {
        cum += H[open[k]];
        ++k;
      }
      /* margins of the prefix cut: the sums on either side of gamma */
      if (k >= 1) mg->cum_margin = fabs(cum - c->entropy_bound);
      if (k < n) {
        double nxt = fabs(cum + H[open[k]] - c->entropy_bound);
        if (nxt < mg->cum_margin) mg->cum_margin = nxt;
      }
      if (c->rule == EBO_RULE_EB) {
        if (k == 0) k = 1; /* at least one position per step */
      } else {
        k = k + 1 < n ? k + 1 : n; /* sum minus the largest: one more */
      }
      if (k < n) mg->cut_gap = H[open[k]] - H[open[k - 1]];
      for (int i = 0; i < k; ++i) pick[np++] = open[i];
    } else if (n > 0 && c->rule == EBO_RULE_BR) {
      int32_t* rest = (int32_t*)malloc(sizeof(int32_t) * (size_t)n);
      int nr = 0;
      for (int i = 0; i < n; ++i) {
        int l = open[i];
        double d = fabs(pmax[l] - c->threshold);
        if (d < mg->br_margin) mg->br_margin = d;
        if (pmax[l] >= c->threshold) pick[np++] = l;
        else rest[nr++] = l;
      }
      g_sort_key = pmax;
      qsort(rest, (size_t)nr, sizeof(int32_t), cmp_key_desc);
      int q = c->quota < nr ? c->quota : nr;
      if (q < 0) q = 0;
      if (q >= 1 && q < nr) {
        double a = pmax[rest[q - 1]], b2 = pmax[rest[q]];
        mg->quota_gap = (a - b2) / (a > 0.0 ? a : 1.0);
      }
      for (int i = 0; i < q; ++i) pick[np++] = rest[i];
      free(rest);
    }
    for (int i = 0; i < np; ++i) {
      int l = pick[i];
      canvas[l] = c->greedy ? amax[l] : sample[l];
      committed[l] = 1;
    }
    mg->n_commit = np;
    free(pick);
    free(open);

    /* 4. last step / nothing left */
    if (s == c->num_steps - 1) {
      for (int l = 0; l < L; ++l) {
        if (!committed[l]) {
          canvas[l] = c->greedy ? amax[l] : sample[l];
          committed[l] = 1;
          mg->n_commit++;
        }
      }
      *stop = EBO_STOP_LAST_STEP;
    } else {
      int left = 0;
      for (int l = 0; l < L; ++l) left += !committed[l];
      if (left == 0) *stop = EBO_STOP_ALL_COMMITTED;
    }

    /* 5. renoise */
    for (int l = 0; l < L; ++l) {
      if (!committed[l]) {
        uint32_t x = ebo_draw_word(c->seed, (uint32_t)l >> 2, 0u, (uint32_t)s,
                                   bg | ((uint32_t)EBO_STREAM_RENOISE << 24), l & 3);
        canvas[l] = (int32_t)ebo_uniform_token(x, (uint32_t)c->V);
      }
    }
  }

  /* 6. */
  for (int l = 0; l < L; ++l) prev_amax[l] = amax[l];
}

/* ------------------------------------------------------------------------- */
/* One full step of one canvas                                               */
/* ------------------------------------------------------------------------- */

int ebo_step_canvas(const ebo_config_t* c, const void* logits, int dtype, int bl, int s,
                    int32_t* canvas, uint8_t* committed, uint8_t* stop,
                    int32_t* prev_amax, int32_t* stable,
                    double* H, int32_t* amax, double* pmax, int32_t* sample,
                    double* sample_margin, int32_t* sample_group, ebo_margins_t* mg) {
  if (*stop != EBO_STOP_ACTIVE) return 0; /* frozen canvases are skipped */
  const size_t elt = dtype == EBO_F32 ? 4 : 2;
  const double inv_T = 1.0 / ebo_temperature(c, s);
  for (int l = 0; l < c->L; ++l) {
    const void* row = (const char*)logits + (size_t)l * (size_t)c->V * elt;
    ebo_row_stats(row, dtype, c->V, inv_T, &H[l], &pmax[l], &amax[l], NULL);
    sample_margin[l] = INFINITY;
    sample_group[l] = -1;
    if (committed[l]) {
      sample[l] = -1;
    } else if (c->greedy) {
      sample[l] = amax[l];
    } else {
      sample[l] = ebo_sample(c, row, dtype, inv_T, bl, l, s, &sample_margin[l], &sample_group[l]);
    }
  }
  ebo_canvas_decide(c, bl, s, H, amax, pmax, sample, canvas, committed, stop, prev_amax,
                    stable, mg);
  return 1;
}
