/*
 * eb_oracle.h -- CPU reference ("oracle") for the entropy-bound canvas sampler.
 *
 * TEST INFRASTRUCTURE ONLY.  This is a plain, slow, single-threaded float64
 * restatement of what one denoising step of the sampler computes.  It exists
 * so that tests and the benchmark's CPU-baseline leg can check the CUDA
 * implementation; the product path never links, loads or calls it, and it
 * shares no source with the CUDA library (the two agree only on the published
 * definitions they both follow: Philox4x32-10 and the counter layout below).
 *
 * Sources (the pages this follows; cited by title and section):
 *   [MC-BP]    DiffusionGemma model card (Hugging Face mirror; ai.google.dev in
 *              German and Japanese), "Best practices, 1. Diffusion sampling
 *              settings": at most 48 steps, temperature falling linearly
 *              0.8 -> 0.4 for logit shaping, pick the lowest-entropy tokens
 *              while the bound stays at entropy_bound = 0.1, fully renoise
 *              the rest, stop early when the canvas mean entropy is below
 *              0.005 and the top prediction is unchanged over two steps.
 *   [MC-SPEC]  same card, model summary table: canvas length 256,
 *              vocabulary about 262K.
 *   [DP-SCHED] diffusers v0.43.0 "DiffusionGemma" pipeline page, section
 *              "Schedulers": EntropyBoundScheduler commits the lowest-entropy
 *              positions whose joint entropy stays under entropy_bound,
 *              accepting roughly independent tokens together, with the
 *              temperature annealed from t_max (0.8) at the first step to
 *              t_min (0.4) at the last; BlockRefinementScheduler commits the
 *              tokens above `threshold` plus a uniform per-step quota;
 *              DiscreteDDIM commits its predictions at the last step.
 *   [DP-INTRO] same page, introduction: the model samples candidate tokens
 *              each step, commits, and renoises the rest under uniform
 *              corruption (mask_token_id=None).
 *   [DP-STOP]  same page, "Adaptive stopping": a sample is frozen once its
 *              argmax has been stable for `stability_threshold` steps and
 *              its mean per-token entropy of the scheduler-shaped logits is
 *              below `confidence_threshold` (0.005).
 *   [DP-CALL]  same page, DiffusionGemmaPipeline.__call__ parameters
 *              (temperature 0.0 = greedy; stability_threshold = 1;
 *              confidence_threshold = None disables the stop).
 *   [NEWS]     zhiding.cn news article on DiffusionGemma: generation starts
 *              from a canvas of random placeholder tokens.
 *   [SALMON11] J. Salmon, M. Moraes, R. Dror, D. Shaw, "Parallel random
 *              numbers: as easy as 1, 2, 3", SC'11: the Philox4x32-10
 *              counter-based generator.
 *
 * Readings where the pages are silent or ambiguous are stated at each
 * function; the full list lives with the design notes of the repository.
 *
 * Counter layout of every random draw (fixed before either implementation):
 *   key = (seed & 0xffffffff, seed >> 32)
 *   element Gumbel  : ctr = (v >> 2, l, s, b | 0 << 24), word v & 3
 *   group Gumbel    : ctr = (j >> 2, l, s, b | 3 << 24), word j & 3
 *   renoise         : ctr = (l >> 2, 0, s, b | 1 << 24), word l & 3
 *   initial canvas  : ctr = (l >> 2, 0, 0, b | 2 << 24), word l & 3
 *   (b = global canvas index < 2^24, l = position, s = step, v = vocab id,
 *    j = group index = v / group_size.)
 *   uniform u = (2 * (x >> 9) + 1) * 2^-24, Gumbel g = -log(-log u),
 *   uniform token = (x * V) >> 32 (64-bit product).
 */
#ifndef EB_ORACLE_H
#define EB_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { EBO_F32 = 0, EBO_BF16 = 1 };
enum { EBO_RULE_EB = 0, EBO_RULE_BR = 1, EBO_RULE_EB_MI = 2 };
enum { EBO_STREAM_GUMBEL = 0, EBO_STREAM_RENOISE = 1, EBO_STREAM_INIT = 2, EBO_STREAM_GROUP = 3 };
enum { EBO_STOP_ACTIVE = 0, EBO_STOP_ADAPTIVE = 1, EBO_STOP_ALL_COMMITTED = 2, EBO_STOP_LAST_STEP = 3 };

typedef struct {
  int32_t B, L, V, num_steps;
  double t_max, t_min;        /* temperature endpoints (ignored when greedy) */
  double entropy_bound;       /* gamma */
  double stop_entropy;        /* tau; < 0 disables the adaptive stop */
  int32_t stability_steps;    /* consecutive unchanged-argmax steps required */
  int32_t rule;               /* EBO_RULE_* */
  double threshold;           /* block refinement confidence threshold */
  int32_t quota;              /* block refinement per-step quota */
  int32_t greedy;             /* 1: temperature 0.0, argmax instead of a draw */
  int32_t group_size;         /* elements per Gumbel group (64 in the library) */
  int32_t canvas_offset;      /* global index of local canvas 0 */
  uint64_t seed;
  double editing_threshold;   /* BR: re-edit a committed token when the argmax
                                 differs and pmax >= this; < 0 disables */
} ebo_config_t;

/* What one vocabulary slice [v_off, v_off + V_slice) of a position's logits
   contributes when the vocabulary is sharded (one slice per device):
   its maximum, the sums relative to it, its argmax, and its part of the
   two-level Gumbel-max draw (best group score and the element drawn in that
   group), all with global vocabulary indices. */
typedef struct {
  double S, W;        /* sum exp(y - y_max), sum exp(y - y_max)(y - y_max) over the slice */
  double zmax;        /* raw maximum logit of the slice */
  double gscore;      /* best perturbed group log-partition LSE_j + g_j (-inf if none) */
  int32_t amax;       /* lowest global id holding zmax */
  int32_t sample;     /* global id drawn in the best group (-1 if none) */
} ebo_slice_t;

/* Per-canvas decision margins: how far each decision was from flipping. */
typedef struct {
  double cum_margin;   /* EB: min |cumulative H - gamma| at the cut (inf if n/a) */
  double cut_gap;      /* EB: H(first left out) - H(last committed) (inf if n/a) */
  double stop_margin;  /* |mean H - tau| when the stability part holds (inf otherwise) */
  double br_margin;    /* BR: min |pmax - threshold| over open positions (inf if n/a) */
  double quota_gap;    /* BR: relative pmax gap at the quota cut (inf if n/a) */
  double mean_H;       /* canvas mean entropy (all positions) */
  int32_t n_commit;    /* positions committed this step */
  int32_t fired;       /* 1 if the adaptive stop fired */
  double edit_margin;  /* BR editing: min |pmax - editing_threshold| over committed
                          positions whose argmax differs from their token */
  int32_t n_edit;      /* committed positions re-edited this step */
  int32_t pad;
} ebo_margins_t;

void     ebo_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]);
uint32_t ebo_draw_word(uint64_t seed, uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3, int word);
double   ebo_uniform(uint32_t x);
double   ebo_gumbel(uint32_t x);
uint32_t ebo_uniform_token(uint32_t x, uint32_t V);
double   ebo_temperature(const ebo_config_t* c, int s);

/* Statistics of one position's logits row (V values, dtype EBO_*). */
void ebo_row_stats(const void* row, int dtype, int V, double inv_T,
                   double* H, double* pmax, int32_t* amax, double* H_direct);

/* Two-level Gumbel-max draw for position (b, l) at step s.  Returns the
   sampled vocab id; *margin is the smallest relative top-2 gap of the two
   decisions (group choice, element choice), *group the winning group. */
void ebo_slice_record(const ebo_config_t* c, const void* row_slice, int dtype, int V_slice,
                      int v_off, double inv_T, int b, int l, int s, ebo_slice_t* out);
void ebo_combine_slices(const ebo_slice_t* sl, int n, double inv_T, double* H, double* pmax,
                        int32_t* amax, int32_t* sample);
int32_t ebo_sample(const ebo_config_t* c, const void* row, int dtype, double inv_T,
                   int b, int l, int s, double* margin, int32_t* group);

/* Flat (single-level) Gumbel-max with the element stream; used by the pins
   to show the two-level draw equals it when group_size >= V. */
int32_t ebo_sample_flat(const ebo_config_t* c, const void* row, int dtype, double inv_T,
                        int b, int l, int s, double* margin);

/* Initial canvas of local canvas bl: uniform tokens, nothing committed. */
void ebo_init_canvas(const ebo_config_t* c, int bl, int32_t* canvas, uint8_t* committed,
                     uint8_t* stop, int32_t* stable);

/* Per-canvas decisions of one step, given the per-position quantities.
   H/amax/pmax/sample have L entries; canvas/committed/prev_amax L entries of
   this canvas; stop/stable point at this canvas' scalars. */
void ebo_canvas_decide(const ebo_config_t* c, int bl, int s,
                       const double* H, const int32_t* amax, const double* pmax,
                       const int32_t* sample,
                       int32_t* canvas, uint8_t* committed, uint8_t* stop,
                       int32_t* prev_amax, int32_t* stable, ebo_margins_t* mg);

/* One full step for local canvas bl: logits is that canvas' [L, V] block.
   Outputs H/amax/pmax/sample (L each) and the sample margins (L each).
   A canvas whose stop flag is set is left untouched (returns 0). */
int ebo_step_canvas(const ebo_config_t* c, const void* logits, int dtype, int bl, int s,
                    int32_t* canvas, uint8_t* committed, uint8_t* stop,
                    int32_t* prev_amax, int32_t* stable,
                    double* H, int32_t* amax, double* pmax, int32_t* sample,
                    double* sample_margin, int32_t* sample_group, ebo_margins_t* mg);

#ifdef __cplusplus
}
#endif
#endif
