/*
 * eb_sampler.h -- C ABI of the B200 entropy-bound (EB) canvas sampler.
 *
 * One call of eb_sampler_step performs one denoising step of DiffusionGemma's
 * multi-canvas sampler on decoder logits [B canvases, L positions, V vocab]:
 * tempered softmax entropy and argmax of every position, a categorical draw
 * for every open position, the commit rule, the adaptive stop and the
 * renoise of every position left open.
 *
 * Where the operation is defined (pages cited by title and section):
 *   DiffusionGemma model card (Hugging Face / ai.google.dev), "Best
 *   practices, 1. Diffusion sampling settings": at most 48 denoising steps,
 *   temperature falling linearly 0.8 -> 0.4 for logit shaping, each step
 *   selects the lowest-entropy tokens while the bound stays at
 *   entropy_bound = 0.1, unselected tokens are fully renoised, and sampling
 *   stops early once the canvas mean entropy is below 0.005 and the top
 *   prediction is unchanged over two consecutive steps.
 *   Same card, model summary table: canvas length 256, vocabulary ~262K.
 *   diffusers v0.43.0 "DiffusionGemma" pipeline page, "Schedulers":
 *   EntropyBoundScheduler (joint entropy of the committed positions under
 *   entropy_bound; t_max 0.8 at the first step to t_min 0.4 at the last),
 *   BlockRefinementScheduler (commit above `threshold` plus a uniform
 *   per-step quota; greedy at temperature 0.0); "Adaptive stopping"
 *   (stability_threshold, confidence_threshold on the scheduler-shaped
 *   logits, per-sample freeze); "Static cache and compilation" (fixed shapes,
 *   graph capture, the logits buffer is reused and must not be modified);
 *   "Callbacks" (the canvas lives in caller tensors between steps).
 *
 * Conventions shared by every entry point:
 *   - Every tensor argument is a DEVICE pointer owned by the caller (e.g. a
 *     torch tensor's data_ptr()), row-major and contiguous:
 *       logits     [B][L][V]  fp32 or bf16, read-only, 16-byte aligned for the
 *                  bulk-copy path (other alignments use a slower load path)
 *       canvas     [B][L] int32 tokens in [0, V), in/out
 *       committed  [B][L] uint8 0/1, in/out, never reverts within a canvas
 *       entropies  [B][L] fp32 out, nats, of softmax(logits / T_step)
 *       argmax     [B][L] int32 out, lowest id among equal maxima
 *       stop_flags [B] uint8 in/out: 0 active, else an EB_STOP_* reason
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy stream).
 *   - Every function returns an int status (EB_OK = 0); nothing throws.
 *   - A handle owns its device workspace; one handle per stream at a time;
 *     handles are not thread-safe.
 *   - Canvas b of a handle is canvas (canvas_offset + b) of the whole job;
 *     all random draws are keyed by that global index, so a batch split
 *     across devices gives the same bits as one device.
 */
#ifndef EB_SAMPLER_H
#define EB_SAMPLER_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct eb_sampler eb_sampler_t;

typedef enum { EB_F32 = 0, EB_BF16 = 1 } eb_dtype_t;

/* Commit rules.  ENTROPY_BOUND: sort open positions by (entropy, position)
   and commit the longest prefix whose entropy sum stays <= entropy_bound,
   at least one position.  ENTROPY_BOUND_MI: the prefix's entropy sum minus
   its largest entropy stays <= entropy_bound (the model cards' "mutual
   information bound" wording).  BLOCK_REFINEMENT: open positions with
   max probability >= threshold plus the next `quota` by (-pmax, position). */
typedef enum {
  EB_RULE_ENTROPY_BOUND = 0,
  EB_RULE_BLOCK_REFINEMENT = 1,
  EB_RULE_ENTROPY_BOUND_MI = 2
} eb_rule_t;

enum {
  EB_OK = 0,
  EB_ERR_INVALID_ARG = 1,    /* null pointer, bad size, bad config value */
  EB_ERR_CUDA = 2,           /* a CUDA runtime call failed */
  EB_ERR_OUT_OF_MEMORY = 3,  /* workspace allocation failed */
  EB_ERR_STEP_ORDER = 4,     /* step is neither 0 nor previous step + 1 */
  EB_ERR_UNSUPPORTED = 5,    /* unsupported dtype or device */
  EB_ERR_OVERFLOW = 6,       /* sizes exceed the documented limits */
  EB_ERR_DEVICE_STATUS = 7   /* a kernel reported a problem (see eb_sampler_status) */
};

/* Bits of the device status word. */
enum {
  EB_STATUS_BAD_TOKEN = 1,   /* a committed position held a token outside [0, V) */
  EB_STATUS_NONFINITE = 2,   /* a row produced a non-finite softmax sum */
  EB_STATUS_TIMEOUT = 4      /* an internal bounded wait gave up */
};

/* Stop reasons written to stop_flags. */
enum {
  EB_STOP_ACTIVE = 0,
  EB_STOP_ADAPTIVE = 1,      /* adaptive stop fired; open positions took the argmax */
  EB_STOP_ALL_COMMITTED = 2, /* the commit rule left nothing open */
  EB_STOP_LAST_STEP = 3      /* step num_steps-1 committed every open position */
};

/* Size of the vocabulary groups of the two-level Gumbel-max draw. */
#define EB_GUMBEL_GROUP 64

/* Limits checked by eb_sampler_init. */
#define EB_MAX_CANVASES 4096
#define EB_MAX_POSITIONS 1024

typedef struct {
  int32_t B;               /* canvases in this handle, 1..EB_MAX_CANVASES */
  int32_t L;               /* positions per canvas (256 on the model card), 1..EB_MAX_POSITIONS */
  int32_t V;               /* vocabulary size (262144), >= 1 */
  int32_t num_steps;       /* N, at most 48 on the model card, >= 1 */
  double t_max, t_min;     /* temperature at step 0 and at step N-1 (0.8, 0.4), > 0 */
  double entropy_bound;    /* gamma (0.1), >= 0 */
  double stop_entropy;     /* tau (0.005); < 0 disables the adaptive stop */
  int32_t stability_steps; /* consecutive unchanged-argmax steps required (1), >= 0 */
  int32_t rule;            /* eb_rule_t */
  double threshold;        /* block refinement confidence threshold (0.9) */
  int32_t quota;           /* block refinement per-step quota (ceil(L/N) = 6), >= 0 */
  int32_t greedy;          /* 1: temperature 0.0 -- shape with T = 1, commit argmax, no draw */
  int32_t canvas_offset;   /* global index of canvas 0; offset + B <= 2^24 */
  uint64_t seed;           /* key of every Philox4x32-10 draw */
  double editing_threshold; /* block refinement re-editing (diffusers "DiffusionGemma",
                               Schedulers: editing_threshold lets the scheduler re-edit
                               committed tokens).  Read here as: at a step where the stop
                               did not fire, a position committed before the step takes
                               this step's argmax when the argmax differs from its token
                               and pmax >= editing_threshold; it stays committed.  < 0
                               (the default) disables it; other rules ignore it.  Not NaN. */
  int32_t vocab_offset;    /* vocabulary-sharded logits: global id of this handle's first
                              logit, a multiple of EB_GUMBEL_GROUP (0 when not sharded) */
  int32_t vocab_total;     /* vocabulary-sharded logits: the full vocabulary size, >= 
                              vocab_offset + V; 0 when not sharded (then V is the vocabulary) */
} eb_config_t;

/* Fill *cfg with the model card's settings for B canvases of L x V. */
void eb_config_default(eb_config_t* cfg, int32_t B, int32_t L, int32_t V);

/* Create a sampler on CUDA device `device` (the device must be sm_100).
   Validates cfg, allocates and zeroes the workspace (the per-(position,
   stream CTA) records and per-position counters of the stream pass, the
   active-canvas list, previous argmax, stability counters, per-position
   draws and max probabilities, status word) in one allocation.  The first
   handle on a device also sets the kernels' shared-memory attributes for
   that device (once, to the device maximum).
   On success *out owns the handle (release with eb_sampler_destroy).
   Errors: INVALID_ARG, OVERFLOW, UNSUPPORTED, OUT_OF_MEMORY, CUDA. */
int eb_sampler_init(eb_sampler_t** out, const eb_config_t* cfg, int device);

/* Start new canvases: canvas <- uniform-random tokens (generation starts from
   a canvas of random placeholder tokens; uniform corruption, no mask token),
   committed <- 0, stop_flags <- 0, and reset the stability state.  Enqueued
   on `stream`, no host synchronisation. */
int eb_sampler_init_canvas(eb_sampler_t* h, int32_t* canvas, uint8_t* committed,
                           uint8_t* stop_flags, void* stream);

/* One denoising step `step` (0 .. num_steps-1) on `stream`: one kernel,
   launched as a programmatic dependent of the stream's previous kernel
   (its shared-memory set-up overlaps that kernel's end; it reads nothing
   before that kernel has completed).  `step` must be
   0 (which restarts the step sequence) or the previous step + 1, else
   EB_ERR_STEP_ORDER.  Canvases whose stop flag is set are skipped: their
   logits are not read and their buffers are left untouched.  For every
   other canvas: entropies/argmax of all L positions are written, open
   positions are committed by the rule or renoised, and stop_flags[b] is set
   when the canvas finishes.  Never synchronises the host, allocates nothing,
   so a sequence of steps can be captured in a CUDA graph.  Kernel-side
   problems set the status word instead of faulting (see eb_sampler_status).
   Errors: INVALID_ARG, STEP_ORDER, UNSUPPORTED (dtype), CUDA (launch). */
int eb_sampler_step(eb_sampler_t* h, const void* logits, int dtype, int step,
                    int32_t* canvas, uint8_t* committed, float* entropies,
                    int32_t* argmax, uint8_t* stop_flags, void* stream);

/* Synchronise `stream`, then report whether canvas b (or, for b = -1, every
   canvas) has stopped, reading the device stop flags.  The only call that
   waits for the device.  Returns EB_ERR_DEVICE_STATUS if the status word is
   non-zero (the flags are still reported). */
int eb_canvas_done(eb_sampler_t* h, const uint8_t* stop_flags, int b, int* done, void* stream);

/* Synchronise `stream` and read the device status word (EB_STATUS_* bits);
   clear it when `clear` is non-zero. */
int eb_sampler_status(eb_sampler_t* h, uint32_t* status, int clear, void* stream);

/* Copy the last step's per-position categorical draws ([B][L] int32, -1 for
   positions that were committed before the step) and max probabilities
   ([B][L] fp32) into caller device buffers on `stream`.  Either may be NULL. */
int eb_sampler_draws(eb_sampler_t* h, int32_t* sample, float* pmax, void* stream);

/* Resume support: overwrite the previous-step argmax ([B][L] int32, device)
   and the per-canvas stability counters ([B] int32, device; NULL = zeros)
   so that a trajectory checkpointed in caller buffers can continue at any
   step.  Enqueued on `stream`. */
int eb_sampler_set_state(eb_sampler_t* h, const int32_t* prev_argmax, const int32_t* stable,
                         int next_step, void* stream);

/* Allocation-free per-row statistics.  For `rows` rows of `V` logits
   (dtype EB_F32 / EB_BF16, [rows][V] row-major, device memory, caller-owned)
   writes each row's entropy in nats of softmax(z / temperature) into
   `entropies` ([rows] fp32, device) and its argmax (lowest index on ties)
   into `argmax` ([rows] int32, device), enqueued on `stream`.  These are the
   entropies and argmax that eb_sampler_step computes for a position at the
   same temperature (bit for bit against a one-canvas sampler with L = rows,
   which splits the work across the GPU the same way).

   For callers that cannot allocate device memory, or must not: code that
   runs under a hard device-memory budget, a plugin handed raw pointers by a
   host that owns the allocator, or a caller that has no eb_sampler_t
   (eb_sampler_init allocates its workspace).  This call allocates nothing:
   its scratch (the stream pass's per-(row, stream CTA) records, per-row
   counters and side outputs) is a static device array of
   EB_NOALLOC_SCRATCH_BYTES bytes in the library, which every GPU that loads
   the library holds until the process exits.
     - The first call on a device performs a one-time setup on it (the
       scratch's device address, kernel attributes); make it before any
       stream capture.
     - Sizes beyond the scratch return EB_ERR_OVERFLOW: 256 + rows x (48 x
       the stream CTAs a row can span + 12) bytes must fit (about 50000 rows
       of 262144 logits).
     - Every call clears what must start at zero; calls that overlap in time
       (different streams or threads) share the scratch and race: serialise
       them.
   If an internal wait of the pass gives up (EB_STATUS_TIMEOUT in the
   scratch status word), every row's entropy is written as NaN and its
   argmax as -1 instead of being left stale.  Non-finite softmax sums set
   EB_STATUS_NONFINITE in that word, which is cleared at the start of every
   call and not otherwise reported.  Returns EB_ERR_INVALID_ARG for NULL
   pointers, rows or V < 1, a temperature that is not finite and positive,
   or logits not aligned to their element size.  No counterpart in the
   DiffusionGemma pages: it exposes the sampler's row reduction on its own,
   for deployment. */
#define EB_NOALLOC_SCRATCH_BYTES (8u << 20)
int eb_row_stats_noalloc(const void* logits, int dtype, int32_t rows, int32_t V,
                         double temperature, float* entropies, int32_t* argmax, void* stream);

/* Vocabulary-sharded logits (a tensor-parallel LM head gives each device a
   contiguous slice of the vocabulary).  Each device's handle is configured
   with its slice (V = slice width, vocab_offset, vocab_total); all keep the
   same canvas state.  A step is then three calls, the middle one the
   caller's collective:
     1. eb_sampler_step_slice on every device: reads the slice's logits
        ([B][L][V], dtype as in eb_sampler_step) and writes one
        eb_slice_record_bytes() record per position ([B][L], device memory,
        8-byte aligned, caller-owned) -- the slice's maximum, sums, argmax and
        its part of the two-level draw, with global ids;
     2. the caller all-gathers the records of every device into one buffer
        [n_slices][B][L], slices in increasing vocab_offset (rank order of a
        torch.distributed all_gather_into_tensor with ranks ordered by slice);
     3. eb_sampler_combine on every device: combines each position's records
        in slice order (the same arithmetic everywhere, so every device
        computes the same results) and runs the canvas decisions; outputs as
        in eb_sampler_step.
   The results equal eb_sampler_step over the full vocabulary: the maximum,
   argmax and draw exactly (the draw's groups never straddle slices and
   every Philox counter uses global ids), the entropies to rounding.
   eb_sampler_step refuses a slice handle (EB_ERR_INVALID_ARG).  Step order
   as in eb_sampler_step; eb_sampler_combine needs this handle's
   eb_sampler_step_slice of the same step first (EB_ERR_STEP_ORDER).  The
   split follows the pages' model size (one accelerator) only as an
   extension: no counterpart in the DiffusionGemma pages. */
int eb_sampler_step_slice(eb_sampler_t* h, const void* logits, int dtype, int step,
                          const uint8_t* committed, const uint8_t* stop_flags, void* records,
                          void* stream);
int eb_sampler_combine(eb_sampler_t* h, const void* records, int n_slices, int step,
                       int32_t* canvas, uint8_t* committed, float* entropies, int32_t* argmax,
                       uint8_t* stop_flags, void* stream);
size_t eb_slice_record_bytes(void);

/* The sampler fused into the decoder's LM head: a step from the last hidden
   states instead of from logits.  The logits z = h W^T are formed on the
   tensor cores (tcgen05, bf16 in, fp32 accumulate) tile by tile and reduced
   on chip -- maximum, argmax, the entropy sums, the two-level Gumbel draw --
   so they never reach HBM; then the canvas decisions run as in
   eb_sampler_step (diffusers "DiffusionGemma" page, `__call__` parameters:
   the pipeline's logits are the decoder's [batch, canvas_length,
   vocab_size] output; model card, summary table: vocabulary about 262K).
     hidden  [B*L][d] bf16, device memory, 16-byte aligned, row-major (row =
             canvas b, position l in the handle's order), read only;
     weight  [V][d] bf16, device memory, 16-byte aligned, row-major (the LM
             head, one row per vocabulary id), read only;
     d       hidden size, a multiple of 64; V (the handle's) a multiple of
             256; the handle must cover the whole vocabulary (no slice);
     canvas .. stop_flags, stream: as in eb_sampler_step.
   The results equal eb_sampler_step on the logits z computed in fp32: the
   argmax and the draw exactly wherever z is (for example when every partial
   sum of h W^T is exactly representable), the entropies to rounding.
   eb_lmhead_reserve(h, d) allocates the handle's per-(position, vocabulary
   range) records once, before the first eb_lmhead_step (EB_ERR_INVALID_ARG
   otherwise); eb_lmhead_step itself allocates nothing and never
   synchronises.  Step order as in eb_sampler_step.  Errors:
   EB_ERR_UNSUPPORTED for d or V not multiples of 64 / 256 or a slice
   handle, EB_ERR_INVALID_ARG for NULL or misaligned pointers, bad steps.
   A pipeline wait that runs out sets EB_STATUS_TIMEOUT as in the stream
   kernel.  No counterpart in the pages' pipeline, which forms the logits
   first; this is the same step with the logits kept on chip. */
int eb_lmhead_reserve(eb_sampler_t* h, int32_t d);
int eb_lmhead_step(eb_sampler_t* h, const void* hidden, const void* weight, int32_t d, int step,
                   int32_t* canvas, uint8_t* committed, float* entropies, int32_t* argmax,
                   uint8_t* stop_flags, void* stream);

/* Diagnostic form of the LM-head kernel's contraction: logits [rows][V]
   fp32 (device memory, 16-byte aligned, caller-owned) = hidden [rows][d] x
   weight[V][d]^T, both bf16 as in eb_lmhead_step, on the current device and
   `stream`.  Same size rules; no handle.  It lets a caller (and the tests)
   check the tensor-core contraction apart from the sampler. */
int eb_lmhead_logits(const void* hidden, const void* weight, int32_t rows, int32_t V, int32_t d,
                     float* logits, void* stream);

/* Profiling hook.  When `event` (a cudaEvent_t passed as void*, owned by
   the caller) is non-NULL, every following eb_sampler_step records it on
   its stream right after the step's kernel, so that the caller can time that
   kernel with an event recorded before the call.  Recording it keeps the
   next kernel on the stream from starting early (programmatic dependent
   launch), so set it only for timing; NULL turns it off.  No counterpart in
   the method: it measures the implementation. */
int eb_sampler_set_split_event(eb_sampler_t* h, void* event);

/* Diagnostic hook: the limit, in nanoseconds, of every wait of the stream
   kernel's pipeline (a consumer waiting for a copy, a producer waiting for a
   free stage, the hand-off of row records); 0 restores the default of 2 s.
   A wait that runs out sets EB_STATUS_TIMEOUT, ends the step's stream pass
   early (the step's outputs are then not valid) and leaves the device
   usable; the wait for copies still in flight when the kernel exits keeps
   its own 2 s limit.  A waiting thread is suspended until the awaited
   event happens, so the limit bounds waits for events that do not happen;
   below 20 us the start-up wait (every role waiting for the first copy to
   be issued) tests without suspending, so a tiny limit runs out there.
   Tests use a tiny limit to drive that error path without a fault.  The
   LM-head step's waits use the same limit.  After a timeout, start the canvases again with
   eb_sampler_init_canvas (which also clears the row counters a cut-short
   step may leave).  No counterpart in the method. */
int eb_sampler_set_wait_limit(eb_sampler_t* h, uint64_t limit_ns);

/* Bytes of device workspace the handle holds. */
size_t eb_sampler_workspace_bytes(const eb_sampler_t* h);

/* Release the workspace and the handle (NULL is allowed). */
void eb_sampler_destroy(eb_sampler_t* h);

/* Static description of a status code. */
const char* eb_strerror(int code);

/* ABI version (major * 100 + minor). */
int eb_version(void);

#ifdef __cplusplus
}
#endif
#endif
