/*
 * eb_synth.h -- seeded synthetic decoder logits for the sampler's tests and
 * benchmark.  Stands in for the decoder forward pass, which needs trained
 * weights: it produces [B, L, V] logits with the shapes of the model card
 * (canvas of 256 positions, vocabulary of about 262K) and a controllable mix
 * of confident and uncertain positions.
 *
 * This module holds none of the sampler's arithmetic.  Its only randomness is
 * a SplitMix64-style counter hash of (seed, tag, b, s, l, v).  One element
 * function is compiled both for the GPU and for the host with no fused
 * multiply-add contraction, IEEE division and square root, and a log of its
 * own (no libm), so both produce the same bits.
 *
 * Kinds:
 *   EBS_TARGET_BOOST: z = noise_sd * N(0,1) + boost * [v == t_{b,l}], with a
 *     per-position target t fixed over steps, a per-position rank r ~ U(0,1)
 *     fixed over steps, and the position "confident" at step s iff
 *     r < f_b(s) = min(1, f0 + (f1 - f0) * s / e_b), e_b = ramp_base +
 *     ramp_per_canvas * b.  boost ~ U(conf_lo, conf_hi) if confident, else
 *     U(unc_lo, unc_hi), drawn afresh per (b, s, l).
 *   EBS_ZIPF: z = -zipf_scale * ln(rank_{b,l}(v)) + zipf_noise_sd * N(0,1)
 *     + U(boost_lo, boost_hi) * [v == t_{b,l}], with rank_{b,l} a keyed
 *     permutation of [1, V] (4-round Feistel with cycle walking).
 */
#ifndef EB_SYNTH_H
#define EB_SYNTH_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { EBS_TARGET_BOOST = 0, EBS_ZIPF = 1 };
enum { EBS_F32 = 0, EBS_BF16 = 1 };

typedef struct {
  int32_t kind;
  int32_t dtype;
  int32_t B, L, V, num_steps;
  uint64_t seed;
  float f0, f1, ramp_base, ramp_per_canvas;
  float conf_lo, conf_hi, unc_lo, unc_hi, noise_sd;
  float zipf_scale, zipf_noise_sd, boost_lo, boost_hi;
} ebs_params_t;

/* Canvases b0 .. b0+nb-1 (global indices), all L rows, at step s, written
   row-major [nb, L, V] to device memory `out` on `stream` (a cudaStream_t).
   Returns 0 or a CUDA error code. */
int ebs_generate_device(const ebs_params_t* p, int b0, int nb, int s, void* out, void* stream);

/* The same values on the host, rows l0 .. l0+nl-1 of canvases b0 .. b0+nb-1,
   written [nb, nl, V] to host memory `out`.  Returns 0. */
int ebs_generate_host(const ebs_params_t* p, int b0, int nb, int s, int l0, int nl, void* out);

/* Host-side helpers exposed for tests of the generator itself. */
float ebs_log(float x);
uint32_t ebs_target(const ebs_params_t* p, int b, int l);

#ifdef __cplusplus
}
#endif
#endif
