// eb_common.cuh -- definitions shared by the two kernels of a sampler step:
// arguments, the per-(row, segment) partial record and its merge, and the
// 64-logit group reduction.
//
// Quantities, for one position (row) of logits z_0 .. z_{V-1} at temperature
// T (DiffusionGemma model card, "Best practices, 1. Diffusion sampling
// settings": logits are shaped by a temperature falling linearly 0.8 -> 0.4;
// diffusers "DiffusionGemma" page, "Schedulers", "Adaptive stopping"):
//   c2 = log2(e) / T, d_v = (z_v - zmax) c2      (log2 units, d_v <= 0)
//   S = sum_v 2^d_v, W = sum_v 2^d_v d_v,
//   entropy H = ln S - ln2 W / S (nats), max probability pmax = 1 / S.
#pragma once

#include <cuda_bf16.h>

#include "eb_device.cuh"

namespace ebk {

constexpr int kGroup = 64;  // vocabulary ids per Gumbel group (EB_GUMBEL_GROUP)
constexpr int kMaxL = 1024;

enum : uint32_t { kStatusBadToken = 1, kStatusNonFinite = 2, kStatusTimeout = 4 };
enum : int { kF32 = 0, kBF16 = 1 };
enum : int { kRuleEB = 0, kRuleBR = 1, kRuleMI = 2 };

__host__ __device__ constexpr int elt_bytes(int dt) { return dt == kF32 ? 4 : 2; }

// Per-(row, stream-CTA segment) partial, relative to the segment's maximum
// logit zmax: the fp32 sums of the group that holds the maximum (Stop, Wtop)
// kept apart from the sums of everything else (Srest, Wrest), so that the
// finish kernel can replace the top group by an exact recomputation; the
// lowest group holding zmax; and the best Gumbel-perturbed group.
struct Partial {
  float zmax;
  int agrp;
  float Stop, Wtop;
  float Srest, Wrest;
  float gscore;
  int gidx;
};

// What one vocabulary slice contributes to a position (vocabulary-sharded
// logits): sums relative to the slice maximum (d = (z - zmax) c2, log2
// units), its argmax and its part of the draw, with global ids.  40 bytes.
struct SliceRecord {
  double S, W;
  float zmax;
  float gscore;  // best group score of the slice (-inf: none)
  int32_t amax;
  int32_t sample;  // element drawn in the slice's best group (-1: none)
  int32_t pad0, pad1;
};
static_assert(sizeof(SliceRecord) == 40, "slice record layout");

struct StepArgs {
  const void* logits;
  int32_t* canvas;
  uint8_t* committed;
  float* H_out;
  int32_t* amax_out;
  uint8_t* stop_flags;
  Partial* partials;
  int32_t* prev_amax;
  int32_t* stable;
  int32_t* sample;
  float* pmax;
  uint32_t* status;
  int32_t* act_index;  // [B] written by the stream kernel: active index or -1
  int32_t* n_act;      // [1] written by the stream kernel
  int B, L, V, ng, s, N;
  int max_segs;  // stream CTAs that can share one row
  int nw;        // Partial records per (row, stream CTA): its consumer warps
  int G1;        // grid size of the stream kernel (its group split)
  int vec_ok;    // rows start on 16-byte boundaries (vector loads allowed)
  int rule, quota, stability_steps, greedy, stop_enabled;
  int canvas_offset;
  float c2, iT;
  double gamma, tau, theta;
  double eps_edit;  // block refinement editing threshold; < 0: no editing
  int v_off;        // global id of local logit 0 (vocabulary slice; a multiple of 64)
  int V_tot;        // global vocabulary size (renoise range, token check)
  uint32_t key0, key1;
};

// Stream CTA of G that owns group g among NG: the largest c with
// floor(c NG / G) <= g.
__device__ __forceinline__ int cta_of(unsigned long long g, unsigned long long NG, int G) {
  return (int)(((g + 1ull) * (unsigned long long)G - 1ull) / NG);
}
__device__ __forceinline__ unsigned long long range_start(int c, unsigned long long NG, int G) {
  return (unsigned long long)c * NG / (unsigned long long)G;
}

// ---------------------------------------------------------------------------
// Partials
// ---------------------------------------------------------------------------
__device__ __forceinline__ Partial empty_partial() {
  Partial p;
  p.zmax = -INFINITY;
  p.agrp = 0x7fffffff;
  p.Stop = 0.f;
  p.Wtop = 0.f;
  p.Srest = 0.f;
  p.Wrest = 0.f;
  p.gscore = -INFINITY;
  p.gidx = 0x7fffffff;
  return p;
}

// Everything of `o` (top and rest), rescaled from o.zmax to a.zmax
// (>= o.zmax), added to the rest sums of `a`.
__device__ __forceinline__ void add_to_rest(Partial& a, const Partial& o, float c2) {
  const float d = (o.zmax - a.zmax) * c2;
  const float f = ex2(d);
  const float S = o.Stop + o.Srest;
  const float W = o.Wtop + o.Wrest;
  a.Srest = fmaf(f, S, a.Srest);
  a.Wrest = fmaf(f, fmaf(d, S, W), a.Wrest);
}

__device__ __forceinline__ void merge(Partial& a, const Partial& b, float c2) {
  if (b.gscore > a.gscore || (b.gscore == a.gscore && b.gidx < a.gidx)) {
    a.gscore = b.gscore;
    a.gidx = b.gidx;
  }
  if (!(b.zmax > -INFINITY)) return;
  if (!(a.zmax > -INFINITY)) {
    const float gs = a.gscore;
    const int gi = a.gidx;
    a = b;
    a.gscore = gs;
    a.gidx = gi;
    return;
  }
  const bool b_top = b.zmax > a.zmax || (b.zmax == a.zmax && b.agrp < a.agrp);
  if (b_top) {
    Partial t = b;
    t.gscore = a.gscore;
    t.gidx = a.gidx;
    add_to_rest(t, a, c2);
    a = t;
  } else {
    add_to_rest(a, b, c2);
  }
}

__device__ __forceinline__ Partial shfl_partial(const Partial& p, int mask_lane) {
  Partial q;
  q.zmax = __shfl_xor_sync(0xffffffffu, p.zmax, mask_lane);
  q.agrp = __shfl_xor_sync(0xffffffffu, p.agrp, mask_lane);
  q.Stop = __shfl_xor_sync(0xffffffffu, p.Stop, mask_lane);
  q.Wtop = __shfl_xor_sync(0xffffffffu, p.Wtop, mask_lane);
  q.Srest = __shfl_xor_sync(0xffffffffu, p.Srest, mask_lane);
  q.Wrest = __shfl_xor_sync(0xffffffffu, p.Wrest, mask_lane);
  q.gscore = __shfl_xor_sync(0xffffffffu, p.gscore, mask_lane);
  q.gidx = __shfl_xor_sync(0xffffffffu, p.gidx, mask_lane);
  return q;
}

// All lanes end with the merge of all 32 partials.  The merge is
// commutative up to rounding; maxima, argmax groups and Gumbel winners are
// order independent.
__device__ __forceinline__ void warp_merge(Partial& p, float c2) {
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    Partial q = shfl_partial(p, o);
    merge(p, q, c2);
  }
}

// ---------------------------------------------------------------------------
// Packed arithmetic and group reductions
// ---------------------------------------------------------------------------
// Lane-wise maximum of two packed bf16 pairs.
__device__ __forceinline__ uint32_t bf16x2_max(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Packed fp32 pair arithmetic (sm_100): one instruction for two lanes.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 r;
  asm("{\n\t.reg .b64 a, b, c, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "mov.b64 c, {%6, %7};\n\tfma.rn.f32x2 d, a, b, c;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return r;
}

__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 r;
  asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "add.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}

// One pair of logits: d = z c2 - r c2, p = 2^d, S += p, W += p d.  An element
// equal to the reference r gets d = the rounding residue of r c2 rather than
// 0; the finish kernel recomputes the group holding the row maximum exactly.
__device__ __forceinline__ void acc_pair(float2 z, float2 c2v, float2 nmc, float2& S, float2& W) {
  const float2 d = ffma2(z, c2v, nmc);
  float2 p;
  p.x = ex2(d.x);
  p.y = ex2(d.y);
  S = fadd2(S, p);
  W = ffma2(p, d, W);
}

__device__ __forceinline__ float sum4(const float2 (&v)[4]) {
  return ((v[0].x + v[0].y) + (v[1].x + v[1].y)) + ((v[2].x + v[2].y) + (v[3].x + v[3].y));
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// ---------------------------------------------------------------------------
// Group reductions.  A consumer lane reduces whole 64-logit groups that sit in
// shared memory.  Max pass: the raw group maximum m_g.  Exponential pass,
// relative to a reference Mref >= m_g: S_g = sum 2^d, W_g = sum 2^d d with
// d = (z - Mref) c2.  Pieces of 16 bytes are read in an order rotated by the
// lane index, so the eight lanes of a shared-memory phase hit eight different
// bank quads.
// ---------------------------------------------------------------------------
template <int DT>
struct GroupIO;

template <>
struct GroupIO<kBF16> {
  static constexpr int kPieces = 8;  // 16-byte pieces per group
  __device__ __forceinline__ static float max_of(const unsigned char* gp, int rot) {
    const uint4* q = reinterpret_cast<const uint4*>(gp);
    uint32_t t[16];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint4 v = q[(k + rot) & 7];
      t[2 * k] = bf16x2_max(v.x, v.y);
      t[2 * k + 1] = bf16x2_max(v.z, v.w);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) t[i] = bf16x2_max(t[2 * i], t[2 * i + 1]);
#pragma unroll
    for (int i = 0; i < 4; ++i) t[i] = bf16x2_max(t[2 * i], t[2 * i + 1]);
    const uint32_t m = bf16x2_max(bf16x2_max(t[0], t[1]), bf16x2_max(t[2], t[3]));
    return fmaxf(bf16_lo(m), bf16_hi(m));
  }
  __device__ __forceinline__ static void exp1_of(const unsigned char* g0, int rot, float c2,
                                                 float r0, float& S0, float& W0) {
    const uint4* q0 = reinterpret_cast<const uint4*>(g0);
    const float2 c2v = make_float2(c2, c2);
    const float2 n0 = make_float2(-r0 * c2, -r0 * c2);
    float2 s0[4], w0[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) s0[i] = w0[i] = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint4 a = q0[(k + rot) & 7];
      const uint32_t wa[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
        acc_pair(make_float2(bf16_lo(wa[i]), bf16_hi(wa[i])), c2v, n0, s0[i], w0[i]);
    }
    S0 = sum4(s0);
    W0 = sum4(w0);
  }
  // Exponential pass of two groups at once (independent chains interleave).
  __device__ __forceinline__ static void exp2_of(const unsigned char* g0, const unsigned char* g1,
                                                 int rot, float c2, float r0, float r1,
                                                 float& S0, float& W0, float& S1, float& W1) {
    const uint4* q0 = reinterpret_cast<const uint4*>(g0);
    const uint4* q1 = reinterpret_cast<const uint4*>(g1);
    const float2 c2v = make_float2(c2, c2);
    const float2 n0 = make_float2(-r0 * c2, -r0 * c2), n1 = make_float2(-r1 * c2, -r1 * c2);
    float2 s0[4], w0[4], s1[4], w1[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      s0[i] = w0[i] = s1[i] = w1[i] = make_float2(0.f, 0.f);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint4 a = q0[(k + rot) & 7];
      const uint4 b = q1[(k + rot) & 7];
      const uint32_t wa[4] = {a.x, a.y, a.z, a.w};
      const uint32_t wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc_pair(make_float2(bf16_lo(wa[i]), bf16_hi(wa[i])), c2v, n0, s0[i], w0[i]);
        acc_pair(make_float2(bf16_lo(wb[i]), bf16_hi(wb[i])), c2v, n1, s1[i], w1[i]);
      }
    }
    S0 = sum4(s0);
    W0 = sum4(w0);
    S1 = sum4(s1);
    W1 = sum4(w1);
  }
};

template <>
struct GroupIO<kF32> {
  __device__ __forceinline__ static void exp1_of(const unsigned char* g0, int rot, float c2,
                                                 float r0, float& S0, float& W0) {
    const float4* q0 = reinterpret_cast<const float4*>(g0);
    const float2 c2v = make_float2(c2, c2);
    const float2 n0 = make_float2(-r0 * c2, -r0 * c2);
    float2 s0[4], w0[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) s0[i] = w0[i] = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const float4 a = q0[(k + rot) & 15];
      acc_pair(make_float2(a.x, a.y), c2v, n0, s0[(2 * k) & 3], w0[(2 * k) & 3]);
      acc_pair(make_float2(a.z, a.w), c2v, n0, s0[(2 * k + 1) & 3], w0[(2 * k + 1) & 3]);
    }
    S0 = sum4(s0);
    W0 = sum4(w0);
  }
  static constexpr int kPieces = 16;
  __device__ __forceinline__ static float max_of(const unsigned char* gp, int rot) {
    const float4* q = reinterpret_cast<const float4*>(gp);
    float t[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const float4 v = q[(k + rot) & 15];
      t[k] = fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w));
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) t[i] = fmaxf(t[2 * i], t[2 * i + 1]);
#pragma unroll
    for (int i = 0; i < 4; ++i) t[i] = fmaxf(t[2 * i], t[2 * i + 1]);
    return fmaxf(fmaxf(t[0], t[1]), fmaxf(t[2], t[3]));
  }
  __device__ __forceinline__ static void exp2_of(const unsigned char* g0, const unsigned char* g1,
                                                 int rot, float c2, float r0, float r1,
                                                 float& S0, float& W0, float& S1, float& W1) {
    const float4* q0 = reinterpret_cast<const float4*>(g0);
    const float4* q1 = reinterpret_cast<const float4*>(g1);
    const float2 c2v = make_float2(c2, c2);
    const float2 n0 = make_float2(-r0 * c2, -r0 * c2), n1 = make_float2(-r1 * c2, -r1 * c2);
    float2 s0[2], w0[2], s1[2], w1[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      s0[i] = w0[i] = s1[i] = w1[i] = make_float2(0.f, 0.f);
    }
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const float4 a = q0[(k + rot) & 15];
      const float4 b = q1[(k + rot) & 15];
      acc_pair(make_float2(a.x, a.y), c2v, n0, s0[0], w0[0]);
      acc_pair(make_float2(a.z, a.w), c2v, n0, s0[1], w0[1]);
      acc_pair(make_float2(b.x, b.y), c2v, n1, s1[0], w1[0]);
      acc_pair(make_float2(b.z, b.w), c2v, n1, s1[1], w1[1]);
    }
    S0 = (s0[0].x + s0[0].y) + (s0[1].x + s0[1].y);
    W0 = (w0[0].x + w0[0].y) + (w0[1].x + w0[1].y);
    S1 = (s1[0].x + s1[0].y) + (s1[1].x + s1[1].y);
    W1 = (w1[0].x + w1[0].y) + (w1[1].x + w1[1].y);
  }
};

template <int DT>
__device__ __forceinline__ float load_elem(const void* p, int e) {
  if (DT == kF32) return reinterpret_cast<const float*>(p)[e];
  return __uint_as_float((uint32_t) reinterpret_cast<const uint16_t*>(p)[e] << 16);
}

// Any group element by element (a partial last group of a row, rows that are
// not 16-byte aligned, or a group whose fast-path sums were not finite).
template <int DT>
__device__ __noinline__ float group_max_safe(const void* gp, int glen) {
  float m = -INFINITY;
  for (int e = 0; e < glen; ++e) m = fmaxf(m, load_elem<DT>(gp, e));
  return m;
}

// Sums relative to the reference r over the elements whose term is nonzero,
// so that a -inf logit contributes nothing (rather than 0 * -inf).
template <int DT>
__device__ __noinline__ float2 group_sums_safe(const void* gp, int glen, float c2, float r) {
  float S = 0.f, W = 0.f;
  if (r > -INFINITY) {
    for (int e = 0; e < glen; ++e) {
      const float d = (load_elem<DT>(gp, e) - r) * c2;
      const float p = ex2(d);
      if (p > 0.f) {
        S += p;
        W = fmaf(p, d, W);
      }
    }
  }
  return make_float2(S, W);
}

__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ int warp_min_i(int v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Running state of one warp over the groups of one row segment.  Every lane
// holds the same M (largest logit so far), tgrp (lowest group holding M), R
// (best Gumbel ratio) and gbest (its group); each lane holds its own sums,
// relative to M, of the groups it reduced: those of group tgrp (top) apart
// from all others (rest).  Group j's Gumbel-perturbed log-partition is
// ln Z_j + M / T - ln E_j, with Z_j its S relative to M and E_j = -ln u_j, so
// the winning group is the one with the largest ratio Z_j / E_j.
struct WarpAcc {
  float M, R;
  int tgrp, gbest;
  float Stop, Wtop, Srest, Wrest;
};

__device__ __forceinline__ void warp_reset(WarpAcc& A) {
  A.M = -INFINITY;
  A.R = 0.f;
  A.tgrp = 0x7fffffff;
  A.gbest = 0x7fffffff;
  A.Stop = A.Wtop = A.Srest = A.Wrest = 0.f;
}

// Before the exponential pass of a sub-tile: this lane's largest group
// maximum m_loc (first reached at group j_loc) joins the warp's M.  On a new
// maximum every sum (and R) is rescaled to it, the old top group joins the
// rest, and the lowest group holding the new maximum becomes the top group.
__device__ __forceinline__ void warp_raise(WarpAcc& A, float m_loc, int j_loc, float c2) {
  const float Mn = warp_max_f(fmaxf(A.M, m_loc));
  if (Mn > A.M) {  // warp-uniform
    if (A.M > -INFINITY) {
      const float dd = (A.M - Mn) * c2;
      const float f = ex2(dd);
      const float S = A.Stop + A.Srest;
      const float W = A.Wtop + A.Wrest;
      A.Srest = f * S;
      A.Wrest = f * fmaf(dd, S, W);
      A.R *= f;
    }
    A.Stop = A.Wtop = 0.f;
    A.M = Mn;
    A.tgrp = warp_min_i(m_loc == Mn ? j_loc : 0x7fffffff);
  }
}

// One group's sums (relative to M) into the lane's top or rest.
__device__ __forceinline__ void warp_fold(WarpAcc& A, float S, float W, int j) {
  if (j == A.tgrp) {
    A.Stop = S;
    A.Wtop = W;
  } else {
    A.Srest += S;
    A.Wrest += W;
  }
}

// Gumbel race of one group (Z = its S relative to M, group-stream word x)
// against the lane's running best (Rl, gl), which starts at the warp's R.
// Since E = -ln u >= 1 - u, a group with Z <= R (1 - u) cannot beat R
// (checked with a 1e-4 relative margin): its logarithm is skipped.
__device__ __forceinline__ void lane_race(float& Rl, int& gl, float Z, uint32_t x, int j) {
  if (Z * 1.0001f <= Rl * one_minus_u(x)) return;
  const float E = -logf(uniform_open(x));
  if (Z > Rl * E) {
    Rl = __fdividef(Z, E);
    gl = j;
  }
}

// After the race of a sub-tile: the warp's best ratio (ties: lower group).
__device__ __forceinline__ void warp_race_merge(WarpAcc& A, float Rl, int gl) {
  if (!__any_sync(0xffffffffu, gl != 0x7fffffff)) return;
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const float oR = __shfl_xor_sync(0xffffffffu, Rl, o);
    const int og = __shfl_xor_sync(0xffffffffu, gl, o);
    if (oR > Rl || (oR == Rl && og < gl)) {
      Rl = oR;
      gl = og;
    }
  }
  A.R = Rl;
  A.gbest = gl;
}

// The warp's state as one Partial record (absolute Gumbel score ln R + M/T).
__device__ __forceinline__ Partial warp_record(const WarpAcc& A, float iT) {
  Partial p;
  p.zmax = A.M;
  p.agrp = A.tgrp;
  p.Stop = warp_sum_f(A.Stop);
  p.Wtop = warp_sum_f(A.Wtop);
  p.Srest = warp_sum_f(A.Srest);
  p.Wrest = warp_sum_f(A.Wrest);
  if (A.R > 0.f && A.M > -INFINITY) {
    p.gscore = fmaf(A.M, iT, logf(A.R));
    p.gidx = A.gbest;
  } else {
    p.gscore = -INFINITY;
    p.gidx = 0x7fffffff;
  }
  return p;
}

}  // namespace ebk
