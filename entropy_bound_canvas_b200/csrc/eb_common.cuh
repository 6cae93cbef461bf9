// eb_common.cuh -- definitions shared by the kernels of a sampler step:
// arguments, the running accumulator of a row segment and its merge, the
// 64-logit group reductions (one shared-memory pass for bf16 logits held in
// registers; a polynomial exp2 on the FMA pipe for part of the terms) and
// the exact slow paths.
//
// Quantities, for one position (row) of logits z_0 .. z_{V-1} at temperature
// T (DiffusionGemma model card, "Best practices, 1. Diffusion sampling
// settings": logits are shaped by a temperature falling linearly 0.8 -> 0.4;
// diffusers "DiffusionGemma" page, "Schedulers", "Adaptive stopping"):
//   c2 = log2(e) / T, d_v = (z_v - M) c2 relative to a reference M >= z_v
//   (log2 units, d_v <= 0), S = sum_v 2^d_v, W = sum_v 2^d_v d_v,
//   entropy H = ln S - ln2 W / S (nats), max probability pmax = 1 / S
//   when M is the row maximum.
#pragma once

#include <cuda_bf16.h>

#include "eb_device.cuh"

namespace ebk {

constexpr int kGroup = 64;  // vocabulary ids per Gumbel group (EB_GUMBEL_GROUP)
constexpr int kMaxL = 1024;
constexpr int kNone = 0x7fffffff;

enum : uint32_t { kStatusBadToken = 1, kStatusNonFinite = 2, kStatusTimeout = 4 };
enum : int { kF32 = 0, kBF16 = 1 };
enum : int { kRuleEB = 0, kRuleBR = 1, kRuleMI = 2 };

__host__ __device__ constexpr int elt_bytes(int dt) { return dt == kF32 ? 4 : 2; }

// ---------------------------------------------------------------------------
// Running state of a row segment: a lane's groups, then a warp's, then a
// stream CTA's.  Sums are relative to M, the largest logit seen.  The sums
// of the group holding M (the lowest such group) are kept apart, so that the
// position's final step can replace them by an exact recomputation of that
// group (its elements equal to the row maximum count exactly 1 each, and
// only its smaller elements are summed): a confident row's entropy is then
// not lost in the rounding of a sum near 1.  Gumbel race (two-level draw,
// group level): group j's perturbed log-partition is
// ln Z_j + M / T - ln E_j with Z_j its S relative to M and E_j = -ln u_j,
// so the winning group has the largest ratio R = Z_j / E_j.
// ---------------------------------------------------------------------------
struct Acc {
  float M;       // largest logit seen (-inf: none)
  float tS, tW;  // sums of the top group
  float Sr, Wr;  // sums of every other group
  float R;       // best Gumbel ratio Z_j / E_j relative to M (0: none)
  int tj;        // top group: lowest group holding M (kNone: none)
  int gb;        // group of R (kNone: none)
};

// A stream CTA's record of one row, final for its part of the row: sums
// relative to its maximum M, the exact form of its top group (elements equal
// to M counted, the smaller ones summed), its best Gumbel group and the
// element drawn inside that group.  48 bytes.
struct Rec {
  float M;
  float Sr, Wr;  // every group but the top group
  float tS, tW;  // the top group's elements below M
  float R;       // best Gumbel ratio relative to M (0: none)
  int tn;        // elements of the top group equal to M
  int ta;        // lowest local id holding M (kNone: no finite logit)
  int gb;        // group of R (kNone: none)
  int xs;        // element drawn in group gb (local id; kNone: none)
  int pad0, pad1;
};
static_assert(sizeof(Rec) == 48, "row record layout");

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
  Rec* recs;            // [B * L][max_segs]: per (row, stream CTA) records
  int32_t* row_cnt;     // [B * L]: stream CTAs done with the row (zero between steps)
  SliceRecord* slice_out;  // vocabulary slice: the per-position records (else null)
  int32_t* prev_amax;
  int32_t* stable;
  int32_t* sample;
  float* pmax;
  uint32_t* status;
  int32_t* act_index;  // [B] written by the stream kernel: active index or -1
  int32_t* n_act;      // [1] written by the stream kernel
  int32_t* canvas_cnt;  // [B]: positions of the canvas finished (zero between steps)
  int32_t* sync_cnt;    // [2]: stream CTAs started, exited (zero between steps)
  int run_epilogue;     // the stream kernel runs each finished canvas's decisions
  uint64_t wait_ns;    // limit of the stream kernel's pipeline waits
  int B, L, V, ng, s, N;
  int max_segs;  // stream CTAs that can share one row
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
__host__ __device__ __forceinline__ int cta_of(unsigned long long g, unsigned long long NG, int G) {
  return (int)(((g + 1ull) * (unsigned long long)G - 1ull) / NG);
}
__host__ __device__ __forceinline__ unsigned long long range_start(int c, unsigned long long NG,
                                                                   int G) {
  return (unsigned long long)c * NG / (unsigned long long)G;
}

// ---------------------------------------------------------------------------
// Accumulators
// ---------------------------------------------------------------------------
__device__ __forceinline__ void acc_reset(Acc& a) {
  a.M = -INFINITY;
  a.tS = a.tW = a.Sr = a.Wr = 0.f;
  a.R = 0.f;
  a.tj = a.gb = kNone;
}

// a absorbs b.  The higher maximum (the lower group on equal maxima) keeps
// its top group; the other state joins the rest, rescaled to that maximum.
__device__ __forceinline__ void acc_merge(Acc& a, const Acc& b, float c2) {
  if (!(b.M > -INFINITY)) return;  // b saw no finite logit (and raced no group)
  if (!(a.M > -INFINITY)) {
    a = b;
    return;
  }
  const bool b_top = b.M > a.M || (b.M == a.M && b.tj < a.tj);
  Acc t = b_top ? b : a;
  const Acc o = b_top ? a : b;
  const bool tie = o.M == t.M;
  const float dd = tie ? 0.f : (o.M - t.M) * c2;
  const float f = tie ? 1.f : ex2(dd);
  const float So = o.tS + o.Sr;
  const float Wo = o.tW + o.Wr;
  t.Sr = fmaf(f, So, t.Sr);
  t.Wr = fmaf(f, fmaf(dd, So, Wo), t.Wr);
  const float Ro = o.R * f;
  if (Ro > t.R || (Ro == t.R && Ro > 0.f && o.gb < t.gb)) {
    t.R = Ro;
    t.gb = o.gb;
  }
  a = t;
}

__device__ __forceinline__ Acc shfl_acc(const Acc& p, int lane_mask) {
  Acc q;
  q.M = __shfl_xor_sync(0xffffffffu, p.M, lane_mask);
  q.tS = __shfl_xor_sync(0xffffffffu, p.tS, lane_mask);
  q.tW = __shfl_xor_sync(0xffffffffu, p.tW, lane_mask);
  q.Sr = __shfl_xor_sync(0xffffffffu, p.Sr, lane_mask);
  q.Wr = __shfl_xor_sync(0xffffffffu, p.Wr, lane_mask);
  q.R = __shfl_xor_sync(0xffffffffu, p.R, lane_mask);
  q.tj = __shfl_xor_sync(0xffffffffu, p.tj, lane_mask);
  q.gb = __shfl_xor_sync(0xffffffffu, p.gb, lane_mask);
  return q;
}

// Every lane ends with the merge of the lanes below `width` (a power of two
// <= 32) in a fixed butterfly order, so the result is deterministic.
__device__ __forceinline__ void warp_merge_acc(Acc& p, float c2, int width = 32) {
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    if (o < width) {
      const Acc q = shfl_acc(p, o);
      acc_merge(p, q, c2);
    }
  }
}

// ---------------------------------------------------------------------------
// Packed fp32 pair arithmetic (sm_100): one instruction for two lanes.
// ---------------------------------------------------------------------------
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

__device__ __forceinline__ float2 fsub2(float2 a, float2 b) {
  float2 r;
  asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "sub.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}

// 2^d for a pair on the FMA pipe (the MUFU pipe is the step's busiest; this
// moves part of its work).  Method: d = n + f with n = round(d), found by
// adding and subtracting 1.5 * 2^23 (exact: in base 2 the reduction needs no
// extended-precision constant), f in [-1/2, 1/2]; 2^f = 1 + f q(f) with q a
// degree-4 polynomial fitted to (2^f - 1) / f on [-1/2, 1/2] (weighted least
// squares on Chebyshev nodes, iterated toward equal relative error; maximum
// relative error 9e-8 in exact arithmetic, 1.9e-7 evaluated by fp32 Horner
// steps, against 2^-22 for ex2.approx); 2^n is added to the exponent field
// as an integer.  d is clamped to >= -126, so a term below 2^-126 of the
// reference comes out at most 2^-126 instead of 0 (ex2.approx.ftz gives 0):
// a difference of < 2^-120 relative to S.
__device__ __forceinline__ float2 ex2_poly2(float2 d) {
  d.x = fmaxf(d.x, -126.f);
  d.y = fmaxf(d.y, -126.f);
  const float2 magic = make_float2(12582912.f, 12582912.f);
  const float2 t = fadd2(d, magic);
  const float2 n = fsub2(t, magic);
  const float2 f = fsub2(d, n);
  float2 p = ffma2(make_float2(1.326472731307149e-3f, 1.326472731307149e-3f), f,
                   make_float2(9.671512991189957e-3f, 9.671512991189957e-3f));
  p = ffma2(p, f, make_float2(5.550733581185341e-2f, 5.550733581185341e-2f));
  p = ffma2(p, f, make_float2(2.4022242426872253e-1f, 2.4022242426872253e-1f));
  p = ffma2(p, f, make_float2(6.931470036506653e-1f, 6.931470036506653e-1f));
  p = ffma2(p, f, make_float2(1.f, 1.f));
  p.x = __int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23));
  p.y = __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23));
  return p;
}

__device__ __forceinline__ float sum4(const float2 (&v)[4]) {
  return ((v[0].x + v[0].y) + (v[1].x + v[1].y)) + ((v[2].x + v[2].y) + (v[3].x + v[3].y));
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Lane-wise maximum of two packed bf16 pairs.
__device__ __forceinline__ uint32_t bf16x2_max(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// ---------------------------------------------------------------------------
// bf16 groups held in registers.  A lane reads its group's eight 16-byte
// pieces in an order rotated by its lane index (the eight lanes of a
// shared-memory phase then hit eight different bank quads):
// A[4 k + i] is word i of piece (k + rot) & 7, i.e. elements
// 8 ((k + rot) & 7) + 2 i (low half) and + 1 (high half).
// ---------------------------------------------------------------------------
#ifndef EB_POLY_PER8
#define EB_POLY_PER8 0  // words of every 8 whose exponentials use ex2_poly2
#endif
constexpr int kPolyPer8 = EB_POLY_PER8;

__device__ __forceinline__ void load_group_bf16(const unsigned char* gp, int rot, uint32_t (&A)[32]) {
  const uint4* q = reinterpret_cast<const uint4*>(gp);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint4 v = q[(k + rot) & 7];
    A[4 * k] = v.x;
    A[4 * k + 1] = v.y;
    A[4 * k + 2] = v.z;
    A[4 * k + 3] = v.w;
  }
}

__device__ __forceinline__ float group_max_bf16(const uint32_t (&A)[32]) {
  uint32_t t[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) t[i] = bf16x2_max(A[2 * i], A[2 * i + 1]);
#pragma unroll
  for (int i = 0; i < 8; ++i) t[i] = bf16x2_max(t[2 * i], t[2 * i + 1]);
#pragma unroll
  for (int i = 0; i < 4; ++i) t[i] = bf16x2_max(t[2 * i], t[2 * i + 1]);
  const uint32_t m = bf16x2_max(bf16x2_max(t[0], t[1]), bf16x2_max(t[2], t[3]));
  return fmaxf(bf16_lo(m), bf16_hi(m));
}

// S = sum 2^d, W = sum 2^d d over the group, d = (z - ref) c2 (ref >= every
// element, so every term is <= 1).  An element equal to ref gets d = the
// rounding residue of ref c2 instead of 0: the position's final step
// recomputes the row's top group exactly.  A -inf logit gives 0 * -inf in W;
// for such a group (non-finite sums) the caller reruns the loop with
// CLAMP: every logit below -1e30 is raised to -1e30 first (packed bf16
// maximum), whose term is exactly 0 as well, with a finite d.
template <bool CLAMP = false>
__device__ __forceinline__ void group_sums_bf16(const uint32_t (&A)[32], float c2, float ref,
                                                float& S, float& W) {
  const float2 c2v = make_float2(c2, c2);
  const float2 nrc = make_float2(-ref * c2, -ref * c2);
  float2 s[4], w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) s[i] = w[i] = make_float2(0.f, 0.f);
#pragma unroll
  for (int q = 0; q < 32; ++q) {
    const uint32_t aw = CLAMP ? bf16x2_max(A[q], 0xF149F149u) : A[q];  // -9.96e29 in each half
    const float2 z = make_float2(bf16_lo(aw), bf16_hi(aw));
    const float2 d = ffma2(z, c2v, nrc);
    float2 p;
    if ((q & 7) < kPolyPer8) {
      p = ex2_poly2(d);
    } else {
      p.x = ex2(d.x);
      p.y = ex2(d.y);
    }
    s[q & 3] = fadd2(s[q & 3], p);
    w[q & 3] = ffma2(p, d, w[q & 3]);
  }
  S = sum4(s);
  W = sum4(w);
}

// The sums of two groups relative to one reference, interleaved word by
// word: twice the independent exponentials in flight of one group's loop.
// Per group, the same terms and rules as group_sums_bf16.
__device__ __forceinline__ void group_sums2_bf16(const uint32_t (&A)[32], const uint32_t (&B)[32],
                                                 float c2, float ref, float& SA, float& WA,
                                                 float& SB, float& WB) {
  const float2 c2v = make_float2(c2, c2);
  const float2 nrc = make_float2(-ref * c2, -ref * c2);
  float2 sa[2], wa[2], sb[2], wb[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) sa[i] = wa[i] = sb[i] = wb[i] = make_float2(0.f, 0.f);
#pragma unroll
  for (int q = 0; q < 32; ++q) {
    const float2 za = make_float2(bf16_lo(A[q]), bf16_hi(A[q]));
    const float2 zb = make_float2(bf16_lo(B[q]), bf16_hi(B[q]));
    const float2 da = ffma2(za, c2v, nrc);
    const float2 db = ffma2(zb, c2v, nrc);
    const float2 pa = make_float2(ex2(da.x), ex2(da.y));
    const float2 pb = make_float2(ex2(db.x), ex2(db.y));
    sa[q & 1] = fadd2(sa[q & 1], pa);
    wa[q & 1] = ffma2(pa, da, wa[q & 1]);
    sb[q & 1] = fadd2(sb[q & 1], pb);
    wb[q & 1] = ffma2(pb, db, wb[q & 1]);
  }
  SA = (sa[0].x + sa[0].y) + (sa[1].x + sa[1].y);
  WA = (wa[0].x + wa[0].y) + (wa[1].x + wa[1].y);
  SB = (sb[0].x + sb[0].y) + (sb[1].x + sb[1].y);
  WB = (wb[0].x + wb[0].y) + (wb[1].x + wb[1].y);
}

// Exact form of a group relative to ref >= every element: n = elements equal
// to ref, amin = the lowest of them (kNone if none), S and W over the
// others with d = (z - ref) c2 (the difference is exact for bf16 values of
// like magnitude), skipping zero terms (-inf logits contribute nothing).
struct Exact {
  float S, W;
  int n, amin;
};

__device__ __forceinline__ void exact_elem(float z, int v, float ref, float c2, Exact& e) {
  if (z == ref) {
    ++e.n;
    e.amin = min(e.amin, v);
  } else {
    const float d = (z - ref) * c2;
    const float p = ex2(d);
    if (p > 0.f) {
      e.S += p;
      e.W = fmaf(p, d, e.W);
    }
  }
}

// ---------------------------------------------------------------------------
// Groups read from shared memory: fp32 logits (two 16-byte-vector passes),
// and element by element (a partial last group, rows that are not 16-byte
// aligned).
// ---------------------------------------------------------------------------
template <int DT>
__device__ __forceinline__ float load_elem(const void* p, int e) {
  if (DT == kF32) return reinterpret_cast<const float*>(p)[e];
  return __uint_as_float((uint32_t) reinterpret_cast<const uint16_t*>(p)[e] << 16);
}

template <int DT>
__device__ __noinline__ float elem_max(const void* gp, int len) {
  float m = -INFINITY;
  for (int e = 0; e < len; ++e) m = fmaxf(m, load_elem<DT>(gp, e));
  return m;
}

template <int DT>
__device__ __noinline__ Exact elem_exact(const void* gp, int len, float ref, float c2) {
  Exact e{0.f, 0.f, 0, kNone};
  for (int v = 0; v < len; ++v) exact_elem(load_elem<DT>(gp, v), v, ref, c2, e);
  return e;
}

__device__ __forceinline__ float group_max_f32(const unsigned char* gp, int rot) {
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

__device__ __forceinline__ void group_sums_f32(const unsigned char* gp, int rot, float c2,
                                               float ref, float& S, float& W) {
  const float4* q = reinterpret_cast<const float4*>(gp);
  const float2 c2v = make_float2(c2, c2);
  const float2 nrc = make_float2(-ref * c2, -ref * c2);
  float2 s[4], w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) s[i] = w[i] = make_float2(0.f, 0.f);
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const float4 a = q[(k + rot) & 15];
    const float2 d0 = ffma2(make_float2(a.x, a.y), c2v, nrc);
    const float2 d1 = ffma2(make_float2(a.z, a.w), c2v, nrc);
    const float2 p0 = make_float2(ex2(d0.x), ex2(d0.y));
    const float2 p1 = make_float2(ex2(d1.x), ex2(d1.y));
    s[(2 * k) & 3] = fadd2(s[(2 * k) & 3], p0);
    w[(2 * k) & 3] = ffma2(p0, d0, w[(2 * k) & 3]);
    s[(2 * k + 1) & 3] = fadd2(s[(2 * k + 1) & 3], p1);
    w[(2 * k + 1) & 3] = ffma2(p1, d1, w[(2 * k + 1) & 3]);
  }
  S = sum4(s);
  W = sum4(w);
}

// ---------------------------------------------------------------------------
// A lane's group step
// ---------------------------------------------------------------------------
// Group j (maximum mg > A.M) becomes the lane's top group: the old state is
// rescaled to mg (its top group joins the rest) and the group's sums (S, W),
// relative to mg, become the top sums.  Returns the group's Z = S.
__device__ __forceinline__ float lane_new_top(Acc& A, float mg, int j, float S, float W,
                                              float c2) {
  if (A.M > -INFINITY) {
    const float dd = (A.M - mg) * c2;
    const float f = ex2(dd);
    const float So = A.tS + A.Sr;
    const float Wo = A.tW + A.Wr;
    A.Sr = f * So;
    A.Wr = f * fmaf(dd, So, Wo);
    A.R *= f;
  }
  A.M = mg;
  A.tj = j;
  A.tS = S;
  A.tW = W;
  return S;
}

// Group-level Gumbel race of group j (Z relative to the lane's M, group-stream
// word x).  Since E = -ln u >= 1 - u, a group with Z <= R (1 - u) cannot beat
// R (checked with a 1e-4 relative margin): its logarithm is skipped.  Strict
// comparison: on equal ratios the earlier (lower) group stays.
// Returns true when group j becomes the lane's best.
__device__ __forceinline__ bool lane_race(Acc& A, float Z, uint32_t x, int j) {
  if (Z * 1.0001f <= A.R * one_minus_u(x)) return false;
  const float E = -logf(uniform_open(x));
  if (Z > A.R * E) {
    A.R = __fdividef(Z, E);
    A.gb = j;
    return true;
  }
  return false;
}

}  // namespace ebk
