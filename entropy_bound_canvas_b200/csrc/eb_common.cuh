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
  int B, L, V, ng, s, N, max_segs;
  int G1;      // grid size of the stream kernel (its group split)
  int vec_ok;  // rows start on 16-byte boundaries (vector loads allowed)
  int rule, quota, stability_steps, greedy, stop_enabled;
  int canvas_offset;
  float c2, iT;
  double gamma, tau, theta;
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
struct GroupStat {
  float m;  // raw maximum
  float S;  // sum 2^d, d = (z - m) c2
  float W;  // sum 2^d d
};

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

// One pair of logits: d = z c2 - m c2, p = 2^d, S += p, W += p d.  The
// maximum itself gets d = the rounding residue of m c2 rather than 0; the
// finish kernel recomputes the group holding the argmax exactly.
__device__ __forceinline__ void acc_pair(float2 z, float2 c2v, float2 nmc, float2& S, float2& W) {
  const float2 d = ffma2(z, c2v, nmc);
  float2 p;
  p.x = ex2(d.x);
  p.y = ex2(d.y);
  S = fadd2(S, p);
  W = ffma2(p, d, W);
}

__device__ __forceinline__ float tree8(const float (&v)[8]) {
  return ((v[0] + v[1]) + (v[2] + v[3])) + ((v[4] + v[5]) + (v[6] + v[7]));
}

__device__ __forceinline__ float sum4(const float2 (&v)[4]) {
  return ((v[0].x + v[0].y) + (v[1].x + v[1].y)) + ((v[2].x + v[2].y) + (v[3].x + v[3].y));
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Full 64-element bf16 group in shared memory (128 bytes), read twice (max,
// then exponentials) to keep register use low.  Pieces of 16 bytes are read
// in an order rotated by the thread index so that the eight threads of a
// shared-memory phase hit eight different bank quads.
__device__ __forceinline__ GroupStat group_bf16_full(const unsigned char* gp, int rot, float c2) {
  const uint4* q = reinterpret_cast<const uint4*>(gp);
  uint32_t mx0, mx1;
  {
    const uint4 v = q[rot & 7];
    mx0 = bf16x2_max(v.x, v.y);
    mx1 = bf16x2_max(v.z, v.w);
  }
#pragma unroll
  for (int k = 1; k < 8; ++k) {
    const uint4 v = q[(k + rot) & 7];
    mx0 = bf16x2_max(mx0, bf16x2_max(v.x, v.y));
    mx1 = bf16x2_max(mx1, bf16x2_max(v.z, v.w));
  }
  const uint32_t mx = bf16x2_max(mx0, mx1);
  const float m = fmaxf(bf16_lo(mx), bf16_hi(mx));
  const float2 c2v = make_float2(c2, c2);
  const float2 nmc = make_float2(-m * c2, -m * c2);

  float2 S[4], W[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    S[i] = make_float2(0.f, 0.f);
    W[i] = make_float2(0.f, 0.f);
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint4 v = q[(k + rot) & 7];
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      acc_pair(make_float2(bf16_lo(w4[i]), bf16_hi(w4[i])), c2v, nmc, S[i], W[i]);
  }
  GroupStat g;
  g.m = m;
  g.S = sum4(S);
  g.W = sum4(W);
  return g;
}

// Full 64-element fp32 group in shared memory (256 bytes), read twice.
__device__ __forceinline__ GroupStat group_f32_full(const unsigned char* gp, int rot, float c2) {
  const float4* q = reinterpret_cast<const float4*>(gp);
  float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const float4 v = q[(k + rot) & 15];
    m0 = fmaxf(m0, fmaxf(v.x, v.y));
    m1 = fmaxf(m1, fmaxf(v.z, v.w));
  }
  const float m = fmaxf(m0, m1);
  const float2 c2v = make_float2(c2, c2);
  const float2 nmc = make_float2(-m * c2, -m * c2);
  float2 S[4], W[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    S[i] = make_float2(0.f, 0.f);
    W[i] = make_float2(0.f, 0.f);
  }
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const float4 v = q[(k + rot) & 15];
    acc_pair(make_float2(v.x, v.y), c2v, nmc, S[(2 * k) & 3], W[(2 * k) & 3]);
    acc_pair(make_float2(v.z, v.w), c2v, nmc, S[(2 * k + 1) & 3], W[(2 * k + 1) & 3]);
  }
  GroupStat g;
  g.m = m;
  g.S = sum4(S);
  g.W = sum4(W);
  return g;
}

template <int DT>
__device__ __forceinline__ float load_elem(const void* p, int e) {
  if (DT == kF32) return reinterpret_cast<const float*>(p)[e];
  return __uint_as_float((uint32_t) reinterpret_cast<const uint16_t*>(p)[e] << 16);
}

// Any group (partial last group of a row, or unaligned rows): element by
// element through a generic pointer (shared or global memory).
template <int DT>
__device__ __noinline__ GroupStat group_scalar(const void* gp, int glen, float c2) {
  float m = -INFINITY;
  for (int e = 0; e < glen; ++e) m = fmaxf(m, load_elem<DT>(gp, e));
  float s[8], ws[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    s[i] = 0.f;
    ws[i] = 0.f;
  }
  for (int e = 0; e < glen; ++e) {
    const float d = (load_elem<DT>(gp, e) - m) * c2;
    const float p = ex2(d);
    s[e & 7] += p;
    ws[e & 7] = fmaf(p, d, ws[e & 7]);
  }
  GroupStat g;
  g.m = m;
  g.S = tree8(s);
  g.W = tree8(ws);
  return g;
}

// Fold one group into a thread's running partial (a thread sees the groups
// of a row segment in increasing index order, so a tie never moves the
// maximum's group).
__device__ __forceinline__ void fold_group(Partial& t, const GroupStat& g, int j, float c2) {
  if (g.m > t.zmax) {
    if (t.zmax > -INFINITY) {
      const float d = (t.zmax - g.m) * c2;
      const float f = ex2(d);
      const float S = t.Stop + t.Srest;
      const float W = t.Wtop + t.Wrest;
      t.Srest = f * S;
      t.Wrest = f * fmaf(d, S, W);
    }
    t.Stop = g.S;
    t.Wtop = g.W;
    t.zmax = g.m;
    t.agrp = j;
  } else {
    const float d = (g.m - t.zmax) * c2;
    const float f = ex2(d);
    t.Srest = fmaf(f, g.S, t.Srest);
    t.Wrest = fmaf(f, fmaf(d, g.S, g.W), t.Wrest);
  }
}

}  // namespace ebk
