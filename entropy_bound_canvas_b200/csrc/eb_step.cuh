// eb_step.cuh -- the fused sampler step kernel.
//
// One launch performs one denoising step for every active canvas:
//   stream every logit of every active canvas once (HBM -> shared memory by
//   1-D bulk copies), reduce each 64-logit vocabulary group to its maximum,
//   sum of 2^d and sum of 2^d d (d = (z - max) log2(e) / T) and, for open
//   positions, a Gumbel-perturbed group log-partition; merge groups into
//   per-row partials; the last CTA to finish a row combines its partials into
//   the entropy, argmax, max probability and categorical draw; the last row
//   of a canvas runs the canvas epilogue (adaptive stop, commit rule,
//   renoise).  Cross-CTA hand-off uses atomic tickets only: no CTA ever waits
//   for another.
//
// Work split: the active rows' groups are numbered g = row * ng + j and CTA c
// of G owns the contiguous range [c NG / G, (c + 1) NG / G), processed in
// tiles of up to 128 groups that never straddle a row.  Every CTA therefore
// streams the same number of bytes (to within one group).
//
// Roles inside a CTA: warp 4 lane 0 issues the bulk copies into a ring of
// kStages tiles; warps 0-3 (128 "consumer" threads) each reduce one group of
// every tile.
//
// Source of the arithmetic (pages cited by title and section): DiffusionGemma
// model card, "Best practices, 1. Diffusion sampling settings" (temperature
// schedule, lowest-entropy selection under entropy_bound, full renoise,
// adaptive stop); diffusers "DiffusionGemma" pipeline page, "Schedulers"
// (entropy-bound and block-refinement commit, t_max -> t_min), "Adaptive
// stopping" (stability_threshold, confidence_threshold on the scheduler-
// shaped logits).
#pragma once

#include <cuda_bf16.h>

#include "eb_device.cuh"

namespace ebk {

constexpr int kGroup = 64;
constexpr int kConsumerWarps = 4;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;
constexpr int kTileGroups = kConsumers;
constexpr int kStages = 3;
constexpr int kMaxL = 1024;

enum : uint32_t { kStatusBadToken = 1, kStatusNonFinite = 2, kStatusTimeout = 4 };
enum : int { kF32 = 0, kBF16 = 1 };
enum : int { kRuleEB = 0, kRuleBR = 1, kRuleMI = 2 };

__host__ __device__ constexpr int elt_bytes(int dt) { return dt == kF32 ? 4 : 2; }
__host__ __device__ constexpr int tile_bytes(int dt) { return kTileGroups * kGroup * elt_bytes(dt); }

// Per-(row, CTA segment) partial, relative to the segment's maximum logit
// zmax with d = (z - zmax) c2 (log2 units): the fp32 sums of the group that
// holds the argmax (Stop = sum 2^d, Wtop = sum 2^d d) kept apart from the sums
// of everything else (Srest, Wrest), so that the row combine can replace the
// top group by an exact recomputation; plus the best Gumbel group.
struct Partial {
  float zmax;
  int agrp;  // lowest group index holding zmax
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
  uint32_t* row_ticket;
  uint32_t* canvas_ticket;
  uint32_t* exit_ticket;
  int32_t* prev_amax;
  int32_t* stable;
  int32_t* sample;
  float* pmax;
  uint8_t* stop_next;
  uint32_t* status;
  int B, L, V, ng, s, N, max_segs;
  int rule, quota, stability_steps, greedy, stop_enabled;
  int canvas_offset;
  float c2, iT;
  double gamma, tau, theta;
  uint32_t key0, key1;
};

struct Ctrl {
  int n_act;
  int abort;
  int issued;
  int row_last;
  int canvas_last;
  int exit_last;
  int kpref;
  int pad;
  int wcnt[kThreads / 32];
  double dscr[kConsumerWarps];
  int iscr[kConsumerWarps];
  unsigned long long uscr[kConsumerWarps];
};

struct Layout {
  uint32_t bars, ctrl, red, act, keys, skeys, pick, ring, total;
};

__host__ __device__ inline uint32_t align_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline Layout make_layout(int dt, int B, int L) {
  Layout y;
  uint32_t o = 0;
  y.bars = o;
  o = align_up(o + 16u * kStages, 16);
  y.ctrl = o;
  o = align_up(o + (uint32_t)sizeof(Ctrl), 16);
  y.red = o;
  o = align_up(o + (uint32_t)sizeof(Partial) * kConsumerWarps, 16);
  y.act = o;
  o = align_up(o + 2u * (uint32_t)B, 16);
  y.keys = o;
  o = align_up(o + 8u * (uint32_t)L, 16);
  y.skeys = o;
  o = align_up(o + 8u * (uint32_t)L, 16);
  y.pick = o;
  o = align_up(o + (uint32_t)L, 128);
  y.ring = o;
  o += (uint32_t)kStages * (uint32_t)tile_bytes(dt);
  y.total = o;
  return y;
}

// CTA of G that owns group g among NG: the largest c with floor(c NG / G) <= g.
__device__ __forceinline__ int cta_of(unsigned long long g, unsigned long long NG, int G) {
  return (int)(((g + 1ull) * (unsigned long long)G - 1ull) / NG);
}
__device__ __forceinline__ unsigned long long range_start(int c, unsigned long long NG, int G) {
  return (unsigned long long)c * NG / (unsigned long long)G;
}

struct Tile {
  long long r;  // active row index
  int j0;       // first group of the tile within the row
  int cnt;      // groups in the tile
  int ai;       // index of the row's canvas in the active list
  int l;        // position of the row
};

// Walks a CTA's group range tile by tile; divides only once, at the start.
struct TileIter {
  unsigned long long g, g_hi;
  int ng, L;
  long long r;
  int j0, ai, l;
  __device__ __forceinline__ TileIter(unsigned long long lo, unsigned long long hi, int ng_, int L_)
      : g(lo), g_hi(hi), ng(ng_), L(L_) {
    r = (long long)(lo / (unsigned long long)ng_);
    j0 = (int)(lo - (unsigned long long)r * (unsigned long long)ng_);
    ai = (int)(r / L_);
    l = (int)(r - (long long)ai * L_);
  }
  __device__ __forceinline__ bool next(Tile& t) {
    if (g >= g_hi) return false;
    int cnt = ng - j0;
    if (cnt > kTileGroups) cnt = kTileGroups;
    if ((unsigned long long)cnt > g_hi - g) cnt = (int)(g_hi - g);
    t.r = r;
    t.j0 = j0;
    t.cnt = cnt;
    t.ai = ai;
    t.l = l;
    g += (unsigned long long)cnt;
    j0 += cnt;
    if (j0 == ng) {
      j0 = 0;
      ++r;
      if (++l == L) {
        l = 0;
        ++ai;
      }
    }
    return true;
  }
};

// ---------------------------------------------------------------------------
// Partials: merge and warp reduction
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

// Everything of `o` (top and rest), rescaled from o.zmax to zmax, added to
// the rest sums of `a` (whose maximum zmax >= o.zmax).
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

// All lanes end with the merge of all 32 partials.  merge() is commutative
// up to rounding; the argmax and Gumbel winners are order independent.
__device__ __forceinline__ void warp_merge(Partial& p, float c2) {
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    Partial q = shfl_partial(p, o);
    merge(p, q, c2);
  }
}

// ---------------------------------------------------------------------------
// Group reductions
// ---------------------------------------------------------------------------
struct GroupStat {
  float m;    // raw maximum
  float S;    // sum 2^d, d = (z - m) c2
  float W;    // sum 2^d d
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

// Accumulates one pair of logits: d = z c2 - m c2, p = 2^d, S += p, W += p d.
// The maximum itself gets d = the rounding residue of m c2 rather than 0;
// the row combine recomputes the group holding the argmax exactly.
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
  const float m = fmaxf(__uint_as_float(mx << 16), __uint_as_float(mx & 0xffff0000u));
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
    for (int i = 0; i < 4; ++i) {
      const float2 z = make_float2(__uint_as_float(w4[i] << 16), __uint_as_float(w4[i] & 0xffff0000u));
      acc_pair(z, c2v, nmc, S[i], W[i]);
    }
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

// Fold one group into a thread's running partial (groups arrive in
// increasing index order within a row segment, so a tie never moves the
// argmax).
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

// ---------------------------------------------------------------------------
// 128-thread block helpers (consumer warps, named barrier 1)
// ---------------------------------------------------------------------------
__device__ __forceinline__ double block_sum(double v, Ctrl* c, int tid) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((tid & 31) == 0) c->dscr[tid >> 5] = v;
  consumer_sync(kConsumers);
  const double r = (c->dscr[0] + c->dscr[1]) + (c->dscr[2] + c->dscr[3]);
  consumer_sync(kConsumers);
  return r;
}

__device__ __forceinline__ int block_sum_int(int v, Ctrl* c, int tid) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((tid & 31) == 0) c->iscr[tid >> 5] = v;
  consumer_sync(kConsumers);
  const int r = c->iscr[0] + c->iscr[1] + c->iscr[2] + c->iscr[3];
  consumer_sync(kConsumers);
  return r;
}

__device__ __forceinline__ unsigned long long block_min_u64(unsigned long long v, Ctrl* c,
                                                            int tid) {
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const unsigned long long w = __shfl_xor_sync(0xffffffffu, v, o);
    v = w < v ? w : v;
  }
  if ((tid & 31) == 0) c->uscr[tid >> 5] = v;
  consumer_sync(kConsumers);
  unsigned long long r = c->uscr[0];
  for (int i = 1; i < kConsumerWarps; ++i) r = c->uscr[i] < r ? c->uscr[i] : r;
  consumer_sync(kConsumers);
  return r;
}

// Exclusive prefix of v over the 128 threads; *total gets the sum.
__device__ __forceinline__ int block_excl_scan(int v, Ctrl* c, int tid, int* total) {
  const int lane = tid & 31;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) c->iscr[tid >> 5] = x;
  consumer_sync(kConsumers);
  int off = 0, tot = 0;
  for (int i = 0; i < kConsumerWarps; ++i) {
    if (i < (tid >> 5)) off += c->iscr[i];
    tot += c->iscr[i];
  }
  consumer_sync(kConsumers);
  *total = tot;
  return off + x - v;
}

// Sort key of an entropy (>= 0, so its float bits order like the value) and
// its position: ascending (H, l).
__device__ __forceinline__ unsigned long long key_asc(float H, int l) {
  const float h = H > 0.f ? H : 0.f;
  return ((unsigned long long)__float_as_uint(h) << 32) | (unsigned)l;
}
// Descending probability, ascending position.
__device__ __forceinline__ unsigned long long key_desc(float p, int l) {
  const float q = p > 0.f ? p : 0.f;
  return ((unsigned long long)(~__float_as_uint(q)) << 32) | (unsigned)l;
}

// ---------------------------------------------------------------------------
// Canvas epilogue: stability, adaptive stop, commit rule, finalisation,
// renoise.  Runs on the 128 consumer threads of the CTA that completed the
// canvas's last row.  Kept compact (positions in rolled loops, values
// re-read from L2) because it runs from a cold instruction cache.
// ---------------------------------------------------------------------------
__device__ __noinline__ void canvas_epilogue(const StepArgs a, int bi, Ctrl* ctrl,
                                             unsigned long long* keys, unsigned long long* skeys,
                                             uint8_t* pick, int tid) {
  const int L = a.L;
  const size_t row0 = (size_t)bi * (size_t)L;
  const int lane = tid & 31, warp = tid >> 5;
  const bool br = a.rule == kRuleBR;

  // Pass 1: entropy sum, argmax stability, candidate counts.
  double sumH = 0.0;
  int neq = a.s < 1 ? 1 : 0;
  int ncand = 0;
#pragma unroll 1
  for (int l = tid; l < L; l += kConsumers) {
    const float H = __ldcg(a.H_out + row0 + l);
    const int am = __ldcg(a.amax_out + row0 + l);
    const bool open = a.committed[row0 + l] == 0;
    pick[l] = 0;
    sumH += (double)H;
    if (a.s >= 1 && am != a.prev_amax[row0 + l]) neq = 1;
    if (!open) {
      const int tok = a.canvas[row0 + l];
      if (tok < 0 || tok >= a.V) atomicOr(a.status, kStatusBadToken);
    } else if (!br) {
      ncand += (double)H <= a.gamma ? 1 : 0;
    } else if ((double)__ldcg(a.pmax + row0 + l) >= a.theta) {
      pick[l] = 1;
    } else {
      ++ncand;
    }
  }
  const double totH = block_sum(sumH, ctrl, tid);
  const int any_neq = block_sum_int(neq, ctrl, tid);
  const int stable_new = any_neq ? 0 : a.stable[bi] + 1;
  const double meanH = totH / (double)L;
  const bool fired = a.stop_enabled && stable_new >= a.stability_steps && meanH < a.tau;
  const bool last_step = a.s == a.N - 1;

  if (!fired) {
    // Candidates: EB -- open positions with H <= gamma (no other can be in the
    // prefix); BR -- open positions below the threshold (quota competitors).
    int n_c = 0;
    int pos = block_excl_scan(ncand, ctrl, tid, &n_c);
#pragma unroll 1
    for (int l = tid; l < L; l += kConsumers) {
      if (a.committed[row0 + l] != 0) continue;
      if (!br) {
        const float H = __ldcg(a.H_out + row0 + l);
        if ((double)H <= a.gamma) keys[pos++] = key_asc(H, l);
      } else {
        const float p = __ldcg(a.pmax + row0 + l);
        if (!((double)p >= a.theta)) keys[pos++] = key_desc(p, l);
      }
    }
    consumer_sync(kConsumers);
#pragma unroll 1
    for (int c = tid; c < n_c; c += kConsumers) {
      const unsigned long long kc = keys[c];
      int rank = 0;
#pragma unroll 4
      for (int j = 0; j < n_c; ++j) rank += keys[j] < kc;
      if (!br) skeys[rank] = kc;
      else if (rank < a.quota) pick[(int)(kc & 0xffffffffu)] = 1;
    }
    consumer_sync(kConsumers);
    if (!br) {
      // Longest prefix of the sorted candidates with cumulative H <= gamma.
      if (warp == 0) {
        const int chunk = (n_c + 31) / 32;
        const int lo = lane * chunk;
        const int hi = lo + chunk < n_c ? lo + chunk : n_c;
        double part = 0.0;
        for (int i = lo; i < hi; ++i) part += (double)__uint_as_float((uint32_t)(skeys[i] >> 32));
        double x = part;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const double y = __shfl_up_sync(0xffffffffu, x, o);
          if (lane >= o) x += y;
        }
        double cum = x - part;
        int cnt = 0;
        for (int i = lo; i < hi; ++i) {
          cum += (double)__uint_as_float((uint32_t)(skeys[i] >> 32));
          if (cum <= a.gamma) ++cnt;
          else break;
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
        if (lane == 0) ctrl->kpref = cnt;
      }
      consumer_sync(kConsumers);
      const int kpref = ctrl->kpref;
      for (int i = tid; i < kpref; i += kConsumers) pick[(int)(skeys[i] & 0xffffffffu)] = 1;
      // EB with an empty prefix: the single lowest (H, l).  MI: the prefix
      // plus the next position in (H, l) order.
      const bool mi = a.rule == kRuleMI;
      if (mi && kpref < n_c) {
        if (tid == 0) pick[(int)(skeys[kpref] & 0xffffffffu)] = 1;
      } else if (kpref == 0 || mi) {
        unsigned long long best = ~0ull;
#pragma unroll 1
        for (int l = tid; l < L; l += kConsumers) {
          if (a.committed[row0 + l] != 0) continue;
          const float H = __ldcg(a.H_out + row0 + l);
          if (mi && (double)H <= a.gamma) continue;
          const unsigned long long kk = key_asc(H, l);
          best = kk < best ? kk : best;
        }
        best = block_min_u64(best, ctrl, tid);
        if (tid == 0 && best != ~0ull) pick[(int)(best & 0xffffffffu)] = 1;
      }
    }
    consumer_sync(kConsumers);
  }

  // Final pass: commit, renoise, remember the argmax.
  const uint32_t bg = (uint32_t)(a.canvas_offset + bi);
  int left = 0;
#pragma unroll 1
  for (int l = tid; l < L; l += kConsumers) {
    const int am = __ldcg(a.amax_out + row0 + l);
    if (a.committed[row0 + l] == 0) {
      if (fired) {
        a.canvas[row0 + l] = am;
        a.committed[row0 + l] = 1;
      } else if (pick[l] || last_step) {
        a.canvas[row0 + l] = a.greedy ? am : __ldcg(a.sample + row0 + l);
        a.committed[row0 + l] = 1;
      } else {
        ++left;
        const Words4 r = philox((uint32_t)l >> 2, 0u, (uint32_t)a.s, bg | (kStreamRenoise << 24),
                                a.key0, a.key1);
        a.canvas[row0 + l] = (int32_t)uniform_token(pick_word(r, (uint32_t)l & 3u), (uint32_t)a.V);
      }
    }
    a.prev_amax[row0 + l] = am;
  }
  const int left_tot = block_sum_int(left, ctrl, tid);
  if (tid == 0) {
    a.stable[bi] = stable_new;
    a.stop_next[bi] = (uint8_t)(fired ? 1 : last_step ? 3 : left_tot == 0 ? 2 : 0);
  }
}

// ---------------------------------------------------------------------------
// Row combine: merge the row's partials, recompute the argmax group exactly,
// draw the categorical sample.  Runs on warp 0 of the CTA that completed the
// row.  Returns (in lane 0) whether this row completed its canvas.
// ---------------------------------------------------------------------------
template <int DT>
__device__ __noinline__ bool row_combine(const StepArgs a, unsigned long long r, int bi, int l,
                            unsigned long long NG, int lane) {
  const size_t grow = (size_t)bi * (size_t)a.L + (size_t)l;
  const int G = gridDim.x;
  const unsigned long long g_first = r * (unsigned long long)a.ng;
  const int c_first = cta_of(g_first, NG, G);
  const int c_last = cta_of(g_first + (unsigned long long)a.ng - 1ull, NG, G);
  Partial R = empty_partial();
  for (int i = lane; i <= c_last - c_first; i += 32) {
    const int c = c_first + i;
    if (range_start(c, NG, G) < range_start(c + 1, NG, G)) {
      const Partial* src = a.partials + grow * (size_t)a.max_segs + (size_t)i;
      Partial q;
      q.zmax = __ldcg(&src->zmax);
      q.agrp = __ldcg(&src->agrp);
      q.Stop = __ldcg(&src->Stop);
      q.Wtop = __ldcg(&src->Wtop);
      q.Srest = __ldcg(&src->Srest);
      q.Wrest = __ldcg(&src->Wrest);
      q.gscore = __ldcg(&src->gscore);
      q.gidx = __ldcg(&src->gidx);
      merge(R, q, a.c2);
    }
  }
  warp_merge(R, a.c2);

  const char* rowp = reinterpret_cast<const char*>(a.logits) + grow * (size_t)a.V * elt_bytes(DT);
  // Exact (f64) recomputation of the group holding the argmax: its fp32 sums
  // (Stop, Wtop) carry the maximum's own term, whose rounding would dominate
  // the entropy of a confident row, and are replaced.
  // Exact recomputation of the group holding the argmax: its fp32 sums
  // (Stop, Wtop) carry the maximum's own term, whose rounding would dominate
  // the entropy of a confident row.  Here every element equal to the maximum
  // contributes exactly 1 (d = (z - zmax) c2 = 0) and is counted apart from
  // the smaller terms, which keep full relative precision.
  const int jt = R.agrp;
  float ss = 0.f, wsum = 0.f;
  int nmax = 0;
  int am = 0x7fffffff;  // lowest index of the maximum (it lies in the top group)
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int v = jt * kGroup + lane + 32 * h;
    if (v < a.V) {
      const float z = load_elem<DT>(rowp, v);
      const float d = (z - R.zmax) * a.c2;
      if (d == 0.f) {
        ++nmax;
        am = min(am, v);
      } else {
        const float p = ex2(d);
        ss += p;
        wsum = fmaf(p, d, wsum);
      }
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
    wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
    nmax += __shfl_xor_sync(0xffffffffu, nmax, o);
    am = min(am, __shfl_xor_sync(0xffffffffu, am, o));
  }
  const double S = (double)nmax + ((double)ss + (double)R.Srest);
  const double W = (double)wsum + (double)R.Wrest;
  const double H = log(S) - 0.6931471805599453 * (W / S);

  const bool open = a.committed[grow] == 0;
  int smp = -1;
  if (open) {
    if (a.greedy || R.gidx == 0x7fffffff) {
      smp = am;
    } else {
      // Element-level Gumbel-max inside the winning group.
      const uint32_t bg = (uint32_t)(a.canvas_offset + bi);
      float best = -INFINITY;
      int barg = 0x7fffffff;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int v = R.gidx * kGroup + lane + 32 * h;
        if (v < a.V) {
          const Words4 w = philox((uint32_t)v >> 2, (uint32_t)l, (uint32_t)a.s,
                                  bg | (kStreamGumbel << 24), a.key0, a.key1);
          const float sc = load_elem<DT>(rowp, v) * a.iT + gumbel(pick_word(w, (uint32_t)v & 3u));
          if (sc > best || (sc == best && v < barg)) {
            best = sc;
            barg = v;
          }
        }
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int oa = __shfl_xor_sync(0xffffffffu, barg, o);
        if (ob > best || (ob == best && oa < barg)) {
          best = ob;
          barg = oa;
        }
      }
      smp = barg;
    }
  }
  bool canvas_done = false;
  if (lane == 0) {
    a.H_out[grow] = (float)H;
    a.amax_out[grow] = am;
    a.sample[grow] = smp;
    a.pmax[grow] = (float)(1.0 / S);
    if (!isfinite(S) || !isfinite(W)) atomicOr(a.status, kStatusNonFinite);
    __threadfence();
    const unsigned old = atomicAdd(a.canvas_ticket + bi, 1u);
    if (old == (unsigned)a.L - 1u) {
      a.canvas_ticket[bi] = 0u;
      __threadfence();
      canvas_done = true;
    }
  }
  return canvas_done;
}

// End of a row segment: reduce the 128 thread partials, publish the CTA's
// partial for the row, take a ticket; the CTA that completes the row combines
// it, and the one that completes the canvas runs the canvas epilogue.
template <int DT>
__device__ __forceinline__ void flush_segment(const StepArgs& a, Partial& acc, long long cur_r,
                                              int bi, int l, int seg_groups,
                                              unsigned long long NG, Partial* red, Ctrl* ctrl,
                                              unsigned long long* keys,
                                              unsigned long long* skeys, uint8_t* pick,
                                              int tid) {
  const int lane = tid & 31, warp = tid >> 5;
  const int G = gridDim.x;
  warp_merge(acc, a.c2);
  if (lane == 0) red[warp] = acc;
  consumer_sync(kConsumers);
  if (tid == 0) {
    Partial P = red[0];
    for (int w = 1; w < kConsumerWarps; ++w) merge(P, red[w], a.c2);
    const size_t grow = (size_t)bi * (size_t)a.L + (size_t)l;
    const unsigned long long g_first = (unsigned long long)cur_r * (unsigned long long)a.ng;
    const int slot = (int)blockIdx.x - cta_of(g_first, NG, G);
    a.partials[grow * (size_t)a.max_segs + (size_t)slot] = P;
    __threadfence();
    const unsigned old = atomicAdd(a.row_ticket + grow, (unsigned)seg_groups);
    const bool last = old + (unsigned)seg_groups == (unsigned)a.ng;
    if (last) {
      a.row_ticket[grow] = 0u;
      __threadfence();
    }
    ctrl->row_last = last ? 1 : 0;
  }
  consumer_sync(kConsumers);
  if (ctrl->row_last) {
    if (warp == 0) {
      const bool done = row_combine<DT>(a, (unsigned long long)cur_r, bi, l, NG, lane);
      if (lane == 0) ctrl->canvas_last = done ? 1 : 0;
    }
    consumer_sync(kConsumers);
    if (ctrl->canvas_last) canvas_epilogue(a, bi, ctrl, keys, skeys, pick, tid);
    consumer_sync(kConsumers);
  }
}

// ---------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------
template <int DT, bool TMA>
__global__ void __launch_bounds__(kThreads, DT == kBF16 ? 4 : 3) step_kernel(const StepArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const Layout lay = make_layout(DT, a.B, a.L);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + lay.bars);
  uint64_t* empty = full + kStages;
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + lay.ctrl);
  Partial* red = reinterpret_cast<Partial*>(smem + lay.red);
  uint16_t* act = reinterpret_cast<uint16_t*>(smem + lay.act);
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(smem + lay.keys);
  unsigned long long* skeys = reinterpret_cast<unsigned long long*>(smem + lay.skeys);
  uint8_t* pick = smem + lay.pick;
  unsigned char* ring = smem + lay.ring;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int st = 0; st < kStages; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], kConsumerWarps);
    }
    ctrl->abort = 0;
    ctrl->issued = 0;
    fence_mbar_init();
  }
  // Active canvases, in index order (each CTA computes the same list from the
  // stop flags as they were when the step began; flags are only published by
  // the last CTA to exit).
  {
    int base = 0;
    for (int b0 = 0; b0 < a.B; b0 += kThreads) {
      const int b = b0 + tid;
      const bool on = b < a.B && __ldcg(a.stop_flags + b) == 0;
      const unsigned bal = __ballot_sync(0xffffffffu, on);
      if (lane == 0) ctrl->wcnt[warp] = __popc(bal);
      __syncthreads();
      int off = base;
      for (int w = 0; w < warp; ++w) off += ctrl->wcnt[w];
      if (on) act[off + __popc(bal & ((1u << lane) - 1u))] = (uint16_t)b;
      for (int w = 0; w < kThreads / 32; ++w) base += ctrl->wcnt[w];
      __syncthreads();
    }
    if (tid == 0) ctrl->n_act = base;
  }
  __syncthreads();

  const int n_act = ctrl->n_act;
  const int G = gridDim.x;
  const unsigned long long NG =
      (unsigned long long)n_act * (unsigned long long)a.L * (unsigned long long)a.ng;
  const unsigned long long g_lo = range_start(blockIdx.x, NG, G);
  const unsigned long long g_hi = range_start(blockIdx.x + 1, NG, G);
  const size_t row_bytes = (size_t)a.V * (size_t)elt_bytes(DT);
  const char* logits = reinterpret_cast<const char*>(a.logits);

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (TMA && lane == 0) {
      const uint64_t policy = evict_first_policy();
      TileIter it(g_lo, g_hi, a.ng, a.L);
      Tile t;
      int k = 0;
      while (it.next(t)) {
        const int st = k % kStages;
        if (k >= kStages) {
          if (!mbar_wait(&empty[st], (uint32_t)((k / kStages) - 1) & 1u)) {
            atomicOr(a.status, kStatusTimeout);
            *(volatile int*)&ctrl->abort = 1;
          }
        }
        if (*(volatile int*)&ctrl->abort) break;
        const size_t grow = (size_t)act[t.ai] * (size_t)a.L + (size_t)t.l;
        const size_t e0 = (size_t)t.j0 * kGroup;
        size_t nel = (size_t)t.cnt * kGroup;
        if (e0 + nel > (size_t)a.V) nel = (size_t)a.V - e0;
        const uint32_t bytes = (uint32_t)(nel * elt_bytes(DT));
        mbar_arrive_expect_tx(&full[st], bytes);
        bulk_load(ring + (size_t)st * tile_bytes(DT), logits + grow * row_bytes + e0 * elt_bytes(DT),
                  bytes, &full[st], policy);
        ++k;
        *(volatile int*)&ctrl->issued = k;
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    TileIter it(g_lo, g_hi, a.ng, a.L);
    Tile t;
    int k = 0;
    long long cur_r = -1;
    int seg_groups = 0;
    int bi = 0, l = 0;
    bool sampling = false;
    Partial acc = empty_partial();
    const int rot = tid;  // piece rotation for bank-conflict-free reads

    while (it.next(t)) {
      if (t.r != cur_r) {
        if (cur_r >= 0)
          flush_segment<DT>(a, acc, cur_r, bi, l, seg_groups, NG, red, ctrl, keys, skeys, pick, tid);
        cur_r = t.r;
        seg_groups = 0;
        acc = empty_partial();
        bi = act[t.ai];
        l = t.l;
        const size_t grow = (size_t)bi * (size_t)a.L + (size_t)l;
        sampling = !a.greedy && a.committed[grow] == 0;
      }
      const int st = k % kStages;
      const size_t grow = (size_t)bi * (size_t)a.L + (size_t)l;
      const int j = t.j0 + tid;
      float lse = -INFINITY;
      if (TMA) {
        bool ok = true;
        if (!*(volatile int*)&ctrl->abort) ok = mbar_wait(&full[st], (uint32_t)(k / kStages) & 1u);
        if (!ok) {
          atomicOr(a.status, kStatusTimeout);
          *(volatile int*)&ctrl->abort = 1;
        }
      }
      if (tid < t.cnt) {
        const int glen = (a.V - j * kGroup) < kGroup ? (a.V - j * kGroup) : kGroup;
        GroupStat gs;
        if (TMA) {
          const unsigned char* gp =
              ring + (size_t)st * tile_bytes(DT) + (size_t)tid * kGroup * elt_bytes(DT);
          if (glen == kGroup) {
            gs = DT == kBF16 ? group_bf16_full(gp, rot, a.c2) : group_f32_full(gp, rot, a.c2);
          } else {
            gs = group_scalar<DT>(gp, glen, a.c2);
          }
        } else {
          const char* gp = logits + grow * row_bytes + (size_t)j * kGroup * elt_bytes(DT);
          gs = group_scalar<DT>(gp, glen, a.c2);
        }
        fold_group(acc, gs, j, a.c2);
        if (sampling) lse = 0.6931471805599453f * fmaf(gs.m, a.c2, lg2(gs.S));
      }
      if (TMA) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
      }
      if (sampling) {
        // Group-level Gumbel: the 32 groups of this warp need at most 9
        // Philox calls (4 words each); lanes 0-8 compute them and every lane
        // picks its word by shuffle.
        const bool need = tid < t.cnt && lse + kGumbelMax >= acc.gscore;
        if (__ballot_sync(0xffffffffu, need)) {
          const uint32_t jw = (uint32_t)(t.j0 + warp * 32);
          const uint32_t cbase = jw >> 2;
          Words4 w{};
          if (lane < 9)
            w = philox(cbase + (uint32_t)lane, (uint32_t)l, (uint32_t)a.s,
                       (uint32_t)(a.canvas_offset + bi) | (kStreamGroup << 24), a.key0, a.key1);
          const int src = (int)(((jw + (uint32_t)lane) >> 2) - cbase);
          const uint32_t x0 = __shfl_sync(0xffffffffu, w.w[0], src);
          const uint32_t x1 = __shfl_sync(0xffffffffu, w.w[1], src);
          const uint32_t x2 = __shfl_sync(0xffffffffu, w.w[2], src);
          const uint32_t x3 = __shfl_sync(0xffffffffu, w.w[3], src);
          if (need) {
            const uint32_t sel = (uint32_t)j & 3u;
            const uint32_t x = sel == 0 ? x0 : sel == 1 ? x1 : sel == 2 ? x2 : x3;
            const float sc = lse + gumbel(x);
            if (sc > acc.gscore) {
              acc.gscore = sc;
              acc.gidx = j;
            }
          }
        }
      }
      seg_groups += t.cnt;
      ++k;
    }
    if (cur_r >= 0)
      flush_segment<DT>(a, acc, cur_r, bi, l, seg_groups, NG, red, ctrl, keys, skeys, pick, tid);

    // After an abort, wait (bounded) for bulk copies still in flight into
    // this CTA's shared memory before it may exit.
    if (TMA && tid == 0 && *(volatile int*)&ctrl->abort) {
      const int issued = *(volatile int*)&ctrl->issued;
      for (int st = 0; st < kStages && st < issued; ++st) {
        const int n = (issued - st + kStages - 1) / kStages;
        mbar_wait(&full[st], (uint32_t)(n - 1) & 1u);
      }
    }
  }

  // Last CTA out publishes the new stop flags of the canvases finished in
  // this step (no CTA can still be reading the old flags by then).
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const unsigned old = atomicAdd(a.exit_ticket, 1u);
    ctrl->exit_last = old == (unsigned)G - 1u ? 1 : 0;
    if (ctrl->exit_last) {
      *a.exit_ticket = 0u;
      __threadfence();
    }
  }
  __syncthreads();
  if (ctrl->exit_last) {
    for (int i = tid; i < n_act; i += kThreads) {
      const int b = act[i];
      a.stop_flags[b] = __ldcg(a.stop_next + b);
    }
  }
}

// Initial canvas: uniform-random tokens (stream 2), nothing committed.
__global__ void init_canvas_kernel(int32_t* canvas, uint8_t* committed, uint8_t* stop_flags,
                                   int32_t* stable, uint8_t* stop_next, int L, int V,
                                   int canvas_offset, uint32_t key0, uint32_t key1) {
  const int bi = blockIdx.x;
  const uint32_t bg = (uint32_t)(canvas_offset + bi);
  for (int l = threadIdx.x; l < L; l += blockDim.x) {
    const Words4 r = philox((uint32_t)l >> 2, 0u, 0u, bg | (kStreamInit << 24), key0, key1);
    const size_t i = (size_t)bi * (size_t)L + (size_t)l;
    canvas[i] = (int32_t)uniform_token(pick_word(r, (uint32_t)l & 3u), (uint32_t)V);
    committed[i] = 0;
  }
  if (threadIdx.x == 0) {
    stop_flags[bi] = 0;
    stable[bi] = 0;
    stop_next[bi] = 0;
  }
}

}  // namespace ebk
