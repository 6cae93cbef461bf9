// eb_stream.cuh -- first kernel of a sampler step: one pass over every logit
// of every active canvas, and each position's results.
//
// Work split.  The active rows' 64-logit groups are numbered g = row ng + j
// (row = active canvas index * L + position).  Stream CTA c of G (one per SM)
// owns the contiguous range [c NG / G, (c + 1) NG / G): every CTA reads the
// same number of bytes to within one group, and a row meets only a few CTAs.
//
// Inside a CTA (one CTA per SM):
//   - the copy producer (one lane) walks the range in tiles of up to
//     kStageGroups groups that never straddle a row, writes each tile's
//     description and copies it into a kStages-deep ring with one 1-D bulk
//     copy (the TMA engine, into this CTA only, L2 evict-first);
//   - the word producer computes the group-stream Philox words of an open
//     position's tiles;
//   - twelve consumer warps take the tiles' 64-group sub-tiles round-robin
//     (a fixed assignment, so every run sums in the same order).  A lane
//     reduces two groups per sub-tile into its own running state (Acc): for
//     bf16 logits it copies both groups into registers and releases the
//     stage before any arithmetic, so the ring refills while it computes.
//     When a warp leaves a row it merges its lanes and deposits one record
//     per row of the CTA's range into a shared-memory slot;
//   - two finisher warps (alternating rows) merge the twelve deposits of
//     each row into the CTA's part of the row, made final (the exact top
//     group and the element drawn in its best Gumbel group).  A row spread
//     over several CTAs exchanges these records through global memory: each
//     CTA writes its record and counts itself in the row's counter (or sees
//     that the others are done already); the last one combines them (in CTA
//     order) and writes the position's entropy, max probability, argmax and
//     draw.
// The roles hand work to one another through mbarrier phases, in which a
// waiting thread is suspended rather than polling shared memory: the
// start-up publication (ready), a tile's description (described), a
// stage's copy and header (full), its release (empty) and a row's twelve
// deposits (the row slot's barrier).
// The CTA that finishes a canvas's last position then runs that canvas's
// decisions with all its threads (eb_finish.cuh), once every CTA of the
// grid has read the stop flags.  Consecutive steps' kernels are chained by
// programmatic dependent launch: a CTA sets up its shared memory while the
// previous step's kernel drains, then waits for it (griddepcontrol.wait).
#pragma once

#include "eb_common.cuh"
#include "eb_finish.cuh"

namespace ebk {

#ifndef EB_STREAM_CONSUMER_WARPS
#define EB_STREAM_CONSUMER_WARPS 12
#endif
#ifndef EB_STREAM_STAGES
#define EB_STREAM_STAGES 3
#endif
#ifndef EB_STREAM_STAGE_KB
#define EB_STREAM_STAGE_KB 64
#endif
#ifndef EB_STREAM_FINISHERS
#define EB_STREAM_FINISHERS 2
#endif

constexpr int kStages = EB_STREAM_STAGES;
constexpr int kSlots = 8;  // row slots of the consumer -> finisher hand-off

template <int DT>
struct StreamShape {
  static constexpr int kConsumerWarps = EB_STREAM_CONSUMER_WARPS;
  static constexpr int kFinishers = EB_STREAM_FINISHERS;  // finisher warps, alternating rows
  // + copy producer, word producer, finishers
  static constexpr int kThreads = (kConsumerWarps + 2 + kFinishers) * 32;
  static constexpr int kStageBytes = EB_STREAM_STAGE_KB * 1024;
  // room for a copy widened to 16-byte boundaries; 128-byte aligned stages
  static constexpr int kStageStride = kStageBytes + 128;
  static constexpr int kStageGroups = kStageBytes / (kGroup * elt_bytes(DT));
  static constexpr int kSubGroups = 64;  // groups per sub-tile: two per lane
  static constexpr int kSubPerStage = kStageGroups / kSubGroups;
  static_assert(kSubPerStage >= 1 && (kSubPerStage & (kSubPerStage - 1)) == 0,
                "sub-tiles per stage must be a power of two");
  static_assert(kConsumerWarps <= 16, "the finisher merges at most 16 deposits per row");
};

__host__ __device__ constexpr int stream_threads(int dt) {
  return dt == kBF16 ? StreamShape<kBF16>::kThreads : StreamShape<kF32>::kThreads;
}

struct StreamCtrl {
  int abort;
  int issued;  // tiles whose bulk copy has been issued (the exit drain's count)
  int n_sub;   // sub-tiles of this CTA's range
  int words_arrived;  // tiles whose second (header) arrival was made
  int n_epi;          // canvases whose decisions this CTA runs
  int epi_ok;         // every CTA of the grid has read the stop flags
  int nread;          // warps that have read the stop flags
};

// What the producer tells the consumers about the tile in a stage.
struct TileMeta {
  int r;         // active row index
  int j0;        // first group of the tile within the row
  int cnt;       // groups in the tile
  int bi;        // canvas
  int l;         // position
  int sampling;  // open position of a sampled (not greedy) run
  int delta;     // byte offset of the tile's first logit in the stage
  int whole;     // every group whole and 16-byte aligned: the vector path
};

// A row slot: the consumer warps' deposits for one row of the CTA's range.
struct RowSlot {
  int q;  // CTA-relative row the slot accepts deposits for
  int pad0;
  uint64_t full;  // one arrival per consumer warp's deposit
  Acc rec[EB_STREAM_CONSUMER_WARPS];
};

struct StreamLayout {
  uint32_t bars, ctrl, meta, words, slots, act, epi, ring, total;
};

__host__ __device__ inline uint32_t align_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

template <int DT>
__host__ __device__ inline StreamLayout stream_layout(int B) {
  using Sh = StreamShape<DT>;
  StreamLayout y;
  uint32_t o = 0;
  y.bars = o;
  o = align_up(o + 24u * kStages + 8u, 16);  // full, empty, described; ready
  y.ctrl = o;
  o = align_up(o + (uint32_t)sizeof(StreamCtrl), 16);
  y.meta = o;
  o = align_up(o + (uint32_t)sizeof(TileMeta) * kStages, 16);
  y.words = o;
  o = align_up(o + 4u * (uint32_t)Sh::kStageGroups * kStages, 16);
  y.slots = o;
  o = align_up(o + (uint32_t)sizeof(RowSlot) * kSlots, 16);
  y.act = o;
  o = align_up(o + 2u * (uint32_t)B, 16);
  y.epi = o;
  o = align_up(o + 2u * (uint32_t)B, 128);
  y.ring = o;
  o += (uint32_t)kStages * (uint32_t)Sh::kStageStride;
  y.total = o;
  return y;
}

struct Tile {
  long long r;  // active row index
  int j0;       // first group of the tile within the row
  int cnt;      // groups in the tile
  int ai;       // index of the row's canvas in the active list
  int l;        // position of the row
};

// Walks a CTA's group range in tiles that end at the row's multiples of tg
// groups (so a tile after the first of a row segment starts on a Philox
// call boundary); divides only once, at the start.
struct TileIter {
  unsigned long long g, g_hi;
  int ng, L, tg;
  long long r;
  int j0, ai, l;
  __device__ __forceinline__ TileIter(unsigned long long lo, unsigned long long hi, int ng_, int L_,
                                      int tg_)
      : g(lo), g_hi(hi), ng(ng_), L(L_), tg(tg_) {
    r = (long long)(lo / (unsigned long long)ng_);
    j0 = (int)(lo - (unsigned long long)r * (unsigned long long)ng_);
    ai = (int)(r / L_);
    l = (int)(r - (long long)ai * L_);
  }
  __device__ __forceinline__ bool next(Tile& t) {
    if (g >= g_hi) return false;
    int cnt = ng - j0;
    const int to_edge = tg - j0 % tg;  // tiles end on multiples of tg within a row
    if (cnt > to_edge) cnt = to_edge;
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

// Tiles of the range [lo, hi), the same cut as TileIter: a row segment
// covering groups [a, b) of its row has ceil(b / tg) - floor(a / tg) tiles.
__device__ __forceinline__ int count_tiles(unsigned long long lo, unsigned long long hi, int ng,
                                           int tg) {
  int n = 0;
  while (lo < hi) {
    const unsigned long long r = lo / (unsigned long long)ng;
    unsigned long long e = (r + 1ull) * (unsigned long long)ng;
    if (e > hi) e = hi;
    const int a = (int)(lo - r * (unsigned long long)ng), b = (int)(e - r * (unsigned long long)ng);
    n += (b + tg - 1) / tg - a / tg;
    lo = e;
  }
  return n;
}

// Active canvases (stop flag clear) counted by one warp from the stop flags
// as they were when the step began (only this kernel's canvas decisions, at
// its end, write them); with act != nullptr the warp also lists them in index
// order, and with act_index != nullptr writes every canvas's place in that
// list (-1: stopped).
__device__ __forceinline__ int warp_active_list(const uint8_t* stop_flags, int B, uint16_t* act,
                                                int32_t* act_index) {
  const int lane = threadIdx.x & 31;
  int n = 0;
  for (int b0 = 0; b0 < B; b0 += 32) {
    const int b = b0 + lane;
    const bool on = b < B && __ldcg(stop_flags + b) == 0;
    const unsigned bal = __ballot_sync(0xffffffffu, on);
    const int rank = n + __popc(bal & ((1u << lane) - 1u));
    if (on && act != nullptr) act[rank] = (uint16_t)b;
    if (b < B && act_index != nullptr) act_index[b] = on ? rank : -1;
    n += __popc(bal);
  }
  return n;
}

// Where row r's records live: the stream CTAs that own part of it are
// c_first .. c_last; with at least one group per CTA (NG >= G) record `seg`
// of CTA c is c - c_first, otherwise every CTA owns at most one group and
// the record index is that group's index in the row.
struct RowSpan {
  int seg, nseg;
};
__device__ __forceinline__ RowSpan row_span(unsigned long long r, int ng, unsigned long long NG,
                                            int G, int c) {
  const unsigned long long g0 = r * (unsigned long long)ng;
  RowSpan s;
  if (NG >= (unsigned long long)G) {
    const int c0 = cta_of(g0, NG, G);
    const int c1 = cta_of(g0 + (unsigned long long)ng - 1ull, NG, G);
    s.seg = c - c0;
    s.nseg = c1 - c0 + 1;
  } else {
    s.seg = (int)(range_start(c, NG, G) - g0);
    s.nseg = ng;
  }
  return s;
}

// ---------------------------------------------------------------------------
// A stream CTA's part of a row, made final (one warp): the exact form of its
// top group and the element draw inside its best Gumbel group, from those
// two groups' logits (global memory) and their element-stream Philox words.
// ---------------------------------------------------------------------------
// This lane's two elements 2 lane, 2 lane + 1 of group j of a row (local
// ids; those at or beyond V read as -inf).
template <int DT>
__device__ __forceinline__ float2 load_pair(const StepArgs& a, const char* rowp, int j) {
  const int v0 = j * kGroup + 2 * (threadIdx.x & 31);
  float2 z = make_float2(-INFINITY, -INFINITY);
  if (a.vec_ok && v0 + 1 < a.V) {
    if (DT == kF32) {
      z = __ldg(reinterpret_cast<const float2*>(rowp) + (v0 >> 1));
    } else {
      const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(rowp) + (v0 >> 1));
      z = make_float2(bf16_lo(w), bf16_hi(w));
    }
  } else {
    if (v0 < a.V) z.x = load_elem<DT>(rowp, v0);
    if (v0 + 1 < a.V) z.y = load_elem<DT>(rowp, v0 + 1);
  }
  return z;
}

// Element draw inside group j (local group id), whose elements this lane
// holds as (z.x, z.y) = elements 2 lane, 2 lane + 1.  Every lane returns the
// drawn local id (kNone if the group holds no finite logit).  The largest
// tempered logit is drawn first, and the logarithms of every element that
// provably cannot beat it are skipped.
__device__ __forceinline__ int draw_in_group(const StepArgs& a, float2 z, int j, int bi, int l) {
  const int lane = threadIdx.x & 31;
  const int v0 = j * kGroup + 2 * lane;
  // element-stream words: lane k < 16 computes call k of the group (global
  // ids: the group starts on a multiple of 64, so on a call boundary)
  const uint32_t gv0 = (uint32_t)(a.v_off + j * kGroup);
  Words4 w4{{0u, 0u, 0u, 0u}};
  if (lane < 16)
    w4 = philox((gv0 >> 2) + (uint32_t)lane, (uint32_t)l, (uint32_t)a.s,
                (uint32_t)(a.canvas_offset + bi) | (kStreamGumbel << 24), a.key0, a.key1);
  const int src = lane >> 1;
  const uint32_t s0 = __shfl_sync(0xffffffffu, w4.w[0], src);
  const uint32_t s1 = __shfl_sync(0xffffffffu, w4.w[1], src);
  const uint32_t s2 = __shfl_sync(0xffffffffu, w4.w[2], src);
  const uint32_t s3 = __shfl_sync(0xffffffffu, w4.w[3], src);
  const uint32_t x0 = (lane & 1) ? s2 : s0, x1 = (lane & 1) ? s3 : s1;
  const float y0 = z.x * a.iT, y1 = z.y * a.iT;
  float ym = y0;
  int vm = v0;
  uint32_t xm = x0;
  if (y1 > ym) {
    ym = y1;
    vm = v0 + 1;
    xm = x1;
  }
  if (!(ym > -INFINITY)) vm = kNone;
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const float oy = __shfl_xor_sync(0xffffffffu, ym, o);
    const int ov = __shfl_xor_sync(0xffffffffu, vm, o);
    const uint32_t ox = __shfl_xor_sync(0xffffffffu, xm, o);
    if (oy > ym || (oy == ym && ov < vm)) {
      ym = oy;
      vm = ov;
      xm = ox;
    }
  }
  if (vm == kNone) return kNone;
  const float seed = ym + gumbel(xm);
  float best = seed;
  int barg = vm;
  auto consider = [&](float y, int v, uint32_t x) {
    if (v == vm || !(y > -INFINITY)) return;
    // can v beat the seed?  It needs g > seed - y, i.e. -ln u < e^-(seed - y);
    // -ln u >= 1 - u, so 1 - u >= e^-(seed - y) (1e-4 relative margin) rules it out.
    const float tgap = seed - y;
    if (tgap > -2.0f && one_minus_u(x) >= ex2(-1.4426950408889634f * tgap) * 1.0001f) return;
    const float sc = y + gumbel(x);
    if (sc > best || (sc == best && v < barg)) {
      best = sc;
      barg = v;
    }
  };
  consider(y0, v0, x0);
  consider(y1, v0 + 1, x1);
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const float ob = __shfl_xor_sync(0xffffffffu, best, o);
    const int oa = __shfl_xor_sync(0xffffffffu, barg, o);
    if (ob > best || (ob == best && oa < barg)) {
      best = ob;
      barg = oa;
    }
  }
  return barg;
}

// The CTA's merged state of its part of a row -> its final record, in two
// halves so that other memory traffic can be issued between them: the loads
// of the part's top group and best Gumbel group, then the arithmetic.  The
// top group is recomputed exactly relative to M: elements equal to M count 1
// each (d = (z - M) c2 from the exact difference), the smaller ones are
// summed, zero terms skipped.  Every lane returns the record.
struct PartLoads {
  float2 zt, zd;
  bool has, drw;
};

template <int DT>
__device__ __forceinline__ PartLoads part_loads(const StepArgs& a, const Acc& A, const char* rowp,
                                                bool draw) {
  PartLoads p;
  p.has = A.M > -INFINITY && A.tj != kNone;
  p.drw = draw && p.has && A.gb != kNone;
  p.zt = p.zd = make_float2(-INFINITY, -INFINITY);
  if (p.has) p.zt = load_pair<DT>(a, rowp, A.tj);
  if (p.drw) p.zd = load_pair<DT>(a, rowp, A.gb);
  return p;
}

__device__ __forceinline__ Rec part_finalize(const StepArgs& a, const Acc& A, const PartLoads& p,
                                             int bi, int l) {
  const int lane = threadIdx.x & 31;
  Exact e{0.f, 0.f, 0, kNone};
  if (p.has) {
    exact_elem(p.zt.x, A.tj * kGroup + 2 * lane, A.M, a.c2, e);
    exact_elem(p.zt.y, A.tj * kGroup + 2 * lane + 1, A.M, a.c2, e);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    e.S += __shfl_xor_sync(0xffffffffu, e.S, o);
    e.W += __shfl_xor_sync(0xffffffffu, e.W, o);
    e.n += __shfl_xor_sync(0xffffffffu, e.n, o);
    e.amin = min(e.amin, __shfl_xor_sync(0xffffffffu, e.amin, o));
  }
  Rec r;
  r.M = p.has ? A.M : -INFINITY;
  r.Sr = A.Sr;
  r.Wr = A.Wr;
  r.tS = e.S;
  r.tW = e.W;
  r.R = A.R;
  r.tn = e.n;
  r.ta = e.amin;
  r.gb = A.gb;
  r.xs = p.drw ? draw_in_group(a, p.zd, A.gb, bi, l) : kNone;
  r.pad0 = r.pad1 = 0;
  return r;
}

__device__ __forceinline__ Rec ld_rec(const Rec* p) {
  Rec r;
  const float4 u = __ldcg(reinterpret_cast<const float4*>(p));
  const float4 v = __ldcg(reinterpret_cast<const float4*>(p) + 1);
  const int4 w = __ldcg(reinterpret_cast<const int4*>(p) + 2);
  r.M = u.x;
  r.Sr = u.y;
  r.Wr = u.z;
  r.tS = u.w;
  r.tW = v.x;
  r.R = v.y;
  r.tn = __float_as_int(v.z);
  r.ta = __float_as_int(v.w);
  r.gb = w.x;
  r.xs = w.y;
  r.pad0 = r.pad1 = 0;
  return r;
}

// The row's n records in stream-CTA order (which is group order), combined
// in float64: the row maximum M; the first record attaining it gives the
// argmax; every record's sums are rescaled to M (a record whose maximum
// equals M adds its count of maxima exactly); the best Gumbel ratio (lower
// group on equal ratios) gives the draw.  `rec(i)` returns record i; every
// lane returns the same values.
struct RowFinal {
  double S, W;  // relative to M, W in log2 units
  float M, R;
  int amax, gb, xs;  // local ids
};

template <class Load>
__device__ __forceinline__ RowFinal combine_records(int n, Load rec, float c2) {
  const int lane = threadIdx.x & 31;
  float M = -INFINITY;
  for (int i = lane; i < n; i += 32) M = fmaxf(M, rec(i).M);
#pragma unroll
  for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  double S = 0.0, W = 0.0;
  float Rl = 0.f;
  int gl = kNone, xl = kNone, top = kNone, ta = kNone;
  for (int i = lane; i < n; i += 32) {
    const Rec c = rec(i);
    if (!(c.M > -INFINITY)) continue;
    const bool tie = c.M == M;
    if (tie && i < top) {
      top = i;
      ta = c.ta;
    }
    const double dd = tie ? 0.0 : (double)((c.M - M) * c2);
    const double f = tie ? 1.0 : exp2(dd);
    const double So = (double)c.tn + ((double)c.tS + (double)c.Sr);
    const double Wo = (double)c.tW + (double)c.Wr;
    S += f * So;
    W += f * (Wo + dd * So);
    const float Rc = c.R * (float)f;
    if (Rc > Rl || (Rc == Rl && Rc > 0.f && c.gb < gl)) {
      Rl = Rc;
      gl = c.gb;
      xl = c.xs;
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    S += __shfl_xor_sync(0xffffffffu, S, o);
    W += __shfl_xor_sync(0xffffffffu, W, o);
    const float oR = __shfl_xor_sync(0xffffffffu, Rl, o);
    const int og = __shfl_xor_sync(0xffffffffu, gl, o);
    const int ox = __shfl_xor_sync(0xffffffffu, xl, o);
    if (oR > Rl || (oR == Rl && oR > 0.f && og < gl)) {
      Rl = oR;
      gl = og;
      xl = ox;
    }
    const int ot = __shfl_xor_sync(0xffffffffu, top, o);
    const int oa = __shfl_xor_sync(0xffffffffu, ta, o);
    if (ot < top) {
      top = ot;
      ta = oa;
    }
  }
  RowFinal f;
  f.S = S;
  f.W = W;
  f.M = M;
  f.R = Rl;
  f.amax = ta;
  f.gb = gl;
  f.xs = xl;
  return f;
}

// The position's outputs from its combined records (lane 0 writes): the
// entropy and max probability in float64, the argmax, the draw -- or, for a
// vocabulary slice, its slice record.
__device__ __forceinline__ void write_position(const StepArgs& a, const RowFinal& F, int bi, int l,
                                               bool open) {
  if ((threadIdx.x & 31) != 0) return;
  const size_t grow = (size_t)bi * (size_t)a.L + (size_t)l;
  const double S = F.S, W = F.W;
  if (!isfinite(S) || !isfinite(W) || F.amax == kNone) atomicOr(a.status, kStatusNonFinite);
  const int amax = F.amax == kNone ? kNone : F.amax + a.v_off;
  const bool drawn = open && !a.greedy && F.xs != kNone;
  const int smp = drawn ? F.xs + a.v_off : amax;
  if (a.slice_out != nullptr) {
    SliceRecord r;
    r.S = S;
    r.W = W;
    r.zmax = F.M;
    r.gscore = (F.R > 0.f && F.gb != kNone) ? fmaf(F.M, a.iT, logf(F.R)) : -INFINITY;
    r.amax = amax;
    r.sample = drawn ? smp : -1;
    r.pad0 = r.pad1 = 0;
    a.slice_out[grow] = r;
    return;
  }
  a.H_out[grow] = (float)(log(S) - 0.6931471805599453 * (W / S));
  a.amax_out[grow] = amax;
  a.pmax[grow] = (float)(1.0 / S);
  a.sample[grow] = open ? smp : -1;
}

// One CTA per SM: the register cap is the register file over the block.
template <int DT>
__global__ void __launch_bounds__(StreamShape<DT>::kThreads, 1) stream_kernel(const StepArgs a) {
  using Sh = StreamShape<DT>;
  constexpr int NW = Sh::kConsumerWarps;
  extern __shared__ __align__(128) unsigned char smem[];
  const StreamLayout lay = stream_layout<DT>(a.B);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + lay.bars);
  uint64_t* empty = full + kStages;
  uint64_t* described = empty + kStages;  // a tile's copy issued, its description written
  uint64_t* ready = described + kStages;  // the active list and sub-tile count published
  StreamCtrl* ctrl = reinterpret_cast<StreamCtrl*>(smem + lay.ctrl);
  TileMeta* meta = reinterpret_cast<TileMeta*>(smem + lay.meta);
  uint32_t* words = reinterpret_cast<uint32_t*>(smem + lay.words);
  RowSlot* slots = reinterpret_cast<RowSlot*>(smem + lay.slots);
  uint16_t* act = reinterpret_cast<uint16_t*>(smem + lay.act);
  uint16_t* epi = reinterpret_cast<uint16_t*>(smem + lay.epi);
  unsigned char* ring = smem + lay.ring;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int st = 0; st < kStages; ++st) {
      mbar_init(&full[st], 2);  // the copy's arrival (+ bytes) and the header's
      mbar_init(&empty[st], Sh::kSubPerStage);
      mbar_init(&described[st], 1);
    }
    mbar_init(ready, 1);
    ctrl->abort = 0;
    ctrl->issued = 0;
    ctrl->words_arrived = 0;
    ctrl->n_epi = 0;
    ctrl->epi_ok = 0;
    ctrl->nread = 0;
    for (int i = 0; i < kSlots; ++i) {
      slots[i].q = i;
      mbar_init(&slots[i].full, NW);
    }
    fence_mbar_init();
  }
  // Barriers and slots initialized before any warp uses them.
  block_sync();
  // Everything above is this CTA's own shared memory; from here on the
  // kernel reads what the previous step's kernel wrote (stop flags, canvas
  // state, counters): wait until that grid has completed.  The next kernel
  // on the stream may be scheduled from now on, wherever an SM has room: it
  // waits for this grid's completion in turn before reading anything this
  // grid writes.
  const int G = gridDim.x;
  griddep_wait();
  griddep_launch_dependents();
  // Every warp counts the active canvases itself (no block barrier); the
  // producer warp also lists them for the others (published with `ready`),
  // and in block 0 writes the list's index for the split-vocabulary combine.
  const int n_act = warp_active_list(
      a.stop_flags, a.B, warp == NW ? act : nullptr,
      (warp == NW && blockIdx.x == 0) ? a.act_index : nullptr);
  if (lane == 0) {
    if (warp == NW && blockIdx.x == 0) *a.n_act = n_act;
    // the last warp of the CTA to have read the stop flags says so
    if (atomicAdd(&ctrl->nread, 1) == Sh::kThreads / 32 - 1 && a.run_epilogue)
      atomicAdd(a.sync_cnt, 1);
  }
  const unsigned long long NG =
      (unsigned long long)n_act * (unsigned long long)a.L * (unsigned long long)a.ng;
  const unsigned long long g_lo = range_start(blockIdx.x, NG, G);
  const unsigned long long g_hi = range_start(blockIdx.x + 1, NG, G);
  // The other roles start once the producer has published the active list
  // and the range's sub-tile count (right after its first copy).
  auto wait_ready = [&]() -> bool {
    const bool ok = __all_sync(0xffffffffu, mbar_wait_timed(ready, 0, a.wait_ns, &ctrl->abort));
    if (!ok && lane == 0) {
      atomicOr(a.status, kStatusTimeout);
      *(volatile int*)&ctrl->abort = 1;
    }
    return ok;
  };

  const size_t row_bytes = (size_t)a.V * (size_t)elt_bytes(DT);
  const char* logits = reinterpret_cast<const char*>(a.logits);
  // the range's first row and one past its last (roles that need them)
  auto row_range = [&](long long& r_first, long long& r_end) {
    r_first = (long long)(g_lo / (unsigned long long)a.ng);
    r_end = g_hi > g_lo ? (long long)((g_hi - 1ull) / (unsigned long long)a.ng) + 1 : r_first;
  };
  auto row_of = [&](long long r, int& bi, int& l) {
    const int ai = (int)(r / a.L);
    l = (int)(r - (long long)ai * a.L);
    bi = act[ai];
  };

  if (warp == NW) {
    // ------------------------------------------------------- copy producer
    // Lane 0 alone: waits for a free stage, issues the tile's bulk copy (the
    // stage's first arrival, with the bytes) and writes its description.  No
    // global load ever delays the next copy.  Right after its first copy it
    // publishes the range's sub-tile count and the active list (`ready`).
    __syncwarp();  // the warp's active list before lane 0 publishes it
    if (lane == 0) {
      bool published = false;
      auto publish = [&]() {
        ctrl->n_sub = count_tiles(g_lo, g_hi, a.ng, Sh::kStageGroups) * Sh::kSubPerStage;
        mbar_arrive(ready);
        published = true;
      };
      // Logits are read once: L2 evict-first, so that the stream does not push
      // out the kernel's code and small state.
      const uint64_t policy = evict_first_policy();
      TileIter it(g_lo, g_hi, a.ng, a.L, Sh::kStageGroups);
      Tile t;
      int k = 0, st = 0;
      uint32_t ph = 0;  // parity of the current pass over the ring
      long long row_seen = -1;
      int bi = 0;
      while (it.next(t)) {
        if (k >= kStages && !mbar_wait(&empty[st], ph ^ 1u, a.wait_ns)) {
          atomicOr(a.status, kStatusTimeout);
          *(volatile int*)&ctrl->abort = 1;
          break;
        }
        if (*(volatile int*)&ctrl->abort) break;
        if (t.r != row_seen) {
          row_seen = t.r;
          bi = act[t.ai];
        }
        const char* src = logits + ((size_t)bi * (size_t)a.L + (size_t)t.l) * row_bytes +
                          (size_t)t.j0 * kGroup * elt_bytes(DT);
        size_t nel = (size_t)t.cnt * kGroup;
        if ((size_t)t.j0 * kGroup + nel > (size_t)a.V) nel = (size_t)a.V - (size_t)t.j0 * kGroup;
        // The copy is widened to 16-byte boundaries: at most 15 bytes on each
        // side, inside the 16-byte blocks that hold the tile's first and last
        // logits.
        const uintptr_t a0 = reinterpret_cast<uintptr_t>(src) & ~(uintptr_t)15;
        const uintptr_t a1 =
            (reinterpret_cast<uintptr_t>(src) + nel * elt_bytes(DT) + 15) & ~(uintptr_t)15;
        mbar_arrive_expect_tx(&full[st], (uint32_t)(a1 - a0));
        bulk_load(ring + (size_t)st * Sh::kStageStride, reinterpret_cast<const void*>(a0),
                  (uint32_t)(a1 - a0), &full[st], policy);
        TileMeta m;
        m.r = (int)t.r;
        m.j0 = t.j0;
        m.cnt = t.cnt;
        m.bi = bi;
        m.l = t.l;
        m.sampling = 0;  // set by the word producer
        m.delta = (int)(reinterpret_cast<uintptr_t>(src) - a0);
        m.whole = a.vec_ok && (t.j0 + t.cnt) * kGroup <= a.V;
        meta[st] = m;
        st_release_shared(&ctrl->issued, k + 1);
        mbar_arrive(&described[st]);
        if (!published) publish();
        ++k;
        if (++st == kStages) {
          st = 0;
          ph ^= 1u;
        }
      }
      if (!published) publish();
      // Have all CTAs of the grid read the stop flags?  (Checked here, long
      // before this CTA can need it, so that a canvas's decisions at the end
      // rarely wait for the round trip.)
      if (a.run_epilogue && ld_acquire_gpu(a.sync_cnt) >= (int)gridDim.x) ctrl->epi_ok = 1;
    }
  } else if (warp == NW + 1) {
    // ------------------------------------------------------- word producer
    // Once tile k is issued (its stage free and its description written),
    // decides whether its position draws (open, not greedy), computes the
    // group-stream Philox words of a drawing position's groups into the
    // stage's header and makes the stage's second arrival.  The committed
    // flags of the range's first 32 rows are loaded at once, at the start.
    const int n_tiles = wait_ready() ? ctrl->n_sub / Sh::kSubPerStage : 0;
    long long r_first, r_end;
    row_range(r_first, r_end);
    uint32_t open_bits = 0;
    if (!a.greedy) {
      const long long r = r_first + lane;
      bool o = false;
      if (r < r_end) {
        int bi, l;
        row_of(r, bi, l);
        o = a.committed[(size_t)bi * (size_t)a.L + (size_t)l] == 0;
      }
      open_bits = __ballot_sync(0xffffffffu, o);
    }
    int st = 0, words_done = 0;
    long long row_seen = -1;
    int samp = 0;
    for (int k = 0; k < n_tiles; ++k, words_done = k) {
      // every lane waits (bounded, suspended in the barrier rather than
      // polling); the warp acts on the vote, so that a limit running out for
      // some lanes only still ends the loop for all.  The phase is this
      // warp's own next one: it waited for the stage's previous tile itself,
      // and the stage's next tile needs this tile's header first.
      if (!__all_sync(0xffffffffu, mbar_wait(&described[st], (uint32_t)(k / kStages) & 1u, a.wait_ns,
                                             &ctrl->abort))) {
        if (lane == 0) {
          atomicOr(a.status, kStatusTimeout);
          *(volatile int*)&ctrl->abort = 1;
        }
        break;
      }
      TileMeta* mp = &meta[st];
      const int mr = mp->r, mj0 = mp->j0, mcnt = mp->cnt, mbi = mp->bi, ml = mp->l;
      if (mr != row_seen) {
        row_seen = mr;
        const long long q = mr - r_first;
        samp = !a.greedy &&
               (q < 32 ? (open_bits >> q) & 1u
                       : a.committed[(size_t)mbi * (size_t)a.L + (size_t)ml] == 0);
      }
      if (samp) {
        uint32_t* wd = words + st * Sh::kStageGroups;
        const int gj0 = (a.v_off >> 6) + mj0;  // global group id of the tile's first group
        const int c0 = gj0 >> 2, c1 = (gj0 + mcnt - 1) >> 2;
        const uint32_t c3 = (uint32_t)(a.canvas_offset + mbi) | (kStreamGroup << 24);
        for (int c = c0 + lane; c <= c1; c += 32) {
          const Words4 w = philox((uint32_t)c, (uint32_t)ml, (uint32_t)a.s, c3, a.key0, a.key1);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int j = 4 * c + q - gj0;
            if (j >= 0 && j < mcnt) wd[j] = w.w[q];
          }
        }
      }
      __syncwarp();
      if (lane == 0) {
        mp->sampling = samp;
        mbar_arrive(&full[st]);  // header (words, draw flag) complete
      }
      if (++st == kStages) st = 0;
    }
    if (lane == 0) ctrl->words_arrived = words_done;
  } else if (warp >= NW + 2) {
    // ----------------------------------------------------------- finishers
    // Finisher f takes the rows q = f, f + kFinishers, ... of the range, so
    // that rows completed close together (at the end of the range) are
    // finished in parallel.
    long long r_first, r_end;
    row_range(r_first, r_end);
    const int nrows = wait_ready() ? (int)(r_end - r_first) : 0;
    const int f = warp - (NW + 2);
    static_assert(kSlots % Sh::kFinishers == 0, "a slot's rows must all go to one finisher");
    for (int q = f; q < nrows; q += Sh::kFinishers) {
      RowSlot* sl = &slots[q % kSlots];
      const long long r = r_first + q;
      int bi, l;
      row_of(r, bi, l);
      const size_t grow = (size_t)bi * (size_t)a.L + (size_t)l;
      const bool open = a.committed != nullptr && a.committed[grow] == 0;
      const RowSpan sp = row_span((unsigned long long)r, a.ng, NG, G, blockIdx.x);
      Rec* rr = a.recs + grow * (size_t)a.max_segs;
      // Are the row's other stream CTAs done already?  (Read before this
      // CTA's part is ready; if so, this CTA finishes the row without the
      // counter's round trip.)
      int pre = 0;
      if (sp.nseg > 1 && lane == 0) pre = ld_acquire_gpu(a.row_cnt + grow);
      // the twelve deposits of row q: use q / kSlots of the slot, whose
      // previous use this finisher waited for itself (a slot's rows all go
      // to one finisher), and whose next needs this row's release first
      const bool ok = mbar_wait(&sl->full, (uint32_t)(q / kSlots) & 1u, a.wait_ns, &ctrl->abort);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) {
          atomicOr(a.status, kStatusTimeout);
          *(volatile int*)&ctrl->abort = 1;
        }
        break;
      }
      Acc mine;
      if (lane < NW) {
        mine = sl->rec[lane];
      } else {
        acc_reset(mine);
      }
      warp_merge_acc(mine, a.c2);  // every lane ends with the CTA's merged state
      __syncwarp();
      if (lane == 0) st_release_shared(&sl->q, q + kSlots);
      const char* rowp = logits + grow * row_bytes;
      // this part's candidate groups: loads in flight first
      const PartLoads pl = part_loads<DT>(a, mine, rowp, open && !a.greedy);
      // then the row's counter again if the early read did not show the other
      // CTAs done (they usually are by now), and their records
      if (sp.nseg > 1 && lane == 0 && pre != sp.nseg - 1) pre = ld_acquire_gpu(a.row_cnt + grow);
      const bool others_done =
          sp.nseg > 1 && __shfl_sync(0xffffffffu, pre, 0) == sp.nseg - 1;
      Rec other;
      other.M = -INFINITY;
      __syncwarp();  // lane 0's acquire before the other lanes' record loads
      if (others_done && lane < sp.nseg && lane != sp.seg) other = ld_rec(rr + lane);
      const Rec own = part_finalize(a, mine, pl, bi, l);
      // the canvas's finished positions; the CTA finishing its last one runs
      // the canvas's decisions after its roles are done
      auto count_canvas = [&]() {
        if (!a.run_epilogue || lane != 0) return;
        if (atom_add_acq_rel_gpu(a.canvas_cnt + bi, 1) == a.L - 1)
          epi[atomicAdd(&ctrl->n_epi, 1)] = (uint16_t)bi;
      };
      if (sp.nseg == 1) {
        const RowFinal F = combine_records(1, [&](int) { return own; }, a.c2);
        write_position(a, F, bi, l, open);
        count_canvas();
        continue;
      }
      bool last = others_done;
      if (!last) {
        int old = 0;
        if (lane == 0) {
          rr[sp.seg] = own;
          old = atom_add_acq_rel_gpu(a.row_cnt + grow, 1);
        }
        last = __shfl_sync(0xffffffffu, old, 0) == sp.nseg - 1;
        if (!last) continue;
        __syncwarp();  // lane 0's acquire before the other lanes' record loads
        if (lane < sp.nseg && lane != sp.seg) other = ld_rec(rr + lane);
      }
      auto rec = [&](int i) -> Rec {
        if (i == sp.seg) return own;
        if (i < 32) return other;  // lane i holds record i
        return ld_rec(rr + i);
      };
      const RowFinal F = combine_records(sp.nseg, rec, a.c2);
      if (lane == 0) a.row_cnt[grow] = 0;  // zero again for the next step
      write_position(a, F, bi, l, open);
      count_canvas();
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int n_sub = wait_ready() ? ctrl->n_sub : 0;
    long long r_first, r_end;
    row_range(r_first, r_end);
    long long cur_r = -1;
    long long next_r = r_first;  // first row of the range this warp still owes a deposit
    int sampling = 0;
    Acc A;
    acc_reset(A);
    const int rot = lane;
    bool fail = false;

    // This warp's record of row r into its slot (after the finisher has
    // released the slot's previous row).
    auto deposit = [&](long long r, bool empty_rec) -> bool {
      Acc w = A;
      if (!empty_rec) warp_merge_acc(w, a.c2);
      const int q = (int)(r - r_first);
      RowSlot* sl = &slots[q % kSlots];
      int ok = 1;
      if (lane == 0) {
        const uint64_t t0 = global_ns();
        while (ld_acquire_shared(&sl->q) != q) {
          if (*(volatile int*)&ctrl->abort || global_ns() - t0 > a.wait_ns) {
            ok = 0;
            break;
          }
          __nanosleep(32);
        }
        if (ok) {
          if (empty_rec) {
            sl->rec[warp].M = -INFINITY;
          } else {
            sl->rec[warp] = w;
          }
          mbar_arrive(&sl->full);
        }
      }
      return __shfl_sync(0xffffffffu, ok, 0) != 0;
    };
    auto owe_empty = [&](long long upto) -> bool {
      for (; next_r < upto; ++next_r)
        if (!deposit(next_r, true)) return false;
      return true;
    };
    // A row change: this warp's deposit of the row it leaves, empty ones for
    // the rows of the range it skipped, and a fresh state.
    auto enter_row = [&](const TileMeta& m) -> bool {
      if (m.r == cur_r) return true;
      if (cur_r >= 0) {
        if (!deposit(cur_r, false)) return false;
        next_r = cur_r + 1;
      }
      if (!owe_empty(m.r)) return false;
      cur_r = m.r;
      next_r = cur_r + 1;
      sampling = m.sampling;
      acc_reset(A);
      return true;
    };

    // Sub-tiles are dealt round-robin: warp w takes w, w + NW, w + 2 NW, ...
    // The four sub-tiles of a tile go to four warps that also share every
    // tile k +- 3 NW / kSubPerStage ...; a warp has consumed the stage's
    // previous tile (k - kStages) itself before it waits for tile k, so the
    // parity of the stage's full barrier is unambiguous, and once it has
    // completed the tile's description and header are in place.
    for (int u = warp; u < n_sub; u += NW) {
      const int k = u / Sh::kSubPerStage;
      const int sub = u & (Sh::kSubPerStage - 1);
      const int st = k % kStages;
      // one try in every lane, agreed by a vote; when it is not yet
      // complete, a bounded wait in every lane and a second vote
      {
        const uint32_t par = (uint32_t)(k / kStages) & 1u;
        if (!__all_sync(0xffffffffu, mbar_try_wait(&full[st], par)) &&
            !__all_sync(0xffffffffu, mbar_wait(&full[st], par, a.wait_ns, &ctrl->abort))) {
          fail = true;
          break;
        }
      }
      const int gl0 = sub * Sh::kSubGroups + lane, gl1 = gl0 + 32;
      const uint32_t* wd = words + st * Sh::kStageGroups;
      if (DT == kBF16 && a.vec_ok) {
        // Rows on 16-byte boundaries: every tile's copy starts at the stage's
        // first byte, so the lane's two groups and their race words are
        // loaded together with the tile's description (one shared-memory
        // round trip after the wait).  Both groups lie inside the stage
        // whatever the tile's count; a group past the count is ignored.
        const unsigned char* sb = ring + (size_t)st * Sh::kStageStride;
        uint32_t G0[32], G1[32];
        load_group_bf16(sb + (size_t)gl0 * 128, rot, G0);
        load_group_bf16(sb + (size_t)gl1 * 128, rot, G1);
        const uint32_t x0 = wd[gl0], x1 = wd[gl1];
        const TileMeta m = meta[st];
        if (m.whole) {
          // the stage goes back to the producer; the row change (which may
          // wait for a row slot) comes after the release
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[st]);
          if (!enter_row(m)) {
            fail = true;
            break;
          }
          const bool has0 = gl0 < m.cnt, has1 = gl1 < m.cnt;  // has1 implies has0
          if (!has0) continue;
          const int j0 = m.j0 + gl0, j1 = m.j0 + gl1;
          // Both groups against one reference, the larger of the lane's
          // maximum and theirs: a group raising it becomes the top group (the
          // first on equal maxima), the other joins the rest; then the race,
          // group 0 first.
          const float mg0 = group_max_bf16(G0);
          const float mg1 = has1 ? group_max_bf16(G1) : -INFINITY;
          const bool v0 = mg0 > -INFINITY, v1 = mg1 > -INFINITY;  // not every logit -inf
          if (!(v0 || v1)) continue;
          const float mg = fmaxf(mg0, mg1);
          const bool new_top = mg > A.M;
          const float ref = new_top ? mg : A.M;
          float S0, W0, S1, W1;
          group_sums2_bf16(G0, G1, a.c2, ref, S0, W0, S1, W1);
          if (v0 && !(W0 >= -3.0e38f && S0 <= 3.0e38f)) group_sums_bf16<true>(G0, a.c2, ref, S0, W0);
          if (v1 && !(W1 >= -3.0e38f && S1 <= 3.0e38f)) group_sums_bf16<true>(G1, a.c2, ref, S1, W1);
          if (new_top) {
            const bool top0 = mg0 == mg;
            lane_new_top(A, mg, top0 ? j0 : j1, top0 ? S0 : S1, top0 ? W0 : W1, a.c2);
            const bool rest = top0 ? v1 : v0;
            if (rest) {
              A.Sr += top0 ? S1 : S0;
              A.Wr += top0 ? W1 : W0;
            }
          } else {
            if (v0) {
              A.Sr += S0;
              A.Wr += W0;
            }
            if (v1) {
              A.Sr += S1;
              A.Wr += W1;
            }
          }
          if (sampling) {
            if (v0) lane_race(A, S0, x0, j0);
            if (v1) lane_race(A, S1, x1, j1);
          }
          continue;
        }
      }
      // Any other tile (fp32 logits; bf16 rows off 16-byte boundaries or a
      // row's partial last group): its description first.
      const TileMeta m = meta[st];
      const unsigned char* sbase = ring + (size_t)st * Sh::kStageStride + m.delta;
      const bool any = sub * Sh::kSubGroups < m.cnt;  // warp-uniform
      const bool has0 = gl0 < m.cnt, has1 = gl1 < m.cnt;
      const int j0 = m.j0 + gl0, j1 = m.j0 + gl1;
      // fp32: whole 16-byte-aligned groups in the whole tile take the vector
      // path; every other group is read element by element
      const bool fast = m.whole != 0;
      uint32_t x0 = 0, x1 = 0;
      if (m.sampling) {
        if (has0) x0 = wd[gl0];
        if (has1) x1 = wd[gl1];
      }
      // The lane's step for group j with maximum mg: a new maximum makes it
      // the lane's top group; otherwise its sums join the rest.
      // sums(ref, S, W): the group's sums relative to ref.
      auto fold = [&](float mg, int j, uint32_t x, auto sums) {
        if (!(mg > -INFINITY)) return;  // every logit -inf: nothing, never drawn
        const bool new_top = mg > A.M;
        float S, W;
        sums(new_top ? mg : A.M, S, W);
        float Z;
        if (new_top) {
          Z = lane_new_top(A, mg, j, S, W, a.c2);
        } else {
          A.Sr += S;
          A.Wr += W;
          Z = S;
        }
        if (sampling) lane_race(A, Z, x, j);
      };
      if (!enter_row(m)) {
        fail = true;
        break;
      }
      if (any) {
        auto group = [&](bool has, int gl, int len, int j, uint32_t x) {
          if (!has) return;
          const unsigned char* gp = sbase + (size_t)gl * kGroup * elt_bytes(DT);
          const bool vec = DT == kF32 && fast;
          fold(vec ? group_max_f32(gp, rot) : elem_max<DT>(gp, len), j, x,
               [&](float ref, float& S, float& W) {
                 if (vec) {
                   group_sums_f32(gp, rot, a.c2, ref, S, W);
                   if (W >= -3.0e38f && S <= 3.0e38f) return;
                 }
                 const Exact e = elem_exact<DT>(gp, len, ref, a.c2);  // term by term
                 S = (float)e.n + e.S;
                 W = e.W;
               });
        };
        const int len0 = has0 ? min(kGroup, a.V - j0 * kGroup) : 0;
        const int len1 = has1 ? min(kGroup, a.V - j1 * kGroup) : 0;
        group(has0, gl0, len0, j0, x0);
        group(has1, gl1, len1, j1, x1);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }
    // The abort flag may change while the lanes read it: the warp acts on
    // one vote (the deposits below are warp-wide).
    if (__all_sync(0xffffffffu, !fail && !*(volatile int*)&ctrl->abort)) {
      if (cur_r >= 0) {
        if (!deposit(cur_r, false)) fail = true;
        next_r = cur_r + 1;
      }
      if (!fail && !owe_empty(r_end)) fail = true;
    }
    if (fail && lane == 0) {
      atomicOr(a.status, kStatusTimeout);
      *(volatile int*)&ctrl->abort = 1;
    }
  }

  // Every warp reaches the block barrier converged (the copy producer's lane
  // 0 leaves its loop long after lanes 1-31).
  block_sync();
  // After an abort, wait (bounded) for bulk copies still in flight into this
  // CTA's shared memory before it may exit.  Every role has left its loop, so
  // the issued count is final: first make the second arrival of every issued
  // tile the word producer did not reach, so each stage's last phase can
  // complete once its copy lands.
  const bool aborted = *(volatile int*)&ctrl->abort != 0;
  if (tid == 0 && aborted) {
    const int issued = ld_acquire_shared(&ctrl->issued);
    for (int k = ctrl->words_arrived; k < issued; ++k) mbar_arrive(&full[k % kStages]);
    for (int st = 0; st < kStages && st < issued; ++st) {
      const int n2 = (issued - st + kStages - 1) / kStages;
      mbar_wait(&full[st], (uint32_t)(n2 - 1) & 1u, kDrainLimitNs);
    }
  }
  if (!a.run_epilogue) return;
  // The decisions of the canvases this CTA completed, with every thread and
  // the ring's shared memory; they write stop flags, so first every CTA of
  // the grid must have read them (the started counter).
  const int n_epi = ctrl->n_epi;
  if (n_epi > 0 && !aborted) {
    if (tid == 0 && !ctrl->epi_ok) {
      const uint64_t t0 = global_ns();
      bool ok = true;
      while (ld_acquire_gpu(a.sync_cnt) < (int)gridDim.x) {
        if (global_ns() - t0 > a.wait_ns) {
          ok = false;
          break;
        }
        __nanosleep(64);
      }
      if (!ok) atomicOr(a.status, kStatusTimeout);
      ctrl->epi_ok = ok;
    }
    block_sync();
    if (ctrl->epi_ok) {
      const EpiSmem m = epi_smem(ring, a.L);
      for (int e = 0; e < n_epi; ++e) {
        const int bi = epi[e];
        epi_load<Sh::kThreads>(a, bi, m);
        block_sync();
        canvas_epilogue<Sh::kThreads>(a, bi, m);
        if (tid == 0) a.canvas_cnt[bi] = 0;  // zero again for the next step
        block_sync();
      }
    }
  }
  // The last CTA to leave zeroes the grid counters for the next step (the
  // release orders this CTA's reads of them before its count; the acquire,
  // everyone's before the reset).
  if (tid == 0) {
    if (atom_add_acq_rel_gpu(a.sync_cnt + 1, 1) == (int)gridDim.x - 1) {
      a.sync_cnt[0] = 0;
      a.sync_cnt[1] = 0;
    }
  }
}

}  // namespace ebk
