// eb_stream.cuh -- first kernel of a sampler step: one pass over every logit
// of every active canvas.
//
// Work split.  The active rows' 64-logit groups are numbered g = row ng + j
// (row = active canvas index * L + position).  Stream CTA c of G (one per SM)
// owns the contiguous range [c NG / G, (c + 1) NG / G): every CTA reads the
// same number of bytes to within one group, and a row meets only a few CTAs.
//
// Inside a CTA.  The producer warp walks the range in tiles of up to
// kStageGroups groups that never straddle a row.  For each tile it writes the
// tile's description and, for an open position, the group-stream Philox
// words of the tile's groups into the stage's header in shared memory; lane 0
// then copies the tile into a kStages-deep ring with one 1-D bulk copy (the
// TMA engine, no multicast, L2 evict-first).  A tile is cut into sub-tiles of
// 64 groups, dealt round-robin to the consumer warps (a fixed assignment, so
// every run sums in the same order).  A lane reduces two groups of its warp's
// sub-tile; the warp shares one running maximum per row (WarpAcc), so its
// lanes' sums stay relative to the same reference and the Gumbel race runs
// against the warp's best.  When a warp moves on to another row it sums its
// lanes and writes one Partial record for (row, CTA, warp); it writes an
// empty record for
// each row of its CTA's range that it never touched, so the finish kernel
// only ever reads records written during this step.
#pragma once

#include "eb_common.cuh"

namespace ebk {

#ifndef EB_STREAM_CONSUMER_WARPS
#define EB_STREAM_CONSUMER_WARPS 12
#endif
#ifndef EB_STREAM_STAGES
#define EB_STREAM_STAGES 6
#endif
#ifndef EB_STREAM_STAGE_KB
#define EB_STREAM_STAGE_KB 32
#endif
#ifndef EB_STREAM_GROUPS_PER_LANE
#define EB_STREAM_GROUPS_PER_LANE 2
#endif

constexpr int kStages = EB_STREAM_STAGES;

// Shape of the stream CTA: kConsumerWarps consumer warps + 2 producer warps,
// a ring of kStages stages of kStageBytes each (192 KB with the defaults:
// one CTA per SM).  Twelve consumer warps, each lane reducing two groups at
// a time, keep the SM's MUFU and FMA pipes busy.
template <int DT>
struct StreamShape {
  static constexpr int kConsumerWarps = EB_STREAM_CONSUMER_WARPS;
  static constexpr int kThreads = (kConsumerWarps + 2) * 32;  // + copy and word producers
  static constexpr int kStageBytes = EB_STREAM_STAGE_KB * 1024;
  // room for a copy widened to 16-byte boundaries; 128-byte aligned stages
  static constexpr int kStageStride = kStageBytes + 128;
  static constexpr int kStageGroups = kStageBytes / (kGroup * elt_bytes(DT));
  static constexpr int kGroupsPerLane = EB_STREAM_GROUPS_PER_LANE;
  static constexpr int kSubGroups = 32 * kGroupsPerLane;  // groups per sub-tile
  static constexpr int kSubPerStage = kStageGroups / kSubGroups;
  static_assert(kSubPerStage >= 1 && (kSubPerStage & (kSubPerStage - 1)) == 0,
                "sub-tiles per stage must be a power of two");
};

__host__ __device__ constexpr int stream_threads(int dt) {
  return dt == kBF16 ? StreamShape<kBF16>::kThreads : StreamShape<kF32>::kThreads;
}
__host__ __device__ constexpr int stream_consumer_warps() { return EB_STREAM_CONSUMER_WARPS; }

struct StreamCtrl {
  int abort;
  int issued;  // tiles whose bulk copy has been issued
  int n_sub;   // sub-tiles of this CTA's range
  int wcnt[32];
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
  int pad;
};

struct StreamLayout {
  uint32_t bars, ctrl, meta, words, act, ring, total;
};

__host__ __device__ inline uint32_t align_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

template <int DT>
__host__ __device__ inline StreamLayout stream_layout(int B) {
  using Sh = StreamShape<DT>;
  StreamLayout y;
  uint32_t o = 0;
  y.bars = o;
  o = align_up(o + 16u * kStages, 16);
  y.ctrl = o;
  o = align_up(o + (uint32_t)sizeof(StreamCtrl), 16);
  y.meta = o;
  o = align_up(o + (uint32_t)sizeof(TileMeta) * kStages, 16);
  y.words = o;
  o = align_up(o + 4u * (uint32_t)Sh::kStageGroups * kStages, 16);
  y.act = o;
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

// Active canvases in index order, from the stop flags as they were when the
// step began (only the finish kernel, after this one, writes them).
__device__ __forceinline__ int build_active_list(const uint8_t* stop_flags, int B, uint16_t* act,
                                                 int* wcnt, int nthreads) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nwarps = nthreads / 32;
  int base = 0;
  for (int b0 = 0; b0 < B; b0 += nthreads) {
    const int b = b0 + tid;
    const bool on = b < B && __ldcg(stop_flags + b) == 0;
    const unsigned bal = __ballot_sync(0xffffffffu, on);
    if (lane == 0) wcnt[warp] = __popc(bal);
    __syncthreads();
    int off = base;
    for (int w = 0; w < warp; ++w) off += wcnt[w];
    if (on) act[off + __popc(bal & ((1u << lane) - 1u))] = (uint16_t)b;
    for (int w = 0; w < nwarps; ++w) base += wcnt[w];
    __syncthreads();
  }
  return base;
}

// One CTA per SM: the register cap is the register file over the block.
template <int DT>
__global__ void __launch_bounds__(StreamShape<DT>::kThreads, 1) stream_kernel(const StepArgs a) {
  using Sh = StreamShape<DT>;
  using IO = GroupIO<DT>;
  extern __shared__ __align__(128) unsigned char smem[];
  const StreamLayout lay = stream_layout<DT>(a.B);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + lay.bars);
  uint64_t* empty = full + kStages;
  StreamCtrl* ctrl = reinterpret_cast<StreamCtrl*>(smem + lay.ctrl);
  TileMeta* meta = reinterpret_cast<TileMeta*>(smem + lay.meta);
  uint32_t* words = reinterpret_cast<uint32_t*>(smem + lay.words);
  uint16_t* act = reinterpret_cast<uint16_t*>(smem + lay.act);
  unsigned char* ring = smem + lay.ring;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int st = 0; st < kStages; ++st) {
      mbar_init(&full[st], 2);  // the copy's arrival (+ bytes) and the header's
      mbar_init(&empty[st], Sh::kSubPerStage);
    }
    ctrl->abort = 0;
    ctrl->issued = 0;
    fence_mbar_init();
  }
  const int n_act = build_active_list(a.stop_flags, a.B, act, ctrl->wcnt, Sh::kThreads);
  if (blockIdx.x == 0) {  // publish the active list for the finish kernel
    for (int b = tid; b < a.B; b += Sh::kThreads) a.act_index[b] = -1;
    __syncthreads();
    for (int i = tid; i < n_act; i += Sh::kThreads) a.act_index[act[i]] = i;
    if (tid == 0) *a.n_act = n_act;
  }
  const int G = gridDim.x;
  const unsigned long long NG =
      (unsigned long long)n_act * (unsigned long long)a.L * (unsigned long long)a.ng;
  const unsigned long long g_lo = range_start(blockIdx.x, NG, G);
  const unsigned long long g_hi = range_start(blockIdx.x + 1, NG, G);
  if (tid == 0) ctrl->n_sub = count_tiles(g_lo, g_hi, a.ng, Sh::kStageGroups) * Sh::kSubPerStage;
  __syncthreads();
  // The finish kernel may be scheduled from now on, wherever an SM has room:
  // its CTAs load what the previous step left and then wait for this grid's
  // completion (griddepcontrol.wait) before reading anything it writes.
  griddep_launch_dependents();

  const size_t row_bytes = (size_t)a.V * (size_t)elt_bytes(DT);
  const char* logits = reinterpret_cast<const char*>(a.logits);

  if (warp == Sh::kConsumerWarps) {
    // ------------------------------------------------------- copy producer
    // Lane 0 alone: waits for a free stage, writes the tile's description
    // and issues its bulk copy (the stage's first arrival, with the bytes).
    if (lane == 0) {
      const uint64_t policy = evict_first_policy();
      TileIter it(g_lo, g_hi, a.ng, a.L, Sh::kStageGroups);
      Tile t;
      int k = 0, st = 0;
      uint32_t ph = 0;  // parity of the current pass over the ring
      long long row_seen = -1;
      int bi = 0, samp = 0;
      while (it.next(t)) {
        if (k >= kStages && !mbar_wait(&empty[st], ph ^ 1u)) {
          atomicOr(a.status, kStatusTimeout);
          *(volatile int*)&ctrl->abort = 1;
          break;
        }
        if (*(volatile int*)&ctrl->abort) break;
        const bool new_row = t.r != row_seen;
        if (new_row) {
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
        // The position's committed flag is read while the copy is in flight.
        // Nothing reads the description before the release of `issued`, and
        // the stage cannot fill before the word producer's arrival, which
        // follows that release.
        if (new_row)
          samp = !a.greedy && a.committed[(size_t)bi * (size_t)a.L + (size_t)t.l] == 0;
        TileMeta m;
        m.r = (int)t.r;
        m.j0 = t.j0;
        m.cnt = t.cnt;
        m.bi = bi;
        m.l = t.l;
        m.sampling = samp;
        m.delta = (int)(reinterpret_cast<uintptr_t>(src) - a0);
        m.pad = 0;
        meta[st] = m;
        st_release_shared(&ctrl->issued, k + 1);
        ++k;
        if (++st == kStages) {
          st = 0;
          ph ^= 1u;
        }
      }
    }
  } else if (warp == Sh::kConsumerWarps + 1) {
    // ------------------------------------------------------- word producer
    // Follows the copy producer: once tile k is issued (so its stage is free
    // and its description written), computes the group-stream Philox words
    // of an open position's groups into the stage's header and makes the
    // stage's second arrival.  Kept off the copy producer so that copies are
    // never issued late.
    const int n_tiles = ctrl->n_sub / Sh::kSubPerStage;
    int st = 0, words_done = 0;
    for (int k = 0; k < n_tiles; ++k, words_done = k) {
      if (!wait_counter_above(&ctrl->issued, k)) {
        if (lane == 0) {
          atomicOr(a.status, kStatusTimeout);
          *(volatile int*)&ctrl->abort = 1;
        }
        break;
      }
      const TileMeta m = meta[st];
      if (m.sampling) {
        uint32_t* wd = words + st * Sh::kStageGroups;
        const int gj0 = (a.v_off >> 6) + m.j0;  // global group id of the tile's first group
        const int c0 = gj0 >> 2, c1 = (gj0 + m.cnt - 1) >> 2;
        const uint32_t c3 = (uint32_t)(a.canvas_offset + m.bi) | (kStreamGroup << 24);
        for (int c = c0 + lane; c <= c1; c += 32) {
          const Words4 w = philox((uint32_t)c, (uint32_t)m.l, (uint32_t)a.s, c3, a.key0, a.key1);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int j = 4 * c + q - gj0;
            if (j >= 0 && j < m.cnt) wd[j] = w.w[q];
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&full[st]);  // header (words) complete
      if (++st == kStages) st = 0;
    }
    // After an abort: the second arrival of every tile already issued, so
    // that the drain below sees each copy complete.
    if (lane == 0 && *(volatile int*)&ctrl->abort) {
      const int issued = ld_acquire_shared(&ctrl->issued);
      for (int k = words_done; k < issued; ++k) mbar_arrive(&full[k % kStages]);
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int n_sub = ctrl->n_sub;
    const long long r_first = (long long)(g_lo / (unsigned long long)a.ng);
    const long long r_end =
        g_hi > g_lo ? (long long)((g_hi - 1ull) / (unsigned long long)a.ng) + 1 : r_first;
    // slot of this CTA among the CTAs of its first row; later rows start in it
    const int seg_first =
        (int)blockIdx.x - cta_of((unsigned long long)r_first * (unsigned long long)a.ng, NG, G);
    const size_t spr = (size_t)(a.max_segs * a.nw);
    auto record_of = [&](long long r, int bi, int l) {
      const int seg = r == r_first ? seg_first : 0;
      return ((size_t)bi * (size_t)a.L + (size_t)l) * spr + (size_t)(seg * a.nw + warp);
    };
    long long cur_r = -1;
    long long next_r = r_first;  // first row of the range this warp still owes a record
    size_t cur_rec = 0;
    int sampling = 0;
    WarpAcc A;
    warp_reset(A);
    const int rot = lane;

    auto owe_empty = [&](long long upto) {
      for (; next_r < upto; ++next_r) {
        if (lane == 0) {
          const int ai = (int)(next_r / a.L);
          const int l = (int)(next_r - (long long)ai * a.L);
          a.partials[record_of(next_r, act[ai], l)] = empty_partial();
        }
      }
    };
    auto flush = [&]() {
      const Partial P = warp_record(A, a.iT);
      if (lane == 0) a.partials[cur_rec] = P;
    };

    // Sub-tiles are dealt round-robin: warp w takes w, w + nw, w + 2 nw, ...
    for (int u = warp; u < n_sub; u += Sh::kConsumerWarps) {
      if (*(volatile int*)&ctrl->abort) break;
      const int k = u / Sh::kSubPerStage;
      const int sub = u & (Sh::kSubPerStage - 1);
      const int st = k % kStages;
      // A warp may run up to a few sub-tiles ahead of the ring, past the
      // stage's current phase; the parity of the full barrier is only
      // unambiguous once the producer has issued tile k (which it does after
      // the stage's previous tile, k - kStages, was released).
      if (!wait_counter_above(&ctrl->issued, k) ||
          !mbar_wait(&full[st], (uint32_t)(k / kStages) & 1u)) {
        if (lane == 0) {
          atomicOr(a.status, kStatusTimeout);
          *(volatile int*)&ctrl->abort = 1;
        }
        break;
      }
      const TileMeta m = meta[st];
      if (m.r != cur_r) {
        if (cur_r >= 0) flush();
        owe_empty(m.r);
        cur_r = m.r;
        next_r = cur_r + 1;
        cur_rec = record_of(cur_r, m.bi, m.l);
        sampling = m.sampling;
        warp_reset(A);
      }
      const int gl0 = sub * Sh::kSubGroups + lane, gl1 = gl0 + 32;
      if (sub * Sh::kSubGroups < m.cnt) {  // warp-uniform
        const bool has0 = gl0 < m.cnt, has1 = Sh::kGroupsPerLane == 2 && gl1 < m.cnt;
        const unsigned char* sbase = ring + (size_t)st * Sh::kStageStride + m.delta;
        const unsigned char* gp0 = sbase + (size_t)(has0 ? gl0 : 0) * kGroup * elt_bytes(DT);
        const unsigned char* gp1 = has1 ? sbase + (size_t)gl1 * kGroup * elt_bytes(DT) : gp0;
        const int j0 = m.j0 + gl0, j1 = m.j0 + gl1;
        const int len0 = has0 ? min(kGroup, a.V - j0 * kGroup) : 0;
        const int len1 = has1 ? min(kGroup, a.V - j1 * kGroup) : 0;
        const bool fast = a.vec_ok && (!has0 || len0 == kGroup) && (!has1 || len1 == kGroup);
        float mg0, mg1;
        if (fast) {
          mg0 = IO::max_of(gp0, rot);
          mg1 = Sh::kGroupsPerLane == 2 ? IO::max_of(gp1, rot) : -INFINITY;
        } else {
          mg0 = has0 ? group_max_safe<DT>(gp0, len0) : -INFINITY;
          mg1 = has1 ? group_max_safe<DT>(gp1, len1) : -INFINITY;
        }
        if (!has0) mg0 = -INFINITY;
        if (!has1) mg1 = -INFINITY;
        warp_raise(A, fmaxf(mg0, mg1), mg0 >= mg1 ? j0 : j1, a.c2);
        float S0 = 0.f, W0 = 0.f, S1 = 0.f, W1 = 0.f;
        if (fast) {
          if constexpr (Sh::kGroupsPerLane == 2) {
            IO::exp2_of(gp0, gp1, rot, a.c2, A.M, A.M, S0, W0, S1, W1);
          } else {
            IO::exp1_of(gp0, rot, a.c2, A.M, S0, W0);
          }
          // -inf (or other non-finite) logits: redo the group term by term
          if (!(W0 >= -3.0e38f)) {
            const float2 q = group_sums_safe<DT>(gp0, kGroup, a.c2, A.M);
            S0 = q.x;
            W0 = q.y;
          }
          if (has1 && !(W1 >= -3.0e38f)) {
            const float2 q = group_sums_safe<DT>(gp1, kGroup, a.c2, A.M);
            S1 = q.x;
            W1 = q.y;
          }
        } else {
          if (has0) {
            const float2 q = group_sums_safe<DT>(gp0, len0, a.c2, A.M);
            S0 = q.x;
            W0 = q.y;
          }
          if (has1) {
            const float2 q = group_sums_safe<DT>(gp1, len1, a.c2, A.M);
            S1 = q.x;
            W1 = q.y;
          }
        }
        if (has0) warp_fold(A, S0, W0, j0);
        if (has1) warp_fold(A, S1, W1, j1);
        if (sampling) {
          const uint32_t* wd = words + st * Sh::kStageGroups;
          float Rl = A.R;
          int gbl = 0x7fffffff;
          if (has0) lane_race(Rl, gbl, S0, wd[gl0], j0);
          if (has1) lane_race(Rl, gbl, S1, wd[gl1], j1);
          warp_race_merge(A, Rl, gbl);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }
    if (cur_r >= 0) flush();
    owe_empty(r_end);
  }

  __syncthreads();
  // After an abort, wait (bounded) for bulk copies still in flight into this
  // CTA's shared memory before it may exit.
  if (tid == 0 && *(volatile int*)&ctrl->abort) {
    const int issued = ld_acquire_shared(&ctrl->issued);
    for (int st = 0; st < kStages && st < issued; ++st) {
      const int n2 = (issued - st + kStages - 1) / kStages;
      mbar_wait(&full[st], (uint32_t)(n2 - 1) & 1u);
    }
  }
}

}  // namespace ebk
