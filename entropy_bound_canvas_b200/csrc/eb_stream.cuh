// eb_stream.cuh -- first kernel of a sampler step: one pass over every logit
// of every active canvas.
//
// The active rows' 64-logit groups are numbered g = row * ng + j; stream CTA
// c of G owns the contiguous range [c NG / G, (c + 1) NG / G), so every CTA
// reads the same number of bytes (to within one group).  A range is walked in
// tiles of up to kTileGroups groups that never straddle a row.  Lane 0 of the
// last warp copies tiles into a kStages-deep shared-memory ring with 1-D bulk
// copies (the TMA engine, no multicast, L2 evict-first); the other warps (the
// "consumer" threads) reduce one group each per tile: the group maximum,
// sum 2^d, sum 2^d d and, for open positions, a Gumbel-perturbed group
// log-partition.  At the end of each row segment the consumer partials are
// merged and written as one Partial record; nothing else crosses CTAs, and no
// CTA waits for another.
#pragma once

#include "eb_common.cuh"

namespace ebk {

#ifndef EB_STREAM_WARPS_BF16
#define EB_STREAM_WARPS_BF16 4
#endif
#ifndef EB_STREAM_WARPS_F32
#define EB_STREAM_WARPS_F32 4
#endif
#ifndef EB_STREAM_CTAS_BF16
#define EB_STREAM_CTAS_BF16 4
#endif
#ifndef EB_STREAM_CTAS_F32
#define EB_STREAM_CTAS_F32 2
#endif

constexpr int kStages = 3;

// Shape of a stream CTA per logits dtype: consumer warps (one 64-logit group
// per consumer thread per tile), tile size, threads (consumers + 1 producer
// warp) and the CTAs meant to share an SM.  bf16: 4 consumer warps, 16 KB
// tiles, a 48 KB ring, 4 CTAs per SM.  Measured on the 1 x 256 x 262144 bf16
// canvas this beat one 16-warp CTA per SM (64 KB tiles) by 11 %: four
// independent rings keep more bulk copies in flight per SM, and a CTA that
// falls behind holds back only its own quarter of the SM.  fp32: 4 consumer
// warps, 32 KB tiles, 2 CTAs per SM (the fp32 consumer needs ~160 registers).
template <int DT>
struct StreamShape {
  static constexpr int kWarps = DT == kBF16 ? EB_STREAM_WARPS_BF16 : EB_STREAM_WARPS_F32;
  static constexpr int kCtasPerSM = DT == kBF16 ? EB_STREAM_CTAS_BF16 : EB_STREAM_CTAS_F32;
  static constexpr int kConsumers = kWarps * 32;
  static constexpr int kThreads = kConsumers + 32;
  static constexpr int kTileGroups = kConsumers;
  static constexpr int kTileBytes = kTileGroups * kGroup * elt_bytes(DT);
};

__host__ __device__ constexpr int stream_threads(int dt) {
  return dt == kBF16 ? StreamShape<kBF16>::kThreads : StreamShape<kF32>::kThreads;
}
__host__ __device__ constexpr int stream_tile_groups(int dt) {
  return dt == kBF16 ? StreamShape<kBF16>::kTileGroups : StreamShape<kF32>::kTileGroups;
}

struct StreamCtrl {
  int n_act;
  int abort;
  int issued;
  int pad;
  int wcnt[32];
};

struct StreamLayout {
  uint32_t bars, ctrl, red, act, ring, total;
};

__host__ __device__ inline uint32_t align_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

template <int DT>
__host__ __device__ inline StreamLayout stream_layout(int B) {
  StreamLayout y;
  uint32_t o = 0;
  y.bars = o;
  o = align_up(o + 16u * kStages, 16);
  y.ctrl = o;
  o = align_up(o + (uint32_t)sizeof(StreamCtrl), 16);
  y.red = o;
  o = align_up(o + (uint32_t)sizeof(Partial) * StreamShape<DT>::kWarps, 16);
  y.act = o;
  o = align_up(o + 2u * (uint32_t)B, 128);
  y.ring = o;
  o += (uint32_t)kStages * (uint32_t)StreamShape<DT>::kTileBytes;
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

// Walks a CTA's group range in tiles of up to tg groups; divides only once,
// at the start.
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
    if (cnt > tg) cnt = tg;
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

// End of a row segment: merge the 128 thread partials and write the CTA's
// partial for the row into its slot (CTA index minus the row's first CTA).
template <int DT>
__device__ __forceinline__ void flush_segment(const StepArgs& a, Partial& acc, long long r, int bi,
                                              int l, unsigned long long NG, Partial* red, int tid) {
  using Sh = StreamShape<DT>;
  const int lane = tid & 31, warp = tid >> 5;
  warp_merge(acc, a.c2);
  if (lane == 0) red[warp] = acc;
  consumer_sync(Sh::kConsumers);
  if (tid == 0) {
    Partial P = red[0];
    for (int w = 1; w < Sh::kWarps; ++w) merge(P, red[w], a.c2);
    const size_t grow = (size_t)bi * (size_t)a.L + (size_t)l;
    const int slot =
        (int)blockIdx.x - cta_of((unsigned long long)r * (unsigned long long)a.ng, NG, gridDim.x);
    a.partials[grow * (size_t)a.max_segs + (size_t)slot] = P;
  }
  consumer_sync(Sh::kConsumers);
}

template <int DT, bool TMA>
__global__ void __launch_bounds__(StreamShape<DT>::kThreads, StreamShape<DT>::kCtasPerSM)
    stream_kernel(const StepArgs a) {
  using Sh = StreamShape<DT>;
  extern __shared__ __align__(128) unsigned char smem[];
  const StreamLayout lay = stream_layout<DT>(a.B);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + lay.bars);
  uint64_t* empty = full + kStages;
  StreamCtrl* ctrl = reinterpret_cast<StreamCtrl*>(smem + lay.ctrl);
  Partial* red = reinterpret_cast<Partial*>(smem + lay.red);
  uint16_t* act = reinterpret_cast<uint16_t*>(smem + lay.act);
  unsigned char* ring = smem + lay.ring;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int st = 0; st < kStages; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], Sh::kWarps);
    }
    ctrl->abort = 0;
    ctrl->issued = 0;
    fence_mbar_init();
  }
  const int n = build_active_list(a.stop_flags, a.B, act, ctrl->wcnt, Sh::kThreads);
  if (tid == 0) ctrl->n_act = n;
  if (blockIdx.x == 0) {  // publish the active list for the finish kernel
    for (int b = tid; b < a.B; b += Sh::kThreads) a.act_index[b] = -1;
    __syncthreads();
    for (int i = tid; i < n; i += Sh::kThreads) a.act_index[act[i]] = i;
    if (tid == 0) *a.n_act = n;
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

  if (warp == Sh::kWarps) {
    // ------------------------------------------------------------ producer
    if (TMA && lane == 0) {
      const uint64_t policy = evict_first_policy();
      TileIter it(g_lo, g_hi, a.ng, a.L, Sh::kTileGroups);
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
        bulk_load(ring + (size_t)st * Sh::kTileBytes, logits + grow * row_bytes + e0 * elt_bytes(DT),
                  bytes, &full[st], policy);
        ++k;
        *(volatile int*)&ctrl->issued = k;
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    TileIter it(g_lo, g_hi, a.ng, a.L, Sh::kTileGroups);
    Tile t;
    int k = 0;
    long long cur_r = -1;
    int bi = 0, l = 0;
    bool sampling = false;
    Partial acc = empty_partial();
    // Per-warp cache of group-stream Philox words for three tiles of a row.
    Words4 wc{};
    bool wc_valid = false;
    int wc_jw0 = 0;
    const int rot = tid;  // piece rotation for bank-conflict-free reads

    while (it.next(t)) {
      if (t.r != cur_r) {
        if (cur_r >= 0) flush_segment<DT>(a, acc, cur_r, bi, l, NG, red, tid);
        cur_r = t.r;
        acc = empty_partial();
        wc_valid = false;
        bi = act[t.ai];
        l = t.l;
        sampling = !a.greedy && a.committed[(size_t)bi * (size_t)a.L + (size_t)l] == 0;
      }
      const int st = k % kStages;
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
              ring + (size_t)st * Sh::kTileBytes + (size_t)tid * kGroup * elt_bytes(DT);
          if (glen == kGroup) {
            gs = DT == kBF16 ? group_bf16_full(gp, rot, a.c2) : group_f32_full(gp, rot, a.c2);
          } else {
            gs = group_scalar<DT>(gp, glen, a.c2);
          }
        } else {
          const char* gp = logits + ((size_t)bi * (size_t)a.L + (size_t)l) * row_bytes +
                           (size_t)j * kGroup * elt_bytes(DT);
          gs = group_scalar<DT>(gp, glen, a.c2);
        }
        fold_group(acc, gs, j, a.c2);
        // group log-partition in natural units: ln2 (m c2 + log2 S)
        if (sampling) lse = 0.6931471805599453f * fmaf(gs.m, a.c2, lg2(gs.S));
      }
      if (TMA) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
      }
      if (sampling) {
        // Group-level Gumbel.  The 32 groups of this warp in one tile need at
        // most 9 Philox calls (4 words each); lanes 0-26 compute the calls of
        // this and the next two tiles of the row segment at once (the warp's
        // groups advance by one tile, 128 groups, per tile) and every lane
        // picks its word by shuffle.
        const bool need = tid < t.cnt && lse + kGumbelMax >= acc.gscore;
        if (__ballot_sync(0xffffffffu, need)) {
          const int jw = t.j0 + warp * 32;
          int dj = jw - wc_jw0;
          if (!wc_valid || dj < 0 || dj >= 3 * Sh::kTileGroups || (dj % Sh::kTileGroups) != 0) {
            wc_valid = true;
            wc_jw0 = jw;
            dj = 0;
            if (lane < 27)
              wc = philox((uint32_t)(jw >> 2) + 32u * (uint32_t)(lane / 9) + (uint32_t)(lane % 9),
                          (uint32_t)l, (uint32_t)a.s,
                          (uint32_t)(a.canvas_offset + bi) | (kStreamGroup << 24), a.key0, a.key1);
          }
          const int src = 9 * (dj / Sh::kTileGroups) + (((jw & 3) + lane) >> 2);
          const uint32_t x0 = __shfl_sync(0xffffffffu, wc.w[0], src);
          const uint32_t x1 = __shfl_sync(0xffffffffu, wc.w[1], src);
          const uint32_t x2 = __shfl_sync(0xffffffffu, wc.w[2], src);
          const uint32_t x3 = __shfl_sync(0xffffffffu, wc.w[3], src);
          if (need) {
            const uint32_t sel = (uint32_t)j & 3u;
            const uint32_t x = sel == 0 ? x0 : sel == 1 ? x1 : sel == 2 ? x2 : x3;
            // This group wins only if g > t = best - lse, i.e. E = -ln u <
            // e^-t.  Since E >= 1 - u, a group with 1 - u >= e^-t (checked
            // with a 1e-4 relative margin) cannot win: skip its logarithms.
            const float tgap = acc.gscore - lse;
            bool cand = true;
            if (tgap > -2.0f) cand = one_minus_u(x) < ex2(-1.4426950408889634f * tgap) * 1.0001f;
            if (cand) {
              const float sc = lse + gumbel(x);
              if (sc > acc.gscore) {
                acc.gscore = sc;
                acc.gidx = j;
              }
            }
          }
        }
      }
      ++k;
    }
    if (cur_r >= 0) flush_segment<DT>(a, acc, cur_r, bi, l, NG, red, tid);

    // After an abort, wait (bounded) for bulk copies still in flight into
    // this CTA's shared memory before it may exit.
    if (TMA && tid == 0 && *(volatile int*)&ctrl->abort) {
      const int issued = *(volatile int*)&ctrl->issued;
      for (int st = 0; st < kStages && st < issued; ++st) {
        const int n2 = (issued - st + kStages - 1) / kStages;
        mbar_wait(&full[st], (uint32_t)(n2 - 1) & 1u);
      }
    }
  }
  // Let the finish kernel's CTAs be scheduled; it still waits for this
  // grid's completion (and memory) before reading anything.
  griddep_launch_dependents();
}

}  // namespace ebk
