// eb_finish.cuh -- the per-canvas decisions of a sampler step (the canvas
// epilogue), the combine of vocabulary-slice records, and the initial canvas.
//
// Every position's entropy, argmax, max probability and draw are in global
// memory when a canvas's decisions run: argmax stability, adaptive stop,
// commit rule, last-step / all-committed finalisation and renoise.  The
// stream kernel runs them in the CTA that finishes the canvas's last
// position; the combine kernel runs them for vocabulary-sharded logits.  The
// entropy-bound rule sorts the candidates by (entropy, position) with a
// bitonic sort in shared memory and commits the prefix whose float64 running
// sum stays within the bound.
//
// Pages (cited by title and section): DiffusionGemma model card, "Best
// practices, 1. Diffusion sampling settings" (lowest-entropy selection under
// entropy_bound = 0.1, full renoise of unselected tokens, stop when the mean
// entropy is below 0.005 and the top prediction is unchanged over two steps);
// diffusers "DiffusionGemma" page, "Schedulers" (EntropyBoundScheduler joint
// entropy bound, BlockRefinementScheduler threshold plus per-step quota,
// DiscreteDDIM committing its predictions at the last step) and "Adaptive
// stopping" (stability_threshold, confidence_threshold, per-sample freeze).
#pragma once

#include "eb_common.cuh"

namespace ebk {

constexpr int kEpiThreads = 256;  // the combine kernel's block

// Scratch of the block-wide helpers (up to 32 warps).
struct EpiCtrl {
  int stable_prev;
  int pad;
  double dscr[32];
  int iscr[32];
  int cscr[32];
  unsigned long long uscr[32];
};

__host__ __device__ inline int pow2_at_least(int n) {
  int p = 1;
  while (p < n) p <<= 1;
  return p;
}

struct EpiLayout {
  uint32_t ctrl, keys, cum, H, am, smp, pm, prev, tok, open, pick, total;
};

__host__ __device__ inline EpiLayout epi_layout(int L) {
  EpiLayout y;
  uint32_t o = 0;
  const uint32_t l = (uint32_t)L, P = (uint32_t)pow2_at_least(L);
  y.ctrl = o;
  o += (uint32_t)((sizeof(EpiCtrl) + 15) / 16 * 16);
  y.keys = o;
  o += 8u * P;
  y.cum = o;
  o += 8u * P;
  y.H = o;
  o += 4u * l;
  y.am = o;
  o += 4u * l;
  y.smp = o;
  o += 4u * l;
  y.pm = o;
  o += 4u * l;
  y.prev = o;
  o += 4u * l;
  y.tok = o;
  o += 4u * l;
  y.open = o;
  o += l;
  y.pick = o;
  o += l;
  y.total = (o + 15) / 16 * 16;
  return y;
}

struct EpiSmem {
  EpiCtrl* ctrl;
  unsigned long long* keys;
  double* cum;
  float* H;
  int* am;
  int* smp;
  float* pm;
  int* prev;
  int* tok;
  uint8_t* open;
  uint8_t* pick;
};

__device__ __forceinline__ EpiSmem epi_smem(unsigned char* smem, int L) {
  const EpiLayout y = epi_layout(L);
  EpiSmem m;
  m.ctrl = reinterpret_cast<EpiCtrl*>(smem + y.ctrl);
  m.keys = reinterpret_cast<unsigned long long*>(smem + y.keys);
  m.cum = reinterpret_cast<double*>(smem + y.cum);
  m.H = reinterpret_cast<float*>(smem + y.H);
  m.am = reinterpret_cast<int*>(smem + y.am);
  m.smp = reinterpret_cast<int*>(smem + y.smp);
  m.pm = reinterpret_cast<float*>(smem + y.pm);
  m.prev = reinterpret_cast<int*>(smem + y.prev);
  m.tok = reinterpret_cast<int*>(smem + y.tok);
  m.open = smem + y.open;
  m.pick = smem + y.pick;
  return m;
}

// ---------------------------------------------------------------------------
// Block helpers (NT threads, __syncthreads)
// ---------------------------------------------------------------------------
template <int NT>
__device__ __forceinline__ int epi_block_sum_int(int v, EpiCtrl* c) {
  const int tid = threadIdx.x;
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((tid & 31) == 0) c->iscr[tid >> 5] = v;
  block_sync();
  int r = 0;
  for (int w = 0; w < NT / 32; ++w) r += c->iscr[w];
  block_sync();
  return r;
}

template <int NT>
__device__ __forceinline__ unsigned long long epi_block_min(unsigned long long v, EpiCtrl* c) {
  const int tid = threadIdx.x;
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const unsigned long long w = __shfl_xor_sync(0xffffffffu, v, o);
    v = w < v ? w : v;
  }
  if ((tid & 31) == 0) c->uscr[tid >> 5] = v;
  block_sync();
  unsigned long long r = c->uscr[0];
  for (int w = 1; w < NT / 32; ++w) r = c->uscr[w] < r ? c->uscr[w] : r;
  block_sync();
  return r;
}

// One block-wide pass: sum of a (double), OR of b, exclusive prefix of c
// (*c_total gets the sum of c).
template <int NT>
__device__ __forceinline__ void epi_block_reduce(double& a, int& b, int& c, int* c_total,
                                                 EpiCtrl* ctrl) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  double x = a;
  int y = b, z = c;
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    x += __shfl_xor_sync(0xffffffffu, x, o);
    y |= __shfl_xor_sync(0xffffffffu, y, o);
  }
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, z, o);
    if (lane >= o) z += t;
  }
  if (lane == 31) {
    ctrl->dscr[warp] = x;
    ctrl->iscr[warp] = y;
    ctrl->cscr[warp] = z;
  }
  block_sync();
  double sx = 0.0;
  int sy = 0, off = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) {
    sx += ctrl->dscr[w];
    sy |= ctrl->iscr[w];
    if (w < warp) off += ctrl->cscr[w];
    tot += ctrl->cscr[w];
  }
  block_sync();
  a = sx;
  b = sy;
  c = off + z - c;
  *c_total = tot;
}

// Ascending bitonic sort of keys[0, P) (P a power of two).
template <int NT>
__device__ __forceinline__ void epi_bitonic_sort(unsigned long long* keys, int P) {
  const int tid = threadIdx.x;
  for (int k = 2; k <= P; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < P; i += NT) {
        const int p = i ^ j;
        if (p > i) {
          const unsigned long long x = keys[i], y = keys[p];
          const bool up = (i & k) == 0;
          if ((x > y) == up) {
            keys[i] = y;
            keys[p] = x;
          }
        }
      }
      block_sync();
    }
  }
}

// Inclusive float64 prefix sums cum[i] = sum_{m <= i} val(keys[m]), i < P,
// with P / NT consecutive elements per thread.
template <int NT, class Val>
__device__ __forceinline__ void epi_prefix_sum(const unsigned long long* keys, double* cum, int P,
                                               Val val, EpiCtrl* ctrl) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (P + NT - 1) / NT;
  const int i0 = tid * per;
  double run = 0.0;
  for (int e = 0; e < per && i0 + e < P; ++e) {
    run += val(keys[i0 + e]);
    cum[i0 + e] = run;
  }
  double x = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double t = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += t;
  }
  if (lane == 31) ctrl->dscr[warp] = x;
  block_sync();
  double off = x - run;
  for (int w = 0; w < warp; ++w) off += ctrl->dscr[w];
  for (int e = 0; e < per && i0 + e < P; ++e) cum[i0 + e] += off;
  block_sync();
}

// Ascending bitonic sort of 32 K keys held by one warp, K consecutive keys
// per lane (key index lane K + e); partners within a lane are swapped in
// registers, partners in other lanes are exchanged with shuffles.
template <int K>
__device__ __forceinline__ void warp_bitonic_sort(unsigned long long (&v)[K]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 2; k <= 32 * K; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j < K) {
#pragma unroll
        for (int e = 0; e < K; ++e) {
          if (e & j) continue;
          const int i = lane * K + e;
          const bool up = (i & k) == 0;
          const unsigned long long x = v[e], y = v[e ^ j];
          if ((x > y) == up) {
            v[e] = y;
            v[e ^ j] = x;
          }
        }
      } else {
#pragma unroll
        for (int e = 0; e < K; ++e) {
          const int i = lane * K + e;
          const bool up = (i & k) == 0;
          const bool lower = (i & j) == 0;
          const unsigned long long o = __shfl_xor_sync(0xffffffffu, v[e], j / K);
          v[e] = (lower == up) ? (o < v[e] ? o : v[e]) : (o > v[e] ? o : v[e]);
        }
      }
    }
  }
}

// Sort keys: ascending (H, l) (H >= 0, so its float bits order like the
// value) and descending probability, ascending position.
__device__ __forceinline__ unsigned long long key_asc(float H, int l) {
  const float h = H > 0.f ? H : 0.f;
  return ((unsigned long long)__float_as_uint(h) << 32) | (unsigned)l;
}
__device__ __forceinline__ unsigned long long key_desc(float p, int l) {
  const float q = p > 0.f ? p : 0.f;
  return ((unsigned long long)(~__float_as_uint(q)) << 32) | (unsigned)l;
}
__device__ __forceinline__ float key_value(unsigned long long k) {
  return __uint_as_float((uint32_t)(k >> 32));
}

// The commit selection of n_c <= 32 K candidate keys (keys[0, n_c) in shared
// memory) by one warp: sort, then EB: pick every candidate whose float64
// prefix sum of entropies (in sorted order) stays <= gamma; BR: pick the
// first `quota`.
template <int K>
__device__ __forceinline__ void warp_select(const StepArgs& a, const unsigned long long* keys,
                                            int n_c, bool br, uint8_t* pick) {
  const int lane = threadIdx.x & 31;
  unsigned long long v[K];
#pragma unroll
  for (int e = 0; e < K; ++e) {
    const int i = lane * K + e;
    v[e] = i < n_c ? keys[i] : ~0ull;
  }
  warp_bitonic_sort<K>(v);
  if (br) {
#pragma unroll
    for (int e = 0; e < K; ++e) {
      const int i = lane * K + e;
      if (i < n_c && i < a.quota) pick[(int)(v[e] & 0xffffffffu)] = 1;
    }
    return;
  }
  double c[K];
  double run = 0.0;
#pragma unroll
  for (int e = 0; e < K; ++e) {
    run += v[e] == ~0ull ? 0.0 : (double)key_value(v[e]);
    c[e] = run;
  }
  double x = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double t = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += t;
  }
  const double off = x - run;
#pragma unroll
  for (int e = 0; e < K; ++e) {
    const int i = lane * K + e;
    if (i < n_c && off + c[e] <= a.gamma) pick[(int)(v[e] & 0xffffffffu)] = 1;
  }
}

// ---------------------------------------------------------------------------
// Canvas epilogue (one CTA, values of every position in shared memory)
// ---------------------------------------------------------------------------
template <int NT>
__device__ void canvas_epilogue(const StepArgs& a, int bi, const EpiSmem& m) {
  const int tid = threadIdx.x;
  const int L = a.L;
  const size_t row0 = (size_t)bi * (size_t)L;
  const bool br = a.rule == kRuleBR;
  EpiCtrl* ctrl = m.ctrl;

  // pass 1: entropy sum, argmax stability, candidates (EB: open with
  // H <= gamma, no other can be in the prefix; BR: open below the threshold,
  // which compete for the quota, while those at or above it commit outright)
  double sumH = 0.0;
  int neq = a.s < 1 ? 1 : 0;
  int ncand = 0;
  for (int l = tid; l < L; l += NT) {
    m.pick[l] = 0;
    sumH += (double)m.H[l];
    if (a.s >= 1 && m.am[l] != m.prev[l]) neq = 1;
    if (!m.open[l]) {
      const int tok = m.tok[l];
      if (tok < 0 || tok >= a.V_tot) atomicOr(a.status, kStatusBadToken);
    } else if (!br) {
      ncand += (double)m.H[l] <= a.gamma ? 1 : 0;
    } else if (!((double)m.pm[l] >= a.theta)) {
      ++ncand;
    }
  }
  int n_c = 0;
  int pos = ncand;
  epi_block_reduce<NT>(sumH, neq, pos, &n_c, ctrl);
  const int stable_new = neq ? 0 : ctrl->stable_prev + 1;
  const double meanH = sumH / (double)L;
  const bool fired = a.stop_enabled && stable_new >= a.stability_steps && meanH < a.tau;
  const bool last_step = a.s == a.N - 1;

  if (!fired) {
    const int P = pow2_at_least(n_c > 0 ? n_c : 1);
    for (int l = tid; l < L; l += NT) {
      if (!m.open[l]) continue;
      if (!br) {
        if ((double)m.H[l] <= a.gamma) m.keys[pos++] = key_asc(m.H[l], l);
      } else if ((double)m.pm[l] >= a.theta) {
        m.pick[l] = 1;
      } else {
        m.keys[pos++] = key_desc(m.pm[l], l);
      }
    }
    block_sync();
    if (P <= 256) {
      // one warp sorts and selects in registers
      if (tid < 32) {
        if (P <= 32) {
          warp_select<1>(a, m.keys, n_c, br, m.pick);
        } else if (P <= 64) {
          warp_select<2>(a, m.keys, n_c, br, m.pick);
        } else if (P <= 128) {
          warp_select<4>(a, m.keys, n_c, br, m.pick);
        } else {
          warp_select<8>(a, m.keys, n_c, br, m.pick);
        }
      }
    } else {
      for (int i = n_c + tid; i < P; i += NT) m.keys[i] = ~0ull;
      block_sync();
      epi_bitonic_sort<NT>(m.keys, P);
      if (!br) {
        // EB: the longest prefix in (H, l) order whose entropy sum stays
        // within gamma (the sums grow along the order)
        epi_prefix_sum<NT>(
            m.keys, m.cum, P,
            [](unsigned long long k) { return k == ~0ull ? 0.0 : (double)key_value(k); }, ctrl);
        for (int i = tid; i < n_c; i += NT)
          if (m.cum[i] <= a.gamma) m.pick[(int)(m.keys[i] & 0xffffffffu)] = 1;
      } else {
        // BR: the quota goes to the first candidates in (-pmax, l) order
        for (int i = tid; i < n_c && i < a.quota; i += NT)
          m.pick[(int)(m.keys[i] & 0xffffffffu)] = 1;
      }
    }
    block_sync();
    // EB with no candidate: the single lowest (H, l).  MI: the prefix plus
    // the next open position in (H, l) order.  Candidates (H <= gamma) come
    // before every other open position, so both are the lowest open
    // position left out of the prefix.
    if (!br && (a.rule == kRuleMI || n_c == 0)) {
      unsigned long long best = ~0ull;
      for (int l = tid; l < L; l += NT) {
        if (!m.open[l] || m.pick[l]) continue;
        const unsigned long long kk = key_asc(m.H[l], l);
        best = kk < best ? kk : best;
      }
      best = epi_block_min<NT>(best, ctrl);
      if (tid == 0 && best != ~0ull) m.pick[(int)(best & 0xffffffffu)] = 1;
      block_sync();
    }
  }

  // commit, renoise, remember the argmax
  const uint32_t bg = (uint32_t)(a.canvas_offset + bi);
  int left = 0;
  const bool edit = !fired && a.eps_edit >= 0.0;
  for (int l = tid; l < L; l += NT) {
    if (!m.open[l]) {
      // block refinement editing: a committed position whose argmax moved
      // takes it when the argmax is confident enough
      if (edit && m.am[l] != m.tok[l] && (double)m.pm[l] >= a.eps_edit) a.canvas[row0 + l] = m.am[l];
    } else {
      if (fired) {
        a.canvas[row0 + l] = m.am[l];
        a.committed[row0 + l] = 1;
      } else if (m.pick[l] || last_step) {
        a.canvas[row0 + l] = a.greedy ? m.am[l] : m.smp[l];
        a.committed[row0 + l] = 1;
      } else {
        ++left;
        const Words4 r = philox((uint32_t)l >> 2, 0u, (uint32_t)a.s, bg | (kStreamRenoise << 24),
                                a.key0, a.key1);
        a.canvas[row0 + l] =
            (int32_t)uniform_token(pick_word(r, (uint32_t)l & 3u), (uint32_t)a.V_tot);
      }
    }
    a.prev_amax[row0 + l] = m.am[l];
  }
  const int left_tot = epi_block_sum_int<NT>(left, ctrl);
  if (tid == 0) {
    a.stable[bi] = stable_new;
    a.stop_flags[bi] = (uint8_t)(fired ? 1 : last_step ? 3 : left_tot == 0 ? 2 : 0);
  }
}

// What the previous step left: argmax, tokens, open flags, stability.
template <int NT>
__device__ __forceinline__ void epi_load_state(const StepArgs& a, int bi, const EpiSmem& m) {
  const size_t row0 = (size_t)bi * (size_t)a.L;
  for (int l = threadIdx.x; l < a.L; l += NT) {
    m.prev[l] = a.prev_amax[row0 + l];
    m.tok[l] = a.canvas[row0 + l];
    m.open[l] = a.committed[row0 + l] == 0;
  }
  if (threadIdx.x == 0) m.ctrl->stable_prev = a.stable[bi];
}

// What the previous step left and this step's per-position results of
// canvas bi (written by other CTAs: read through L2), all of a position's
// loads issued before its shared-memory stores.
template <int NT>
__device__ __forceinline__ void epi_load(const StepArgs& a, int bi, const EpiSmem& m) {
  const size_t row0 = (size_t)bi * (size_t)a.L;
  if (threadIdx.x == 0) m.ctrl->stable_prev = a.stable[bi];
  for (int l = threadIdx.x; l < a.L; l += NT) {
    const int prev = a.prev_amax[row0 + l];
    const int tok = a.canvas[row0 + l];
    const uint8_t cm = a.committed[row0 + l];
    const float H = __ldcg(a.H_out + row0 + l);
    const int am = __ldcg(a.amax_out + row0 + l);
    const int smp = __ldcg(a.sample + row0 + l);
    const float pm = __ldcg(a.pmax + row0 + l);
    m.prev[l] = prev;
    m.tok[l] = tok;
    m.open[l] = cm == 0;
    m.H[l] = H;
    m.am[l] = am;
    m.smp[l] = smp;
    m.pm[l] = pm;
  }
}

// ---------------------------------------------------------------------------
// Vocabulary-sharded logits: the n slices' records of each position, in
// slice order, give the position's entropy, max probability, argmax and draw
// (the largest slice maximum; the sums rescaled to it; the first slice
// attaining it for the argmax; the best slice score, earlier slice on a tie,
// for the draw); then the canvas epilogue.  One CTA per canvas.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kEpiThreads) combine_kernel(const StepArgs a,
                                                              const int32_t* act_index,
                                                              const SliceRecord* records,
                                                              int n_slices) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int bi = blockIdx.x;
  if (act_index[bi] < 0) return;  // a stopped canvas is untouched
  const EpiSmem m = epi_smem(smem, a.L);
  epi_load_state<kEpiThreads>(a, bi, m);
  const size_t stride = (size_t)a.B * (size_t)a.L;
  for (int l = threadIdx.x; l < a.L; l += kEpiThreads) {
    const size_t grow = (size_t)bi * (size_t)a.L + (size_t)l;
    float M = -INFINITY;
    int am = kNone;
    for (int g = 0; g < n_slices; ++g) {
      const SliceRecord& r = records[(size_t)g * stride + grow];
      if (r.zmax > M) {
        M = r.zmax;
        am = r.amax;
      }
    }
    double S = 0.0, W = 0.0;
    float best = -INFINITY;
    int x = -1;
    for (int g = 0; g < n_slices; ++g) {
      const SliceRecord r = records[(size_t)g * stride + grow];
      if (r.gscore > best) {
        best = r.gscore;
        x = r.sample;
      }
      if (!(r.zmax > -INFINITY)) continue;
      const double dd = (double)(r.zmax - M) * (double)a.c2;
      const double f = exp2(dd);
      S += f * r.S;
      W += f * (r.W + dd * r.S);
    }
    const float H = (float)(log(S) - 0.6931471805599453 * (W / S));
    const float pm = (float)(1.0 / S);
    if (!isfinite(S) || !isfinite(W) || am == kNone) atomicOr(a.status, kStatusNonFinite);
    const bool open = m.open[l] != 0;
    const int smp = open ? (a.greedy || x < 0 ? am : x) : -1;
    a.H_out[grow] = H;
    a.amax_out[grow] = am;
    a.sample[grow] = smp;
    a.pmax[grow] = pm;
    m.H[l] = H;
    m.am[l] = am;
    m.smp[l] = smp;
    m.pm[l] = pm;
  }
  block_sync();
  canvas_epilogue<kEpiThreads>(a, bi, m);
}

// Initial canvas: uniform-random tokens (stream 2), nothing committed; the
// stability state and the row and canvas counters of the stream kernel
// start at zero.
__global__ void init_canvas_kernel(int32_t* canvas, uint8_t* committed, uint8_t* stop_flags,
                                   int32_t* stable, int32_t* row_cnt, int32_t* canvas_cnt, int L,
                                   int V, int canvas_offset, uint32_t key0, uint32_t key1) {
  const int bi = blockIdx.x;
  const uint32_t bg = (uint32_t)(canvas_offset + bi);
  for (int l = threadIdx.x; l < L; l += blockDim.x) {
    const Words4 r = philox((uint32_t)l >> 2, 0u, 0u, bg | (kStreamInit << 24), key0, key1);
    const size_t i = (size_t)bi * (size_t)L + (size_t)l;
    canvas[i] = (int32_t)uniform_token(pick_word(r, (uint32_t)l & 3u), (uint32_t)V);
    committed[i] = 0;
    row_cnt[i] = 0;
  }
  if (threadIdx.x == 0) {
    stop_flags[bi] = 0;
    stable[bi] = 0;
    canvas_cnt[bi] = 0;
  }
}

}  // namespace ebk
