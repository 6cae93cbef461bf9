// eb_finish.cuh -- second kernel of a sampler step: per-position results and
// the per-canvas decisions.
//
// One thread-block cluster of kFinCluster CTAs per canvas.  Cluster rank r
// owns a contiguous slice of the canvas's L positions; each position is
// handled by a power-of-two subgroup of lanes that
//   1. merges the position's Partial records written by the stream kernel,
//   2. recomputes the group holding the maximum exactly (every element equal
//      to the maximum contributes exactly 1, the smaller terms are summed
//      apart) -> entropy H, max probability, argmax,
//   3. for an open position, draws the element within the winning Gumbel
//      group (element-stream Philox words; the element with the largest
//      logit is drawn first and the logarithms of every element that cannot
//      beat it are skipped exactly),
// then the cluster synchronises and rank 0 gathers the slice results from its
// peers' shared memory and runs the canvas epilogue: argmax stability,
// adaptive stop, commit rule, last-step / all-committed finalisation and
// renoise.  Only hardware barriers (CTA and cluster) are used.
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

#include <cooperative_groups.h>

#include "eb_common.cuh"

namespace ebk {

namespace cgr = cooperative_groups;

constexpr int kFinCluster = 8;
constexpr int kFinThreads = 256;
constexpr int kFinWarps = kFinThreads / 32;

struct FinCtrl {
  int kpref;
  int pad;
  double dscr[kFinWarps];
  int iscr[kFinWarps];
  unsigned long long uscr[kFinWarps];
};

struct FinLayout {
  uint32_t ctrl, H, am, smp, pm, open, pick, keys, skeys, total;
};

__host__ __device__ inline FinLayout fin_layout(int L) {
  FinLayout y;
  uint32_t o = 0;
  const uint32_t l = (uint32_t)L;
  y.ctrl = o;
  o += (uint32_t)((sizeof(FinCtrl) + 15) / 16 * 16);
  y.keys = o;
  o += 8u * l;
  y.skeys = o;
  o += 8u * l;
  y.H = o;
  o += 4u * l;
  y.am = o;
  o += 4u * l;
  y.smp = o;
  o += 4u * l;
  y.pm = o;
  o += 4u * l;
  y.open = o;
  o += l;
  y.pick = o;
  o += l;
  y.total = (o + 15) / 16 * 16;
  return y;
}

// Rows per cluster rank and lanes per row (power of two, 2 .. 32).
__host__ __device__ inline int fin_rows_per_cta(int L) { return (L + kFinCluster - 1) / kFinCluster; }
__host__ __device__ inline int fin_lanes_per_row(int L) {
  const int rpc = fin_rows_per_cta(L);
  int t = 32;
  while (t > 2 && t * rpc > kFinThreads) t >>= 1;
  return t;
}

// ---------------------------------------------------------------------------
// 256-thread block helpers (whole CTA, __syncthreads)
// ---------------------------------------------------------------------------
__device__ __forceinline__ double fin_block_sum(double v, FinCtrl* c) {
  const int tid = threadIdx.x;
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((tid & 31) == 0) c->dscr[tid >> 5] = v;
  __syncthreads();
  double r = 0.0;
  for (int w = 0; w < kFinWarps; ++w) r += c->dscr[w];
  __syncthreads();
  return r;
}

__device__ __forceinline__ int fin_block_sum_int(int v, FinCtrl* c) {
  const int tid = threadIdx.x;
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((tid & 31) == 0) c->iscr[tid >> 5] = v;
  __syncthreads();
  int r = 0;
  for (int w = 0; w < kFinWarps; ++w) r += c->iscr[w];
  __syncthreads();
  return r;
}

__device__ __forceinline__ unsigned long long fin_block_min(unsigned long long v, FinCtrl* c) {
  const int tid = threadIdx.x;
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const unsigned long long w = __shfl_xor_sync(0xffffffffu, v, o);
    v = w < v ? w : v;
  }
  if ((tid & 31) == 0) c->uscr[tid >> 5] = v;
  __syncthreads();
  unsigned long long r = c->uscr[0];
  for (int w = 1; w < kFinWarps; ++w) r = c->uscr[w] < r ? c->uscr[w] : r;
  __syncthreads();
  return r;
}

// Exclusive prefix of v over the CTA; *total gets the sum.
__device__ __forceinline__ int fin_excl_scan(int v, FinCtrl* c, int* total) {
  const int tid = threadIdx.x, lane = tid & 31;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) c->iscr[tid >> 5] = x;
  __syncthreads();
  int off = 0, tot = 0;
  for (int w = 0; w < kFinWarps; ++w) {
    if (w < (tid >> 5)) off += c->iscr[w];
    tot += c->iscr[w];
  }
  __syncthreads();
  *total = tot;
  return off + x - v;
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

// ---------------------------------------------------------------------------
// Per-position work of one subgroup of `tpr` lanes (all lanes of a warp
// execute it; `valid` is false for lanes without a position).
// ---------------------------------------------------------------------------
struct RowOut {
  float H, pmax;
  int amax, sample;
};

template <int DT>
__device__ __forceinline__ RowOut finish_row(const StepArgs& a, int bi, int ai, int l, bool valid,
                                             int tpr, int sl, unsigned long long NG) {
  RowOut out;
  const size_t grow = (size_t)bi * (size_t)a.L + (size_t)(valid ? l : 0);
  // 1. merge the row's partials
  Partial R = empty_partial();
  if (valid) {
    const unsigned long long r = (unsigned long long)ai * (unsigned long long)a.L + (unsigned long long)l;
    const unsigned long long g_first = r * (unsigned long long)a.ng;
    const int c_first = cta_of(g_first, NG, a.G1);
    const int c_last = cta_of(g_first + (unsigned long long)a.ng - 1ull, NG, a.G1);
    for (int i = sl; i <= c_last - c_first; i += tpr) {
      const int c = c_first + i;
      if (range_start(c, NG, a.G1) < range_start(c + 1, NG, a.G1))
        merge(R, a.partials[grow * (size_t)a.max_segs + (size_t)i], a.c2);
    }
  }
  for (int o = 1; o < tpr; o <<= 1) {
    Partial q = shfl_partial(R, o);
    merge(R, q, a.c2);
  }

  const char* rowp = reinterpret_cast<const char*>(a.logits) + grow * (size_t)a.V * elt_bytes(DT);
  const int per = kGroup / tpr;  // elements of a group per lane
  // 2. exact recomputation of the top group
  float ss = 0.f, wsum = 0.f;
  int nmax = 0, am = 0x7fffffff;
  if (valid && R.agrp != 0x7fffffff) {
    const int e0 = R.agrp * kGroup + sl * per;
#pragma unroll 4
    for (int e = 0; e < per; ++e) {
      const int v = e0 + e;
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
  }
  for (int o = 1; o < tpr; o <<= 1) {
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
    wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
    nmax += __shfl_xor_sync(0xffffffffu, nmax, o);
    am = min(am, __shfl_xor_sync(0xffffffffu, am, o));
  }
  const double S = (double)nmax + ((double)ss + (double)R.Srest);
  const double W = (double)wsum + (double)R.Wrest;
  out.H = (float)(log(S) - 0.6931471805599453 * (W / S));
  out.pmax = (float)(1.0 / S);
  out.amax = am;
  if (valid && (!isfinite(S) || !isfinite(W))) atomicOr(a.status, kStatusNonFinite);

  // 3. the categorical draw of an open position
  const bool open = valid && a.committed[grow] == 0;
  const bool draw = open && !a.greedy && R.gidx != 0x7fffffff;
  out.sample = open ? am : -1;
  if (__any_sync(0xffffffffu, draw)) {
    const int jg = draw ? R.gidx : 0;
    const int e0 = jg * kGroup + sl * per;
    // largest tempered logit of the group and its lowest index
    float ymax = -INFINITY;
    int vmax = 0x7fffffff;
    if (draw) {
      for (int e = 0; e < per; ++e) {
        const int v = e0 + e;
        if (v < a.V) {
          const float y = load_elem<DT>(rowp, v) * a.iT;
          if (y > ymax) {
            ymax = y;
            vmax = v;
          }
        }
      }
    }
    for (int o = 1; o < tpr; o <<= 1) {
      const float oy = __shfl_xor_sync(0xffffffffu, ymax, o);
      const int ov = __shfl_xor_sync(0xffffffffu, vmax, o);
      if (oy > ymax || (oy == ymax && ov < vmax)) {
        ymax = oy;
        vmax = ov;
      }
    }
    const uint32_t c3 = (uint32_t)(a.canvas_offset + bi) | (kStreamGumbel << 24);
    float best = -INFINITY;
    int barg = 0x7fffffff;
    if (draw && vmax != 0x7fffffff) {
      // every lane evaluates the seed element's score identically
      const Words4 w = philox((uint32_t)vmax >> 2, (uint32_t)l, (uint32_t)a.s, c3, a.key0, a.key1);
      best = ymax + gumbel(pick_word(w, (uint32_t)vmax & 3u));
      barg = vmax;
      const float s0 = best;
      uint32_t cur_call = 0xffffffffu;
      Words4 cw{};
      for (int e = 0; e < per; ++e) {
        const int v = e0 + e;
        if (v >= a.V || v == vmax) continue;
        if (((uint32_t)v >> 2) != cur_call) {
          cur_call = (uint32_t)v >> 2;
          cw = philox(cur_call, (uint32_t)l, (uint32_t)a.s, c3, a.key0, a.key1);
        }
        const uint32_t x = pick_word(cw, (uint32_t)v & 3u);
        const float y = load_elem<DT>(rowp, v) * a.iT;
        // can v beat the seed?  It needs g > s0 - y, i.e. -ln u < e^-(s0 - y);
        // -ln u >= 1 - u, so 1 - u >= e^-(s0 - y) (1e-4 relative margin) rules it out.
        const float tgap = s0 - y;
        if (tgap > -2.0f && one_minus_u(x) >= ex2(-1.4426950408889634f * tgap) * 1.0001f) continue;
        const float sc = y + gumbel(x);
        if (sc > best || (sc == best && v < barg)) {
          best = sc;
          barg = v;
        }
      }
    }
    for (int o = 1; o < tpr; o <<= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oa = __shfl_xor_sync(0xffffffffu, barg, o);
      if (ob > best || (ob == best && oa < barg)) {
        best = ob;
        barg = oa;
      }
    }
    if (draw) out.sample = barg;
  }
  return out;
}

// ---------------------------------------------------------------------------
// Canvas epilogue (cluster rank 0, 256 threads, values in shared memory)
// ---------------------------------------------------------------------------
__device__ void canvas_epilogue(const StepArgs& a, int bi, FinCtrl* ctrl, const float* sH,
                                const int* sAm, const int* sSmp, const float* sPm,
                                const uint8_t* sOpen, uint8_t* pick, unsigned long long* keys,
                                unsigned long long* skeys) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int L = a.L;
  const size_t row0 = (size_t)bi * (size_t)L;
  const bool br = a.rule == kRuleBR;

  double sumH = 0.0;
  int neq = a.s < 1 ? 1 : 0;
  int ncand = 0;
  for (int l = tid; l < L; l += kFinThreads) {
    pick[l] = 0;
    sumH += (double)sH[l];
    if (a.s >= 1 && sAm[l] != a.prev_amax[row0 + l]) neq = 1;
    if (!sOpen[l]) {
      const int tok = a.canvas[row0 + l];
      if (tok < 0 || tok >= a.V) atomicOr(a.status, kStatusBadToken);
    } else if (!br) {
      ncand += (double)sH[l] <= a.gamma ? 1 : 0;
    } else if (!((double)sPm[l] >= a.theta)) {
      ++ncand;
    }
  }
  const double totH = fin_block_sum(sumH, ctrl);
  const int any_neq = fin_block_sum_int(neq, ctrl);
  const int stable_new = any_neq ? 0 : a.stable[bi] + 1;
  const double meanH = totH / (double)L;
  const bool fired = a.stop_enabled && stable_new >= a.stability_steps && meanH < a.tau;
  const bool last_step = a.s == a.N - 1;

  if (!fired) {
    // Candidates.  EB: open positions with H <= gamma (no other can be in
    // the prefix).  BR: open positions below the threshold compete for the
    // quota; those at or above it are committed outright.
    int n_c = 0;
    int pos = fin_excl_scan(ncand, ctrl, &n_c);
    for (int l = tid; l < L; l += kFinThreads) {
      if (!sOpen[l]) continue;
      if (!br) {
        if ((double)sH[l] <= a.gamma) keys[pos++] = key_asc(sH[l], l);
      } else if ((double)sPm[l] >= a.theta) {
        pick[l] = 1;
      } else {
        keys[pos++] = key_desc(sPm[l], l);
      }
    }
    __syncthreads();
    for (int c = tid; c < n_c; c += kFinThreads) {
      const unsigned long long kc = keys[c];
      int rank = 0;
#pragma unroll 4
      for (int j = 0; j < n_c; ++j) rank += keys[j] < kc;
      if (!br) skeys[rank] = kc;
      else if (rank < a.quota) pick[(int)(kc & 0xffffffffu)] = 1;
    }
    __syncthreads();
    if (!br) {
      // longest prefix of the sorted candidates with cumulative H <= gamma
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
      __syncthreads();
      const int kpref = ctrl->kpref;
      for (int i = tid; i < kpref; i += kFinThreads) pick[(int)(skeys[i] & 0xffffffffu)] = 1;
      // EB with an empty prefix: the single lowest (H, l).  MI: the prefix
      // plus the next position in (H, l) order.
      const bool mi = a.rule == kRuleMI;
      if (mi && kpref < n_c) {
        if (tid == 0) pick[(int)(skeys[kpref] & 0xffffffffu)] = 1;
      } else if (kpref == 0 || mi) {
        unsigned long long best = ~0ull;
        for (int l = tid; l < L; l += kFinThreads) {
          if (!sOpen[l] || (mi && (double)sH[l] <= a.gamma)) continue;
          const unsigned long long kk = key_asc(sH[l], l);
          best = kk < best ? kk : best;
        }
        best = fin_block_min(best, ctrl);
        if (tid == 0 && best != ~0ull) pick[(int)(best & 0xffffffffu)] = 1;
      }
    }
    __syncthreads();
  }

  // commit, renoise, remember the argmax
  const uint32_t bg = (uint32_t)(a.canvas_offset + bi);
  int left = 0;
  for (int l = tid; l < L; l += kFinThreads) {
    if (sOpen[l]) {
      if (fired) {
        a.canvas[row0 + l] = sAm[l];
        a.committed[row0 + l] = 1;
      } else if (pick[l] || last_step) {
        a.canvas[row0 + l] = a.greedy ? sAm[l] : sSmp[l];
        a.committed[row0 + l] = 1;
      } else {
        ++left;
        const Words4 r = philox((uint32_t)l >> 2, 0u, (uint32_t)a.s, bg | (kStreamRenoise << 24),
                                a.key0, a.key1);
        a.canvas[row0 + l] = (int32_t)uniform_token(pick_word(r, (uint32_t)l & 3u), (uint32_t)a.V);
      }
    }
    a.prev_amax[row0 + l] = sAm[l];
  }
  const int left_tot = fin_block_sum_int(left, ctrl);
  if (tid == 0) {
    a.stable[bi] = stable_new;
    a.stop_flags[bi] = (uint8_t)(fired ? 1 : last_step ? 3 : left_tot == 0 ? 2 : 0);
  }
}

// act_index[b]: index of canvas b among the canvases active at the start of
// the step (-1 if it had stopped), written by the stream kernel.
template <int DT>
__global__ void __cluster_dims__(kFinCluster, 1, 1) __launch_bounds__(kFinThreads)
    finish_kernel(const StepArgs a, const int32_t* act_index, const int32_t* n_act_ptr) {
  griddep_wait();  // the stream kernel has completed and its writes are visible
  extern __shared__ __align__(16) unsigned char smem[];
  const FinLayout lay = fin_layout(a.L);
  FinCtrl* ctrl = reinterpret_cast<FinCtrl*>(smem + lay.ctrl);
  float* sH = reinterpret_cast<float*>(smem + lay.H);
  int* sAm = reinterpret_cast<int*>(smem + lay.am);
  int* sSmp = reinterpret_cast<int*>(smem + lay.smp);
  float* sPm = reinterpret_cast<float*>(smem + lay.pm);
  uint8_t* sOpen = smem + lay.open;
  uint8_t* pick = smem + lay.pick;
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(smem + lay.keys);
  unsigned long long* skeys = reinterpret_cast<unsigned long long*>(smem + lay.skeys);

  cgr::cluster_group cluster = cgr::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int bi = blockIdx.x / kFinCluster;
  const int ai = act_index[bi];
  if (ai < 0) return;  // uniform over the cluster: a stopped canvas is untouched
  const int n_act = *n_act_ptr;
  const unsigned long long NG =
      (unsigned long long)n_act * (unsigned long long)a.L * (unsigned long long)a.ng;

  const int rpc = fin_rows_per_cta(a.L);
  const int tpr = fin_lanes_per_row(a.L);
  const int tid = threadIdx.x;
  const int sub = tid / tpr, sl = tid % tpr;
  const int l = rank * rpc + sub;
  const bool valid = sub < rpc && l < a.L;
  const RowOut ro = DT == kBF16 ? finish_row<kBF16>(a, bi, ai, l, valid, tpr, sl, NG)
                                : finish_row<kF32>(a, bi, ai, l, valid, tpr, sl, NG);
  if (valid && sl == 0) {
    const size_t grow = (size_t)bi * (size_t)a.L + (size_t)l;
    a.H_out[grow] = ro.H;
    a.amax_out[grow] = ro.amax;
    a.sample[grow] = ro.sample;
    a.pmax[grow] = ro.pmax;
    sH[l] = ro.H;
    sAm[l] = ro.amax;
    sSmp[l] = ro.sample;
    sPm[l] = ro.pmax;
    sOpen[l] = a.committed[grow] == 0 ? 1 : 0;
  }
  cluster.sync();
  if (rank == 0) {  // gather the other slices from the peers' shared memory
    for (int i = tid; i < a.L; i += kFinThreads) {
      const int owner = i / rpc;
      if (owner == 0) continue;
      sH[i] = *cluster.map_shared_rank(sH + i, owner);
      sAm[i] = *cluster.map_shared_rank(sAm + i, owner);
      sSmp[i] = *cluster.map_shared_rank(sSmp + i, owner);
      sPm[i] = *cluster.map_shared_rank(sPm + i, owner);
      sOpen[i] = *cluster.map_shared_rank(sOpen + i, owner);
    }
  }
  cluster.sync();  // peers stay resident until rank 0 has read them
  if (rank == 0) canvas_epilogue(a, bi, ctrl, sH, sAm, sSmp, sPm, sOpen, pick, keys, skeys);
}

// Initial canvas: uniform-random tokens (stream 2), nothing committed.
__global__ void init_canvas_kernel(int32_t* canvas, uint8_t* committed, uint8_t* stop_flags,
                                   int32_t* stable, int L, int V, int canvas_offset,
                                   uint32_t key0, uint32_t key1) {
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
  }
}

}  // namespace ebk
