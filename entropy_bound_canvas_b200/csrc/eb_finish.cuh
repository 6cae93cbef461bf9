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
// and writes its results straight into cluster rank 0's shared memory; after
// one cluster barrier rank 0 runs the canvas epilogue: argmax stability,
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
  int stable_prev;
  double dscr[kFinWarps];
  int iscr[kFinWarps];
  int cscr[kFinWarps];
  unsigned long long uscr[kFinWarps];
};

struct FinLayout {
  uint32_t ctrl, H, am, smp, pm, prev, tok, open, pick, keys, total;
};

__host__ __device__ inline FinLayout fin_layout(int L) {
  FinLayout y;
  uint32_t o = 0;
  const uint32_t l = (uint32_t)L;
  y.ctrl = o;
  o += (uint32_t)((sizeof(FinCtrl) + 15) / 16 * 16);
  y.keys = o;
  o += 8u * l;
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
// Per-position work of one subgroup of TPR lanes (all lanes of a warp
// execute it; `valid` is false for lanes without a position).
// ---------------------------------------------------------------------------
struct RowOut {
  float H, pmax;
  int amax, sample;  // global vocabulary ids
  // the same sums before the entropy, for a vocabulary slice's record:
  // S = sum 2^d, W = sum 2^d d, d = (z - zmax) c2, and the best group score
  double S, W;
  float zmax, gscore;
};

// The PER logits v0 .. v0 + PER - 1 of one row (those >= V read as -inf):
// vector loads when the row is 16-byte aligned and the chunk is whole.
template <int DT, int PER>
__device__ __forceinline__ void load_chunk(const char* rowp, int v0, int V, bool vec, float (&z)[PER]) {
  constexpr int kBytes = PER * elt_bytes(DT);
  const char* p = rowp + (size_t)v0 * elt_bytes(DT);
  if (vec && v0 + PER <= V && kBytes >= 4) {
    uint32_t w[kBytes / 4];
    if constexpr (kBytes >= 16) {
#pragma unroll
      for (int i = 0; i < kBytes / 16; ++i) {
        const uint4 q = __ldg(reinterpret_cast<const uint4*>(p) + i);
        w[4 * i] = q.x;
        w[4 * i + 1] = q.y;
        w[4 * i + 2] = q.z;
        w[4 * i + 3] = q.w;
      }
    } else if constexpr (kBytes == 8) {
      const uint2 q = __ldg(reinterpret_cast<const uint2*>(p));
      w[0] = q.x;
      w[1] = q.y;
    } else {
      w[0] = __ldg(reinterpret_cast<const uint32_t*>(p));
    }
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      if (DT == kF32) {
        z[e] = __uint_as_float(w[e]);
      } else {
        z[e] = (e & 1) ? bf16_hi(w[e >> 1]) : bf16_lo(w[e >> 1]);
      }
    }
  } else {
#pragma unroll
    for (int e = 0; e < PER; ++e) z[e] = v0 + e < V ? load_elem<DT>(rowp, v0 + e) : -INFINITY;
  }
}

template <int DT, int TPR>
__device__ __forceinline__ RowOut finish_row(const StepArgs& a, int bi, int ai, int l, bool valid,
                                             bool open, int sl, unsigned long long NG) {
  constexpr int PER = kGroup / TPR;  // elements of a group per lane
  RowOut out;
  const size_t grow = (size_t)bi * (size_t)a.L + (size_t)(valid ? l : 0);
  // 1. merge the row's records: (stream CTAs that own part of the row) x nw
  Partial R = empty_partial();
  if (valid) {
    const unsigned long long r = (unsigned long long)ai * (unsigned long long)a.L + (unsigned long long)l;
    const unsigned long long g_first = r * (unsigned long long)a.ng;
    const int c_first = cta_of(g_first, NG, a.G1);
    const int c_last = cta_of(g_first + (unsigned long long)a.ng - 1ull, NG, a.G1);
    const int nrec = (c_last - c_first + 1) * a.nw;
    const Partial* rec = a.partials + grow * (size_t)(a.max_segs * a.nw);
    if (NG >= (unsigned long long)a.G1) {
      // every stream CTA owns at least one group, so every CTA from c_first
      // to c_last wrote its records for this row: load four at a time
      const char* rowp = reinterpret_cast<const char*>(a.logits) + grow * (size_t)a.V * elt_bytes(DT);
      for (int i0 = sl; i0 < nrec; i0 += 4 * TPR) {
        Partial q[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = i0 + u * TPR;
          q[u] = i < nrec ? rec[i] : empty_partial();
        }
        // every record's top group and draw group may be the row's: start
        // bringing their logits into L1 while the records merge
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (q[u].agrp != 0x7fffffff)
            prefetch_l1(rowp + (size_t)q[u].agrp * kGroup * elt_bytes(DT));
          if (q[u].gidx != 0x7fffffff && !a.greedy)
            prefetch_l1(rowp + (size_t)q[u].gidx * kGroup * elt_bytes(DT));
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) merge(R, q[u], a.c2);
      }
    } else {
      for (int i = sl; i < nrec; i += TPR) {
        const int c = c_first + i / a.nw;
        if (range_start(c, NG, a.G1) < range_start(c + 1, NG, a.G1)) merge(R, rec[i], a.c2);
      }
    }
  }
#pragma unroll
  for (int o = 1; o < TPR; o <<= 1) {
    Partial q = shfl_partial(R, o);
    merge(R, q, a.c2);
  }

  // 2. the lane's slices of the group holding the maximum and of the winning
  //    Gumbel group, loaded together
  const char* rowp = reinterpret_cast<const char*>(a.logits) + grow * (size_t)a.V * elt_bytes(DT);
  const bool has_top = valid && R.agrp != 0x7fffffff;
  const bool draw = open && !a.greedy && R.gidx != 0x7fffffff;
  const int vt0 = (has_top ? R.agrp : 0) * kGroup + sl * PER;
  const int vs0 = (draw ? R.gidx : 0) * kGroup + sl * PER;
  float zt[PER], zs[PER];
  if (has_top) load_chunk<DT, PER>(rowp, vt0, a.V, a.vec_ok != 0, zt);
  if (draw) load_chunk<DT, PER>(rowp, vs0, a.V, a.vec_ok != 0, zs);
  // element-stream words of the sample slice (independent of the loads)
  constexpr int NC = PER >= 4 ? PER / 4 : 1;
  uint32_t xw[NC * 4];
  const uint32_t c3 = (uint32_t)(a.canvas_offset + bi) | (kStreamGumbel << 24);
  if (draw) {
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      const Words4 w = philox(((uint32_t)(a.v_off + vs0) >> 2) + (uint32_t)c, (uint32_t)l,
                              (uint32_t)a.s, c3,
                              a.key0, a.key1);
#pragma unroll
      for (int q = 0; q < 4; ++q) xw[4 * c + q] = w.w[q];
    }
  }

  // 3. exact recomputation of the top group: an element equal to the
  //    maximum contributes exactly 1, the others 2^d (-inf logits nothing)
  float ss = 0.f, wsum = 0.f;
  int nmax = 0, am = 0x7fffffff;
  if (has_top) {
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      const float d = (zt[e] - R.zmax) * a.c2;
      if (d == 0.f) {
        ++nmax;
        am = min(am, vt0 + e);
      } else {
        const float p = ex2(d);
        if (p > 0.f) {
          ss += p;
          wsum = fmaf(p, d, wsum);
        }
      }
    }
  }
#pragma unroll
  for (int o = 1; o < TPR; o <<= 1) {
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
    wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
    nmax += __shfl_xor_sync(0xffffffffu, nmax, o);
    am = min(am, __shfl_xor_sync(0xffffffffu, am, o));
  }
  const double S = (double)nmax + ((double)ss + (double)R.Srest);
  const double W = (double)wsum + (double)R.Wrest;
  out.H = (float)(log(S) - 0.6931471805599453 * (W / S));
  out.pmax = (float)(1.0 / S);
  out.amax = am == 0x7fffffff ? am : am + a.v_off;
  out.S = S;
  out.W = W;
  out.zmax = R.zmax;
  out.gscore = R.gscore;
  if (valid && (!isfinite(S) || !isfinite(W) || am == 0x7fffffff))
    atomicOr(a.status, kStatusNonFinite);

  // 4. the categorical draw within the winning group: the largest tempered
  //    logit is drawn first; the logarithms of every element that cannot
  //    beat it are skipped exactly
  out.sample = open ? out.amax : -1;
  if (__any_sync(0xffffffffu, draw)) {
    float ymax = -INFINITY;
    int emax = -1;
    if (draw) {
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        const float y = zs[e] * a.iT;
        if (y > ymax) {
          ymax = y;
          emax = e;
        }
      }
    }
    // word of element e of the slice (PER >= 4: slices start on a call)
    auto word_at = [&](int e) -> uint32_t {
      if constexpr (PER >= 4) {
        return xw[e];
      } else {
        return (vs0 & 2) ? xw[2 + e] : xw[e];
      }
    };
    int vmax = emax >= 0 ? vs0 + emax : 0x7fffffff;
    uint32_t xmax = 0;
#pragma unroll
    for (int e = 0; e < PER; ++e)
      if (e == emax) xmax = word_at(e);
#pragma unroll
    for (int o = 1; o < TPR; o <<= 1) {
      const float oy = __shfl_xor_sync(0xffffffffu, ymax, o);
      const int ov = __shfl_xor_sync(0xffffffffu, vmax, o);
      const uint32_t ox = __shfl_xor_sync(0xffffffffu, xmax, o);
      if (oy > ymax || (oy == ymax && ov < vmax)) {
        ymax = oy;
        vmax = ov;
        xmax = ox;
      }
    }
    float best = -INFINITY;
    int barg = 0x7fffffff;
    if (draw && vmax != 0x7fffffff) {
      best = ymax + gumbel(xmax);
      barg = vmax;
      const float s0 = best;
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        const int v = vs0 + e;
        if (v >= a.V || v == vmax) continue;
        const uint32_t x = word_at(e);
        const float y = zs[e] * a.iT;
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
#pragma unroll
    for (int o = 1; o < TPR; o <<= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oa = __shfl_xor_sync(0xffffffffu, barg, o);
      if (ob > best || (ob == best && oa < barg)) {
        best = ob;
        barg = oa;
      }
    }
    if (draw) out.sample = barg == 0x7fffffff ? barg : barg + a.v_off;
  }
  return out;
}

// ---------------------------------------------------------------------------
// Canvas epilogue (cluster rank 0, 256 threads, values in shared memory)
// ---------------------------------------------------------------------------
// One block-wide pass: sum of a (double), OR of b, exclusive prefix of c
// (*c_total gets the sum of c).
__device__ __forceinline__ void fin_block_reduce(double& a, int& b, int& c, int* c_total,
                                                 FinCtrl* ctrl) {
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
  __syncthreads();
  double sx = 0.0;
  int sy = 0, off = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kFinWarps; ++w) {
    sx += ctrl->dscr[w];
    sy |= ctrl->iscr[w];
    if (w < warp) off += ctrl->cscr[w];
    tot += ctrl->cscr[w];
  }
  __syncthreads();
  a = sx;
  b = sy;
  c = off + z - c;
  *c_total = tot;
}

__device__ void canvas_epilogue(const StepArgs& a, int bi, FinCtrl* ctrl, const float* sH,
                                const int* sAm, const int* sSmp, const float* sPm,
                                const int* sPrev, const int* sTok, const uint8_t* sOpen,
                                uint8_t* pick, unsigned long long* keys) {
  const int tid = threadIdx.x;
  const int L = a.L;
  const size_t row0 = (size_t)bi * (size_t)L;
  const bool br = a.rule == kRuleBR;

  // pass 1: entropy sum, argmax stability, candidates (EB: open with
  // H <= gamma, no other can be in the prefix; BR: open below the threshold,
  // which compete for the quota, while those at or above it commit outright)
  double sumH = 0.0;
  int neq = a.s < 1 ? 1 : 0;
  int ncand = 0;
  for (int l = tid; l < L; l += kFinThreads) {
    pick[l] = 0;
    sumH += (double)sH[l];
    if (a.s >= 1 && sAm[l] != sPrev[l]) neq = 1;
    if (!sOpen[l]) {
      const int tok = sTok[l];
      if (tok < 0 || tok >= a.V_tot) atomicOr(a.status, kStatusBadToken);
    } else if (!br) {
      ncand += (double)sH[l] <= a.gamma ? 1 : 0;
    } else if (!((double)sPm[l] >= a.theta)) {
      ++ncand;
    }
  }
  int n_c = 0;
  int pos = ncand;
  fin_block_reduce(sumH, neq, pos, &n_c, ctrl);
  const int stable_new = neq ? 0 : ctrl->stable_prev + 1;
  const double meanH = sumH / (double)L;
  const bool fired = a.stop_enabled && stable_new >= a.stability_steps && meanH < a.tau;
  const bool last_step = a.s == a.N - 1;

  if (!fired) {
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
    // EB: candidate c is in the lowest-entropy prefix iff the entropies of all
    // candidates at or before it in (H, l) order sum to <= gamma (the sums
    // grow along the order).  BR: the quota goes to the first candidates in
    // (-pmax, l) order.
    for (int c = tid; c < n_c; c += kFinThreads) {
      const unsigned long long kc = keys[c];
      if (!br) {
        double cum = (double)__uint_as_float((uint32_t)(kc >> 32));
        for (int j = 0; j < n_c; ++j) {
          const unsigned long long kj = keys[j];
          if (kj < kc) cum += (double)__uint_as_float((uint32_t)(kj >> 32));
        }
        if (cum <= a.gamma) pick[(int)(kc & 0xffffffffu)] = 1;
      } else {
        int rank = 0;
#pragma unroll 4
        for (int j = 0; j < n_c; ++j) rank += keys[j] < kc;
        if (rank < a.quota) pick[(int)(kc & 0xffffffffu)] = 1;
      }
    }
    __syncthreads();
    // EB with no candidate: the single lowest (H, l).  MI: the prefix plus
    // the next open position in (H, l) order.  Candidates (H <= gamma) come
    // before every other open position, so both are the lowest open
    // position left out of the prefix.
    if (!br && (a.rule == kRuleMI || n_c == 0)) {
      unsigned long long best = ~0ull;
      for (int l = tid; l < L; l += kFinThreads) {
        if (!sOpen[l] || pick[l]) continue;
        const unsigned long long kk = key_asc(sH[l], l);
        best = kk < best ? kk : best;
      }
      best = fin_block_min(best, ctrl);
      if (tid == 0 && best != ~0ull) pick[(int)(best & 0xffffffffu)] = 1;
      __syncthreads();
    }
  }

  // commit, renoise, remember the argmax
  const uint32_t bg = (uint32_t)(a.canvas_offset + bi);
  int left = 0;
  const bool edit = !fired && a.eps_edit >= 0.0;
  for (int l = tid; l < L; l += kFinThreads) {
    if (!sOpen[l]) {
      // block refinement editing: a committed position whose argmax moved
      // takes it when the argmax is confident enough
      if (edit && sAm[l] != sTok[l] && (double)sPm[l] >= a.eps_edit) a.canvas[row0 + l] = sAm[l];
    } else {
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
        a.canvas[row0 + l] =
            (int32_t)uniform_token(pick_word(r, (uint32_t)l & 3u), (uint32_t)a.V_tot);
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
template <int DT, int TPR>
__device__ __forceinline__ void finish_rows(const StepArgs& a, const FinLayout& lay,
                                            unsigned char* smem, cgr::cluster_group& cluster,
                                            int bi, int ai, int rank, bool open,
                                            unsigned long long NG) {
  const int rpc = fin_rows_per_cta(a.L);
  const int tid = threadIdx.x;
  const int sub = tid / TPR, sl = tid % TPR;
  const int l = rank * rpc + sub;
  const bool valid = sub < rpc && l < a.L;
  const RowOut ro = finish_row<DT, TPR>(a, bi, ai, l, valid, open, sl, NG);
  if (valid && sl == 0) {
    const size_t grow = (size_t)bi * (size_t)a.L + (size_t)l;
    a.H_out[grow] = ro.H;
    a.amax_out[grow] = ro.amax;
    a.sample[grow] = ro.sample;
    a.pmax[grow] = ro.pmax;
    // straight into cluster rank 0's shared memory
    *cluster.map_shared_rank(reinterpret_cast<float*>(smem + lay.H) + l, 0) = ro.H;
    *cluster.map_shared_rank(reinterpret_cast<int*>(smem + lay.am) + l, 0) = ro.amax;
    *cluster.map_shared_rank(reinterpret_cast<int*>(smem + lay.smp) + l, 0) = ro.sample;
    *cluster.map_shared_rank(reinterpret_cast<float*>(smem + lay.pm) + l, 0) = ro.pmax;
    *cluster.map_shared_rank(smem + lay.open + l, 0) = open ? 1 : 0;
  }
}

template <int DT>
__global__ void __cluster_dims__(kFinCluster, 1, 1) __launch_bounds__(kFinThreads, 2)
    finish_kernel(const StepArgs a, const int32_t* act_index, const int32_t* n_act_ptr) {
  extern __shared__ __align__(128) unsigned char smem[];
  const FinLayout lay = fin_layout(a.L);
  FinCtrl* ctrl = reinterpret_cast<FinCtrl*>(smem + lay.ctrl);
  cgr::cluster_group cluster = cgr::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int bi = blockIdx.x / kFinCluster;
  const int tid = threadIdx.x;
  const int rpc = fin_rows_per_cta(a.L);
  const int tpr = fin_lanes_per_row(a.L);

  // Before the stream kernel has finished: what the previous step left (the
  // canvas state is written only by finish kernels, never by the stream
  // kernel that runs now).
  const int my_l = rank * rpc + tid / tpr;
  const bool open = tid / tpr < rpc && my_l < a.L &&
                    a.committed[(size_t)bi * (size_t)a.L + (size_t)my_l] == 0;
  if (rank == 0) {
    const size_t row0 = (size_t)bi * (size_t)a.L;
    int* sPrev = reinterpret_cast<int*>(smem + lay.prev);
    int* sTok = reinterpret_cast<int*>(smem + lay.tok);
    for (int i = tid; i < a.L; i += kFinThreads) {
      sPrev[i] = a.prev_amax[row0 + i];
      sTok[i] = a.canvas[row0 + i];
    }
    if (tid == 0) ctrl->stable_prev = a.stable[bi];
  }
  cluster.sync();  // every CTA of the cluster runs: its shared memory may be written

  griddep_wait();  // the stream kernel has completed and its writes are visible
  const int ai = act_index[bi];
  if (ai < 0) return;  // uniform over the cluster: a stopped canvas is untouched
  const int n_act = *n_act_ptr;
  const unsigned long long NG =
      (unsigned long long)n_act * (unsigned long long)a.L * (unsigned long long)a.ng;
  switch (tpr) {
    case 2: finish_rows<DT, 2>(a, lay, smem, cluster, bi, ai, rank, open, NG); break;
    case 4: finish_rows<DT, 4>(a, lay, smem, cluster, bi, ai, rank, open, NG); break;
    case 8: finish_rows<DT, 8>(a, lay, smem, cluster, bi, ai, rank, open, NG); break;
    case 16: finish_rows<DT, 16>(a, lay, smem, cluster, bi, ai, rank, open, NG); break;
    default: finish_rows<DT, 32>(a, lay, smem, cluster, bi, ai, rank, open, NG); break;
  }
  cluster.sync();  // rank 0 now holds every position's results
  if (rank == 0)
    canvas_epilogue(a, bi, ctrl, reinterpret_cast<const float*>(smem + lay.H),
                    reinterpret_cast<const int*>(smem + lay.am),
                    reinterpret_cast<const int*>(smem + lay.smp),
                    reinterpret_cast<const float*>(smem + lay.pm),
                    reinterpret_cast<const int*>(smem + lay.prev),
                    reinterpret_cast<const int*>(smem + lay.tok), smem + lay.open,
                    smem + lay.pick, reinterpret_cast<unsigned long long*>(smem + lay.keys));
}

// ---------------------------------------------------------------------------
// Vocabulary-sharded logits
// ---------------------------------------------------------------------------
// Slice records: after the stream kernel ran over this device's slice, every
// position of an active canvas gets its SliceRecord (8-lane subgroups, the
// same per-position work as the finish kernel, without the epilogue).
template <int DT>
__global__ void __launch_bounds__(256) slice_finish_kernel(const StepArgs a,
                                                           const int32_t* act_index,
                                                           const int32_t* n_act_ptr,
                                                           SliceRecord* records) {
  constexpr int kTPR = 8;
  const int bi = blockIdx.y;
  const int tid = threadIdx.x;
  const int l = blockIdx.x * (256 / kTPR) + tid / kTPR;
  const int sl = tid % kTPR;
  const bool in_range = l < a.L;
  const bool open = in_range && a.committed[(size_t)bi * (size_t)a.L + (size_t)l] == 0;
  griddep_wait();  // the stream kernel's records and active list are visible
  const int ai = act_index[bi];
  if (ai < 0) return;  // uniform over the CTA: a stopped canvas has no records
  const unsigned long long NG =
      (unsigned long long)(*n_act_ptr) * (unsigned long long)a.L * (unsigned long long)a.ng;
  const RowOut ro = finish_row<DT, kTPR>(a, bi, ai, in_range ? l : 0, in_range, open, sl, NG);
  if (in_range && sl == 0) {
    SliceRecord r;
    r.S = ro.S;
    r.W = ro.W;
    r.zmax = ro.zmax;
    r.gscore = ro.gscore;
    r.amax = ro.amax;
    r.sample = open && !a.greedy ? ro.sample : -1;
    r.pad0 = r.pad1 = 0;
    records[(size_t)bi * (size_t)a.L + (size_t)l] = r;
  }
}

// Combine: the n slices' records of each position, in slice order, give the
// position's entropy, max probability, argmax and draw (the largest slice
// maximum; the sums rescaled to it; the first slice attaining it for the
// argmax; the best slice score, earlier slice on a tie, for the draw);
// then the canvas epilogue, as in finish_kernel.
template <int DT>
__global__ void __cluster_dims__(kFinCluster, 1, 1) __launch_bounds__(kFinThreads, 2)
    combine_kernel(const StepArgs a, const int32_t* act_index, const SliceRecord* records,
                   int n_slices) {
  extern __shared__ __align__(128) unsigned char smem[];
  const FinLayout lay = fin_layout(a.L);
  FinCtrl* ctrl = reinterpret_cast<FinCtrl*>(smem + lay.ctrl);
  cgr::cluster_group cluster = cgr::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int bi = blockIdx.x / kFinCluster;
  const int tid = threadIdx.x;
  const int rpc = fin_rows_per_cta(a.L);
  if (act_index[bi] < 0) return;  // uniform over the cluster: a stopped canvas is untouched
  if (rank == 0) {
    const size_t row0 = (size_t)bi * (size_t)a.L;
    int* sPrev = reinterpret_cast<int*>(smem + lay.prev);
    int* sTok = reinterpret_cast<int*>(smem + lay.tok);
    for (int i = tid; i < a.L; i += kFinThreads) {
      sPrev[i] = a.prev_amax[row0 + i];
      sTok[i] = a.canvas[row0 + i];
    }
    if (tid == 0) ctrl->stable_prev = a.stable[bi];
  }
  cluster.sync();  // every CTA of the cluster runs: its shared memory may be written
  for (int k = tid; k < rpc; k += kFinThreads) {
    const int l = rank * rpc + k;
    if (l >= a.L) break;
    const size_t grow = (size_t)bi * (size_t)a.L + (size_t)l;
    const size_t stride = (size_t)a.B * (size_t)a.L;
    float M = -INFINITY;
    int am = 0x7fffffff;
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
    if (!isfinite(S) || !isfinite(W) || am == 0x7fffffff) atomicOr(a.status, kStatusNonFinite);
    const bool open = a.committed[grow] == 0;
    const int smp = open ? (a.greedy || x < 0 ? am : x) : -1;
    a.H_out[grow] = H;
    a.amax_out[grow] = am;
    a.sample[grow] = smp;
    a.pmax[grow] = pm;
    *cluster.map_shared_rank(reinterpret_cast<float*>(smem + lay.H) + l, 0) = H;
    *cluster.map_shared_rank(reinterpret_cast<int*>(smem + lay.am) + l, 0) = am;
    *cluster.map_shared_rank(reinterpret_cast<int*>(smem + lay.smp) + l, 0) = smp;
    *cluster.map_shared_rank(reinterpret_cast<float*>(smem + lay.pm) + l, 0) = pm;
    *cluster.map_shared_rank(smem + lay.open + l, 0) = open ? 1 : 0;
  }
  cluster.sync();  // rank 0 now holds every position's results
  if (rank == 0)
    canvas_epilogue(a, bi, ctrl, reinterpret_cast<const float*>(smem + lay.H),
                    reinterpret_cast<const int*>(smem + lay.am),
                    reinterpret_cast<const int*>(smem + lay.smp),
                    reinterpret_cast<const float*>(smem + lay.pm),
                    reinterpret_cast<const int*>(smem + lay.prev),
                    reinterpret_cast<const int*>(smem + lay.tok), smem + lay.open,
                    smem + lay.pick, reinterpret_cast<unsigned long long*>(smem + lay.keys));
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
