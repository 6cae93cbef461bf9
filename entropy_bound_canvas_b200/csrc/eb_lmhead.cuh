// eb_lmhead.cuh -- the sampler fused into the LM-head contraction: the
// decoder's logits z = h W^T (h: hidden states [rows, d], W: LM head
// [V, d], both bf16, K = d contiguous) are formed tile by tile on the
// 5th-generation tensor cores and reduced on chip, so they never reach HBM
// (diffusers "DiffusionGemma" page, `__call__` parameters: the pipeline's
// logits are the decoder's [batch, canvas_length, vocab_size] output; the
// model card's summary table: a vocabulary of about 262K).
//
// One CTA per SM, six warps:
//   warp 0  producer: TMA (cp.async.bulk.tensor, 128-byte swizzle, each
//           CTA loading for itself) of a 128 x 64 tile of h and a 256 x 64
//           tile of W per stage, into a ring of kLmStages stages;
//   warp 1  MMA issuer: one elected thread issues tcgen05.mma (kind::f16,
//           bf16 in, fp32 accumulate, M = 128, N = 256, K = 16 per
//           instruction) into one of two TMEM accumulators (2 x 256 columns)
//           and commits each stage back to the producer, each finished tile
//           to the epilogue;
//   warps 2-5 epilogue: thread t of the four holds row t of the tile (TMEM
//           lane t); it reads the tile's 256 fp32 logits with tcgen05.ld and
//           folds them, 64 at a time (one Gumbel group), into the row's
//           running state: maximum and its lowest id, S = sum 2^d,
//           W = sum 2^d d with d = (z - M) c2, and the group-level Gumbel race
//           (the winning group's 64 logits kept in shared memory).
// A CTA owns one 128-row tile and a contiguous range of the vocabulary's
// 256-wide tiles; at the end each row draws the element inside its best
// group and writes one slice record (the same record a vocabulary slice of
// the logits gives), which the combine merges in vocabulary order before
// the canvas decisions.
#pragma once

#include <cuda.h>

#include "eb_common.cuh"

namespace ebk {

constexpr int kLmBM = 128;  // rows per tile: the MMA's M, one TMEM lane per row
constexpr int kLmBN = 256;  // vocabulary ids per tile: the MMA's N, four Gumbel groups
constexpr int kLmBK = 64;   // hidden elements per stage: one 128-byte swizzle row
constexpr int kLmStages = 4;
constexpr int kLmThreads = 6 * 32;
constexpr uint32_t kLmABytes = kLmBM * kLmBK * 2;  // 16 KB
constexpr uint32_t kLmBBytes = kLmBN * kLmBK * 2;  // 32 KB
constexpr uint32_t kLmTmemCols = 2 * kLmBN;        // two accumulators
constexpr int kLmZStride = 66;  // floats per row of the race buffer (conflict-free float2 stores)

struct LmArgs {
  StepArgs a;          // temperature, keys, canvas state (read), status
  SliceRecord* rec;    // [n_split][rows]: the sampler's records, or
  float* logits_out;   // [rows][V] fp32: the logits themselves (diagnostic)
  int rows, V, d;
  int n_split;         // vocabulary ranges per 128-row tile
};

struct LmLayout {
  uint32_t a, b, z, bars, total;
};

__host__ __device__ inline LmLayout lm_layout(bool sampler) {
  LmLayout y;
  uint32_t o = 0;
  y.a = o;
  o += kLmStages * kLmABytes;
  y.b = o;
  o += kLmStages * kLmBBytes;
  y.z = o;
  if (sampler) o += (uint32_t)kLmBM * kLmZStride * 4u;
  y.bars = o;
  o += 8u * (2 * kLmStages + 5) + 16u;
  y.total = o + 1024u;  // room to align the base to 1024 bytes
  return y;
}

// ---------------------------------------------------------------------------
// tcgen05 / TMA primitives
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;"
      :
      : "r"(smem_u32(dst)), "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void tc_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               :
               : "r"(smem_u32(dst)), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" : : "r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrives on `bar` once every tcgen05 operation this thread issued so far
// has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               :
               : "r"(smem_u32(bar))
               : "memory");
}
// D[tmem] (+)= A[smem] B[smem]^T, both K-major.
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      :
      : "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tc_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tc_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor of a K-major tile written by TMA with the
// 128-byte swizzle: rows of 128 bytes in groups of 8 (1024 bytes apart),
// descriptor version 1, swizzle mode 2.  `addr` may step inside the first
// 128 bytes (the K slices of one MMA each).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr) {
  uint64_t d = (uint64_t)((addr & 0x3FFFFu) >> 4);
  d |= (uint64_t)1 << 16;            // leading byte offset (not used by this layout)
  d |= (uint64_t)(1024u >> 4) << 32;  // stride byte offset: 8 rows of 128 bytes
  d |= (uint64_t)1 << 46;            // descriptor version
  d |= (uint64_t)2 << 61;            // 128-byte swizzle
  return d;
}

// Instruction descriptor: bf16 x bf16 -> fp32, A and B K-major, M x N.
__host__ __device__ constexpr uint32_t lm_idesc(int M, int N) {
  return (1u << 4) |                 // D fp32
         (1u << 7) | (1u << 10) |    // A, B bf16
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------------------
// Per-row state of the epilogue
// ---------------------------------------------------------------------------
struct LmRow {
  float M, S, W, R;  // maximum; sums relative to it (log2 units); best Gumbel ratio
  int amax, gb;      // global ids: lowest id attaining M; best group (kNone: none)
};

// The element drawn inside group gb from its 64 logits z (shared memory):
// x = argmax (z_v / T + g_v), g_v the element stream's Gumbel (global ids),
// the lowest id on ties; the same pruning as the stream kernel's draw (an
// element that provably cannot beat the largest tempered logit's score is
// skipped).
__device__ __forceinline__ int lm_draw(const StepArgs& a, const float* z, int gb, int bi, int l) {
  const uint32_t gv0 = (uint32_t)gb * (uint32_t)kGroup;
  const uint32_t key3 = (uint32_t)(a.canvas_offset + bi) | (kStreamGumbel << 24);
  float ym = -INFINITY;
  int im = -1;
  for (int i = 0; i < kGroup; ++i) {
    const float y = z[i] * a.iT;
    if (y > ym) {
      ym = y;
      im = i;
    }
  }
  if (im < 0) return kNone;
  const Words4 ws = philox((gv0 >> 2) + (uint32_t)(im >> 2), (uint32_t)l, (uint32_t)a.s, key3,
                           a.key0, a.key1);
  float best = ym + gumbel(pick_word(ws, (uint32_t)im & 3u));
  int barg = im;
  const float seed = best;
  for (int c = 0; c < kGroup / 4; ++c) {
    const Words4 w = philox((gv0 >> 2) + (uint32_t)c, (uint32_t)l, (uint32_t)a.s, key3, a.key0,
                            a.key1);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int i = 4 * c + q;
      if (i == im) continue;
      const float y = z[i] * a.iT;
      if (!(y > -INFINITY)) continue;
      const uint32_t x = w.w[q];
      const float tgap = seed - y;
      if (tgap > -2.0f && one_minus_u(x) >= ex2(-1.4426950408889634f * tgap) * 1.0001f) continue;
      const float sc = y + gumbel(x);
      if (sc > best || (sc == best && i < barg)) {
        best = sc;
        barg = i;
      }
    }
  }
  return (int)gv0 + barg;
}

// ---------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------
template <bool SAMPLER>
__global__ void __launch_bounds__(kLmThreads, 1)
    lmhead_kernel(const __grid_constant__ CUtensorMap tm_h, const __grid_constant__ CUtensorMap tm_w,
                  const LmArgs p) {
  extern __shared__ unsigned char lm_smem_raw[];
  const LmLayout lay = lm_layout(SAMPLER);
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(lm_smem_raw) + 1023) & ~(uintptr_t)1023);
  unsigned char* sa = smem + lay.a;
  unsigned char* sb = smem + lay.b;
  float* zbuf = reinterpret_cast<float*>(smem + lay.z);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + lay.bars);
  uint64_t* empty = full + kLmStages;
  uint64_t* acc_full = empty + kLmStages;  // [2]
  uint64_t* acc_empty = acc_full + 2;      // [2]
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const StepArgs& a = p.a;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_mt = (p.rows + kLmBM - 1) / kLmBM;
  const int n_nt = p.V / kLmBN;  // V is a multiple of kLmBN
  const int mt = blockIdx.x / p.n_split;
  const int ns = blockIdx.x % p.n_split;
  if (mt >= n_mt) return;
  const int nt_lo = (int)((long long)ns * n_nt / p.n_split);
  const int nt_hi = (int)((long long)(ns + 1) * n_nt / p.n_split);
  const int n_tiles = nt_hi - nt_lo;
  const int KB = p.d / kLmBK;

  // A tile whose rows all belong to stopped canvases is not computed (the
  // combine skips those canvases); the records it would write are not read.
  if (SAMPLER) {
    const int r0 = mt * kLmBM, r1 = min(p.rows, r0 + kLmBM) - 1;
    bool any = false;
    for (int b = r0 / a.L; b <= r1 / a.L; ++b) any |= a.stop_flags[b] == 0;
    if (!any) return;
  }

  if (tid == 0) {
    for (int s = 0; s < kLmStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) tc_alloc(tmem_slot, kLmTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto fail = [&]() {
    if (a.status != nullptr) atomicOr(a.status, kStatusTimeout);
    *(volatile int*)abort_flag = 1;
  };

  int issued = 0, consumed = 0;  // stages (producer, MMA issuer)
  if (warp == 0) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      const uint64_t keep = evict_last_policy();   // h: every vocabulary tile reads it again
      const uint64_t once = evict_first_policy();  // W: read once
      for (int t = 0; t < n_tiles && !*(volatile int*)abort_flag; ++t) {
        const int n0 = (nt_lo + t) * kLmBN;
        for (int kb = 0; kb < KB; ++kb, ++issued) {
          const int s = issued % kLmStages;
          if (issued >= kLmStages &&
              !mbar_wait(&empty[s], (uint32_t)(issued / kLmStages - 1) & 1u, a.wait_ns, abort_flag)) {
            fail();
            break;
          }
          mbar_arrive_expect_tx(&full[s], kLmABytes + kLmBBytes);
          tma_load_2d(sa + s * kLmABytes, &tm_h, kb * kLmBK, mt * kLmBM, &full[s], keep);
          tma_load_2d(sb + s * kLmBBytes, &tm_w, kb * kLmBK, n0, &full[s], once);
        }
      }
      // every load issued has landed before the CTA may leave
      for (int i = max(0, issued - kLmStages); i < issued; ++i)
        mbar_wait(&full[i % kLmStages], (uint32_t)(i / kLmStages) & 1u, kDrainLimitNs);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = lm_idesc(kLmBM, kLmBN);
      const uint32_t a0 = smem_u32(sa), b0 = smem_u32(sb);
      for (int t = 0; t < n_tiles && !*(volatile int*)abort_flag; ++t) {
        const int buf = t & 1;
        if (t >= 2 && !mbar_wait(&acc_empty[buf], (uint32_t)(t / 2 - 1) & 1u, a.wait_ns, abort_flag)) {
          fail();
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(buf * kLmBN);
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb, ++consumed) {
          const int s = consumed % kLmStages;
          if (!mbar_wait(&full[s], (uint32_t)(consumed / kLmStages) & 1u, a.wait_ns, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < kLmBK / 16; ++k) {
            const uint64_t ad = sw128_desc(a0 + (uint32_t)(s * kLmABytes + k * 32));
            const uint64_t bd = sw128_desc(b0 + (uint32_t)(s * kLmBBytes + k * 32));
            tc_mma(d_tmem, ad, bd, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          tc_commit(&empty[s]);  // the stage is free once these MMAs have read it
        }
        if (!ok) {
          fail();
          break;
        }
        tc_commit(&acc_full[buf]);  // the tile's accumulator is complete
      }
      // every MMA issued has completed before TMEM is released
      tc_commit(drain);
      mbar_wait(drain, 0u, kDrainLimitNs);
    }
  } else {
    // --------------------------------------------------------- epilogue
    const int q = warp & 3;                  // TMEM lanes 32 q .. 32 q + 31
    const int row_in_tile = 32 * q + lane;
    const int row = mt * kLmBM + row_in_tile;
    const bool valid = row < p.rows;
    const int bi = valid ? row / a.L : 0;
    const int l = valid ? row - bi * a.L : 0;
    const bool samp = SAMPLER && valid && !a.greedy &&
                      a.stop_flags[bi] == 0 && a.committed[(size_t)row] == 0;
    float* zrow = zbuf + (size_t)row_in_tile * kLmZStride;
    LmRow st{-INFINITY, 0.f, 0.f, 0.f, kNone, kNone};
    const float c2 = a.c2;
    for (int t = 0; t < n_tiles; ++t) {
      const int buf = t & 1;
      // a warp-uniform outcome: the TMEM loads below need the whole warp
      if (!__all_sync(0xffffffffu,
                      mbar_wait(&acc_full[buf], (uint32_t)(t / 2) & 1u, a.wait_ns, abort_flag))) {
        if (lane == 0) fail();
        break;
      }
      tc_fence_after();
      const int n0 = (nt_lo + t) * kLmBN;
      Words4 gw{{0u, 0u, 0u, 0u}};
      if (samp)  // the group stream's words of the tile's four groups (one call)
        gw = philox((uint32_t)(n0 / kGroup) >> 2, (uint32_t)l, (uint32_t)a.s,
                    (uint32_t)(a.canvas_offset + bi) | (kStreamGroup << 24), a.key0, a.key1);
      const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * kLmBN);
#pragma unroll 1
      for (int g = 0; g < kLmBN / kGroup; ++g) {
        float z[64];
        {
          float lo[32], hi[32];
          __syncwarp();  // tcgen05.ld is warp-wide: every lane, converged
          tc_ld32(taddr + (uint32_t)(g * kGroup), lo);
          tc_ld32(taddr + (uint32_t)(g * kGroup + 32), hi);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            z[i] = lo[i];
            z[32 + i] = hi[i];
          }
        }
        if (!valid) continue;
        const int v0 = n0 + g * kGroup;
        if constexpr (!SAMPLER) {
          float4* out = reinterpret_cast<float4*>(p.logits_out + (size_t)row * p.V + v0);
#pragma unroll
          for (int i = 0; i < 16; ++i) out[i] = make_float4(z[4 * i], z[4 * i + 1], z[4 * i + 2], z[4 * i + 3]);
          continue;
        }
        if constexpr (SAMPLER) {
          // group maximum and its lowest index
          float m8[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            float m = z[8 * j];
#pragma unroll
            for (int i = 1; i < 8; ++i) m = fmaxf(m, z[8 * j + i]);
            m8[j] = m;
          }
          const float mg = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                 fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
          uint32_t eq_lo = 0u, eq_hi = 0u;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            eq_lo |= (z[i] == mg ? 1u : 0u) << i;
            eq_hi |= (z[32 + i] == mg ? 1u : 0u) << i;
          }
          const int ig = eq_lo ? __ffs(eq_lo) - 1 : 31 + __ffs(eq_hi);
          if (mg > st.M) {  // a new maximum: rescale the state to it
            if (st.M > -INFINITY) {
              const float dd = (st.M - mg) * c2;
              const float f = ex2(dd);
              st.W = f * fmaf(dd, st.S, st.W);
              st.S *= f;
              st.R *= f;
            }
            st.M = mg;
            st.amax = v0 + ig;
          }
          // the group's sums relative to the maximum (z - M exact for the
          // largest terms, so the maximum's own term is exactly 1)
          float s8[8], w8[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) s8[j] = w8[j] = 0.f;
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            const float d = (z[i] - st.M) * c2;
            const float e = ex2(d);
            s8[i & 7] += e;
            w8[i & 7] = fmaf(e, d, w8[i & 7]);
          }
          const float Sg = ((s8[0] + s8[1]) + (s8[2] + s8[3])) + ((s8[4] + s8[5]) + (s8[6] + s8[7]));
          const float Wg = ((w8[0] + w8[1]) + (w8[2] + w8[3])) + ((w8[4] + w8[5]) + (w8[6] + w8[7]));
          st.S += Sg;
          st.W += Wg;
          if (samp) {  // the group-level race (strict: the earlier group keeps a tie)
            const uint32_t x = pick_word(gw, (uint32_t)g);
            if (!(Sg * 1.0001f <= st.R * one_minus_u(x))) {
              const float E = -logf(uniform_open(x));
              if (Sg > st.R * E) {
                st.R = __fdividef(Sg, E);
                st.gb = v0 / kGroup;
#pragma unroll
                for (int i = 0; i < 32; ++i)
                  reinterpret_cast<float2*>(zrow)[i] = make_float2(z[2 * i], z[2 * i + 1]);
              }
            }
          }
              }
}
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
    }
    if (SAMPLER && valid && !*(volatile int*)abort_flag) {
      SliceRecord r;
      r.S = (double)st.S;
      r.W = (double)st.W;
      r.zmax = st.M;
      const bool drawn = samp && st.gb != kNone;
      r.gscore = (drawn && st.R > 0.f) ? fmaf(st.M, a.iT, logf(st.R)) : -INFINITY;
      r.amax = st.amax;
      r.sample = drawn ? lm_draw(a, zrow, st.gb, bi, l) : -1;
      r.pad0 = r.pad1 = 0;
      p.rec[(size_t)ns * (size_t)p.rows + (size_t)row] = r;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) {
    __syncwarp();
    tc_dealloc(tmem, kLmTmemCols);
    tc_relinquish();
  }
}

// Each canvas's place among the active ones (stop flag clear), -1 for a
// stopped one: what the combine reads to skip stopped canvases.  One block.
__global__ void active_index_kernel(const uint8_t* stop_flags, int B, int32_t* act_index) {
  __shared__ int base;
  if (threadIdx.x == 0) base = 0;
  __syncthreads();
  for (int b0 = 0; b0 < B; b0 += blockDim.x) {
    const int b = b0 + threadIdx.x;
    const bool on = b < B && stop_flags[b] == 0;
    const unsigned bal = __ballot_sync(0xffffffffu, on);
    __shared__ int wsum[32];
    if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = __popc(bal);
    __syncthreads();
    int off = base;
    for (int w = 0; w < (int)(threadIdx.x >> 5); ++w) off += wsum[w];
    if (b < B) act_index[b] = on ? off + __popc(bal & ((1u << (threadIdx.x & 31)) - 1u)) : -1;
    __syncthreads();
    if (threadIdx.x == 0)
      for (int w = 0; w < (int)(blockDim.x >> 5); ++w) base += wsum[w];
    __syncthreads();
  }
}

}  // namespace ebk
