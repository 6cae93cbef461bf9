// eb_synth.cu -- seeded synthetic decoder logits (see eb_synth.h).
//
// Build with `-fmad=false` (device) and `-ffp-contract=off` (host) so that
// the element function below rounds identically on both sides: it uses only
// IEEE add/mul/div/sqrt and integer operations.
#include "eb_synth.h"

#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#define EBS_HD __host__ __device__ __forceinline__

namespace {

enum : uint32_t { TAG_TARGET = 1, TAG_RANK = 2, TAG_BOOST = 3, TAG_NOISE = 4, TAG_PERM = 5 };

EBS_HD uint32_t f2u(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
EBS_HD float u2f(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

// SplitMix64 finaliser (Steele, Lea, Flood, "Fast splittable pseudorandom
// number generators", OOPSLA 2014).
EBS_HD uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
  z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
  return z ^ (z >> 31);
}

EBS_HD uint64_t row_key(uint64_t seed, uint32_t tag, uint32_t b, uint32_t s, uint32_t l) {
  uint64_t k = mix64(seed ^ (0x9E3779B97F4A7C15ULL * (uint64_t)(tag + 1)));
  k = mix64(k ^ (((uint64_t)b << 32) | (uint64_t)s));
  return mix64(k ^ (uint64_t)l);
}

// Uniform in (0, 1) on a 2^-24 grid from the top 24 bits.
EBS_HD float u01(uint64_t h) {
  return ((float)(uint32_t)(h >> 40) + 0.5f) * (1.0f / 16777216.0f);
}

// Natural log for positive normal floats: x = 2^e m with m in [sqrt(1/2),
// sqrt(2)), ln m = 2 atanh(t) with t = (m - 1) / (m + 1), |t| <= 0.1716, by
// its odd series to t^9 (truncation below 1e-9), ln x = e ln 2 + ln m.
EBS_HD float my_log(float x) {
  uint32_t bits = f2u(x);
  int e = (int)((bits >> 23) & 0xffu) - 127;
  float m = u2f((bits & 0x7fffffu) | 0x3f800000u);
  if (m > 1.41421356f) {
    m = m * 0.5f;
    e += 1;
  }
  float t = (m - 1.0f) / (m + 1.0f);
  float t2 = t * t;
  float p = 1.0f / 9.0f;
  p = p * t2 + 1.0f / 7.0f;
  p = p * t2 + 0.2f;
  p = p * t2 + 1.0f / 3.0f;
  p = p * t2 + 1.0f;
  float lnm = 2.0f * t * p;
  return (float)e * 0.693147181f + lnm;
}

// Standard normal by Marsaglia's polar method on successive hashes of k.
EBS_HD float normal01(uint64_t k) {
  for (uint64_t i = 0; i < 16; ++i) {
    uint64_t h = mix64(k + i * 0xD1B54A32D192ED03ULL);
    float a = 2.0f * (((float)(uint32_t)(h >> 40) + 0.5f) * (1.0f / 16777216.0f)) - 1.0f;
    float c = 2.0f * (((float)((uint32_t)(h >> 8) & 0xFFFFFFu) + 0.5f) * (1.0f / 16777216.0f)) - 1.0f;
    float s = a * a + c * c;
    if (s < 1.0f && s > 0.0f) {
      float r = -2.0f * my_log(s);
      r = r / s;
      return a * sqrtf(r);
    }
  }
  return 0.0f;
}

EBS_HD uint16_t f2bf(float f) {  // round to nearest even
  uint32_t u = f2u(f);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

EBS_HD int half_bits_for(uint32_t V) {
  int k = 1;
  while ((uint64_t)1 << (2 * k) < (uint64_t)V) ++k;
  return k;
}

// Keyed permutation of [0, V): 4-round Feistel on 2k bits, cycle walking.
EBS_HD uint32_t permute(uint32_t v, uint64_t key, uint32_t V, int hb) {
  const uint32_t mask = (1u << hb) - 1u;
  uint32_t x = v;
  for (int walk = 0; walk < 64; ++walk) {
    uint32_t Lh = x >> hb, R = x & mask;
    for (uint32_t r = 0; r < 4; ++r) {
      uint32_t F = (uint32_t)mix64(key ^ ((uint64_t)r << 32) ^ (uint64_t)R) & mask;
      uint32_t nR = Lh ^ F;
      Lh = R;
      R = nR;
    }
    x = (Lh << hb) | R;
    if (x < V) return x;
  }
  return v;
}

struct Row {
  uint32_t target;
  float boost;
  uint64_t noise_key;
  uint64_t perm_key;
  int hb;
};

EBS_HD Row row_info(const ebs_params_t& p, uint32_t b, uint32_t s, uint32_t l) {
  Row r;
  uint64_t kt = row_key(p.seed, TAG_TARGET, b, 0u, l);
  r.target = (uint32_t)(((kt >> 32) * (uint64_t)(uint32_t)p.V) >> 32);
  float ub = u01(row_key(p.seed, TAG_BOOST, b, s, l));
  if (p.kind == EBS_TARGET_BOOST) {
    float rank = u01(row_key(p.seed, TAG_RANK, b, 0u, l));
    float e = p.ramp_base + p.ramp_per_canvas * (float)b;
    float f = p.f0 + (p.f1 - p.f0) * ((float)s / e);
    if (f > 1.0f) f = 1.0f;
    r.boost = rank < f ? p.conf_lo + (p.conf_hi - p.conf_lo) * ub
                       : p.unc_lo + (p.unc_hi - p.unc_lo) * ub;
  } else {
    r.boost = p.boost_lo + (p.boost_hi - p.boost_lo) * ub;
  }
  r.noise_key = row_key(p.seed, TAG_NOISE, b, s, l);
  r.perm_key = row_key(p.seed, TAG_PERM, b, 0u, l);
  r.hb = half_bits_for((uint32_t)p.V);
  return r;
}

EBS_HD float element(const ebs_params_t& p, const Row& r, uint32_t v) {
  float n = normal01(mix64(r.noise_key ^ (uint64_t)v));
  float z;
  if (p.kind == EBS_TARGET_BOOST) {
    z = p.noise_sd * n;
  } else {
    uint32_t rank = permute(v, r.perm_key, (uint32_t)p.V, r.hb) + 1u;
    float a = -p.zipf_scale * my_log((float)rank);
    z = a + p.zipf_noise_sd * n;
  }
  if (v == r.target) z = z + r.boost;
  return z;
}

constexpr int kThreads = 256;
constexpr int kPerThread = 8;

__global__ void __launch_bounds__(kThreads)
gen_kernel(ebs_params_t p, int b0, int s, void* out) {
  const int l = blockIdx.y, bi = blockIdx.z;
  const uint32_t b = (uint32_t)(b0 + bi);
  const Row r = row_info(p, b, (uint32_t)s, (uint32_t)l);
  const size_t row_off = ((size_t)bi * (size_t)p.L + (size_t)l) * (size_t)p.V;
  const uint32_t base = (uint32_t)blockIdx.x * kThreads * kPerThread + threadIdx.x;
#pragma unroll 1
  for (int k = 0; k < kPerThread; ++k) {
    uint32_t v = base + (uint32_t)k * kThreads;
    if (v >= (uint32_t)p.V) break;
    float z = element(p, r, v);
    if (p.dtype == EBS_F32) ((float*)out)[row_off + v] = z;
    else ((uint16_t*)out)[row_off + v] = f2bf(z);
  }
}

}  // namespace

extern "C" int ebs_generate_device(const ebs_params_t* p, int b0, int nb, int s, void* out,
                                   void* stream) {
  if (!p || !out || nb <= 0 || p->L <= 0 || p->V <= 0 || nb > 65535 || p->L > 65535) return -1;
  dim3 grid((unsigned)((p->V + kThreads * kPerThread - 1) / (kThreads * kPerThread)),
            (unsigned)p->L, (unsigned)nb);
  gen_kernel<<<grid, kThreads, 0, (cudaStream_t)stream>>>(*p, b0, s, out);
  return (int)cudaGetLastError();
}

extern "C" int ebs_generate_host(const ebs_params_t* p, int b0, int nb, int s, int l0, int nl,
                                 void* out) {
  for (int bi = 0; bi < nb; ++bi) {
    for (int li = 0; li < nl; ++li) {
      const Row r = row_info(*p, (uint32_t)(b0 + bi), (uint32_t)s, (uint32_t)(l0 + li));
      const size_t off = ((size_t)bi * (size_t)nl + (size_t)li) * (size_t)p->V;
      for (uint32_t v = 0; v < (uint32_t)p->V; ++v) {
        float z = element(*p, r, v);
        if (p->dtype == EBS_F32) ((float*)out)[off + v] = z;
        else ((uint16_t*)out)[off + v] = f2bf(z);
      }
    }
  }
  return 0;
}

extern "C" float ebs_log(float x) { return my_log(x); }

extern "C" uint32_t ebs_target(const ebs_params_t* p, int b, int l) {
  return row_info(*p, (uint32_t)b, 0u, (uint32_t)l).target;
}
