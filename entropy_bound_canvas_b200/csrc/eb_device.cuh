// eb_device.cuh -- device primitives of the sampler: Philox4x32-10, the
// Gumbel and uniform-token maps, mbarrier / bulk-copy (TMA) wrappers with
// bounded waits, and warp reductions.  sm_100a only.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace ebk {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

// 2^x with the MUFU approximation (relative error ~2^-22); subnormal results
// flush to zero, which only drops terms below 2^-126 of the row maximum.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon et al., "Parallel random numbers: as easy as 1, 2, 3",
// SC'11): ten rounds of two 32x32->64 multiplies, the high halves crossed with
// the other two words and the round key, the key bumped by the Weyl constants.
// ---------------------------------------------------------------------------
struct Words4 {
  uint32_t w[4];
};

__device__ __forceinline__ Words4 philox(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                         uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t hi0 = __umulhi(0xD2511F53u, c0), lo0 = 0xD2511F53u * c0;
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, c2), lo1 = 0xCD9E8D57u * c2;
    const uint32_t n0 = hi1 ^ c1 ^ k0;
    const uint32_t n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
  }
  Words4 o;
  o.w[0] = c0;
  o.w[1] = c1;
  o.w[2] = c2;
  o.w[3] = c3;
  return o;
}

__device__ __forceinline__ uint32_t pick_word(const Words4& r, uint32_t i) {
  return i == 0 ? r.w[0] : i == 1 ? r.w[1] : i == 2 ? r.w[2] : r.w[3];
}

// Streams of the counter layout: ctr = (index >> 2, a, step, b | stream << 24).
enum : uint32_t { kStreamGumbel = 0, kStreamRenoise = 1, kStreamInit = 2, kStreamGroup = 3 };

// The uniform of a word x: u = (2 (x >> 9) + 1) 2^-24, in (0, 1), built
// exactly from bits: 1 + (x >> 9) 2^-23 lies in [1, 2), and subtracting
// 1 - 2^-24 is exact (both operands within a factor of two).
__device__ __forceinline__ float uniform_open(uint32_t x) {
  return __uint_as_float(0x3F800000u | (x >> 9)) - 0.99999994039535522f;
}

// 1 - u for the same word, exactly: (2 (~x >> 9) + 1) 2^-24.
__device__ __forceinline__ float one_minus_u(uint32_t x) {
  return __uint_as_float(0x3F800000u | (~x >> 9)) - 0.99999994039535522f;
}

// Standard Gumbel from one word: g = -ln(-ln u).  The inner log must be
// accurate near u = 1 (logf, ~1 ulp); the outer one only needs absolute
// accuracy, which lg2.approx gives.
__device__ __forceinline__ float gumbel(uint32_t x) {
  const float e = -logf(uniform_open(x));
  return -0.6931471805599453f * lg2(e);
}

// Largest Gumbel value the 23-bit grid can produce, -ln(-ln(1 - 2^-24)) =
// 16.6355..., rounded up; a group whose log-partition plus this bound is
// below the best score so far cannot win.
constexpr float kGumbelMax = 16.64f;

// Uniform token in [0, V): high word of x * V.
__device__ __forceinline__ uint32_t uniform_token(uint32_t x, uint32_t V) { return __umulhi(x, V); }

// ---------------------------------------------------------------------------
// mbarrier + 1-D bulk copy (cp.async.bulk, the TMA engine without a tensor
// map).  Every copy reads this GPU's own memory into the issuing CTA's own
// shared memory and nowhere else.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// One test of the phase that may suspend the thread for up to hint_ns; the
// thread resumes as soon as the phase completes.
__device__ __forceinline__ bool mbar_try_wait_for(uint64_t* bar, uint32_t parity,
                                                  uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Every wait gives up after a limit and reports a timeout: the pipeline
// waits after the step's configured limit (2 s unless a test shortens it),
// the drain of copies still in flight at a kernel's exit after kDrainLimitNs.
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint64_t kDrainLimitNs = 2000000000ull;
// Suspension asked of one test (the limit and the abort flag are looked at
// between tests).
constexpr uint32_t kSuspendHintNs = 20000;

// One test of the phase that never suspends the thread.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Gives up (false) after limit_ns, or once *abort is set when abort is given.
// A suspended test may last until the phase completes (whatever its hint):
// the limit bounds a wait for a phase that does not complete.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          uint64_t limit_ns = kWaitLimitNs,
                                          const int* abort = nullptr) {
  if (mbar_try_wait_for(bar, parity, kSuspendHintNs)) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    if (mbar_try_wait_for(bar, parity, kSuspendHintNs)) return true;
    if (abort != nullptr && *(const volatile int*)abort) return false;
    if (global_ns() - t0 > limit_ns) return false;
  }
}

// mbar_wait, except that a limit shorter than kSuspendHintNs is kept with
// tests that never suspend and the clock read after each: such a limit runs
// out whenever the phase is not complete at the first test.
static __device__ __noinline__ bool mbar_wait_timed(uint64_t* bar, uint32_t parity,
                                                    uint64_t limit_ns, const int* abort) {
  if (limit_ns >= kSuspendHintNs) return mbar_wait(bar, parity, limit_ns, abort);
  const uint64_t t0 = global_ns();
  for (;;) {
    if (mbar_test_wait(bar, parity)) return true;
    if (abort != nullptr && *(const volatile int*)abort) return false;
    if (global_ns() - t0 > limit_ns) return false;
  }
}

// Shared-memory counter published by one thread and polled by others.
__device__ __forceinline__ void st_release_shared(int* p, int v) {
  asm volatile("st.release.cta.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire_shared(const int* p) {
  int v;
  asm volatile("ld.acquire.cta.shared::cta.b32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
  return v;
}

// Global counter read with acquire semantics at GPU scope (pairs with a
// writer's release update).
__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Atomic add at GPU scope with acquire-release semantics: this thread's
// earlier writes are visible to whoever observes the new value, and the
// writes of those whose additions this one observes are visible to it.
// Returns the old value.
__device__ __forceinline__ int atom_add_acq_rel_gpu(int* p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// L2 policy for data read exactly once: evict it first, so that a stream
// larger than L2 does not push out the kernel's code and small shared state.
__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t evict_last_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes,
                                          uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(smem_dst)),
      "l"(gsrc), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Hint: bring the cache line holding p into L1 (no fault on any address the
// caller could load).
__device__ __forceinline__ void prefetch_l1(const void* p) {
  asm volatile("prefetch.global.L1 [%0];" ::"l"(p));
}

// Programmatic dependent launch: the dependent grid may be scheduled once
// every CTA of this grid has signalled (or exited); griddep_wait blocks until
// the prerequisite grid has completed and its memory operations are visible.
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Block barrier entered by converged warps.  The barrier instruction counts
// arrivals per warp-wide instruction, so a warp whose lanes reached it apart
// (after divergent code) would be counted more than once and could let it
// complete early; the warp barrier first reconverges the lanes.
__device__ __forceinline__ void block_sync() {
  __syncwarp();
  __syncthreads();
}

// Named barrier among the consumer warps only (the producer warp never joins).
__device__ __forceinline__ void consumer_sync(int nthreads) {
  asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

}  // namespace ebk
