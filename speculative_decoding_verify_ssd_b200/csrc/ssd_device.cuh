// ssd_device.cuh -- device-side building blocks of libssd (sm_100a only).
//
// Bulk global->shared copies completed on an mbarrier, bounded waits, the
// fast exp2, bf16 unpacking, order-preserving integer keys for logits, and
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As
// Easy as 1, 2, 3", SC'11, section 4).
#pragma once

#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssd {

namespace cg = cooperative_groups;

constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------------------
// Shared-memory addresses, mbarrier and the bulk copy engine.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// Make the initialised barrier visible to the async (bulk copy) proxy.
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_addr(bar)),
      "r"(bytes)
      : "memory");
}

// Adds `bytes` to the current phase's expected transaction count without an
// arrival: the phase cannot complete before its pending arrival comes.
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

// One poll; the thread may be suspended (up to `hint_ns`) until the phase
// completes, so a waiting warp costs almost no issue slots.
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return done != 0;
}

// Nanoseconds of the GPU's global timer.
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait for a phase of an mbarrier.  Each poll suspends the thread in
// hardware until the phase completes (or `kSuspendHintNs` pass), so a waiting
// warp issues almost no instructions and resumes as soon as the bytes land.
// Returns false once `limit_ns` of global time has passed without completion.
constexpr uint32_t kSuspendHintNs = 100000u;
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, unsigned long long limit_ns) {
  if (mbar_try_wait(bar, parity, kSuspendHintNs)) return true;
  const unsigned long long t0 = global_ns();
  for (uint32_t i = 0; i < (1u << 30); ++i) {
    if (mbar_try_wait(bar, parity, kSuspendHintNs)) return true;
    if (global_ns() - t0 > limit_ns) return false;
  }
  return false;
}

// One thread's arrival on a counter in global memory, GPU scope, acquire and
// release at once.  Issued after a CTA barrier, the release publishes what the
// whole CTA wrote before the barrier (the barrier orders those writes before
// this thread's), and after the next barrier the acquire makes what the
// earlier arrivals published visible to the whole CTA.  Returns the old value.
__device__ __forceinline__ int32_t arrive_acq_rel_gpu(int32_t* p) {
  int32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;" : "=r"(old) : "l"(p) : "memory");
  return old;
}

// CTA-scope acquire-release add on a shared-memory counter; returns the old value.
__device__ __forceinline__ uint32_t atom_add_acq_rel_cta_shared(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(smem_addr(p)), "r"(v) : "memory");
  return old;
}

// Orders this thread's view of generic-proxy shared-memory accesses (the
// other warps' reads of a stage, acquired above) before its later
// async-proxy ones (the bulk copy that overwrites the stage).
__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ uint64_t ld_acquire_gpu_u64(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.acquire.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed_gpu_u32(int32_t* p, int32_t v) {
  asm volatile("st.relaxed.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ int32_t ld_relaxed_gpu_u32(const int32_t* p) {
  int32_t v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed_gpu_u64(uint64_t* p, uint64_t v) {
  asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ void st_release_gpu_u64(uint64_t* p, uint64_t v) {
  asm volatile("st.release.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Bounded wait for a 64-bit word whose high half is a tag: true (and the
// word in *out) once the high half equals `tag`; false after `limit_ns`.
__device__ __forceinline__ bool wait_tagged(const uint64_t* word, uint32_t tag, unsigned long long limit_ns,
                                            uint64_t* out, uint32_t max_sleep_ns = 256) {
  const unsigned long long t0 = global_ns();
  uint32_t sleep_ns = 32;
  for (uint32_t i = 0; i < 50000000u; ++i) {
    const uint64_t v = ld_acquire_gpu_u64(word);
    if (static_cast<uint32_t>(v >> 32) == tag) {
      *out = v;
      return true;
    }
    if (global_ns() - t0 > limit_ns) return false;
    __nanosleep(sleep_ns);
    if (sleep_ns < max_sleep_ns) sleep_ns <<= 1;
  }
  return false;
}

// 1-D bulk copy global -> this CTA's shared memory (no multicast).  Both
// addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(static_cast<uint64_t>(__cvta_generic_to_global(src))), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// The same copy with an L2 cache policy (see l2_policy_evict_first).
__device__ __forceinline__ void bulk_copy_g2s_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                                   uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
          "r"(smem_addr(dst)),
      "l"(static_cast<uint64_t>(__cvta_generic_to_global(src))), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

// An L2 policy for data read once: its lines are the first to be evicted, so
// a stream larger than L2 does not push out the small lines that are read
// again soon (workspace records, flags).
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// The default L2 priority, for data that may be read again soon.
__device__ __forceinline__ uint64_t l2_policy_evict_normal() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// ---------------------------------------------------------------------------
// Arithmetic helpers.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// max with NaN propagation (a NaN anywhere makes the result NaN).
// Two fp32 values in one 64-bit register pair, for the packed fp32x2
// arithmetic of sm_100 (one instruction does both lanes, each lane rounded
// exactly like its scalar counterpart).
typedef unsigned long long f32x2;
__device__ __forceinline__ f32x2 f2_pack(float lo, float hi) {
  f32x2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(f32x2 v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ f32x2 f2_fma(f32x2 a, f32x2 b, f32x2 c) {
  f32x2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ f32x2 f2_add(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f32x2 f2_mul(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

__device__ __forceinline__ float fmax_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

__device__ __forceinline__ uint32_t bf16x2_max_nan(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.NaN.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Order-preserving key of a float logit: larger logit -> larger key; -0 and
// +0 map to the same key so that they tie (and the lower token id wins).
__device__ __forceinline__ uint32_t ord_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7FFFFFFFu) == 0u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Composite ranking key: logit descending, then token id ascending.
__device__ __forceinline__ unsigned long long rank_key(float f, int idx) {
  return (static_cast<unsigned long long>(ord_key(f)) << 32) |
         static_cast<unsigned long long>(0xFFFFFFFFu - static_cast<uint32_t>(idx));
}

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon et al., SC'11): ten rounds, key bumped by the Weyl
// constants after each round.
// ---------------------------------------------------------------------------
struct U4 {
  uint32_t x, y, z, w;
};

__device__ __forceinline__ U4 philox4x32_10(U4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t lo0 = 0xD2511F53u * c.x;
    const uint32_t hi0 = __umulhi(0xD2511F53u, c.x);
    const uint32_t lo1 = 0xCD9E8D57u * c.z;
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, c.z);
    c = U4{hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0};
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return c;
}

// Fallback speculator token i of row b: floor(x * V / 2^32), x = word 0 at
// counter (b, i, 2, 0), key = seed.
__device__ __forceinline__ int32_t fallback_token(unsigned long long seed, int b, int i, int V) {
  const U4 o = philox4x32_10(U4{static_cast<uint32_t>(b), static_cast<uint32_t>(i), 2u, 0u},
                             static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32));
  return static_cast<int32_t>((static_cast<unsigned long long>(o.x) * static_cast<uint32_t>(V)) >> 32);
}

// ---------------------------------------------------------------------------
// Warp reductions.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// The F-th largest of n order keys held by one warp (keys[i] for i = lane,
// lane + 32, ...): bitwise search for the largest t with #{key >= t} >= F,
// high bit first.  `bits` = number of significant high bits of the keys.
template <int kPerLane>
__device__ __forceinline__ uint32_t warp_kth_largest(const uint32_t (&keys)[kPerLane], int F, int bits) {
  // two bits per pass: the three extensions of the prefix are counted at once
  // (bits is even), so the dependent chain is bits / 2 warp reductions long
  uint32_t prefix = 0u;
  for (int bit = 30; bit >= 32 - bits; bit -= 2) {
    const uint32_t c1 = prefix | (1u << bit), c2 = prefix | (2u << bit), c3 = prefix | (3u << bit);
    int n1 = 0, n2 = 0, n3 = 0;
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      n1 += keys[i] >= c1;
      n2 += keys[i] >= c2;
      n3 += keys[i] >= c3;
    }
    n1 = __reduce_add_sync(0xFFFFFFFFu, n1);
    n2 = __reduce_add_sync(0xFFFFFFFFu, n2);
    n3 = __reduce_add_sync(0xFFFFFFFFu, n3);
    prefix = n3 >= F ? c3 : (n2 >= F ? c2 : (n1 >= F ? c1 : prefix));
  }
  return prefix;
}

// Inverse of ord_key.
__device__ __forceinline__ float key_to_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

}  // namespace ssd
