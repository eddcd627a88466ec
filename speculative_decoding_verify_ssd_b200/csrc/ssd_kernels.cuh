// ssd_kernels.cuh -- the vocab-wide kernels of libssd.
//
// The step runs as two kernels that talk through the caller's workspace:
//
// Kernel 1 (stats): one CTA per (unit, slice), unit = (row b, position j).
//   The CTA streams its slice of the unit's target row p_j and draft row q_j
//   from HBM exactly once through a ring of 1-D bulk copies into shared
//   memory (cp.async.bulk completed on mbarriers, no multicast) and keeps per
//   thread only running softmax state ([ZH] = "Speculative Speculative
//   Decoding", gist.science Chinese edition, technical summary section 2;
//   [NL] = the Dutch edition, sections 2 and 3A-3C):
//     - online max and rescaled sum of exp2 of p_j and q_j (temperature
//       softmax, one exp per element), or the greedy argmax when T = 0;
//     - the three largest vector maxima of the top-F source row (q_j) and the
//       two vectors holding the largest, so the slice's own top-F (which contains the
//       slice's share of the unit's top-F, [ZH] challenge 2 "top-F tokens")
//       comes from registers: the F-th largest thread maximum bounds it from
//       below.
//   It publishes a small partial and leaves (one thread's release reduction
//   on the unit's counter).  The unit's last slice to arrive (nobody waits)
//   merges the partials, selects the exact
//   top-F by (logit desc, token id asc), forms Q_S and the Saguaro normaliser
//   Z = 1 - (1 - C) Q_S ([ZH] challenge 2; [NL] 3B), and runs the lossless
//   accept test a_j = min(1, p_j(d_j) / q'_j(d_j)).  In verify mode it
//   publishes the unit's result in one tagged word (call epoch, rejected,
//   near-tie, flags) and nobody waits for the rest of the row; in reweight
//   mode the row's last unit to finish publishes the row's per-position words.
//   Units are taken row by row; in verify mode, when every row's unit-K CTAs
//   fit one wave, positions j < K of every row come before any row's unit K.
//
// Kernel 2 (draw): one CTA per (row, slice) of the single unit each row
//   draws from: the residual r = max(0, p_k* - q'_k*) (or p_K after full
//   acceptance, or q' for a draft draw).  It is a programmatic dependent of
//   kernel 1 (scheduled once every kernel-1 CTA has started).  Each CTA polls
//   its own row's unit words and takes k* as soon as positions 0..k* are in
//   (the first rejected one, every earlier one accepted), so the draws of
//   early rows run while kernel 1 finishes.  Each CTA sums its slice of r per
//   (ring chunk, warp); the CTA holding the crossing of u * R in token order
//   (slice, chunk, warp, lane, token) draws the bonus token, reads the words
//   past k* for the row's flags when it has not seen them yet, and finishes
//   the row: outputs, the cache lookup of (k*, bonus) and the random-token
//   fallback ([ZH] basic flow steps 3-4 and challenge 3; [NL] 3C).
#pragma once

#include <limits.h>

#include "../../include/ssd.h"
#include "ssd_device.cuh"

namespace ssd {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
#ifndef SSD_STATS_EVICT_FIRST
#define SSD_STATS_EVICT_FIRST 1
#endif
#ifndef SSD_MIN_BLOCKS
#define SSD_MIN_BLOCKS 5
#endif
#ifndef SSD_STAGES
#define SSD_STAGES 4
#endif
#ifndef SSD_STATS_VPT
#define SSD_STATS_VPT 2
#endif
constexpr int kMinBlocks = SSD_MIN_BLOCKS;  // statistics CTAs per SM the register budget is set for
constexpr int kDrawMinBlocks = 4;      // draw CTAs per SM (their epilogue needs 64 registers)
constexpr int kMaxSlices = 16;         // slices per logit row
constexpr int kStages = SSD_STAGES;    // depth of the bulk-copy ring (32 KB: five CTAs per SM fit)
constexpr int kChunkVecs = kThreads;   // 16-byte vectors per row per ring stage (draw kernel)
constexpr int kStatsVPT = SSD_STATS_VPT;  // stats kernel: vectors per thread per row per stage
constexpr int kStatsChunkVecs = kChunkVecs * kStatsVPT;
constexpr int kStatsStages = kStages * kChunkVecs / kStatsChunkVecs;  // same ring bytes
constexpr int kMaxChunks = 16;         // ring chunks per slice
constexpr int kCandCap = 256;          // local top-F candidates found by a CTA
constexpr int kCandSlice = 128;        // candidates a slice publishes
constexpr int kGatherCap = 1024;       // candidates of a whole unit
constexpr int kSelCap = 512;           // >= SSD_MAX_BUDGET
constexpr int kMaxGroups = kThreads;   // thread maxima per CTA
constexpr unsigned long long kRingWaitNs = 2000000000ull;  // a ring stage's bytes: 2 s at most
constexpr float kNearTie = 1e-5f;
#ifndef SSD_DEP_WAIT_NS
#define SSD_DEP_WAIT_NS 1000000000ull
#endif
// the limit of a wait for another CTA's result (a slice partial, a unit record,
// a row's decision word): 1 s
constexpr unsigned long long kDepWaitNs = SSD_DEP_WAIT_NS;
constexpr int kFlagTimeout = SSD_ROW_DEVICE_TIMEOUT;
constexpr size_t kRingBytes = static_cast<size_t>(kStages) * 2 * kChunkVecs * 16;

static_assert(8 * (kCandCap + kGatherCap + kSelCap) <= kRingBytes, "merge buffers must fit in the idle ring");
static_assert(2 * 4 * kMaxSlices * kMaxChunks * kWarps <= kRingBytes, "draw partial sums must fit in the idle ring");

enum Mode : int { kModeVerify = 0, kModeReweight = 1 };
enum Draw : int { kDrawNone = 0, kDrawResidual = 1, kDrawP = 2, kDrawQ = 3 };

struct Cand {
  float x;
  int32_t idx;
};

// Kernel 1, one per (unit, slice).
struct SlicePart {
  float mP, sP, mQ, sQ;           // running max and exp-sum of the slice
  int32_t argP, argQ;             // greedy: lowest id of the slice maximum
  int32_t n_cand, timeout;        // local candidates found; copy timeout
  float xdP, xdQ;                 // logits of the drafted token (the slice that holds it)
  int32_t pskip, pad2;            // early exit: this slice did not read the target row
  Cand cand[kCandSlice];          // sorted local candidates (at most min(n_cand, F))
};

// Kernel 1, written by the unit's finalizer.
struct UnitState {
  float MP, SP, MQ, SQ;           // unit maxima and exp-sums (relative to the maxima)
  float Z, bx, a, amargin;        // Saguaro normaliser, top-F boundary logit, a_j, |u_j - a_j|
  int32_t bi, argP, argQ, flags;  // top-F boundary id, greedy argmaxes, SSD_ROW_* bits
  int32_t rejected, Fj, seg_off;  // u_j >= a_j; the unit's fan-out; its cache segment
  float dmargin;                  // draft draw: inverse-CDF margin
};

// Kernel 2, one per (draw unit, slice).
struct DrawPart {
  float R, RP;                    // slice mass of the draw's distribution (and of p alone)
  int32_t timeout, pad;
  float rs[kMaxChunks][kWarps];   // per (chunk, warp) partial sums, token order
  float ps[kMaxChunks][kWarps];
};

// Kernel 1, per row: the decision and (verify) the statistics of unit k*,
// so that the draw reads one record.
struct RowState {
  int32_t kstar, flags;
  float amargin;
  int32_t Fj;
  float MP, SP, MQ, SQ;
  float Z, bx;
  int32_t bi, argP;
};

struct UnitOut;  // ssd_cluster.cuh

struct Args {
  const void* target;      // [B, K+1, V]
  const void* draft;       // [B, K, V]
  const void* draft_next;  // [B, V] or null (verify: source of the full-acceptance guesses)
  const void* guess;       // reweight: rows for segment K, or null
  long long guess_stride;
  const int32_t* tokens;   // [B, K]
  const float* uniforms;   // [B, K+1] (verify) or u_draft [B, K] (reweight), may be null
  const int32_t* F;        // [B, K+1] or null
  const float* alpha;      // [B]: plan computed in-kernel when F is null
  int fanout_mode;
  int B, K, V, budget, mode, n_slices, chunk, units_per_row;
  int d_slices, d_chunk;   // kernel 2: slices per drawn row and their length
  int draws;               // kernel 2 runs (verify always; reweight: draft tokens drawn)
  int early_exit;          // verify: the early-exit read schedule
  int lag;                 // early exit: rows between the CTAs of position j and j + 1
  int k_last;              // verify, full read: every row's unit K after all positions j < K
  float T, C;
  // verify outputs
  int32_t* n_accepted;
  int32_t* bonus;
  int32_t* out_tokens;
  float* accept_prob;
  float* residual_mass;
  int32_t* status;
  int32_t* c_offsets;
  int32_t* c_tokens;
  const int32_t* c_payload;
  uint8_t* c_hit;
  int32_t* c_slot;
  int32_t* c_next;
  unsigned long long fallback_seed;
  // reweight outputs
  int32_t* topf_tokens;
  int32_t* offsets;
  float* Z;
  float* q_lse;
  int32_t* draft_tokens;
  // workspace
  SlicePart* parts;
  UnitState* ustate;
  DrawPart* dparts;
  RowState* rstate;
  int32_t* arrive1;
  int32_t* row_arrive;
  int32_t* draw_arrive;    // per draw unit: slices that published their masses
  int32_t* draw_owner;     // per draw unit: the tag of the last call whose row a CTA took to finish
  uint64_t* dtot;          // per (draw unit, slice): (epoch + 1) << 32 | bits of the slice's mass
  int32_t* row_arrive2;
  uint64_t* rflag;         // reweight, per draft position: (epoch + 1) << 32 | flags, once the row is decided
  uint64_t* uword;         // verify, per unit: (epoch + 1) << 32 | near << 17 | rejected << 16 | pflags << 8 | flags
  uint32_t* epoch;         // calls completed on this workspace (kernel 2 advances it)
  int32_t* k2_done;        // kernel 2 CTAs past their wait
  int32_t* error;
  unsigned long long* skipped;  // early exit: target-row bytes not read
  // the one-pass cluster form (ssd_cluster.cuh)
  int cl_size;             // CTAs per unit (the cluster's size)
  int cl_len;              // tokens of a row per CTA (a multiple of 8)
  UnitOut* uout;           // per unit: the record its leader publishes
};

template <typename TIn>
struct Elem;
template <>
struct Elem<uint16_t> {
  static constexpr int VE = 8;  // elements per 16-byte vector
  __device__ static __forceinline__ float at(const uint16_t* p, int i) {
    return __uint_as_float(static_cast<uint32_t>(p[i]) << 16);
  }
  __device__ static __forceinline__ void unpack(const uint4& w, float (&x)[8]) {
    x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x); x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
    x[4] = bf16_lo(w.z); x[5] = bf16_hi(w.z); x[6] = bf16_lo(w.w); x[7] = bf16_hi(w.w);
  }
  __device__ static __forceinline__ uint16_t neg_inf() { return 0xFF80u; }
};

// Streaming loads of one 16-byte vector (read-only path).
__device__ __forceinline__ uint4 ld_vec(const void* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }
template <>
struct Elem<float> {
  static constexpr int VE = 4;
  __device__ static __forceinline__ float at(const float* p, int i) { return p[i]; }
  __device__ static __forceinline__ void unpack(const uint4& w, float (&x)[4]) {
    x[0] = __uint_as_float(w.x); x[1] = __uint_as_float(w.y);
    x[2] = __uint_as_float(w.z); x[3] = __uint_as_float(w.w);
  }
  __device__ static __forceinline__ float neg_inf() { return -__int_as_float(0x7F800000); }
};

// Vocab elements [v0, v0 + VE) of the row that starts at element `rb` of
// `base`; elements at or beyond v_end read as -inf.  Aligned: one 16-byte
// load (rb, v0 multiples of VE and v0 + VE <= v_end).
template <typename TIn, bool kAligned>
__device__ __forceinline__ void load_group(const TIn* __restrict__ base, long long rb, int v0, int v_end,
                                           float (&x)[Elem<TIn>::VE]) {
  constexpr int VE = Elem<TIn>::VE;
  if constexpr (kAligned) {
    Elem<TIn>::unpack(ld_vec(base + rb + v0), x);
  } else {
#pragma unroll
    for (int i = 0; i < VE; ++i)
      x[i] = (v0 + i < v_end) ? Elem<TIn>::at(base + rb, v0 + i) : -INFINITY;
  }
}

// One vector of logits into a thread's running state.  Softmax: the running
// maximum m, the sum s of exp2((x - m) c) rescaled when m grows, and
// nmc = -m c.  Greedy: the running maximum and the lowest id holding it.
template <bool kGreedy>
__device__ __forceinline__ float consume_bf16(const uint4 w, int vbase, float c, f32x2 c2, float& m, f32x2& s2,
                                              f32x2& nm2, int& arg, int& nan_seen) {
  const uint32_t m2 = bf16x2_max_nan(bf16x2_max_nan(w.x, w.y), bf16x2_max_nan(w.z, w.w));
  const float vmax = fmax_nan(bf16_lo(m2), bf16_hi(m2));
  if constexpr (kGreedy) {
    nan_seen |= vmax != vmax;
    if (vmax > m) {
      m = vmax;
      float x[8];
      Elem<uint16_t>::unpack(w, x);
#pragma unroll
      for (int i = 7; i >= 0; --i)
        if (x[i] == vmax) arg = vbase + i;
    }
  } else {
    if (!(vmax <= m)) {  // a new maximum (or a NaN, which then sticks)
      const float nm = fmax_nan(m, vmax);
      const float sc = (m == -INFINITY) ? 0.f : ex2((m - nm) * c);  // s2 is 0 while m = -inf
      s2 = f2_mul(s2, f2_pack(sc, sc));
      m = nm;
      const float nmc = -m * c;
      nm2 = f2_pack(nmc, nmc);
    }
    // two lanes per instruction: lane 0 sums the even tokens, lane 1 the odd
    float a0, a1, a2, a3, a4, a5, a6, a7;
    f2_unpack(f2_fma(f2_pack(bf16_lo(w.x), bf16_hi(w.x)), c2, nm2), a0, a1);
    f2_unpack(f2_fma(f2_pack(bf16_lo(w.y), bf16_hi(w.y)), c2, nm2), a2, a3);
    f2_unpack(f2_fma(f2_pack(bf16_lo(w.z), bf16_hi(w.z)), c2, nm2), a4, a5);
    f2_unpack(f2_fma(f2_pack(bf16_lo(w.w), bf16_hi(w.w)), c2, nm2), a6, a7);
    const f32x2 e01 = f2_pack(ex2(a0), ex2(a1)), e23 = f2_pack(ex2(a2), ex2(a3));
    const f32x2 e45 = f2_pack(ex2(a4), ex2(a5)), e67 = f2_pack(ex2(a6), ex2(a7));
    s2 = f2_add(s2, f2_add(f2_add(e01, e23), f2_add(e45, e67)));
  }
  return vmax;
}

// Two vectors of one row from the same ring stage, softmax: both vector
// maxima (returned for the top-F tracking), ONE rescale check for the pair,
// then the packed exp2 sums.  A vector with ok = false is skipped (its words
// read as -inf).
__device__ __forceinline__ void consume2_bf16(const uint4 w0, const uint4 w1, bool ok0, bool ok1, float c, f32x2 c2,
                                              float& m, f32x2& s2, f32x2& nm2, float& v0, float& v1) {
  const uint32_t a = bf16x2_max_nan(bf16x2_max_nan(w0.x, w0.y), bf16x2_max_nan(w0.z, w0.w));
  const uint32_t b = bf16x2_max_nan(bf16x2_max_nan(w1.x, w1.y), bf16x2_max_nan(w1.z, w1.w));
  v0 = ok0 ? fmax_nan(bf16_lo(a), bf16_hi(a)) : -INFINITY;
  v1 = ok1 ? fmax_nan(bf16_lo(b), bf16_hi(b)) : -INFINITY;
  const float vmax = fmax_nan(v0, v1);
  if (!(vmax <= m)) {  // a new maximum (or a NaN, which then sticks)
    const float nm = fmax_nan(m, vmax);
    const float sc = (m == -INFINITY) ? 0.f : ex2((m - nm) * c);  // s2 is 0 while m = -inf
    s2 = f2_mul(s2, f2_pack(sc, sc));
    m = nm;
    const float nmc = -m * c;
    nm2 = f2_pack(nmc, nmc);
  }
#pragma unroll
  for (int v = 0; v < 2; ++v) {
    if (v == 0 ? !ok0 : !ok1) continue;
    const uint4 w = v == 0 ? w0 : w1;
    float a0, a1, a2, a3, a4, a5, a6, a7;
    f2_unpack(f2_fma(f2_pack(bf16_lo(w.x), bf16_hi(w.x)), c2, nm2), a0, a1);
    f2_unpack(f2_fma(f2_pack(bf16_lo(w.y), bf16_hi(w.y)), c2, nm2), a2, a3);
    f2_unpack(f2_fma(f2_pack(bf16_lo(w.z), bf16_hi(w.z)), c2, nm2), a4, a5);
    f2_unpack(f2_fma(f2_pack(bf16_lo(w.w), bf16_hi(w.w)), c2, nm2), a6, a7);
    const f32x2 e01 = f2_pack(ex2(a0), ex2(a1)), e23 = f2_pack(ex2(a2), ex2(a3));
    const f32x2 e45 = f2_pack(ex2(a4), ex2(a5)), e67 = f2_pack(ex2(a6), ex2(a7));
    s2 = f2_add(s2, f2_add(f2_add(e01, e23), f2_add(e45, e67)));
  }
}

template <int VE, bool kGreedy>
__device__ __forceinline__ float consume_f(const float (&x)[VE], int vbase, float c, float& m, float& s, float& nmc,
                                           int& arg, int& nan_seen) {
  float vmax = x[0];
#pragma unroll
  for (int i = 1; i < VE; ++i) vmax = fmax_nan(vmax, x[i]);
  if constexpr (kGreedy) {
    nan_seen |= vmax != vmax;
    if (vmax > m) {
      m = vmax;
#pragma unroll
      for (int i = VE - 1; i >= 0; --i)
        if (x[i] == vmax) arg = vbase + i;
    }
  } else {
    if (!(vmax <= m)) {
      const float nm = fmax_nan(m, vmax);
      s = (m == -INFINITY) ? 0.f : s * ex2((m - nm) * c);
      m = nm;
      nmc = -m * c;
    }
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < VE; ++i) acc += ex2(fmaf(x[i], c, nmc));
    s += acc;
  }
  return vmax;
}

// Greedy merge: the larger maximum, ties to the lower id (commutative).
__device__ __forceinline__ void merge_arg(float& m, int& arg, float m2, int arg2) {
  if (m2 > m || (m2 == m && arg2 < arg)) { m = m2; arg = arg2; }
  else if (m2 != m2) { m = m2; }
}

// Merge two (max, sum) pairs taken relative to their own maxima.
__device__ __forceinline__ void merge_ms(float& m, float& s, float m2, float s2, float c) {
  const float M = fmax_nan(m, m2);
  const float a = (m == -INFINITY) ? 0.f : s * ex2((m - M) * c);
  const float b = (m2 == -INFINITY) ? 0.f : s2 * ex2((m2 - M) * c);
  m = M;
  s = a + b;
}

// The CTA barrier, and the barrier of the 256 consumer threads of a kernel
// whose last warp only issues copies (named barrier 1).
struct CtaBarrier {
  __device__ __forceinline__ void operator()() const { __syncthreads(); }
};
struct ConsumerBarrier {
  __device__ __forceinline__ void operator()() const { asm volatile("bar.sync 1, 256;" ::: "memory"); }
};

// Exact top-F of a whole row, read from global memory by 256 threads: a radix
// select on the 32-bit order key (four 8-bit digits), ties at the threshold
// taken in token-id order, then the F winners ranked by (key, id) in place.
// Used when the shared-memory candidate filter cannot bound the set (many
// ties, F large).  `hist` needs 256 ints; the result is sel[0 .. F); `bar`
// synchronises the 256 threads.

template <typename TIn, typename Bar>
__device__ void topf_exact_global(const TIn* row, int V, int F, Cand* sel, int32_t* hist, int tid, Bar bar) {
  __shared__ uint32_t s_prefix, s_mask;
  __shared__ int32_t s_remaining, s_napp, s_tie_base[kThreads + 1];
  if (tid == 0) { s_prefix = 0u; s_mask = 0u; s_remaining = F; s_napp = 0; }
  bar();
  for (int level = 0; level < 4; ++level) {
    const int shift = 24 - 8 * level;
    for (int i = tid; i < 256; i += kThreads) hist[i] = 0;
    bar();
    const uint32_t prefix = s_prefix, mask = s_mask;
    for (int v = tid; v < V; v += kThreads) {
      const uint32_t k = ord_key(Elem<TIn>::at(row, v));
      if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1);
    }
    bar();
    if (tid == 0) {
      int cum = 0, rem = s_remaining, d = 255;
      for (; d > 0; --d) {
        if (cum + hist[d] >= rem) break;
        cum += hist[d];
      }
      s_remaining = rem - cum;
      s_prefix = prefix | (static_cast<uint32_t>(d) << shift);
      s_mask = mask | (255u << shift);
    }
    bar();
  }
  const uint32_t t = s_prefix;
  const int need_eq = s_remaining;
  // Ties in token order: each thread owns a contiguous chunk of the row.
  const int per = (V + kThreads - 1) / kThreads;
  const int lo = min(V, tid * per), hi = min(V, lo + per);
  int my_eq = 0;
  for (int v = lo; v < hi; ++v) my_eq += (ord_key(Elem<TIn>::at(row, v)) == t);
  s_tie_base[tid + 1] = my_eq;
  bar();
  if (tid == 0) {
    s_tie_base[0] = 0;
    for (int i = 1; i <= kThreads; ++i) s_tie_base[i] += s_tie_base[i - 1];
  }
  bar();
  int tie_rank = s_tie_base[tid];
  for (int v = lo; v < hi; ++v) {
    const float x = Elem<TIn>::at(row, v);
    const uint32_t k = ord_key(x);
    if (k > t) {
      const int pos = atomicAdd(&s_napp, 1);
      if (pos < F) sel[pos] = Cand{x, v};
    } else if (k == t) {
      if (tie_rank < need_eq) {
        const int pos = atomicAdd(&s_napp, 1);
        if (pos < F) sel[pos] = Cand{x, v};
      }
      ++tie_rank;
    }
  }
  bar();
  // Rank in place: every thread keeps its (at most two) winners in registers.
  constexpr int kPer = kSelCap / kThreads;
  Cand mine[kPer];
  int rk[kPer];
#pragma unroll
  for (int q = 0; q < kPer; ++q) {
    const int i = tid + q * kThreads;
    rk[q] = -1;
    if (i < F) {
      mine[q] = sel[i];
      const unsigned long long key = rank_key(mine[q].x, mine[q].idx);
      int r = 0;
      for (int k2 = 0; k2 < F; ++k2) r += rank_key(sel[k2].x, sel[k2].idx) > key;
      rk[q] = r;
    }
  }
  bar();
#pragma unroll
  for (int q = 0; q < kPer; ++q)
    if (rk[q] >= 0) sel[rk[q]] = mine[q];
  bar();
}

// Fan-out plan of one row ([ZH] section 2 challenge 1; [NL] section 3A):
// P(k) = alpha^k (1 - alpha) for k < K, P(K) = alpha^K, quotas budget * P(k)
// rounded by largest remainder (ties to the smaller k); uniform control:
// floor(budget / (K+1)) each, remainder to the smallest k.  fp64 with every
// product and difference rounded on its own (no fused multiply-add), so the
// result is the same integer plan on every device and host.  alpha outside
// [0, 1] yields F[0] = -1 (a plan the verify rejects).
__device__ __forceinline__ void fanout_row(float alpha_f, int K, int budget, int mode, int32_t* f) {
  if (mode == SSD_FANOUT_UNIFORM) {
    for (int k = 0; k <= K; ++k) f[k] = budget / (K + 1) + (k < budget % (K + 1) ? 1 : 0);
    return;
  }
  const double al = static_cast<double>(alpha_f);
  if (!(al >= 0.0 && al <= 1.0)) {
    f[0] = -1;
    for (int k = 1; k <= K; ++k) f[k] = 0;
    return;
  }
  double frac[SSD_MAX_K + 1];
  bool taken[SSD_MAX_K + 1];
  double run = 1.0;
  long long assigned = 0;
  for (int k = 0; k <= K; ++k) {
    double P;
    if (k < K) {
      P = __dmul_rn(run, __dsub_rn(1.0, al));
      run = __dmul_rn(run, al);
    } else {
      P = run;
    }
    const double quota = __dmul_rn(static_cast<double>(budget), P);
    const double fl = floor(quota);
    f[k] = static_cast<int32_t>(fl);
    frac[k] = __dsub_rn(quota, fl);
    taken[k] = false;
    assigned += f[k];
  }
  long long rem = budget - assigned;
  while (rem > 0) {
    int best = -1;
    for (int k = 0; k <= K; ++k)
      if (!taken[k] && (best < 0 || frac[k] > frac[best])) best = k;
    if (best < 0) {
      for (int k = 0; k <= K; ++k) taken[k] = false;
      continue;
    }
    taken[best] = true;
    f[best] += 1;
    --rem;
  }
}

// Power-law plan ([ZH] section 2 challenge 1, the acceptance's power law;
// [NL] section 3A, a geometric series): F_k proportional to P(k)^gamma,
// gamma = q / 8, the optimum when an outcome's hit rate given F guesses
// follows a power-law curve.  alpha^gamma and (1 - alpha)^gamma are the
// eighth root (three correctly rounded square roots) raised to the q-th power
// by q - 1 rounded products; weights w_k = a^k c (k < K), w_K = a^K; quotas
// budget * w_k / W with W summed in k order; largest remainder as in
// fanout_row.  Every operation is rounded on its own, so the plan is the same
// integers on every device and host.  q = 8 is fanout_row's geometric plan.
__device__ __forceinline__ double eighth_power(double x, int q) {
  const double r = __dsqrt_rn(__dsqrt_rn(__dsqrt_rn(x)));
  double y = r;
  for (int i = 1; i < q; ++i) y = __dmul_rn(y, r);
  return y;
}

__device__ __forceinline__ void fanout_row_power(float alpha_f, int K, int budget, int q, int32_t* f) {
  if (q == 8) {
    fanout_row(alpha_f, K, budget, SSD_FANOUT_GEOMETRIC, f);
    return;
  }
  const double al = static_cast<double>(alpha_f);
  if (!(al >= 0.0 && al <= 1.0)) {
    f[0] = -1;
    for (int k = 1; k <= K; ++k) f[k] = 0;
    return;
  }
  const double a = eighth_power(al, q), c = eighth_power(__dsub_rn(1.0, al), q);
  double w[SSD_MAX_K + 1], frac[SSD_MAX_K + 1];
  bool taken[SSD_MAX_K + 1];
  double run = 1.0, W = 0.0;
  for (int k = 0; k < K; ++k) {
    w[k] = __dmul_rn(run, c);
    run = __dmul_rn(run, a);
  }
  w[K] = run;
  for (int k = 0; k <= K; ++k) W = __dadd_rn(W, w[k]);
  long long assigned = 0;
  for (int k = 0; k <= K; ++k) {
    const double quota = __ddiv_rn(__dmul_rn(static_cast<double>(budget), w[k]), W);
    const double fl = floor(quota);
    f[k] = static_cast<int32_t>(fl);
    frac[k] = __dsub_rn(quota, fl);
    taken[k] = false;
    assigned += f[k];
  }
  long long rem = budget - assigned;
  while (rem > 0) {
    int best = -1;
    for (int k = 0; k <= K; ++k)
      if (!taken[k] && (best < 0 || frac[k] > frac[best])) best = k;
    if (best < 0) {
      for (int k = 0; k <= K; ++k) taken[k] = false;
      continue;
    }
    taken[best] = true;
    f[best] += 1;
    --rem;
  }
}

// Ring of bulk copies that streams one slice of up to two rows of a unit
// through shared memory, chunk by chunk (CV 16-byte vectors per row per
// chunk, ST stages).  Every thread waits on the chunk's full barrier itself;
// after reading a stage, each warp counts its release on the stage's counter,
// and the warp that completes the count refills the stage with the chunk ST
// ahead.  No CTA barrier sits in the stream, and no warp waits for the
// slowest one except through the data it needs.
template <typename TIn, int CV = kChunkVecs, int ST = kStages, bool kEvictFirst = false>
struct Ring {
  unsigned char* buf;
  uint64_t* full;
  uint32_t* rel;  // [ST] warps done with the stage's current chunk
  const TIn* row0;
  const TIn* row1;
  int nrows, e0, nvec, nch, n_issued;  // row0 may be null with nrows = 2: half 0 is not read

  __device__ __forceinline__ unsigned char* stage(int slot, int r) const {
    return buf + (static_cast<size_t>(slot) * 2 + r) * (CV * 16);
  }
  __device__ __forceinline__ void issue(int c) {
    constexpr int VE = 16 / sizeof(TIn);
    const int slot = c % ST;
    const int v0 = c * CV;
    const int nv = min(CV, nvec - v0);
    const int nr = (row0 != nullptr ? 1 : 0) + (nrows > 1 ? 1 : 0);
    mbar_arrive_expect_tx(&full[slot], static_cast<uint32_t>(nv) * 16u * static_cast<uint32_t>(nr));
    if (row0 != nullptr) copy_row(slot, 0, row0 + e0 + v0 * VE, nv);
    if (nrows > 1) copy_row(slot, 1, row1 + e0 + v0 * VE, nv);
    n_issued = c + 1;
  }
  __device__ __forceinline__ void copy_row(int slot, int r, const TIn* src, int nv) {
    if constexpr (kEvictFirst) {
      bulk_copy_g2s_hint(stage(slot, r), src, static_cast<uint32_t>(nv) * 16u, &full[slot], l2_policy_evict_first());
    } else {
      bulk_copy_g2s(stage(slot, r), src, static_cast<uint32_t>(nv) * 16u, &full[slot]);
    }
  }
  // Rows 0 and 1 of the first ST chunks issued separately (two rows only):
  // row 1 now, its bytes expected without an arrival, so no stage can
  // complete before issue_first_row0 has decided on row 0.
  __device__ __forceinline__ void issue_first_row1() {
    constexpr int VE = 16 / sizeof(TIn);
    for (int c = 0; c < min(ST, nch); ++c) {
      const int nv = min(CV, nvec - c * CV);
      mbar_expect_tx(&full[c], static_cast<uint32_t>(nv) * 16u);
      copy_row(c, 1, row1 + e0 + c * CV * VE, nv);
    }
  }
  __device__ __forceinline__ void issue_first_row0(bool read0) {
    constexpr int VE = 16 / sizeof(TIn);
    for (int c = 0; c < min(ST, nch); ++c) {
      const int nv = min(CV, nvec - c * CV);
      mbar_arrive_expect_tx(&full[c], read0 ? static_cast<uint32_t>(nv) * 16u : 0u);
      if (read0) copy_row(c, 0, row0 + e0 + c * CV * VE, nv);
    }
    n_issued = min(ST, nch);
  }
  __device__ __forceinline__ void init(int tid) {
    n_issued = 0;
    if (tid == 0) {
      for (int s = 0; s < ST; ++s) {
        mbar_init(&full[s], 1);
        rel[s] = 0u;
      }
      mbar_init_fence();
    }
    __syncthreads();
  }
  __device__ __forceinline__ void start(int tid) {
    init(tid);
    if (tid == 0)
      for (int c = 0; c < min(ST, nch); ++c) issue(c);
  }
  // Chunk c is ready for this thread.
  __device__ __forceinline__ void acquire(int c, int tid, int& tmo) {
    if (!mbar_wait_bounded(&full[c % ST], (c / ST) & 1, kRingWaitNs)) tmo = 1;
  }
  // This warp is done with chunk c's stage; the last warp to say so refills it.
  __device__ __forceinline__ void release(int c, int lane) {
    __syncwarp();
    if (lane == 0) {
      const int slot = c % ST;
      if (atom_add_acq_rel_cta_shared(&rel[slot], 1u) == static_cast<uint32_t>(kWarps - 1)) {
        rel[slot] = 0u;
        fence_proxy_async_shared();
        if (c + ST < nch) issue(c + ST);
      }
    }
  }
  // Never leave a copy in flight (only a timed-out wait can leave one): every
  // chunk is issued by the time all are released; wait for the last ST.
  __device__ __forceinline__ void drain(int tid, int tmo) {
    if (tmo && tid == 0)
      for (int c = max(0, nch - ST); c < nch; ++c) mbar_wait_bounded(&full[c % ST], (c / ST) & 1, kRingWaitNs);
  }
  __device__ __forceinline__ uint4 vec(int c, int r, int tid) const {
    return *reinterpret_cast<const uint4*>(stage(c % ST, r) + tid * 16);
  }
};

// Roles of a unit: its p row (verify), its q row (draft, draft_next or guess).
template <typename TIn>
__device__ __forceinline__ void unit_rows(const Args& a, int b, int j, const TIn*& baseP, long long& rbP,
                                          const TIn*& baseQ, long long& rbQ) {
  const int K = a.K, V = a.V;
  baseP = nullptr;
  baseQ = nullptr;
  rbP = rbQ = 0;
  if (a.mode == kModeVerify) {
    baseP = static_cast<const TIn*>(a.target);
    rbP = (static_cast<long long>(b) * (K + 1) + j) * V;
    if (j < K) {
      baseQ = static_cast<const TIn*>(a.draft);
      rbQ = (static_cast<long long>(b) * K + j) * V;
    } else if (a.draft_next) {
      baseQ = static_cast<const TIn*>(a.draft_next);
      rbQ = static_cast<long long>(b) * V;
    }
  } else {
    if (j < K) {
      baseQ = static_cast<const TIn*>(a.draft);
      rbQ = (static_cast<long long>(b) * K + j) * V;
    } else {
      baseQ = static_cast<const TIn*>(a.guess);
      rbQ = static_cast<long long>(b) * a.guess_stride;
    }
  }
}

// The same plan on one warp: lane k holds F_k in f[0] and F_{k+32} in f[1].
// Lane k forms alpha^k by k rounded products, so every quota, remainder and
// tie equals the serial one; the repeated largest-remainder picks become a
// rank: a lane of rank r among the remainders (larger first, ties to the
// smaller k) gets rem / (K+1) + (r < rem % (K+1)) extra seats.
__device__ __forceinline__ void fanout_warp(float alpha_f, int K, int budget, int mode, int lane, int (&f)[2]) {
  const int n = K + 1;
  f[0] = f[1] = 0;
  if (mode == SSD_FANOUT_UNIFORM) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int k = lane + 32 * h;
      if (k < n) f[h] = budget / n + (k < budget % n ? 1 : 0);
    }
    return;
  }
  const double al = static_cast<double>(alpha_f);
  if (!(al >= 0.0 && al <= 1.0)) {
    if (lane == 0) f[0] = -1;
    return;
  }
  double frac[2] = {0.0, 0.0};
  int assigned = 0;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int k = lane + 32 * h;
    if (k < n) {
      double run = 1.0;
      for (int i = 0; i < k; ++i) run = __dmul_rn(run, al);
      const double P = k < K ? __dmul_rn(run, __dsub_rn(1.0, al)) : run;
      const double quota = __dmul_rn(static_cast<double>(budget), P);
      const double fl = floor(quota);
      f[h] = static_cast<int>(fl);
      frac[h] = __dsub_rn(quota, fl);
      assigned += f[h];
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) assigned += __shfl_xor_sync(0xFFFFFFFFu, assigned, o);
  const int rem = budget - assigned;
  if (rem <= 0) return;
  int rank[2] = {0, 0};
  for (int i = 0; i < n; ++i) {
    const double src = i < 32 ? frac[0] : frac[1];
    const double fi = __shfl_sync(0xFFFFFFFFu, src, i & 31);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int k = lane + 32 * h;
      if (k < n && i != k && (fi > frac[h] || (fi == frac[h] && i < k))) ++rank[h];
    }
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int k = lane + 32 * h;
    if (k < n) f[h] += rem / n + (rank[h] < rem % n ? 1 : 0);
  }
}

// The row's fan-out plan into shared memory, by one whole warp: F when
// given, else planned from alpha.  Callers check Σ F = budget, 0 <= F <= V.
__device__ __forceinline__ void load_plan(const Args& a, int b, int32_t* s_F, int lane) {
  const int n = a.K + 1;
  int f[2] = {0, 0};
  if (a.F) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int k = lane + 32 * h;
      if (k < n) f[h] = __ldg(a.F + static_cast<long long>(b) * n + k);
    }
  } else {
    const float al = a.fanout_mode == SSD_FANOUT_UNIFORM ? 0.f : __ldg(a.alpha + b);
    fanout_warp(al, a.K, a.budget, a.fanout_mode, lane, f);
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int k = lane + 32 * h;
    if (k < n) s_F[k] = f[h];
  }
}

// Shared memory of kernel 1.
struct Smem1 {
  uint64_t full[kStages];
  uint32_t rel[kStages];
  float wred[kWarps][4];
  int32_t wint[kWarps][2];
  float gmax[kMaxGroups];
  int32_t hist[256];
  int32_t s_F[SSD_MAX_K + 1];
  float tau, MP, SP, MQ, SQ, QS, bx;
  int32_t bi, argP, argQ, n_total, slow, tmo, n_raw, is_last, is_last_row, pad;
  int32_t Fj, seg_off, plan_bad, pskip, d_tok;
  uint32_t epoch0;
  float xdP, xdQ, xdP0, xdQ0;
  int32_t cand_off[kMaxSlices + 1];
  int32_t cnt[kMaxSlices];
};

// One statistics CTA: slice `slice` of unit (row b, position j).
template <typename TIn, bool kAligned, bool kGreedy, bool kEE>
__device__ __forceinline__ void stats_cta(const Args& a, int b, int j, int slice, int S, int chunk) {
  constexpr int VE = Elem<TIn>::VE;
  extern __shared__ __align__(128) unsigned char ring_buf[];
  __shared__ __align__(16) Smem1 sm;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int upr = a.units_per_row;
  const int K = a.K, V = a.V;
  const bool verify = a.mode == kModeVerify;
  const long long u = static_cast<long long>(b) * (K + 1) + j;

  const TIn *baseP, *baseQ;
  long long rbP, rbQ;
  unit_rows<TIn>(a, b, j, baseP, rbP, baseQ, rbQ);

  // ---- slice [e0, e1) of the rows, vectors of VE elements --------------------------
  const int e0 = slice * chunk;
  const int e1 = min(V, e0 + chunk);
  const int n = max(0, e1 - e0);
  const int nvec = (n + VE - 1) / VE;
  const int nch = (nvec + kStatsChunkVecs - 1) / kStatsChunkVecs;
  Ring<TIn, kStatsChunkVecs, kStatsStages, SSD_STATS_EVICT_FIRST != 0> ring;  // read once: first out of L2
  ring.buf = ring_buf;
  ring.full = sm.full;
  ring.rel = sm.rel;
  ring.e0 = e0;
  ring.nvec = nvec;
  ring.nch = nch;

  // Early-exit read schedule: the target row p_j (0 < j < K) is not read
  // once an earlier position of the row is known to be rejected (its unit's
  // tagged word says so).  Then k* < j, and the outcome does not depend on
  // p_j; the CTAs of position j are scheduled a lag of rows after those of
  // position j - 1 so that such rejections are often known in time.  The
  // draft row's first chunks are in flight while the words are read.
  bool pskip = false;
  const bool ee_unit = kEE && verify && j > 0 && j < K;
  if (ee_unit) {
    if constexpr (kAligned) {
      ring.row0 = baseP + rbP;
      ring.row1 = baseQ + rbQ;
      ring.nrows = 2;
      ring.init(tid);
    }
    if (warp == 0) {
      if (kAligned && lane == 0) ring.issue_first_row1();
      const uint32_t tag = *reinterpret_cast<volatile const uint32_t*>(a.epoch) + 1u;
      bool rej = false;
      if (lane < j) {
        const uint64_t w = ld_acquire_gpu_u64(a.uword + static_cast<long long>(b) * (K + 1) + lane);
        rej = static_cast<uint32_t>(w >> 32) == tag && ((w >> 16) & 1u) != 0;
      }
      rej = __any_sync(0xFFFFFFFFu, rej);
      if (kAligned && lane == 0) ring.issue_first_row0(!rej);
      if (lane == 0) sm.pskip = rej ? 1 : 0;
    }
    __syncthreads();
    pskip = sm.pskip != 0;
    if (pskip) {
      baseP = nullptr;
      ring.row0 = nullptr;
      if (tid == 0) atomicAdd(a.skipped, static_cast<unsigned long long>(n) * sizeof(TIn));
    }
  }
  const bool hasP = baseP != nullptr, hasQ = baseQ != nullptr;
  const bool srcQ = hasQ;  // the top-F source row: q_j, else p_j
  const bool has_d = verify && j < K;
  // Thread 0 requests the call's epoch (it cannot advance before every unit
  // of this call has published), the drafted token and, in the slice that
  // holds it, its two logits for the unit's accept test; they land in
  // shared memory while the first chunks are in flight, so the epilogue
  // needs no round trip for them.
  uint32_t epoch_ld = 0;
  int d_ld = -1;
  float xdP_ld = 0.f, xdQ_ld = 0.f;
  if (tid == 0) {
    epoch_ld = *reinterpret_cast<volatile const uint32_t*>(a.epoch);
    if (has_d) d_ld = __ldg(a.tokens + static_cast<long long>(b) * K + j);
    if (!kGreedy && has_d && hasP && d_ld >= e0 && d_ld < e1) {
      xdP_ld = Elem<TIn>::at(baseP + rbP, d_ld);
      xdQ_ld = Elem<TIn>::at(baseQ + rbQ, d_ld);
    }
  }
  // ring stage halves: an early-exit unit keeps p in half 0 and q in half 1
  // whether or not it reads p; otherwise the first row read takes half 0
  const int slotP = 0, slotQ = (hasP || ee_unit) ? 1 : 0;
  if (!ee_unit) {
    ring.row0 = hasP ? baseP + rbP : baseQ + rbQ;
    ring.row1 = baseQ + rbQ;
    ring.nrows = (hasP ? 1 : 0) + (hasQ ? 1 : 0);
    if constexpr (kAligned) ring.start(tid);
  }
  if (tid == 0) {
    sm.epoch0 = epoch_ld;
    sm.d_tok = d_ld;
    sm.xdP0 = xdP_ld;
    sm.xdQ0 = xdQ_ld;
  }

  const bool has_plan = a.F != nullptr || a.alpha != nullptr;
  // Warp 0 forms the plan now, while the first chunks are in flight (only the
  // epilogue reads it; the stream's first barrier publishes it).
  int fplan[2] = {0, 0};
  float alpha_in = 0.f;
  if (warp == 0 && has_plan) {
    if (a.F) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int k = lane + 32 * h;
        if (k <= K) fplan[h] = __ldg(a.F + static_cast<long long>(b) * (K + 1) + k);
      }
    } else if (a.fanout_mode != SSD_FANOUT_UNIFORM && lane == 0) {
      alpha_in = __ldg(a.alpha + b);
    }
    if (!a.F) fanout_warp(__shfl_sync(0xFFFFFFFFu, alpha_in, 0), K, a.budget, a.fanout_mode, lane, fplan);
    // the plan's checks (0 <= F <= V, sum = budget) and this unit's share
    long long sum = 0;
    int bad = 0, pre = 0, fj = 0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int k = lane + 32 * h;
      if (k <= K) {
        const int f = fplan[h];
        sm.s_F[k] = f;
        bad |= (f < 0 || f > V) ? 1 : 0;
        sum += f;
        if (k < j) pre += f;
        if (k == j) fj = f;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
    bad = __reduce_or_sync(0xFFFFFFFFu, bad);
    pre = static_cast<int>(__reduce_add_sync(0xFFFFFFFFu, static_cast<unsigned>(pre)));
    fj = static_cast<int>(__reduce_add_sync(0xFFFFFFFFu, static_cast<unsigned>(fj)));
    if (lane == 0) {
      const int pb = (bad || sum != a.budget) ? 1 : 0;
      sm.plan_bad = pb;
      sm.Fj = pb ? 0 : fj;
      sm.seg_off = pre;
    }
  }
  int flags = 0, d = -1;
  float u_self = 0.f;
  if (verify) {
    u_self = __ldg(a.uniforms + static_cast<long long>(b) * (K + 1) + j);
    if (!(u_self >= 0.f && u_self < 1.f)) flags |= SSD_ROW_BAD_UNIFORM;
  } else if (j < K && a.uniforms) {
    const float ud = __ldg(a.uniforms + static_cast<long long>(b) * K + j);
    if (!(ud >= 0.f && ud < 1.f)) flags |= SSD_ROW_BAD_UNIFORM;
  }
  const float cT = kGreedy ? 0.f : kLog2e / a.T;

  // ---- the stream: online max / exp-sum (or greedy argmax) of both rows ----------
  float mP = -INFINITY, sP = 0.f, nmP1 = 0.f, mQ = -INFINITY, sQ = 0.f, nmQ1 = 0.f;
  f32x2 sP2 = 0ull, sQ2 = 0ull, nmP2 = 0ull, nmQ2 = 0ull;  // packed (even, odd) sums and -m*c: bf16 path
  const f32x2 cT2 = f2_pack(cT, cT);
  int argP = INT_MAX, argQ = INT_MAX, nan_seen = 0, tmo = 0;
  float vm1 = -INFINITY, vm2 = -INFINITY, vm3 = -INFINITY;  // top three vector maxima of the source row
  int g1 = -1, g2 = -1;
  uint4 keep1 = make_uint4(0u, 0u, 0u, 0u), keep2 = keep1;  // the source vectors holding vm1, vm2
  auto track = [&](float vsrc, const uint4& wsrc, int g) {
    if (vsrc > vm3) {
      if (vsrc > vm2) {
        vm3 = vm2;
        if (vsrc > vm1) { vm2 = vm1; keep2 = keep1; g2 = g1; vm1 = vsrc; g1 = g; keep1 = wsrc; }
        else { vm2 = vsrc; g2 = g; keep2 = wsrc; }
      } else {
        vm3 = vsrc;
      }
    }
  };
  for (int c = 0; c < nch; ++c) {
    if constexpr (kAligned) ring.acquire(c, tid, tmo);
    if constexpr (kAligned && sizeof(TIn) == 2 && !kGreedy && kStatsVPT == 2) {
      // both of the thread's vectors of each row in one go: one rescale check
      // per row per stage
      const int g0 = c * kStatsChunkVecs + tid, g1v = g0 + kChunkVecs;
      const bool ok0 = g0 < nvec, ok1 = g1v < nvec;
      const uint4 neg = make_uint4(0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u);
      uint4 wp0 = neg, wp1 = neg, wq0 = neg, wq1 = neg;
      float vp0 = -INFINITY, vp1 = -INFINITY, vq0 = -INFINITY, vq1 = -INFINITY;
      if (hasP) {
        if (ok0) wp0 = ring.vec(c, slotP, tid);
        if (ok1) wp1 = ring.vec(c, slotP, tid + kChunkVecs);
        consume2_bf16(wp0, wp1, ok0, ok1, cT, cT2, mP, sP2, nmP2, vp0, vp1);
      }
      if (hasQ) {
        if (ok0) wq0 = ring.vec(c, slotQ, tid);
        if (ok1) wq1 = ring.vec(c, slotQ, tid + kChunkVecs);
        consume2_bf16(wq0, wq1, ok0, ok1, cT, cT2, mQ, sQ2, nmQ2, vq0, vq1);
      }
      if (ok0) track(srcQ ? vq0 : vp0, srcQ ? wq0 : wp0, g0);
      if (ok1) track(srcQ ? vq1 : vp1, srcQ ? wq1 : wp1, g1v);
    } else {
#pragma unroll
      for (int v = 0; v < kStatsVPT; ++v) {
        const int t = v * kChunkVecs + tid;  // the thread's vector within the chunk
        const int g = c * kStatsChunkVecs + t;
        if (g < nvec) {
          const int vbase = e0 + g * VE;
          float vsrc;
          uint4 wsrc = make_uint4(0u, 0u, 0u, 0u);
          if constexpr (kAligned && sizeof(TIn) == 2) {
            float vp = -INFINITY;
            uint4 wq = make_uint4(0u, 0u, 0u, 0u), wp = wq;
            if (hasP) { wp = ring.vec(c, slotP, t); vp = consume_bf16<kGreedy>(wp, vbase, cT, cT2, mP, sP2, nmP2, argP, nan_seen); }
            float vq = -INFINITY;
            if (hasQ) { wq = ring.vec(c, slotQ, t); vq = consume_bf16<kGreedy>(wq, vbase, cT, cT2, mQ, sQ2, nmQ2, argQ, nan_seen); }
            vsrc = srcQ ? vq : vp;
            wsrc = srcQ ? wq : wp;
          } else {
            float x[VE];
            float vp = -INFINITY, vq = -INFINITY;
            uint4 wp = make_uint4(0u, 0u, 0u, 0u), wq = wp;
            if (hasP) {
              if constexpr (kAligned) { wp = ring.vec(c, slotP, t); Elem<TIn>::unpack(wp, x); }
              else load_group<TIn, false>(baseP, rbP, vbase, e1, x);
              vp = consume_f<VE, kGreedy>(x, vbase, cT, mP, sP, nmP1, argP, nan_seen);
            }
            if (hasQ) {
              if constexpr (kAligned) { wq = ring.vec(c, slotQ, t); Elem<TIn>::unpack(wq, x); }
              else load_group<TIn, false>(baseQ, rbQ, vbase, e1, x);
              vq = consume_f<VE, kGreedy>(x, vbase, cT, mQ, sQ, nmQ1, argQ, nan_seen);
            }
            vsrc = srcQ ? vq : vp;
            wsrc = srcQ ? wq : wp;
          }
          track(vsrc, wsrc, g);
        }
      }
    }
    if constexpr (kAligned) ring.release(c, lane);
  }
  if constexpr (kGreedy) {
    if (nan_seen) { mP = __int_as_float(0x7FC00000); mQ = mP; }
  } else if constexpr (kAligned && sizeof(TIn) == 2) {
    float lo, hi;
    f2_unpack(sP2, lo, hi);
    sP = lo + hi;
    f2_unpack(sQ2, lo, hi);
    sQ = lo + hi;
  }
  sm.gmax[tid] = vm1;
  if (tid == 0) sm.n_raw = 0;

  // The ring is idle from here on: the candidate and merge buffers live in it.
  Cand* const raw = reinterpret_cast<Cand*>(ring_buf);
  Cand* const gbuf = raw + kCandCap;  // the unit's gathered candidates, then its sorted top-F

  // ---- slice reduction: butterfly within each warp, then over the warps ----------
  if constexpr (kGreedy) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      merge_arg(mP, argP, __shfl_xor_sync(0xFFFFFFFFu, mP, o), __shfl_xor_sync(0xFFFFFFFFu, argP, o));
      merge_arg(mQ, argQ, __shfl_xor_sync(0xFFFFFFFFu, mQ, o), __shfl_xor_sync(0xFFFFFFFFu, argQ, o));
    }
    if (lane == 0) {
      sm.wred[warp][0] = mP; sm.wred[warp][2] = mQ;
      sm.wint[warp][0] = argP; sm.wint[warp][1] = argQ;
    }
  } else {
    // the warp's maxima first, then every lane rescales its sum once to them
    float wmP = mP, wmQ = mQ;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      wmP = fmax_nan(wmP, __shfl_xor_sync(0xFFFFFFFFu, wmP, o));
      wmQ = fmax_nan(wmQ, __shfl_xor_sync(0xFFFFFFFFu, wmQ, o));
    }
    sP = (mP == -INFINITY) ? 0.f : sP * ex2((mP - wmP) * cT);
    sQ = (mQ == -INFINITY) ? 0.f : sQ * ex2((mQ - wmQ) * cT);
    mP = wmP;
    mQ = wmQ;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sP += __shfl_xor_sync(0xFFFFFFFFu, sP, o);
      sQ += __shfl_xor_sync(0xFFFFFFFFu, sQ, o);
    }
    if (lane == 0) {
      sm.wred[warp][0] = mP; sm.wred[warp][1] = sP;
      sm.wred[warp][2] = mQ; sm.wred[warp][3] = sQ;
    }
  }
  tmo = __syncthreads_or(tmo);
  if (has_d) {
    d = sm.d_tok;
    if (d < 0 || d >= V) flags |= SSD_ROW_BAD_TOKEN;
  }
  int Fj = 0, seg_off = 0, plan_bad = 0;
  if (has_plan) {
    plan_bad = sm.plan_bad;
    Fj = sm.Fj;
    seg_off = sm.seg_off;
  }
  if (plan_bad) flags |= SSD_ROW_BAD_PLAN;
  const bool want_topf = has_plan && Fj > 0;
  const bool fast_ok = want_topf && Fj <= kMaxGroups;
  SlicePart* part = a.parts + u * a.n_slices + slice;
  if (warp == 0) {
    float m1 = -INFINITY, s1 = 0.f, m2 = -INFINITY, s2 = 0.f;
    int a1 = INT_MAX, a2 = INT_MAX;
    if (lane < kWarps) {
      m1 = sm.wred[lane][0]; s1 = sm.wred[lane][1]; m2 = sm.wred[lane][2]; s2 = sm.wred[lane][3];
      if constexpr (kGreedy) { a1 = sm.wint[lane][0]; a2 = sm.wint[lane][1]; }
    }
#pragma unroll
    for (int o = kWarps / 2; o > 0; o >>= 1) {
      if constexpr (kGreedy) {
        merge_arg(m1, a1, __shfl_xor_sync(0xFFFFFFFFu, m1, o), __shfl_xor_sync(0xFFFFFFFFu, a1, o));
        merge_arg(m2, a2, __shfl_xor_sync(0xFFFFFFFFu, m2, o), __shfl_xor_sync(0xFFFFFFFFu, a2, o));
      } else {
        merge_ms(m1, s1, __shfl_xor_sync(0xFFFFFFFFu, m1, o), __shfl_xor_sync(0xFFFFFFFFu, s1, o), cT);
        merge_ms(m2, s2, __shfl_xor_sync(0xFFFFFFFFu, m2, o), __shfl_xor_sync(0xFFFFFFFFu, s2, o), cT);
      }
    }
    if (lane == 0) {
      part->mP = m1; part->sP = kGreedy ? 0.f : s1;
      part->mQ = m2; part->sQ = kGreedy ? 0.f : s2;
      part->argP = a1; part->argQ = a2;
      part->timeout = tmo;
      part->xdP = sm.xdP0; part->xdQ = sm.xdQ0;
      part->pskip = pskip ? 1 : 0;
    }
  } else if (warp == 1) {
    // This slice's threshold: the F-th largest of its thread maxima bounds the
    // slice's own top-F (hence its share of the unit's top-F) from below.
    float t = -INFINITY;
    if (fast_ok) {
      uint32_t keys[kMaxGroups / 32];
#pragma unroll
      for (int i = 0; i < kMaxGroups / 32; ++i) keys[i] = ord_key(sm.gmax[lane + 32 * i]);
      t = key_to_float(warp_kth_largest(keys, Fj, sizeof(TIn) == 2 ? 16 : 32));
    }
    if (lane == 0) sm.tau = t;
  }
  __syncthreads();
  const float tau = sm.tau;

  // Local candidates: the elements at or above tau.  A thread whose third
  // vector maximum is below tau holds them all in its two kept vectors.
  if (fast_ok && vm1 >= tau && vm1 == vm1) {
    if (kAligned && vm3 < tau) {
      float x[VE];
      Elem<TIn>::unpack(keep1, x);
#pragma unroll
      for (int i = 0; i < VE; ++i) {
        const int v = e0 + g1 * VE + i;
        if (x[i] >= tau && v < e1) {
          const int pos = atomicAdd(&sm.n_raw, 1);
          if (pos < kCandCap) raw[pos] = Cand{x[i], v};
        }
      }
      if (vm2 >= tau && g2 >= 0) {
        Elem<TIn>::unpack(keep2, x);
#pragma unroll
        for (int i = 0; i < VE; ++i) {
          const int v = e0 + g2 * VE + i;
          if (x[i] >= tau && v < e1) {
            const int pos = atomicAdd(&sm.n_raw, 1);
            if (pos < kCandCap) raw[pos] = Cand{x[i], v};
          }
        }
      }
    } else {
      const TIn* bs = srcQ ? baseQ : baseP;
      const long long rs = srcQ ? rbQ : rbP;
      for (int g = tid; g < nvec; g += kThreads) {
        {
          float x[VE];
          load_group<TIn, kAligned>(bs, rs, e0 + g * VE, e1, x);
#pragma unroll
          for (int i = 0; i < VE; ++i) {
            const int v = e0 + g * VE + i;
            if (x[i] >= tau && v < e1) {
              const int pos = atomicAdd(&sm.n_raw, 1);
              if (pos < kCandCap) raw[pos] = Cand{x[i], v};
            }
          }
        }
      }
    }
  }
  __syncthreads();
  {
    // Sort the local candidates; publish the first min(count, F) of them.
    const int nr = min(sm.n_raw, kCandCap);
    const int keepn = min(min(nr, Fj), kCandSlice);
    for (int i = tid; i < nr; i += kThreads) {
      const Cand ci = raw[i];
      const unsigned long long key = rank_key(ci.x, ci.idx);
      int r = 0;
      for (int k2 = 0; k2 < nr; ++k2) r += rank_key(raw[k2].x, raw[k2].idx) > key;
      if (r < keepn) part->cand[r] = ci;
    }
    if (tid == 0) part->n_cand = sm.n_raw;
  }
  __syncthreads();
  if constexpr (kAligned) ring.drain(tid, tmo);
  // The unit's last slice to arrive finalizes; the others leave.  Nobody
  // waits: the arrival is one acquire-release reduction per slice.
  if (tid == 0) sm.is_last = arrive_acq_rel_gpu(a.arrive1 + u) == S - 1 ? 1 : 0;
  __syncthreads();
  if (!sm.is_last) return;

  // =============== the unit's finalizer: its last slice, once all have arrived ======
  const SlicePart* parts = a.parts + u * a.n_slices;
  // Every slice's published candidates, loaded at once with the statistics
  // (slot c * cap + r holds candidate r of slice c; entries past a slice's
  // count are ignored).
  const int cap = min(Fj, kCandSlice);
  const bool one_round = fast_ok && S * cap <= kGatherCap;
  if (one_round && warp != 0) {
    for (int i = tid - 32; i < S * cap; i += kThreads - 32) {
      const Cand* src = &parts[i / cap].cand[i % cap];
      gbuf[i] = Cand{__ldcg(&src->x), __ldcg(&src->idx)};
    }
  }
  if (warp == 0) {
    // Butterfly over the slices (lanes >= S hold neutral values): bit-identical
    // results whichever CTA finalizes.
    float mp = -INFINITY, sp = 0.f, mq = -INFINITY, sq = 0.f;
    int ap = INT_MAX, aq = INT_MAX, nc = 0, to = 0, ps = 0;
    if (lane < S) {
      mp = __ldcg(&parts[lane].mP); sp = __ldcg(&parts[lane].sP);
      mq = __ldcg(&parts[lane].mQ); sq = __ldcg(&parts[lane].sQ);
      ap = __ldcg(&parts[lane].argP); aq = __ldcg(&parts[lane].argQ);
      nc = __ldcg(&parts[lane].n_cand); to = __ldcg(&parts[lane].timeout);
      ps = __ldcg(&parts[lane].pskip);
    }
    float xp = 0.f, xq = 0.f;
    if (!kGreedy && has_d && lane < S) {
      xp = __ldcg(&parts[lane].xdP);
      xq = __ldcg(&parts[lane].xdQ);
    }
    const int cd = (has_d && d >= 0 && d < V) ? d / chunk : 0;  // the slice holding d
    xp = __shfl_sync(0xFFFFFFFFu, xp, cd);
    xq = __shfl_sync(0xFFFFFFFFu, xq, cd);
    const int cnt = min(min(nc, Fj), kCandSlice);
#pragma unroll
    for (int o = kMaxSlices / 2; o > 0; o >>= 1) {
      if constexpr (kGreedy) {
        merge_arg(mp, ap, __shfl_xor_sync(0xFFFFFFFFu, mp, o), __shfl_xor_sync(0xFFFFFFFFu, ap, o));
        merge_arg(mq, aq, __shfl_xor_sync(0xFFFFFFFFu, mq, o), __shfl_xor_sync(0xFFFFFFFFu, aq, o));
      } else {
        merge_ms(mp, sp, __shfl_xor_sync(0xFFFFFFFFu, mp, o), __shfl_xor_sync(0xFFFFFFFFu, sp, o), cT);
        merge_ms(mq, sq, __shfl_xor_sync(0xFFFFFFFFu, mq, o), __shfl_xor_sync(0xFFFFFFFFu, sq, o), cT);
      }
    }
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += y;
    }
    const int total = __shfl_sync(0xFFFFFFFFu, incl, 31);
    const unsigned over = __ballot_sync(0xFFFFFFFFu, nc > kCandCap || (nc > kCandSlice && Fj > kCandSlice));
    const unsigned anyto = __ballot_sync(0xFFFFFFFFu, to != 0);
    const unsigned anyskip = __ballot_sync(0xFFFFFFFFu, ps != 0);
    if (lane < S) {
      sm.cand_off[lane] = incl - cnt;
      sm.cnt[lane] = cnt;
    }
    if (lane == 0) {
      sm.MP = mp; sm.SP = sp; sm.MQ = mq; sm.SQ = sq; sm.argP = ap; sm.argQ = aq;
      sm.xdP = xp; sm.xdQ = xq;
      sm.cand_off[S] = total;
      sm.n_total = total;
      sm.tmo = anyto ? 1 : 0;
      sm.slow = over || total > kGatherCap || total < Fj;
      sm.pskip = anyskip ? 1 : 0;
    }
  }
  __syncthreads();
  const float MP = sm.MP, MQ = sm.MQ, SP = sm.SP, SQ = sm.SQ;
  if (sm.tmo) flags |= kFlagTimeout;
  // Early exit: when a slice skipped p_j, position j lies past k* and its
  // accept test is not taken (a_j is not reported).
  const bool p_read = verify && sm.pskip == 0;
  // a non-finite target row and q'(d_j) = 0 are kept apart (pflags): with the
  // early-exit schedule the row counts them only up to k*
  int pflags = (p_read && !(MP > -INFINITY && MP < INFINITY)) ? SSD_ROW_NONFINITE : 0;
  if (hasQ && !(MQ > -INFINITY && MQ < INFINITY)) flags |= SSD_ROW_NONFINITE;
  const bool valid = ((flags | pflags) & SSD_ROW_INVALID) == 0;
  // the top-F set, Z and the cache segment depend on the source row only (q_j,
  // or p_K for segment K): a bad target row past k* must not void them
  const bool valid_src = ((flags | (srcQ ? 0 : pflags)) & SSD_ROW_INVALID) == 0;
  const bool slow = want_topf && valid_src && (!one_round || sm.slow != 0);
  Cand* sel = gbuf + kGatherCap;
  const float nmP = -MP * cT, nmQ = -MQ * cT;

  // ---- exact top-F: global ranks by binary search in the sorted slice lists --------
  if (want_topf && valid_src && !slow) {
    for (int i = tid; i < S * cap; i += kThreads) {
      const int c = i / cap, r0 = i - c * cap;
      if (r0 >= sm.cnt[c]) continue;
      const Cand ci = gbuf[i];
      const unsigned long long key = rank_key(ci.x, ci.idx);
      int r = r0;  // entries ahead of it in its own list
      for (int c2 = 0; c2 < S; ++c2) {
        if (c2 == c) continue;
        const int base = c2 * cap;
        int lo = base, hi = base + sm.cnt[c2];  // count keys > key (descending list)
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (rank_key(gbuf[mid].x, gbuf[mid].idx) > key) lo = mid + 1;
          else hi = mid;
        }
        r += lo - base;
      }
      if (r < Fj) sel[r] = ci;
    }
  }
  if (slow) {
    const TIn* row = srcQ ? baseQ + rbQ : baseP + rbP;
    topf_exact_global<TIn>(row, V, Fj, sel, sm.hist, tid, CtaBarrier{});
  }
  __syncthreads();

  // Q_S in a fixed order, and the top-F boundary.
  if (warp == 0) {
    float qs = 0.f;
    if (want_topf && valid_src) {
      if constexpr (!kGreedy) {
        for (int i = lane; i < Fj; i += 32) qs += ex2(fmaf(sel[i].x, cT, srcQ ? nmQ : nmP));
      }
    }
    qs = warp_sum(qs);
    if (lane == 0) {
      sm.QS = qs;
      sm.bx = (want_topf && valid_src) ? sel[Fj - 1].x : INFINITY;
      sm.bi = (want_topf && valid_src) ? sel[Fj - 1].idx : -1;
    }
  }
  __syncthreads();

  // ---- Saguaro normaliser and the accept test --------------------------------------
  const float C = a.C;
  float Z = 1.f;
  if (!kGreedy && want_topf && valid_src) Z = 1.f - (1.f - C) * (sm.QS / (srcQ ? SQ : SP));
  const float bx = sm.bx;
  const int bi = sm.bi;
  float acc = 0.f, amargin = INFINITY;
  int rejected = 0;
  if (has_d && valid && !p_read) {
    acc = __int_as_float(0x7FC00000);
    rejected = 1;
  } else if (has_d && valid) {
    if constexpr (kGreedy) {
      acc = (d == sm.argP) ? 1.f : 0.f;
      rejected = d != sm.argP;
    } else {
      const float xdP = sm.xdP, xdQ = sm.xdQ;
      const float pd = ex2(fmaf(xdP, cT, nmP)) / SP;
      const float qd = ex2(fmaf(xdQ, cT, nmQ)) / SQ;
      const bool inS = want_topf && (xdQ > bx || (xdQ == bx && d <= bi));
      const float qpd = (inS ? C : 1.f) * qd / Z;
      if (qpd > 0.f) {
        acc = fminf(1.f, pd / qpd);
      } else {
        acc = pd > 0.f ? 1.f : 0.f;
        pflags |= SSD_ROW_ZERO_Q;
      }
      rejected = !(u_self < acc);
      amargin = fabsf(u_self - acc);
    }
  }

  // ---- unit outputs ------------------------------------------------------------------
  int32_t* segdst = nullptr;
  if (verify) {
    if (a.c_tokens && !plan_bad) segdst = a.c_tokens + static_cast<long long>(b) * a.budget + seg_off;
  } else if (!plan_bad && a.topf_tokens) {
    segdst = a.topf_tokens + static_cast<long long>(b) * a.budget + seg_off;
  }
  if (segdst && has_plan)
    for (int i = tid; i < Fj; i += kThreads) segdst[i] = valid_src ? sel[i].idx : -1;
  if (tid == 0) {
    if (verify && j < K) a.accept_prob[static_cast<long long>(b) * K + j] = valid ? acc : __int_as_float(0x7FC00000);
    if (!verify && j < K) {
      const long long o = static_cast<long long>(b) * K + j;
      const float qlse = kGreedy ? MQ : (MQ * cT + log2f(SQ)) * 0.6931471805599453f;
      if (a.Z) a.Z[o] = valid ? Z : __int_as_float(0x7FC00000);
      if (a.q_lse) a.q_lse[o] = valid ? qlse : __int_as_float(0x7FC00000);
      if (a.draft_tokens && (!valid || !a.draws)) a.draft_tokens[o] = valid ? sm.argQ : -1;
    }
    UnitState st;
    st.MP = MP; st.SP = SP; st.MQ = MQ; st.SQ = SQ;
    st.Z = Z; st.bx = bx; st.a = acc; st.amargin = amargin;
    st.bi = bi; st.argP = sm.argP; st.argQ = sm.argQ; st.flags = flags | pflags;
    st.rejected = rejected; st.Fj = Fj; st.seg_off = seg_off; st.dmargin = INFINITY;
    a.ustate[u] = st;
    a.arrive1[u] = 0;
  }
  __syncthreads();
  if (verify) {
    // The unit's result in one tagged word: the draw CTAs of the row read the
    // row's K+1 words and take the decision themselves (k* = the first
    // rejected position), so no CTA here waits for the rest of the row.
    if (tid == 0) {
      const uint64_t tag = sm.epoch0 + 1u;
      const uint32_t lo = static_cast<uint32_t>(flags & 0xFF) | static_cast<uint32_t>(pflags & 0xFF) << 8 |
                          static_cast<uint32_t>(rejected ? 1 : 0) << 16 |
                          static_cast<uint32_t>(amargin < kNearTie ? 1 : 0) << 17;
      st_release_gpu_u64(a.uword + u, tag << 32 | lo);
    }
    return;
  }
  // Likewise per row: the last unit of the row to arrive decides.
  if (tid == 0) sm.is_last_row = arrive_acq_rel_gpu(a.row_arrive + b) == upr - 1 ? 1 : 0;
  __syncthreads();
  if (!sm.is_last_row) return;

  // =============== the row's decision: unit j = 0, once all units have arrived ======
  // One warp; lane k reads unit k's record (k = 32 only when K = 32), so the
  // whole row costs one round trip.
  if (warp == 0) {
    const UnitState* us = a.ustate + static_cast<long long>(b) * (K + 1);
    int fl = 0;
    if (lane < upr) fl |= __ldcg(&us[lane].flags);
    if (lane + 32 < upr) fl |= __ldcg(&us[lane + 32].flags);
    fl = static_cast<int>(__reduce_or_sync(0xFFFFFFFFu, static_cast<unsigned>(fl)));
    if (verify) {
      // k* = the first rejected position, else K
      const bool rej = lane < K && __ldcg(&us[lane].rejected) != 0;
      const float am_l = lane < K ? __ldcg(&us[lane].amargin) : INFINITY;
      RowState mine = {};
      if (lane < upr) {
        const UnitState* uk = us + lane;
        mine.Fj = __ldcg(&uk->Fj);
        mine.MP = __ldcg(&uk->MP); mine.SP = __ldcg(&uk->SP); mine.MQ = __ldcg(&uk->MQ); mine.SQ = __ldcg(&uk->SQ);
        mine.Z = __ldcg(&uk->Z); mine.bx = __ldcg(&uk->bx); mine.bi = __ldcg(&uk->bi); mine.argP = __ldcg(&uk->argP);
      }
      const unsigned rm = __ballot_sync(0xFFFFFFFFu, rej);
      const int kstar = rm ? __ffs(rm) - 1 : K;
      // the margins of the tests up to and including the first rejection
      float am = lane <= kstar ? am_l : INFINITY;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) am = fminf(am, __shfl_xor_sync(0xFFFFFFFFu, am, o));
      const int src = kstar & 31;
      RowState rs;
      rs.kstar = kstar;
      rs.flags = fl;
      rs.amargin = am;
      rs.Fj = __shfl_sync(0xFFFFFFFFu, mine.Fj, src);
      rs.MP = __shfl_sync(0xFFFFFFFFu, mine.MP, src); rs.SP = __shfl_sync(0xFFFFFFFFu, mine.SP, src);
      rs.MQ = __shfl_sync(0xFFFFFFFFu, mine.MQ, src); rs.SQ = __shfl_sync(0xFFFFFFFFu, mine.SQ, src);
      rs.Z = __shfl_sync(0xFFFFFFFFu, mine.Z, src); rs.bx = __shfl_sync(0xFFFFFFFFu, mine.bx, src);
      rs.bi = __shfl_sync(0xFFFFFFFFu, mine.bi, src); rs.argP = __shfl_sync(0xFFFFFFFFu, mine.argP, src);
      if (lane == 0) {
        if (kstar >= 32) {  // K = 32, every draft accepted: unit 32 is past the warp
          const UnitState* uk = us + kstar;
          rs.Fj = __ldcg(&uk->Fj);
          rs.MP = __ldcg(&uk->MP); rs.SP = __ldcg(&uk->SP); rs.MQ = __ldcg(&uk->MQ); rs.SQ = __ldcg(&uk->SQ);
          rs.Z = __ldcg(&uk->Z); rs.bx = __ldcg(&uk->bx); rs.bi = __ldcg(&uk->bi); rs.argP = __ldcg(&uk->argP);
        }
        a.rstate[b] = rs;
        const uint64_t tag = *reinterpret_cast<volatile uint32_t*>(a.epoch) + 1u;
        st_release_gpu_u64(a.rflag + b, tag << 32 | static_cast<uint64_t>(kstar) << 8 |
                                            static_cast<uint64_t>(fl & 0xFF));
      }
    } else if (lane == 0) {
      const bool pbad = (fl & SSD_ROW_BAD_PLAN) != 0;
      int off = 0;
      if (a.offsets) {
        a.offsets[static_cast<long long>(b) * (K + 2)] = 0;
        for (int k = 0; k <= K; ++k) {
          off += pbad ? 0 : sm.s_F[k];
          a.offsets[static_cast<long long>(b) * (K + 2) + k + 1] = off;
        }
      }
      if (!a.draws) a.status[b] = fl;
      else {
        RowState rs = {};
        rs.flags = fl;
        rs.amargin = INFINITY;
        a.rstate[b] = rs;
        const uint64_t tag = *reinterpret_cast<volatile uint32_t*>(a.epoch) + 1u;
        for (int k = 0; k < K; ++k)
          st_release_gpu_u64(a.rflag + static_cast<long long>(b) * K + k, tag << 32 | static_cast<uint64_t>(fl & 0xFF));
      }
    }
    if (lane == 0) a.row_arrive[b] = 0;
  }
}

// The early-exit order of the units: unit (b, j) has the key b for j = 0 and
// j = K, and b + j * lag for 0 < j < K; units are taken by (key, j), so the
// CTAs of position j come a lag of rows after those of position j - 1.
// One warp maps order index o to (b, j): a 32-way search for the key (the
// count of units below a key is monotone in the key), then the rank among
// the units of that key.
__device__ __noinline__ void lagged_unit_warp(int o, int B, int K, int lag, int lane, int& b, int& j) {
  auto below = [&](int c) {  // units whose key is below c
    long long cnt = 2LL * min(max(c, 0), B);
    for (int jj = 1; jj < K; ++jj) cnt += min(max(c - jj * lag, 0), B);
    return cnt;
  };
  auto off = [&](int jj) { return (jj == 0 || jj == K) ? 0 : jj * lag; };
  int lo = 0, hi = B + (K - 1) * lag;  // the key lies in [lo, hi); below(lo) <= o
  while (hi - lo > 1) {
    const int step = (hi - lo + 31) / 32;
    const int c = lo + step * lane;
    const unsigned ok = __ballot_sync(0xFFFFFFFFu, c < hi && below(c) <= o);
    const int last = 31 - __clz(ok);  // lane 0 (c = lo) always qualifies
    hi = min(hi, lo + step * (last + 1));
    lo += step * last;
  }
  const int r = static_cast<int>(o - below(lo));
  const int bb = lo - off(lane);
  const unsigned has = __ballot_sync(0xFFFFFFFFu, lane <= K && bb >= 0 && bb < B);
  if (r < __popc(has)) {  // the lane holding the r-th unit of the key
    const bool mine = ((has >> lane) & 1u) && __popc(has & ((1u << lane) - 1u)) == r;
    j = __ffs(__ballot_sync(0xFFFFFFFFu, mine)) - 1;
  } else {
    j = 32;  // K = 32: unit 32 sits past the warp's lanes, at key b
  }
  b = lo - off(j);
}

// Kernel 1 of the two-kernel form (the draft side's ssd_saguaro_reweight):
// one CTA per (unit, slice), rows in order so that rows are decided one
// after another.
template <typename TIn, bool kAligned, bool kGreedy, bool kEE>
__global__ void __launch_bounds__(kThreads, kMinBlocks) ssd_stats_kernel(const __grid_constant__ Args a) {
  const int S = a.n_slices;
  const int order = blockIdx.x / S, slice = blockIdx.x % S;
  const int upr = a.units_per_row;
  int b = order / upr, j = order % upr;
  if constexpr (kEE) {
    __shared__ int s_unit[2];
    if (threadIdx.x < 32) {
      int bb, jj;
      lagged_unit_warp(order, a.B, a.K, a.lag, static_cast<int>(threadIdx.x), bb, jj);
      if (threadIdx.x == 0) {
        s_unit[0] = bb;
        s_unit[1] = jj;
      }
    }
    __syncthreads();
    b = s_unit[0];
    j = s_unit[1];
  } else if (a.k_last) {
    // positions j < K of every row first (row by row), then every row's
    // unit K: a row's k* is fixed by its positions up to the first rejection,
    // so most rows are drawn while the short unit-K CTAs (one row each) still
    // stream (the host asks for it when those CTAs fit one wave)
    const int nfirst = a.B * a.K;
    if (order < nfirst) {
      b = order / a.K;
      j = order % a.K;
    } else {
      b = order - nfirst;
      j = a.K;
    }
  }
  // kernel 2 may be scheduled once every CTA of this grid has started; it
  // waits for each of its units' records on its own
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  stats_cta<TIn, kAligned, kGreedy, kEE>(a, b, j, slice, S, a.chunk);
}

// Shared memory of kernel 2.
struct Smem2 {
  uint64_t full[kStages];
  uint32_t rel[kStages];
  int32_t dep_ok, w_kstar, w_flags, w_final, w_flags_all;
  float rs[kMaxChunks][kWarps];
  float ps[kMaxChunks][kWarps];
  int32_t s_F[SSD_MAX_K + 1];
  float tl, total, margin, myR, myRP;
  int32_t cstar, use_p, drawn, is_last, is_last_row, slot, tmo, all_in, own;
};

// The draw's mass at the 8 tokens of one bf16 vector (of p and/or q), token
// v0 first.  The arithmetic of each token is draw_vals' scalar form, two
// tokens per packed instruction; the Saguaro set test runs only for a vector
// whose largest draft logit reaches the set's boundary logit bx.
__device__ __forceinline__ void draw_vals_bf16(int draw, uint4 wp, uint4 wq, int v0, float cT, float nmP, float nmQ,
                                               float invSP, float wS, float wN, bool check_S, float bx, int bi,
                                               bool use_p, float (&val)[8], float (&pv)[8]) {
  const f32x2 c2 = f2_pack(cT, cT);
  const uint32_t wpw[4] = {wp.x, wp.y, wp.z, wp.w};
  const uint32_t wqw[4] = {wq.x, wq.y, wq.z, wq.w};
  float pp[8], qq[8];
  if (draw != kDrawQ) {
    const f32x2 n2 = f2_pack(nmP, nmP), s2 = f2_pack(invSP, invSP);
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      float a0, a1;
      f2_unpack(f2_fma(f2_pack(bf16_lo(wpw[h]), bf16_hi(wpw[h])), c2, n2), a0, a1);
      f2_unpack(f2_mul(f2_pack(ex2(a0), ex2(a1)), s2), pp[2 * h], pp[2 * h + 1]);
    }
  }
  if (draw != kDrawP) {
    bool anyS = false;
    if (check_S) {
      const uint32_t m2 = bf16x2_max_nan(bf16x2_max_nan(wq.x, wq.y), bf16x2_max_nan(wq.z, wq.w));
      anyS = fmax_nan(bf16_lo(m2), bf16_hi(m2)) >= bx;
    }
    const f32x2 n2 = f2_pack(nmQ, nmQ);
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const float x0 = bf16_lo(wqw[h]), x1 = bf16_hi(wqw[h]);
      float w0 = wN, w1 = wN;
      if (anyS) {
        const int v = v0 + 2 * h;
        if (x0 > bx || (x0 == bx && v <= bi)) w0 = wS;
        if (x1 > bx || (x1 == bx && v + 1 <= bi)) w1 = wS;
      }
      float a0, a1;
      f2_unpack(f2_fma(f2_pack(x0, x1), c2, n2), a0, a1);
      f2_unpack(f2_mul(f2_pack(ex2(a0), ex2(a1)), f2_pack(w0, w1)), qq[2 * h], qq[2 * h + 1]);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (draw == kDrawResidual) {
      val[i] = use_p ? pp[i] : fmaxf(pp[i] - qq[i], 0.f);
      pv[i] = pp[i];
    } else if (draw == kDrawP) {
      val[i] = pp[i];
      pv[i] = 0.f;
    } else {
      val[i] = qq[i];
      pv[i] = 0.f;
    }
  }
}

// The draw's mass at VE consecutive tokens of vector g of slice [e0, e1).
template <typename TIn, bool kAligned>
__device__ __forceinline__ void draw_vals(int draw, const TIn* baseP, long long rbP, const TIn* baseQ, long long rbQ,
                                          int e0, int e1, int g, const uint4* wp_ring, const uint4* wq_ring,
                                          float cT, float nmP, float nmQ, float invSP, float wS, float wN, bool check_S,
                                          float bx, int bi, bool use_p, float (&val)[Elem<TIn>::VE],
                                          float (&pv)[Elem<TIn>::VE]) {
  constexpr int VE = Elem<TIn>::VE;
  if constexpr (kAligned && sizeof(TIn) == 2) {
    uint4 wp = make_uint4(0u, 0u, 0u, 0u), wq = wp;
    if (draw != kDrawQ) wp = wp_ring ? *wp_ring : ld_vec(baseP + rbP + e0 + g * VE);
    if (draw != kDrawP) wq = wq_ring ? *wq_ring : ld_vec(baseQ + rbQ + e0 + g * VE);
    draw_vals_bf16(draw, wp, wq, e0 + g * VE, cT, nmP, nmQ, invSP, wS, wN, check_S, bx, bi, use_p, val, pv);
    return;
  }
  float xp[VE], xq[VE];
  if (draw != kDrawQ) {
    if (wp_ring) Elem<TIn>::unpack(*wp_ring, xp);
    else load_group<TIn, kAligned>(baseP, rbP, e0 + g * VE, e1, xp);
  }
  if (draw != kDrawP) {
    if (wq_ring) Elem<TIn>::unpack(*wq_ring, xq);
    else load_group<TIn, kAligned>(baseQ, rbQ, e0 + g * VE, e1, xq);
  }
#pragma unroll
  for (int i = 0; i < VE; ++i) {
    float wq = wN;
    if (check_S) {
      const int v = e0 + g * VE + i;
      if (xq[i] > bx || (xq[i] == bx && v <= bi)) wq = wS;
    }
    if (draw == kDrawResidual) {
      const float pp = ex2(fmaf(xp[i], cT, nmP)) * invSP;
      val[i] = use_p ? pp : fmaxf(pp - ex2(fmaf(xq[i], cT, nmQ)) * wq, 0.f);
      pv[i] = pp;
    } else if (draw == kDrawP) {
      val[i] = ex2(fmaf(xp[i], cT, nmP)) * invSP;
      pv[i] = 0.f;
    } else {
      val[i] = ex2(fmaf(xq[i], cT, nmQ)) * wq;
      pv[i] = 0.f;
    }
  }
}

// One draw CTA: slice `slice` of draw unit du (verify: row du; reweight:
// position du % K of row du / K).
template <typename TIn, bool kAligned, bool kGreedy>
__device__ __forceinline__ void draw_cta(const Args& a, int du, int slice) {
  constexpr int VE = Elem<TIn>::VE;
  extern __shared__ __align__(128) unsigned char ring_buf[];
  __shared__ __align__(16) Smem2 sm;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = a.d_slices;
  const int K = a.K, V = a.V;
  const bool verify = a.mode == kModeVerify;

  // ---- the row decision this CTA needs (kernel 1 may still be running) -------------
  if (verify) {
    // Lane k polls unit k's tagged word (lane 0 also unit 32's when K = 32).
    // k* is fixed as soon as the words of positions 0..j are in with j the
    // first rejected one (or all K+1 words are in, none rejected): the stream
    // of unit k* starts then, and the words past k* are awaited only before
    // the row's flags are written (finish_row).
    if (warp == 0) {
      const uint32_t tag = *reinterpret_cast<volatile const uint32_t*>(a.epoch) + 1u;
      const int upr = K + 1;
      const uint64_t* uw = a.uword + static_cast<long long>(du) * upr;
      uint64_t w0 = 0, w1 = 0;
      bool have0 = lane >= upr, have1 = lane + 32 >= upr;
      int kstar = -1;
      const unsigned long long t0 = global_ns();
      uint32_t sleep_ns = 32;
      for (uint32_t it = 0; it < 50000000u; ++it) {
        if (!have0) {
          const uint64_t v = ld_acquire_gpu_u64(uw + lane);
          if (static_cast<uint32_t>(v >> 32) == tag) { w0 = v; have0 = true; }
        }
        if (!have1) {
          const uint64_t v = ld_acquire_gpu_u64(uw + lane + 32);
          if (static_cast<uint32_t>(v >> 32) == tag) { w1 = v; have1 = true; }
        }
        const unsigned pres = __ballot_sync(0xFFFFFFFFu, have0);
        const unsigned rm = __ballot_sync(0xFFFFFFFFu, have0 && lane < K && ((static_cast<uint32_t>(w0) >> 16) & 1u));
        const bool all1 = __all_sync(0xFFFFFFFFu, have1);
        if (rm) {
          const int js = __ffs(rm) - 1;
          const unsigned below = (1u << js) - 1u;
          if ((pres & below) == below) { kstar = js; break; }
        } else if (pres == 0xFFFFFFFFu && all1) {
          kstar = K;
          break;
        }
        if (global_ns() - t0 > kDepWaitNs) break;
        __nanosleep(sleep_ns);
        if (sleep_ns < 128u) sleep_ns <<= 1;
      }
      const bool ok = kstar >= 0;
      // flags of the units 0..k* only (every CTA of the row has read the
      // same words up to k*, so all take the same stream decision); the
      // flags past k* are added in finish_row
      const uint32_t lo0 = (have0 && lane <= kstar) ? static_cast<uint32_t>(w0) : 0u;
      const uint32_t lo1 = (have1 && lane + 32 <= kstar) ? static_cast<uint32_t>(w1) : 0u;
      uint32_t f = ((lo0 | lo1) & 0xFFu) | ((lo0 >> 8) & 0xFFu) | ((lo1 >> 8) & 0xFFu);
      if ((lo0 >> 17) & 1u) f |= SSD_ROW_NEAR_TIE;
      f = __reduce_or_sync(0xFFFFFFFFu, f);
      // when every word was already in, the row's final flags too (as
      // finish_row would form them), so the finishing CTA need not read again
      const bool all_in = __all_sync(0xFFFFFFFFu, have0 && have1);
      const uint32_t a0 = static_cast<uint32_t>(w0), a1 = static_cast<uint32_t>(w1);
      uint32_t ff = (a0 | a1) & 0xFFu;
      if (!a.early_exit || lane <= kstar || lane == K) ff |= (a0 >> 8) & 0xFFu;
      ff |= (a1 >> 8) & 0xFFu;
      if (lane <= kstar && ((a0 >> 17) & 1u)) ff |= SSD_ROW_NEAR_TIE;
      ff = __reduce_or_sync(0xFFFFFFFFu, ff);
      if (lane == 0) {
        sm.dep_ok = ok ? 1 : 0;
        if (!ok) atomicExch(a.error, 1);
        sm.w_kstar = ok ? kstar : K;
        sm.w_flags = static_cast<int32_t>(f);
        sm.w_final = (ok && all_in) ? 1 : 0;
        sm.w_flags_all = static_cast<int32_t>(ff);
      }
    }
  } else if (tid == 0) {
    const uint32_t epoch = *reinterpret_cast<volatile const uint32_t*>(a.epoch);
    uint64_t word = 0;
    sm.dep_ok = wait_tagged(a.rflag + du, epoch + 1u, kDepWaitNs, &word) ? 1 : 0;
    if (!sm.dep_ok) atomicExch(a.error, 1);
    sm.w_kstar = static_cast<int32_t>((word >> 8) & 0xFF);
    sm.w_flags = static_cast<int32_t>(word & 0xFF);
  }
  // The row's fan-out plan depends on the inputs only: form it while the
  // decision is awaited.
  if (warp == 1 && (a.F != nullptr || a.alpha != nullptr)) load_plan(a, verify ? du : du / K, sm.s_F, lane);
  __syncthreads();
  const bool dep_ok = sm.dep_ok != 0;
  // Every CTA has read the epoch above; the last CTA of the grid to leave
  // advances it for the next call.  Counted at each CTA's exit (thread 0), so
  // the round trip never delays the stream.
  auto leave = [&]() {
    if (tid == 0 && atomicAdd(a.k2_done, 1) == static_cast<int>(gridDim.x) - 1) {
      *a.k2_done = 0;
      __threadfence();
      atomicAdd(a.epoch, 1u);
    }
  };

  // ---- which unit this row (or draft position) draws from ----------------------------
  int b, j, rowflags = 0, draw;
  float amargin = INFINITY;
  UnitState st;
  if (verify) {
    // k* and the row's flags came with the decision word: the stream can start
    // before the row's statistics are read
    b = du;
    j = sm.w_kstar;
    rowflags = sm.w_flags;
    if (!dep_ok || j < 0 || j > K) {  // the decision never came: a timed-out row
      j = K;
      rowflags = kFlagTimeout;
    }
    draw = j < K ? kDrawResidual : kDrawP;
  } else {
    b = du / K;
    j = du % K;
    draw = kDrawQ;
    const UnitState* us = a.ustate + static_cast<long long>(b) * (K + 1) + j;
    st.MQ = __ldcg(&us->MQ); st.SQ = __ldcg(&us->SQ); st.Z = __ldcg(&us->Z); st.bx = __ldcg(&us->bx);
    st.bi = __ldcg(&us->bi); st.argQ = __ldcg(&us->argQ); st.Fj = __ldcg(&us->Fj);
    st.flags = __ldcg(&us->flags) | (dep_ok ? 0 : kFlagTimeout);
    st.MP = 0.f; st.SP = 1.f; st.argP = 0;
  }
  const long long u = static_cast<long long>(b) * (K + 1) + j;
  const bool row_invalid = verify ? (rowflags & SSD_ROW_INVALID) != 0 : (st.flags & SSD_ROW_INVALID) != 0;
  const bool streams = !kGreedy && !row_invalid;
  if (!streams && slice != 0) {
    leave();
    return;
  }

  const TIn *baseP, *baseQ;
  long long rbP, rbQ;
  unit_rows<TIn>(a, b, j, baseP, rbP, baseQ, rbQ);
  if (draw == kDrawP) baseQ = nullptr;  // the full-acceptance draw reads p_K only
  const int e0 = slice * a.d_chunk;
  const int e1 = min(V, e0 + a.d_chunk);
  const int n = max(0, e1 - e0);
  const int nvec = (n + VE - 1) / VE;
  const int nch = (nvec + kChunkVecs - 1) / kChunkVecs;
  const bool useP = draw != kDrawQ, useQ = draw != kDrawP;
  Ring<TIn> ring;
  ring.buf = ring_buf;
  ring.full = sm.full;
  ring.rel = sm.rel;
  ring.row0 = useP ? baseP + rbP : baseQ + rbQ;
  ring.row1 = useQ ? baseQ + rbQ : nullptr;
  ring.nrows = (useP ? 1 : 0) + (useQ ? 1 : 0);
  ring.e0 = e0;
  ring.nvec = nvec;
  ring.nch = nch;
  const int slotP = 0, slotQ = useP ? 1 : 0;
  if (kAligned && streams) ring.start(tid);
  if (verify) {  // the statistics of unit k*, while the first chunks are in flight
    const UnitState* us = a.ustate + static_cast<long long>(b) * (K + 1) + j;
    st.MP = __ldcg(&us->MP); st.SP = __ldcg(&us->SP); st.MQ = __ldcg(&us->MQ); st.SQ = __ldcg(&us->SQ);
    st.Z = __ldcg(&us->Z); st.bx = __ldcg(&us->bx); st.bi = __ldcg(&us->bi); st.argP = __ldcg(&us->argP);
    st.argQ = 0;
    st.Fj = __ldcg(&us->Fj);
    st.flags = rowflags;
  }

  const float cT = kGreedy ? 0.f : kLog2e / a.T;
  const float C = a.C;
  const float nmP = -st.MP * cT, nmQ = -st.MQ * cT;
  const float invSP = 1.f / st.SP;
  const float wS = C / (st.SQ * st.Z), wN = 1.f / (st.SQ * st.Z);
  const bool check_S = st.Fj > 0 && draw != kDrawP;
  const float u_draw = verify ? __ldg(a.uniforms + static_cast<long long>(b) * (K + 1) + K)
                              : __ldg(a.uniforms + static_cast<long long>(b) * K + j);
  int tmo = 0;
  DrawPart* dparts = a.dparts + static_cast<long long>(du) * S;
  int32_t seg_tok0 = -1, seg_tok1 = -1;  // the last slice: cache segment k*, prefetched
  bool late_claim = false;   // resident draw: the crossing CTA claims the row after writing it
  uint32_t claim_tag = 0;

  if (streams) {
    // ---- this slice's mass per (chunk, warp), in token order ------------------------
    for (int c = 0; c < nch; ++c) {
      if constexpr (kAligned) ring.acquire(c, tid, tmo);
      const int g = c * kChunkVecs + tid;
      float rsum = 0.f, psum = 0.f;
      if (g < nvec) {
        float val[VE], pv[VE];
        uint4 wp, wq;
        if constexpr (kAligned) {
          if (useP) wp = ring.vec(c, slotP, tid);
          if (useQ) wq = ring.vec(c, slotQ, tid);
        }
        draw_vals<TIn, kAligned>(draw, baseP, rbP, baseQ, rbQ, e0, e1, g, kAligned ? &wp : nullptr,
                                 kAligned ? &wq : nullptr, cT, nmP, nmQ, invSP, wS, wN, check_S, st.bx, st.bi,
                                 false, val, pv);
#pragma unroll
        for (int i = 0; i < VE; ++i) { rsum += val[i]; psum += pv[i]; }
      }
      rsum = warp_sum(rsum);
      psum = warp_sum(psum);
      if (lane == 0) { sm.rs[c][warp] = rsum; sm.ps[c][warp] = psum; }
      if constexpr (kAligned) ring.release(c, lane);
    }
    tmo = __syncthreads_or(tmo);
    // A slice that never wrapped the ring is still whole in shared memory:
    // its CTA finds the row's crossing there, with no second read.
    const bool resident = kAligned && nch <= kStages;
    if (warp == 0) {  // the slice's masses: lane l sums entries l, l + 32, ... then a butterfly
      float R = 0.f, RP = 0.f;
      for (int i = lane; i < nch * kWarps; i += 32) { R += sm.rs[i / kWarps][i % kWarps]; RP += sm.ps[i / kWarps][i % kWarps]; }
      R = warp_sum(R);
      RP = warp_sum(RP);
      if (lane == 0) {
        dparts[slice].R = R;
        dparts[slice].RP = RP;
        dparts[slice].timeout = tmo;
        sm.myR = tmo ? __int_as_float(0x7FC00000) : R;
        sm.myRP = RP;
      }
    }
    if (!resident) {
      for (int i = tid; i < nch * kWarps; i += kThreads) {
        dparts[slice].rs[i / kWarps][i % kWarps] = sm.rs[i / kWarps][i % kWarps];
        dparts[slice].ps[i / kWarps][i % kWarps] = sm.ps[i / kWarps][i % kWarps];
      }
    }
    // the row's cache segment k*, for the lookup (prefetched by every CTA
    // that may finish the row)
    if (verify && a.c_tokens && !row_invalid) {
      int off = 0;
      for (int k = 0; k < j; ++k) off += sm.s_F[k];
      const int32_t* seg = a.c_tokens + static_cast<long long>(b) * a.budget + off;
      const int Fk = sm.s_F[j];
      if (tid < Fk) seg_tok0 = __ldcg(seg + tid);
      if (tid + kThreads < Fk) seg_tok1 = __ldcg(seg + tid + kThreads);
    }
    __syncthreads();
    if constexpr (kAligned) ring.drain(tid, tmo);

    // Warp 0: the row's total and the slice where the cumulative mass crosses
    // u * total (the first with prefix + part > t, else the last with mass).
    auto find_slice = [&]() {
      float rp = 0.f, pp = 0.f;
      int to = 0;
      if (lane < S) {
        rp = __ldcg(&dparts[lane].R);
        pp = __ldcg(&dparts[lane].RP);
        to = __ldcg(&dparts[lane].timeout);
      }
      float R = 0.f, RP = 0.f;
      for (int c = 0; c < S; ++c) {
        R += __shfl_sync(0xFFFFFFFFu, rp, c);
        RP += __shfl_sync(0xFFFFFFFFu, pp, c);
      }
      const int use_p = (draw == kDrawResidual && !(R > 0.f)) ? 1 : 0;
      const float total = use_p ? RP : R;
      const float t = u_draw * total;
      float run = 0.f, pre = 0.f, prelast = 0.f;
      int cstar = -1, clast = 0;
      for (int c = 0; c < S; ++c) {
        const float part = __shfl_sync(0xFFFFFFFFu, use_p ? pp : rp, c);
        if (part > 0.f) { clast = c; prelast = run; }
        if (cstar < 0 && run + part > t) { cstar = c; pre = run; }
        run += part;
      }
      if (cstar < 0) { cstar = clast; pre = prelast; }
      const unsigned anyto = __ballot_sync(0xFFFFFFFFu, to != 0);
      if (lane == 0) {
        sm.cstar = cstar;
        sm.tl = t - pre;
        sm.total = total;
        sm.use_p = use_p;
        sm.tmo = anyto ? 1 : 0;
      }
    };
    // Warp 0, within slice s_star: chunk, warp, lane and token of the
    // crossing, from that slice's (chunk, warp) sums Ls; the lane level reads
    // the crossing warp-chunk from the ring (resident) or again from memory.
    auto scan_slice = [&](const float* Ls, bool from_ring) {
      const int s_star = sm.cstar;
      const bool use_p = sm.use_p != 0;
      const int e0s = s_star * a.d_chunk;
      const int e1s = min(V, e0s + a.d_chunk);
      const int nvs = (max(0, e1s - e0s) + VE - 1) / VE;
      const int nchs = (nvs + kChunkVecs - 1) / kChunkVecs;
      const float tl = sm.tl;
      // chunk level: lane c holds chunk c's total
      float my = 0.f;
      if (lane < nchs) {
        for (int w = 0; w < kWarps; ++w) my += Ls[lane * kWarps + w];
      }
      float run = 0.f, pre_k = 0.f, pre_last = 0.f;
      int k_star = -1, k_last = 0;
      for (int c = 0; c < nchs; ++c) {
        const float tk = __shfl_sync(0xFFFFFFFFu, my, c);
        if (tk > 0.f) { k_last = c; pre_last = run; }
        if (k_star < 0 && run + tk > tl) { k_star = c; pre_k = run; }
        run += tk;
      }
      if (k_star < 0) { k_star = k_last; pre_k = pre_last; }
      const float tl2 = tl - pre_k;
      float mw = 0.f;
      if (lane < kWarps) mw = Ls[k_star * kWarps + lane];
      run = 0.f;
      float pre_w = 0.f;
      pre_last = 0.f;
      int w_star = -1, w_last = 0;
      for (int w = 0; w < kWarps; ++w) {
        const float tw = __shfl_sync(0xFFFFFFFFu, mw, w);
        if (tw > 0.f) { w_last = w; pre_last = run; }
        if (w_star < 0 && run + tw > tl2) { w_star = w; pre_w = run; }
        run += tw;
      }
      if (w_star < 0) { w_star = w_last; pre_w = pre_last; }
      const float tl3 = tl2 - pre_w;
      // lane level: the 32 vectors of that warp in that chunk
      const int g = k_star * kChunkVecs + w_star * 32 + lane;
      float val[VE], pv[VE];
      if (g < nvs) {
        const uint4* rp = nullptr;
        const uint4* rq = nullptr;
        if (from_ring) {
          if (useP) rp = reinterpret_cast<const uint4*>(ring.stage(k_star % kStages, slotP) + (w_star * 32 + lane) * 16);
          if (useQ) rq = reinterpret_cast<const uint4*>(ring.stage(k_star % kStages, slotQ) + (w_star * 32 + lane) * 16);
        }
        draw_vals<TIn, kAligned>(draw, baseP, rbP, baseQ, rbQ, e0s, e1s, g, rp, rq, cT, nmP, nmQ, invSP, wS, wN,
                                 check_S, st.bx, st.bi, use_p, val, pv);
      } else {
#pragma unroll
        for (int i = 0; i < VE; ++i) val[i] = 0.f;
      }
      float ls = 0.f;
#pragma unroll
      for (int i = 0; i < VE; ++i) ls += val[i];
      float incl = ls;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
      }
      const unsigned cross = __ballot_sync(0xFFFFFFFFu, incl > tl3);
      const unsigned pos = __ballot_sync(0xFFFFFFFFu, ls > 0.f);
      const int l_star = cross ? (__ffs(cross) - 1) : (pos ? (31 - __clz(pos)) : 0);
      if (lane == l_star) {
        const float tl4 = tl3 - (incl - ls);
        float run4 = 0.f, c_prev = 0.f, c_prev_last = 0.f;
        int i_star = -1, i_last = 0;
        for (int i = 0; i < VE; ++i) {
          if (val[i] > 0.f) { i_last = i; c_prev_last = run4; }
          if (i_star < 0 && run4 + val[i] > tl4) { i_star = i; c_prev = run4; }
          run4 += val[i];
        }
        if (i_star < 0) { i_star = i_last; c_prev = c_prev_last; }
        const int v = e0s + g * VE + i_star;
        const float lo = tl4 - c_prev;                // t - CDF before v
        const float hi = c_prev + val[i_star] - tl4;  // CDF at v - t
        sm.drawn = min(max(v, 0), V - 1);
        sm.margin = fminf(fabsf(lo), fabsf(hi)) / sm.total;
      }
    };

    if (resident) {
      // Each slice publishes its mass in one tagged word, (epoch + 1) << 32 |
      // bits(R) (NaN when its copies timed out); every slice of the row polls
      // all S words (bounded), so all find the same crossing slice at once,
      // and its CTA, which still holds the slice, finishes the row.  A CTA
      // whose poll gives up may finish the row instead, as a timed-out row;
      // an atomic maximum with the call's tag on the row's owner word lets
      // exactly one CTA write the row.
      const uint32_t tag = *reinterpret_cast<volatile const uint32_t*>(a.epoch) + 1u;
      uint64_t* const dtot = a.dtot + static_cast<long long>(du) * 2 * S;
      if (warp == 0) {
        // the two words carry everything the others read (no release needed):
        // this slice's residual mass, and its mass of p for a zero residual
        if (lane == 0) {
          st_relaxed_gpu_u64(dtot + slice, static_cast<uint64_t>(tag) << 32 | __float_as_uint(sm.myR));
          st_relaxed_gpu_u64(dtot + S + slice, static_cast<uint64_t>(tag) << 32 | __float_as_uint(sm.myRP));
        }
        uint64_t wv = 0;
        bool ok = true;
        if (lane < S) ok = wait_tagged(dtot + lane, tag, kDepWaitNs, &wv, 64u);
        const bool all_ok = __all_sync(0xFFFFFFFFu, ok);
        if (all_ok) {
          const float rp = lane < S ? __uint_as_float(static_cast<uint32_t>(wv)) : 0.f;
          float R = 0.f;
          for (int c = 0; c < S; ++c) R += __shfl_sync(0xFFFFFFFFu, rp, c);
          const int use_p = (draw == kDrawResidual && !(R > 0.f) && R == R) ? 1 : 0;
          float pp = 0.f;
          if (use_p) {  // rare: the row's residual is 0
            uint64_t wp = 0;
            if (lane < S && wait_tagged(dtot + S + lane, tag, kDepWaitNs, &wp, 64u))
              pp = __uint_as_float(static_cast<uint32_t>(wp));
          }
          float RP = 0.f;
          for (int c = 0; c < S; ++c) RP += __shfl_sync(0xFFFFFFFFu, pp, c);
          const float total = use_p ? RP : R;
          const float t = u_draw * total;
          float run = 0.f, pre = 0.f, prelast = 0.f;
          int cstar = -1, clast = 0;
          for (int c = 0; c < S; ++c) {
            const float part = __shfl_sync(0xFFFFFFFFu, use_p ? pp : rp, c);
            if (part > 0.f) { clast = c; prelast = run; }
            if (cstar < 0 && run + part > t) { cstar = c; pre = run; }
            run += part;
          }
          if (cstar < 0) { cstar = clast; pre = prelast; }
          if (lane == 0) {
            sm.cstar = cstar;
            sm.tl = t - pre;
            sm.total = total;
            sm.use_p = use_p;
            sm.tmo = (R == R) ? 0 : 1;  // a slice's copies timed out
            sm.all_in = 1;
          }
        } else if (lane == 0) {
          atomicExch(a.error, 1);
          sm.cstar = -1;
          sm.tmo = 1;
          sm.total = 1.f;
          sm.use_p = 0;
          sm.all_in = 0;
        }
      }
      __syncthreads();
      const bool clean = sm.all_in != 0 && sm.tmo == 0;
      claim_tag = tag;
      if (clean) {
        // the slice holding the crossing finishes the row, and claims it
        // only after writing (a CTA whose wait gave up may have claimed it
        // first: then the row is rewritten as void)
        if (sm.cstar != slice) {
          leave();
          return;
        }
        if (warp == 0) scan_slice(sm.use_p ? &sm.ps[0][0] : &sm.rs[0][0], true);
        __syncthreads();
        late_claim = true;
      } else {
        if (tid == 0) sm.own = atomicMax(reinterpret_cast<unsigned int*>(a.draw_owner) + du, tag) < tag ? 1 : 0;
        __syncthreads();
        if (!sm.own) {
          leave();
          return;
        }
        if (tid == 0) {
          sm.drawn = -1;
          sm.margin = INFINITY;
          sm.tmo = 1;
        }
        __syncthreads();
      }
    } else {
      if (tid == 0) sm.is_last = arrive_acq_rel_gpu(a.draw_arrive + du) == S - 1;
      __syncthreads();
      if (!sm.is_last) {
        leave();
        return;
      }
      // ============ the draw: the last slice of this unit to arrive ==================
      // Every slice's (chunk, warp) partial sums in one round trip, into the
      // idle ring.
      const int nchm = ((a.d_chunk + VE - 1) / VE + kChunkVecs - 1) / kChunkVecs;  // chunks of a full slice
      float* const Lrs = reinterpret_cast<float*>(ring_buf);
      float* const Lps = Lrs + S * nchm * kWarps;
      for (int i = tid; i < S * nchm * kWarps; i += kThreads) {
        const int s2 = i / (nchm * kWarps), cw = i - s2 * (nchm * kWarps);
        Lrs[i] = __ldcg(&dparts[s2].rs[cw / kWarps][cw % kWarps]);  // past a short slice's chunks: never read
        Lps[i] = __ldcg(&dparts[s2].ps[cw / kWarps][cw % kWarps]);
      }
      if (warp == 0) find_slice();
      __syncthreads();
      if (warp == 0) scan_slice((sm.use_p ? Lps : Lrs) + sm.cstar * nchm * kWarps, false);
      __syncthreads();
      if (tid == 0) a.draw_arrive[du] = 0;
    }
  } else {
    // No stream: greedy (the argmax is the draw) or an invalid row.
    if (tid == 0) {
      sm.drawn = row_invalid ? -1 : (verify ? st.argP : st.argQ);
      sm.margin = INFINITY;
      sm.total = 1.f;
      sm.use_p = 0;
      sm.tmo = 0;
    }
    __syncthreads();
  }
  __syncthreads();

  // ============ finishing the row (verify) or the draft position (reweight) ===========
  const bool tmo_all = sm.tmo != 0;
  if (!verify) {
    if (tid == 0) {
      const bool ok = !row_invalid && !tmo_all;
      a.draft_tokens[static_cast<long long>(b) * K + j] = ok ? sm.drawn : -1;
      UnitState* us = a.ustate + u;
      us->dmargin = sm.margin;
      if (tmo_all) us->flags = st.flags | kFlagTimeout;
      sm.is_last_row = arrive_acq_rel_gpu(a.row_arrive2 + b) == K - 1;
      if (sm.is_last_row) {
        int fl = __ldcg(&a.rstate[b].flags);
        for (int k = 0; k < K; ++k) {
          const UnitState* uk = a.ustate + static_cast<long long>(b) * (K + 1) + k;
          fl |= __ldcg(&uk->flags);
          if (__ldcg(&uk->dmargin) < kNearTie) fl |= SSD_ROW_NEAR_TIE;
        }
        a.status[b] = fl;
        a.row_arrive2[b] = 0;
      }
    }
    leave();
    return;
  }

  const int kstar = j;
  bool flags_final = !dep_ok;  // a row whose decision never came is void anyway
  if (verify && dep_ok && sm.w_final) {  // every word was in when k* was taken
    rowflags = sm.w_flags_all;
    flags_final = true;
  }
  auto finish_row = [&](bool void_row) {
  if (!flags_final) {
    // every unit's word (bounded): the flags of the units past k*
    if (warp == 0) {
      const uint32_t tag = *reinterpret_cast<volatile const uint32_t*>(a.epoch) + 1u;
      const int upr = K + 1;
      const uint64_t* uw = a.uword + static_cast<long long>(b) * upr;
      uint64_t w0 = 0, w1 = 0;
      bool ok = true;
      if (lane < upr) ok = wait_tagged(uw + lane, tag, kDepWaitNs, &w0, 128u);
      if (lane + 32 < upr) ok = wait_tagged(uw + lane + 32, tag, kDepWaitNs, &w1) && ok;
      const bool all_ok = __all_sync(0xFFFFFFFFu, ok);
      const uint32_t lo0 = static_cast<uint32_t>(w0), lo1 = static_cast<uint32_t>(w1);
      uint32_t f = (lo0 | lo1) & 0xFFu;
      if (!a.early_exit || lane <= kstar || lane == K) f |= (lo0 >> 8) & 0xFFu;
      f |= (lo1 >> 8) & 0xFFu;
      if (lane <= kstar && ((lo0 >> 17) & 1u)) f |= SSD_ROW_NEAR_TIE;
      f = __reduce_or_sync(0xFFFFFFFFu, f);
      if (!all_ok) f |= kFlagTimeout;
      if (lane == 0) {
        if (!all_ok) atomicExch(a.error, 1);
        sm.w_flags = static_cast<int32_t>(f);
      }
    }
    __syncthreads();
    rowflags = sm.w_flags;
    flags_final = true;
  }
  int fl = rowflags | ((tmo_all || void_row) ? kFlagTimeout : 0);
  const bool invalid = (fl & SSD_ROW_INVALID) != 0;
  if (tid == 0) {
    if (!kGreedy && (amargin < kNearTie || sm.margin < kNearTie)) fl |= SSD_ROW_NEAR_TIE;
    fl &= ~SSD_ROW_ZERO_RESIDUAL;
    if (sm.use_p) fl |= SSD_ROW_ZERO_RESIDUAL;
    a.status[b] = fl;
    a.n_accepted[b] = invalid ? -1 : kstar;
    a.bonus[b] = invalid ? -1 : sm.drawn;
    a.residual_mass[b] = invalid ? __int_as_float(0x7FC00000) : sm.total;
    sm.slot = -1;
  }
  if (tid <= K) {
    int32_t t = -1;
    if (!invalid) t = tid < kstar ? __ldg(a.tokens + static_cast<long long>(b) * K + tid) : (tid == kstar ? sm.drawn : -1);
    a.out_tokens[static_cast<long long>(b) * (K + 1) + tid] = t;
  }
  if (invalid)
    for (int k = tid; k < K; k += kThreads) a.accept_prob[static_cast<long long>(b) * K + k] = __int_as_float(0x7FC00000);
  else if (a.early_exit)  // no a_j past k*: p_j is not part of the outcome
    for (int k = kstar + 1 + tid; k < K; k += kThreads)
      a.accept_prob[static_cast<long long>(b) * K + k] = __int_as_float(0x7FC00000);
  if (a.c_tokens) {
    const bool pbad = (fl & SSD_ROW_BAD_PLAN) != 0;
    if (tid == 0) {
      int off = 0;
      a.c_offsets[static_cast<long long>(b) * (K + 2)] = 0;
      for (int k = 0; k <= K; ++k) {
        off += pbad ? 0 : sm.s_F[k];
        a.c_offsets[static_cast<long long>(b) * (K + 2) + k + 1] = off;
      }
    }
    __syncthreads();
    if (invalid) {
      for (int s2 = tid; s2 < a.budget; s2 += kThreads) a.c_tokens[static_cast<long long>(b) * a.budget + s2] = -1;
    } else {
      // the key (k*, bonus) in segment k* of the row's cache
      int off = 0;
      for (int k = 0; k < kstar; ++k) off += sm.s_F[k];
      if (streams) {  // the segment was prefetched with the partial sums
        if (seg_tok0 == sm.drawn) sm.slot = off + tid;
        if (seg_tok1 == sm.drawn) sm.slot = off + tid + kThreads;
      } else {
        const int32_t* seg = a.c_tokens + static_cast<long long>(b) * a.budget + off;
        for (int i = tid; i < sm.s_F[kstar]; i += kThreads)
          if (__ldcg(seg + i) == sm.drawn) sm.slot = off + i;
      }
    }
    __syncthreads();
    const int slot = sm.slot;
    if (tid == 0) {
      a.c_hit[b] = slot >= 0 ? 1 : 0;
      a.c_slot[b] = slot;
    }
    for (int i = tid; i < K; i += kThreads) {
      int32_t t;
      if (slot >= 0)
        t = a.c_payload ? __ldg(a.c_payload + (static_cast<long long>(b) * a.budget + slot) * K + i) : -1;
      else
        t = fallback_token(a.fallback_seed, b, i, V);
      a.c_next[static_cast<long long>(b) * K + i] = t;
    }
  }
  };
  finish_row(false);
  if (late_claim) {
    __syncthreads();
    if (tid == 0) sm.own = atomicMax(reinterpret_cast<unsigned int*>(a.draw_owner) + du, claim_tag) < claim_tag ? 1 : 0;
    __syncthreads();
    if (!sm.own) finish_row(true);  // a CTA whose wait gave up claimed the row first
  }
  leave();
}

// Kernel 2 of the two-kernel form: one CTA per (draw unit, slice).
template <typename TIn, bool kAligned, bool kGreedy>
__global__ void __launch_bounds__(kThreads, kDrawMinBlocks) ssd_draw_kernel(const __grid_constant__ Args a) {
  const int S = a.d_slices;
  draw_cta<TIn, kAligned, kGreedy>(a, blockIdx.x / S, blockIdx.x % S);
}

}  // namespace ssd
