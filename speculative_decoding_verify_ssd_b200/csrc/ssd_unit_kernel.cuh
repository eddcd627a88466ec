// ssd_unit_kernel.cuh -- the fused vocab-wide kernel of libssd.
//
// One thread-block cluster handles one "unit" = (row b, position j).  Its CTAs
// split the vocabulary into slices.  Each CTA streams its slice of the unit's
// target row p_j and draft row q_j from HBM exactly once through a ring of
// 1-D bulk copies (cp.async.bulk into shared memory, completed on mbarriers,
// no multicast) and keeps only per-thread running state, so four CTAs share
// an SM and one unit's exchanges overlap other units' streaming.  Cluster-wide
// values are exchanged through distributed shared memory at one barrier.
//
// What one unit computes ([ZH] = "Speculative Speculative Decoding",
// gist.science Chinese edition, technical summary section 2; [NL] = the Dutch
// edition, sections 2 and 3A-3C):
//   pass 1  online max and rescaled sum of exp2 of p_j and q_j (temperature
//           softmax, one exp per element), NaN/+inf detection, a running top-4
//           per thread of the top-F source row (q_j);
//   local   this CTA's candidates for the top-F set ([ZH] challenge 2
//           "top-F tokens"): the F-th largest group maximum of the slice bounds
//           the slice's own top-F from below, so every element of the global
//           top-F in this slice reaches it; the candidates are sorted;
//   B1      one cluster barrier: maxima, sums and sorted candidate lists;
//   select  global ranks by binary search in the other CTAs' sorted lists;
//           the exact top-F by (logit desc, token id asc); Q_S and the Saguaro
//           normaliser Z = 1 - (1 - C) Q_S ([ZH] challenge 2; [NL] 3B);
//   accept  a_j = min(1, p_j(d_j) / q'_j(d_j)), rejected iff u_j >= a_j;
//   pass 2  only where the unit's draw is needed (the first rejection of the
//           row, or full acceptance): residual r = max(0, p - q') (or p_K, or
//           q' for the draft draw) streamed again (from L2), partial sums per
//           (chunk, warp), one barrier, then an inverse-CDF search in token
//           order in the CTA where the cumulative mass crosses u * R;
//   epilogue the CTA that holds the unit's result publishes it; the last unit
//           of a row to finish (arrival counter, no spinning) picks k*, the
//           bonus token, and looks (k*, bonus) up in the cache segment of
//           outcome k* ([ZH] basic flow steps 3-4; [NL] 3C).
#pragma once

#include <limits.h>

#include "../../include/ssd.h"
#include "ssd_device.cuh"

namespace ssd {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMinBlocks = 4;          // CTAs per SM the register budget is set for
constexpr int kMaxCluster = 16;
constexpr int kStages = 4;             // depth of the bulk-copy ring
constexpr int kChunkVecs = kThreads;   // 16-byte vectors per row per ring stage
constexpr int kMaxChunks = 16;         // ring chunks per slice
constexpr int kCandCap = 256;          // local top-F candidates per CTA
constexpr int kGatherCap = 1024;       // candidates of a whole unit (fast path)
constexpr int kSelCap = 512;           // >= SSD_MAX_BUDGET
constexpr int kMaxGroups = kThreads;   // group maxima per CTA
constexpr uint32_t kMaxPolls = 4000000u;  // x ~0.5 us sleep: about 2 s
constexpr float kNearTie = 1e-5f;
constexpr int kFlagTimeout = SSD_ROW_DEVICE_TIMEOUT;

enum Mode : int { kModeVerify = 0, kModeReweight = 1 };
enum Draw : int { kDrawNone = 0, kDrawResidual = 1, kDrawP = 2, kDrawQ = 3 };

// Result of one unit, read by the row epilogue.
struct UnitRes {
  float a;          // acceptance probability a_j (verify, j < K)
  float R;          // mass of the distribution the unit's draw came from
  int32_t draw;     // the unit's drawn / greedy token, -1 if none
  int32_t flags;    // SSD_ROW_* bits of this unit
  float amargin;    // |u_j - a_j|
  float bmargin;    // inverse-CDF margin of the draw, over the mass
  int32_t rejected; // 1 iff u_j >= a_j
  int32_t seg_slot; // index of `draw` in this unit's top-F list, -1 if absent
};

struct UnitArgs {
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
  int B, K, V, budget, mode, n_cta, chunk, units_per_row;
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
  UnitRes* units;
  int32_t* counters;
  int32_t* first_rej;
  int32_t* error;
};

struct Cand {
  float x;
  int32_t idx;
};

// Published to the other CTAs of the cluster (read through DSMEM).
struct Xchg {
  float mP, sP, mQ, sQ;      // this slice's running max and exp-sum
  int32_t argP, argQ;        // greedy: lowest id of the slice maximum
  int32_t hint;              // rank 0: the row's earliest rejection seen so far
  int32_t n_cand;            // local candidates found (may exceed kCandCap)
  int32_t timeout;           // a bulk copy of this CTA did not complete
  float Rpart, RPpart;       // pass 2: mass of this slice (residual, and p alone)
  int32_t timeout2;
  float slow_QS, slow_bx;    // rank 0, slow path
  int32_t slow_bi;
  Cand cand[kCandCap];       // this slice's candidates, sorted by (logit desc, id asc)
};

// CTA-private state.
struct Local {
  uint64_t full[kStages];
  float wred[kWarps][4];
  int32_t wint[kWarps][2];
  float round_sum[kMaxChunks][kWarps];
  float round_sump[kMaxChunks][kWarps];
  float gmax[kMaxGroups];
  // unit-wide values, identical in every CTA of the cluster
  float MP, MQ, SP, SQ, xdP, xdQ, tau, QS, bx, tl, total;
  int32_t bi, argP, argQ, hint, n_total, slow, flags, cstar, use_p, seg_slot, is_last, n_raw, tmo;
  int32_t cand_off[kMaxCluster + 1];
  Cand raw[kCandCap];                 // local candidates before sorting
  Cand buf[kGatherCap + kSelCap];     // gathered lists, then the sorted selection
};
static_assert(2 * kMaxChunks * kWarps >= 256, "round sums double as the slow-path histogram");

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
__device__ __forceinline__ void consume_bf16(const uint4 w, int vbase, float c, float& m, float& s, float& nmc,
                                             int& arg, int& nan_seen) {
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
      s = (m == -INFINITY) ? 0.f : s * ex2((m - nm) * c);
      m = nm;
      nmc = -m * c;
    }
    const float e0 = ex2(fmaf(bf16_lo(w.x), c, nmc)) + ex2(fmaf(bf16_hi(w.x), c, nmc));
    const float e1 = ex2(fmaf(bf16_lo(w.y), c, nmc)) + ex2(fmaf(bf16_hi(w.y), c, nmc));
    const float e2 = ex2(fmaf(bf16_lo(w.z), c, nmc)) + ex2(fmaf(bf16_hi(w.z), c, nmc));
    const float e3 = ex2(fmaf(bf16_lo(w.w), c, nmc)) + ex2(fmaf(bf16_hi(w.w), c, nmc));
    s += (e0 + e1) + (e2 + e3);
  }
}

template <int VE, bool kGreedy>
__device__ __forceinline__ void consume_f(const float (&x)[VE], int vbase, float c, float& m, float& s, float& nmc,
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

// Exact top-F of a whole row, read from global memory by one CTA: a radix
// select on the 32-bit order key (four 8-bit digits), ties at the threshold
// taken in token-id order, then the F winners ranked by (key, id) in place.
// Used when the shared-memory candidate filter cannot bound the set (many
// ties, F large).  `hist` needs 256 ints; the result is sel[0 .. F).
template <typename TIn>
__device__ void topf_exact_global(const TIn* row, int V, int F, Cand* sel, float* hist_f, int tid) {
  __shared__ uint32_t s_prefix, s_mask;
  __shared__ int32_t s_remaining, s_napp, s_tie_base[kThreads + 1];
  int32_t* hist = reinterpret_cast<int32_t*>(hist_f);
  if (tid == 0) { s_prefix = 0u; s_mask = 0u; s_remaining = F; s_napp = 0; }
  __syncthreads();
  for (int level = 0; level < 4; ++level) {
    const int shift = 24 - 8 * level;
    for (int i = tid; i < 256; i += kThreads) hist[i] = 0;
    __syncthreads();
    const uint32_t prefix = s_prefix, mask = s_mask;
    for (int v = tid; v < V; v += kThreads) {
      const uint32_t k = ord_key(Elem<TIn>::at(row, v));
      if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1);
    }
    __syncthreads();
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
    __syncthreads();
  }
  const uint32_t t = s_prefix;
  const int need_eq = s_remaining;
  // Ties in token order: each thread owns a contiguous chunk of the row.
  const int per = (V + kThreads - 1) / kThreads;
  const int lo = min(V, tid * per), hi = min(V, lo + per);
  int my_eq = 0;
  for (int v = lo; v < hi; ++v) my_eq += (ord_key(Elem<TIn>::at(row, v)) == t);
  s_tie_base[tid + 1] = my_eq;
  __syncthreads();
  if (tid == 0) {
    s_tie_base[0] = 0;
    for (int i = 1; i <= kThreads; ++i) s_tie_base[i] += s_tie_base[i - 1];
  }
  __syncthreads();
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
  __syncthreads();
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
  __syncthreads();
#pragma unroll
  for (int q = 0; q < kPer; ++q)
    if (rk[q] >= 0) sel[rk[q]] = mine[q];
  __syncthreads();
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

// The 16-byte vector `g` of a slice row as VE floats: from the ring stage in
// shared memory (bulk-copy path) or straight from global memory.
template <typename TIn, bool kAligned>
__device__ __forceinline__ void fetch(const TIn* __restrict__ base, long long rb, int e0, int e1, int g,
                                      const unsigned char* ring_row, float (&x)[Elem<TIn>::VE]) {
  constexpr int VE = Elem<TIn>::VE;
  if constexpr (kAligned) {
    Elem<TIn>::unpack(*reinterpret_cast<const uint4*>(ring_row + (g % kChunkVecs) * 16), x);
  } else {
    load_group<TIn, false>(base, rb, e0 + g * VE, e1, x);
  }
}

template <typename TIn, bool kAligned, bool kGreedy>
__global__ void __launch_bounds__(kThreads, kMinBlocks) ssd_unit_kernel(const __grid_constant__ UnitArgs a) {
  constexpr int VE = Elem<TIn>::VE;
  extern __shared__ __align__(128) unsigned char ring[];
  __shared__ __align__(16) Xchg xc;
  __shared__ __align__(16) Local lc;
  __shared__ int32_t s_F[SSD_MAX_K + 1];

  cg::cluster_group cluster = cg::this_cluster();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rank = static_cast<int>(cluster.block_rank());
  const int n_cta = a.n_cta;
  const int unit = blockIdx.x / n_cta;
  const int b = unit % a.B, j = unit / a.B;
  const int K = a.K, V = a.V;
  const bool verify = a.mode == kModeVerify;

  // ---- roles of this unit ---------------------------------------------------
  const TIn* baseP = nullptr;
  const TIn* baseQ = nullptr;
  long long rbP = 0, rbQ = 0;
  if (verify) {
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
  const bool hasP = baseP != nullptr, hasQ = baseQ != nullptr;
  const bool has_d = verify && j < K;
  int draw = kDrawNone;
  if (verify) draw = j < K ? kDrawResidual : kDrawP;
  else if (j < K && a.uniforms) draw = kDrawQ;
  const bool srcQ = hasQ;  // the top-F source row: q_j, else p
  // ring layout: row slot 0 = p (if present), the next slot = q
  const int n_rows = (hasP ? 1 : 0) + (hasQ ? 1 : 0);
  const int slotP = 0, slotQ = hasP ? 1 : 0;
  const int ring_rows = verify ? 2 : 1;  // allocated row slots per stage

  // ---- slice of this CTA: vocab [e0, e1) in vectors of VE elements ----------------
  const int e0 = rank * a.chunk;
  const int e1 = min(V, e0 + a.chunk);
  const int n = max(0, e1 - e0);
  const int nvec = (n + VE - 1) / VE;
  const int nch = (nvec + kChunkVecs - 1) / kChunkVecs;

  auto stage_ptr = [&](int slot, int row) -> unsigned char* {
    return ring + (static_cast<size_t>(slot) * ring_rows + row) * (kChunkVecs * 16);
  };
  // Issue ring chunk `c` (pass-local index `k`) of this slice: one bulk copy per row.
  int n_issued = 0;  // chunks issued so far (thread 0)
  auto issue = [&](int c, int k) {
    n_issued = c + 1;
    const int slot = c % kStages;
    const int v0 = k * kChunkVecs;
    const int nv = min(kChunkVecs, nvec - v0);
    const uint32_t bytes = static_cast<uint32_t>(nv) * 16u * static_cast<uint32_t>(n_rows);
    mbar_arrive_expect_tx(&lc.full[slot], bytes);
    if (hasP) bulk_copy_g2s(stage_ptr(slot, slotP), baseP + rbP + e0 + v0 * VE, nv * 16u, &lc.full[slot]);
    if (hasQ) bulk_copy_g2s(stage_ptr(slot, slotQ), baseQ + rbQ + e0 + v0 * VE, nv * 16u, &lc.full[slot]);
  };
  int tmo = 0;  // a bulk copy of this CTA did not complete in time
  // Chunk c (of the pass whose chunks are [c_first, c_end)) is ready for every
  // thread.  Only thread 0 polls the stage's mbarrier, sleeping between polls;
  // the CTA barrier also marks chunk c - 1 consumed, so thread 0 then refills
  // that stage; every other thread takes one acquiring look at the phase.
  auto acquire_chunk = [&](int c, int c_first, int c_end) {
    if (tid == 0 && !mbar_wait_bounded(&lc.full[c % kStages], (c / kStages) & 1, kMaxPolls)) tmo = 1;
    __syncthreads();
    if (tid == 0 && c > c_first && c - 1 + kStages < c_end) issue(c - 1 + kStages, c - 1 + kStages - c_first);
    if (tid != 0 && !mbar_try_wait(&lc.full[c % kStages], (c / kStages) & 1, 0u)) tmo = 1;
  };

  if constexpr (kAligned) {
    if (tid == 0) {
      for (int s2 = 0; s2 < kStages; ++s2) mbar_init(&lc.full[s2], 1);
      mbar_init_fence();
    }
    __syncthreads();
    if (tid == 0)
      for (int k = 0; k < min(kStages, nch); ++k) issue(k, k);
  }

  // ---- fan-out plan of this row -----------------------------------------------
  const bool has_plan = a.F != nullptr || a.alpha != nullptr;
  if (tid == 0 && has_plan) {
    if (a.F) {
      for (int k = 0; k <= K; ++k) s_F[k] = __ldg(a.F + static_cast<long long>(b) * (K + 1) + k);
    } else {
      fanout_row(__ldg(a.alpha + b), K, a.budget, a.fanout_mode, s_F);
    }
  }

  // Per-unit scalars every CTA reads identically.
  int flags = 0;
  int d = -1;
  float u_self = 0.f, u_draw = 0.f;
  if (has_d) {
    d = __ldg(a.tokens + static_cast<long long>(b) * K + j);
    if (d < 0 || d >= V) flags |= SSD_ROW_BAD_TOKEN;
  }
  if (verify) {
    u_self = __ldg(a.uniforms + static_cast<long long>(b) * (K + 1) + j);
    u_draw = __ldg(a.uniforms + static_cast<long long>(b) * (K + 1) + K);
    if (!(u_self >= 0.f && u_self < 1.f)) flags |= SSD_ROW_BAD_UNIFORM;
  } else if (draw == kDrawQ) {
    u_draw = __ldg(a.uniforms + static_cast<long long>(b) * K + j);
    if (!(u_draw >= 0.f && u_draw < 1.f)) flags |= SSD_ROW_BAD_UNIFORM;
  }
  // The logits at the draft token, fetched by every CTA (latency hidden by pass 1).
  float xdP = 0.f, xdQ = 0.f;
  if (tid == 0 && has_d && d >= 0 && d < V) {
    xdP = Elem<TIn>::at(baseP + rbP, d);
    xdQ = Elem<TIn>::at(baseQ + rbQ, d);
  }
  __syncthreads();
  int Fj = 0, seg_off = 0, plan_bad = 0;
  if (has_plan) {
    long long sum = 0;
    for (int k = 0; k <= K; ++k) {
      const int f = s_F[k];
      if (f < 0 || f > V) plan_bad = 1;
      if (k < j) seg_off += f;
      sum += f;
    }
    if (sum != a.budget) plan_bad = 1;
    Fj = plan_bad ? 0 : s_F[j];
  }
  if (plan_bad) flags |= SSD_ROW_BAD_PLAN;
  const bool want_topf = has_plan && Fj > 0;
  const float cT = kGreedy ? 0.f : kLog2e / a.T;

  // ---- pass 1: online max / exp-sum (or greedy argmax) of both rows -------------
  float mP = -INFINITY, sP = 0.f, nmP1 = 0.f, mQ = -INFINITY, sQ = 0.f, nmQ1 = 0.f;
  int argP = INT_MAX, argQ = INT_MAX, nan_seen = 0;
  for (int c = 0; c < nch; ++c) {
    if constexpr (kAligned) acquire_chunk(c, 0, nch);
    const int g = c * kChunkVecs + tid;
    if (g < nvec) {
      const int vbase = e0 + g * VE;
      if constexpr (kAligned && sizeof(TIn) == 2) {
        if (hasP)
          consume_bf16<kGreedy>(*reinterpret_cast<const uint4*>(stage_ptr(c % kStages, slotP) + tid * 16), vbase, cT,
                                mP, sP, nmP1, argP, nan_seen);
        if (hasQ)
          consume_bf16<kGreedy>(*reinterpret_cast<const uint4*>(stage_ptr(c % kStages, slotQ) + tid * 16), vbase, cT,
                                mQ, sQ, nmQ1, argQ, nan_seen);
      } else {
        float x[VE];
        if (hasP) {
          fetch<TIn, kAligned>(baseP, rbP, e0, e1, g, stage_ptr(c % kStages, slotP), x);
          consume_f<VE, kGreedy>(x, vbase, cT, mP, sP, nmP1, argP, nan_seen);
        }
        if (hasQ) {
          fetch<TIn, kAligned>(baseQ, rbQ, e0, e1, g, stage_ptr(c % kStages, slotQ), x);
          consume_f<VE, kGreedy>(x, vbase, cT, mQ, sQ, nmQ1, argQ, nan_seen);
        }
      }
    }
  }
  if constexpr (kGreedy) {
    if (nan_seen) { mP = __int_as_float(0x7FC00000); mQ = mP; }
  }
  const float mSrc = hasQ ? mQ : mP;  // this thread's maximum of the top-F source row
  lc.gmax[tid] = mSrc;
  if (tid == 0) {
    lc.n_raw = 0;
    lc.xdP = xdP;
    lc.xdQ = xdQ;
  }

  // ---- CTA reduction: butterfly within each warp, then over the warps --------------
  if constexpr (kGreedy) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      merge_arg(mP, argP, __shfl_xor_sync(0xFFFFFFFFu, mP, o), __shfl_xor_sync(0xFFFFFFFFu, argP, o));
      merge_arg(mQ, argQ, __shfl_xor_sync(0xFFFFFFFFu, mQ, o), __shfl_xor_sync(0xFFFFFFFFu, argQ, o));
    }
    if (lane == 0) {
      lc.wred[warp][0] = mP; lc.wred[warp][2] = mQ;
      lc.wint[warp][0] = argP; lc.wint[warp][1] = argQ;
    }
  } else {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      merge_ms(mP, sP, __shfl_xor_sync(0xFFFFFFFFu, mP, o), __shfl_xor_sync(0xFFFFFFFFu, sP, o), cT);
      merge_ms(mQ, sQ, __shfl_xor_sync(0xFFFFFFFFu, mQ, o), __shfl_xor_sync(0xFFFFFFFFu, sQ, o), cT);
    }
    if (lane == 0) {
      lc.wred[warp][0] = mP; lc.wred[warp][1] = sP;
      lc.wred[warp][2] = mQ; lc.wred[warp][3] = sQ;
    }
  }
  const bool fast_ok = want_topf && Fj <= kMaxGroups;
  tmo = __syncthreads_or(tmo);
  if (warp == 0) {
    float m1 = -INFINITY, s1 = 0.f, m2 = -INFINITY, s2 = 0.f;
    int a1 = INT_MAX, a2 = INT_MAX;
    if (lane < kWarps) {
      m1 = lc.wred[lane][0]; s1 = lc.wred[lane][1]; m2 = lc.wred[lane][2]; s2 = lc.wred[lane][3];
      if constexpr (kGreedy) { a1 = lc.wint[lane][0]; a2 = lc.wint[lane][1]; }
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
      xc.mP = m1; xc.sP = kGreedy ? 0.f : s1;
      xc.mQ = m2; xc.sQ = kGreedy ? 0.f : s2;
      xc.argP = a1; xc.argQ = a2;
      xc.hint = (rank == 0 && verify) ? __ldcg(a.first_rej + b) : 0;
      xc.timeout = tmo;
    }
  } else if (warp == 1) {
    // This slice's threshold: the F-th largest of its 256 thread maxima bounds
    // the slice's own top-F (hence its share of the global top-F) from below.
    float t = -INFINITY;
    if (fast_ok) {
      uint32_t keys[kMaxGroups / 32];
#pragma unroll
      for (int i = 0; i < kMaxGroups / 32; ++i) keys[i] = ord_key(lc.gmax[lane + 32 * i]);
      t = key_to_float(warp_kth_largest(keys, Fj, sizeof(TIn) == 2 ? 16 : 32));
    }
    if (lane == 0) lc.tau = t;
  }
  __syncthreads();
  const float tau = lc.tau;

  // Local candidates: the elements at or above tau.  Only threads whose
  // maximum reaches tau hold any; they re-read their vectors (from L2).
  if (fast_ok && mSrc >= tau && mSrc == mSrc) {
    const TIn* bs = srcQ ? baseQ : baseP;
    const long long rs = srcQ ? rbQ : rbP;
    for (int c = 0; c < nch; ++c) {
      const int g = c * kChunkVecs + tid;
      if (g < nvec) {
        float x[VE];
        load_group<TIn, kAligned>(bs, rs, e0 + g * VE, e1, x);
#pragma unroll
        for (int i = 0; i < VE; ++i) {
          const int v = e0 + g * VE + i;
          if (x[i] >= tau && v < e1) {
            const int pos = atomicAdd(&lc.n_raw, 1);
            if (pos < kCandCap) lc.raw[pos] = Cand{x[i], v};
          }
        }
      }
    }
  }
  __syncthreads();
  {
    const int nr = min(lc.n_raw, kCandCap);
    for (int i = tid; i < nr; i += kThreads) {
      const Cand ci = lc.raw[i];
      const unsigned long long key = rank_key(ci.x, ci.idx);
      int r = 0;
      for (int k2 = 0; k2 < nr; ++k2) r += rank_key(lc.raw[k2].x, lc.raw[k2].idx) > key;
      xc.cand[r] = ci;
    }
    if (tid == 0) xc.n_cand = lc.n_raw;
  }
  cluster_sync_all();  // ---- B1: every CTA's state and sorted list is published ----

  if (warp == 0) {
    // Butterfly over the CTAs (lanes >= n_cta hold neutral values): every lane,
    // and every CTA, ends with bit-identical unit-wide values.
    float mp = -INFINITY, sp = 0.f, mq = -INFINITY, sq = 0.f;
    int ap = INT_MAX, aq = INT_MAX, nc = 0, to = 0, hint = 0;
    if (lane < n_cta) {
      const Xchg* rx = cluster.map_shared_rank(&xc, lane);
      mp = rx->mP; sp = rx->sP; mq = rx->mQ; sq = rx->sQ; ap = rx->argP; aq = rx->argQ;
      nc = rx->n_cand; to = rx->timeout;
      if (lane == 0) hint = rx->hint;
    }
    const int ncc = min(nc, kCandCap);
#pragma unroll
    for (int o = kMaxCluster / 2; o > 0; o >>= 1) {
      if constexpr (kGreedy) {
        merge_arg(mp, ap, __shfl_xor_sync(0xFFFFFFFFu, mp, o), __shfl_xor_sync(0xFFFFFFFFu, ap, o));
        merge_arg(mq, aq, __shfl_xor_sync(0xFFFFFFFFu, mq, o), __shfl_xor_sync(0xFFFFFFFFu, aq, o));
      } else {
        merge_ms(mp, sp, __shfl_xor_sync(0xFFFFFFFFu, mp, o), __shfl_xor_sync(0xFFFFFFFFu, sp, o), cT);
        merge_ms(mq, sq, __shfl_xor_sync(0xFFFFFFFFu, mq, o), __shfl_xor_sync(0xFFFFFFFFu, sq, o), cT);
      }
    }
    // exclusive offsets of the candidate lists
    int incl = ncc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += y;
    }
    const int total = __shfl_sync(0xFFFFFFFFu, incl, 31);
    const unsigned over = __ballot_sync(0xFFFFFFFFu, nc > kCandCap);
    const unsigned anyto = __ballot_sync(0xFFFFFFFFu, to != 0);
    if (lane < n_cta) lc.cand_off[lane] = incl - ncc;
    if (lane == 0) {
      lc.MP = mp; lc.SP = sp; lc.MQ = mq; lc.SQ = sq; lc.argP = ap; lc.argQ = aq;
      lc.cand_off[n_cta] = total;
      lc.n_total = total;
      lc.tmo = anyto ? 1 : 0;
      lc.hint = hint;
      lc.slow = over || total > kGatherCap || total < Fj;  // refined below with validity
    }
  }
  __syncthreads();
  const float MP = lc.MP, MQ = lc.MQ, SP = lc.SP, SQ = lc.SQ;
  if (lc.tmo) flags |= kFlagTimeout;
  if (hasP && !(MP > -INFINITY && MP < INFINITY)) flags |= SSD_ROW_NONFINITE;
  if (hasQ && !(MQ > -INFINITY && MQ < INFINITY)) flags |= SSD_ROW_NONFINITE;
  const bool valid = (flags & SSD_ROW_INVALID) == 0;
  const bool slow = want_topf && valid && (!fast_ok || lc.slow != 0);
  Cand* sel = lc.buf + kGatherCap;
  const float nmP = -MP * cT, nmQ = -MQ * cT;

  // ---- exact top-F: global ranks by binary search in the sorted lists ---------------
  if (want_topf && valid && !slow) {
    const int N = lc.n_total;
    for (int i = tid; i < N; i += kThreads) {
      int c = 0;
      while (c + 1 < n_cta && lc.cand_off[c + 1] <= i) ++c;
      lc.buf[i] = cluster.map_shared_rank(&xc, c)->cand[i - lc.cand_off[c]];
    }
    __syncthreads();
    for (int i = tid; i < N; i += kThreads) {
      int c = 0;
      while (c + 1 < n_cta && lc.cand_off[c + 1] <= i) ++c;
      const Cand ci = lc.buf[i];
      const unsigned long long key = rank_key(ci.x, ci.idx);
      int r = i - lc.cand_off[c];  // entries ahead of it in its own list
      for (int c2 = 0; c2 < n_cta; ++c2) {
        if (c2 == c) continue;
        int lo = lc.cand_off[c2], hi = lc.cand_off[c2 + 1];  // count keys > key in a descending list
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (rank_key(lc.buf[mid].x, lc.buf[mid].idx) > key) lo = mid + 1;
          else hi = mid;
        }
        r += lo - lc.cand_off[c2];
      }
      if (r < Fj) sel[r] = ci;
    }
  }
  if (slow) {  // uniform: every CTA of the cluster takes this branch or none does
    if (rank == 0) {
      const TIn* row = hasQ ? baseQ + rbQ : baseP + rbP;
      topf_exact_global<TIn>(row, V, Fj, sel, &lc.round_sum[0][0], tid);
    }
    cluster_sync_all();  // ---- B1b (slow path only): rank 0's selection is ready ----
    if (rank != 0) {
      const Cand* s0 = cluster.map_shared_rank(&lc, 0)->buf + kGatherCap;
      for (int i = tid; i < Fj; i += kThreads) sel[i] = s0[i];
    }
  }
  __syncthreads();

  // Q_S in a fixed order (identical in every CTA), the top-F boundary.
  if (warp == 0) {
    float qs = 0.f;
    if (want_topf && valid) {
      if constexpr (!kGreedy) {
        for (int i = lane; i < Fj; i += 32) qs += ex2(fmaf(sel[i].x, cT, hasQ ? nmQ : nmP));
      }
    }
    qs = warp_sum(qs);
    if (lane == 0) {
      lc.QS = qs;
      lc.bx = (want_topf && valid) ? sel[Fj - 1].x : INFINITY;
      lc.bi = (want_topf && valid) ? sel[Fj - 1].idx : -1;
    }
  }
  __syncthreads();

  // ---- Saguaro normaliser and the accept test -------------------------------------
  const float C = a.C;
  float Z = 1.f;
  if (!kGreedy && want_topf && valid) Z = 1.f - (1.f - C) * (lc.QS / (hasQ ? SQ : SP));
  const float bx = lc.bx;
  const int bi = lc.bi;
  float acc = 0.f, amargin = INFINITY;
  int rejected = 0;
  if (has_d && valid) {
    if constexpr (kGreedy) {
      acc = (d == lc.argP) ? 1.f : 0.f;
      rejected = d != lc.argP;
    } else {
      const float xq_d = lc.xdQ;
      const float pd = ex2(fmaf(lc.xdP, cT, nmP)) / SP;
      const float qd = ex2(fmaf(xq_d, cT, nmQ)) / SQ;
      const bool inS = want_topf && (xq_d > bx || (xq_d == bx && d <= bi));
      const float qpd = (inS ? C : 1.f) * qd / Z;
      if (qpd > 0.f) {
        acc = fminf(1.f, pd / qpd);
      } else {
        acc = pd > 0.f ? 1.f : 0.f;
        flags |= SSD_ROW_ZERO_Q;
      }
      rejected = !(u_self < acc);
      amargin = fabsf(u_self - acc);
    }
  }
  if (verify && has_d && valid && rejected && rank == 0 && tid == 0) atomicMax(a.first_rej + b, K + 1 - j);

  bool need_draw = false;
  if (!kGreedy && valid) {
    if (draw == kDrawResidual) need_draw = rejected && !(lc.hint > K + 1 - j);
    else if (draw == kDrawP) need_draw = lc.hint == 0;
    else if (draw == kDrawQ) need_draw = true;
  }

  int owner = 0;  // the CTA that publishes this unit's result
  if (!need_draw) {
    cluster_arrive();  // no more reads of other CTAs' shared memory
  } else {
    // ---- pass 2: the draw (inverse CDF in token order across the cluster) ---------
    const float invSP = 1.f / SP;
    const float wS = C / (SQ * Z), wN = 1.f / (SQ * Z);
    const bool check_S = want_topf && draw != kDrawP;
    if constexpr (kAligned) {
      if (tid == 0)
        for (int k = 0; k < min(kStages, nch); ++k) issue(nch + k, k);
    }
    // the draw's mass of element i of vector g (and p alone, for R = 0)
    auto vals = [&](int g, const unsigned char* rp, const unsigned char* rq, float (&val)[VE], float (&pv)[VE]) {
      float xp[VE], xq[VE];
      if (draw != kDrawQ) fetch<TIn, kAligned>(baseP, rbP, e0, e1, g, rp, xp);
      if (draw != kDrawP) fetch<TIn, kAligned>(baseQ, rbQ, e0, e1, g, rq, xq);
#pragma unroll
      for (int i = 0; i < VE; ++i) {
        float wq = wN;
        if (check_S) {
          const int v = e0 + g * VE + i;
          if (xq[i] > bx || (xq[i] == bx && v <= bi)) wq = wS;
        }
        if (draw == kDrawResidual) {
          const float pp = ex2(fmaf(xp[i], cT, nmP)) * invSP;
          val[i] = fmaxf(pp - ex2(fmaf(xq[i], cT, nmQ)) * wq, 0.f);
          pv[i] = pp;
        } else if (draw == kDrawP) {
          val[i] = ex2(fmaf(xp[i], cT, nmP)) * invSP;
          pv[i] = 0.f;
        } else {
          val[i] = ex2(fmaf(xq[i], cT, nmQ)) * wq;
          pv[i] = 0.f;
        }
      }
    };
    for (int k = 0; k < nch; ++k) {
      const int c = nch + k;
      const int g = k * kChunkVecs + tid;
      if constexpr (kAligned) acquire_chunk(c, nch, 2 * nch);
      float rs = 0.f, ps = 0.f;
      if (g < nvec) {
        float val[VE], pv[VE];
        vals(g, stage_ptr(c % kStages, slotP), stage_ptr(c % kStages, slotQ), val, pv);
#pragma unroll
        for (int i = 0; i < VE; ++i) { rs += val[i]; ps += pv[i]; }
      }
      rs = warp_sum(rs);
      ps = warp_sum(ps);
      if (lane == 0) { lc.round_sum[k][warp] = rs; lc.round_sump[k][warp] = ps; }
    }
    tmo = __syncthreads_or(tmo);
    if (tid == 0) {
      float R = 0.f, RP = 0.f;
      for (int k = 0; k < nch; ++k)
        for (int w = 0; w < kWarps; ++w) { R += lc.round_sum[k][w]; RP += lc.round_sump[k][w]; }
      xc.Rpart = R;
      xc.RPpart = RP;
      xc.timeout2 = tmo;
    }
    cluster_sync_all();  // ---- B2: slice masses published ----
    if (warp == 0) {
      float rp = 0.f, pp = 0.f;
      int to = 0;
      if (lane < n_cta) {
        const Xchg* rx = cluster.map_shared_rank(&xc, lane);
        rp = rx->Rpart;
        pp = rx->RPpart;
        to = rx->timeout2;
      }
      float R = 0.f, RP = 0.f;
      for (int c = 0; c < n_cta; ++c) {
        R += __shfl_sync(0xFFFFFFFFu, rp, c);
        RP += __shfl_sync(0xFFFFFFFFu, pp, c);
      }
      const int use_p = (draw == kDrawResidual && !(R > 0.f)) ? 1 : 0;
      const float total = use_p ? RP : R;
      const float t = u_draw * total;
      // crossing CTA: the first c with prefix + part > t, else the last with mass
      float run = 0.f, pre = 0.f, prelast = 0.f;
      int cstar = -1, clast = 0;
      for (int c = 0; c < n_cta; ++c) {
        const float part = __shfl_sync(0xFFFFFFFFu, use_p ? pp : rp, c);
        if (part > 0.f) { clast = c; prelast = run; }
        if (cstar < 0 && run + part > t) { cstar = c; pre = run; }
        run += part;
      }
      if (cstar < 0) { cstar = clast; pre = prelast; }
      const unsigned anyto = __ballot_sync(0xFFFFFFFFu, to != 0);
      if (lane == 0) {
        lc.cstar = cstar;
        lc.tl = t - pre;
        lc.total = total;
        lc.use_p = use_p;
        lc.tmo = anyto ? 1 : 0;
      }
    }
    __syncthreads();
    cluster_arrive();  // no more reads of other CTAs' shared memory
    if (lc.tmo) flags |= kFlagTimeout;
    owner = lc.cstar;
    if (rank == owner && warp == 0) {
      const bool use_p = lc.use_p != 0;
      const float tl = lc.tl;
      // chunk level, then warp level, in token order
      float run = 0.f, pre_k = 0.f, pre_last = 0.f;
      int k_star = -1, k_last = 0;
      for (int k = 0; k < nch; ++k) {
        float tk = 0.f;
        for (int w = 0; w < kWarps; ++w) tk += use_p ? lc.round_sump[k][w] : lc.round_sum[k][w];
        if (tk > 0.f) { k_last = k; pre_last = run; }
        if (k_star < 0 && run + tk > tl) { k_star = k; pre_k = run; }
        run += tk;
      }
      if (k_star < 0) { k_star = k_last; pre_k = pre_last; }
      const float tl2 = tl - pre_k;
      run = 0.f;
      float pre_w = 0.f;
      pre_last = 0.f;
      int w_star = -1, w_last = 0;
      for (int w = 0; w < kWarps; ++w) {
        const float tw = use_p ? lc.round_sump[k_star][w] : lc.round_sum[k_star][w];
        if (tw > 0.f) { w_last = w; pre_last = run; }
        if (w_star < 0 && run + tw > tl2) { w_star = w; pre_w = run; }
        run += tw;
      }
      if (w_star < 0) { w_star = w_last; pre_w = pre_last; }
      const float tl3 = tl2 - pre_w;
      // lane level: the 32 vectors of that warp in that chunk, re-read from L2
      const int g = k_star * kChunkVecs + w_star * 32 + lane;
      float val[VE], pv[VE];
      float ls = 0.f;
      if (g < nvec) {
        float xp[VE], xq[VE];
        if (draw != kDrawQ) load_group<TIn, kAligned>(baseP, rbP, e0 + g * VE, e1, xp);
        if (draw != kDrawP) load_group<TIn, kAligned>(baseQ, rbQ, e0 + g * VE, e1, xq);
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
          } else if (draw == kDrawP) {
            val[i] = ex2(fmaf(xp[i], cT, nmP)) * invSP;
          } else {
            val[i] = ex2(fmaf(xq[i], cT, nmQ)) * wq;
          }
          pv[i] = 0.f;
        }
      } else {
#pragma unroll
        for (int i = 0; i < VE; ++i) { val[i] = 0.f; pv[i] = 0.f; }
      }
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
        const int v = e0 + g * VE + i_star;
        const float lo = tl4 - c_prev;                // t - CDF before v
        const float hi = c_prev + val[i_star] - tl4;  // CDF at v - t
        lc.seg_slot = min(max(v, 0), V - 1);          // the drawn token (stashed)
        lc.tl = fminf(fabsf(lo), fabsf(hi)) / lc.total;
      }
      (void)pv;
    }
  }
  __syncthreads();

  // ---- the unit's result, published by its owner CTA -------------------------------
  if (rank == owner) {
    int drawn = -1;
    float bmargin = INFINITY, Rout = 1.f;
    if (valid && !(flags & kFlagTimeout)) {
      if constexpr (kGreedy) {
        drawn = verify ? lc.argP : lc.argQ;
      } else if (need_draw) {
        drawn = lc.seg_slot;
        bmargin = lc.tl;
        Rout = lc.total;
      }
    }
    __syncthreads();
    if (tid == 0) lc.seg_slot = -1;
    __syncthreads();
    if (want_topf && valid && drawn >= 0)
      for (int i = tid; i < Fj; i += kThreads)
        if (sel[i].idx == drawn) lc.seg_slot = i;
    __syncthreads();
    if (tid == 0) {
      const bool ok = (flags & SSD_ROW_INVALID) == 0;
      int fl = flags;
      if (need_draw && lc.use_p) fl |= SSD_ROW_ZERO_RESIDUAL;
      if (verify && j < K) a.accept_prob[static_cast<long long>(b) * K + j] = ok ? acc : __int_as_float(0x7FC00000);
      if (!verify && j < K) {
        const long long o = static_cast<long long>(b) * K + j;
        const float qlse = kGreedy ? MQ : (MQ * cT + log2f(SQ)) * 0.6931471805599453f;
        a.Z[o] = ok ? Z : __int_as_float(0x7FC00000);
        a.q_lse[o] = ok ? qlse : __int_as_float(0x7FC00000);
        if (a.draft_tokens) a.draft_tokens[o] = ok ? drawn : -1;
      }
      UnitRes res;
      res.a = acc;
      res.R = Rout;
      res.draw = drawn;
      res.flags = fl;
      res.amargin = amargin;
      res.bmargin = bmargin;
      res.rejected = rejected;
      res.seg_slot = lc.seg_slot;
      a.units[static_cast<long long>(b) * (K + 1) + j] = res;
      __threadfence();  // the unit result is visible before this unit's arrival
      const int old = atomicAdd(a.counters + b, 1);
      lc.is_last = old == a.units_per_row - 1;
    }
  }
  // Segment tokens of this outcome (rank 0 holds the selection in every path).
  if (rank == 0) {
    int32_t* segdst = nullptr;
    if (verify) {
      if (a.c_tokens && !plan_bad) segdst = a.c_tokens + static_cast<long long>(b) * a.budget + seg_off;
    } else if (!plan_bad) {
      segdst = a.topf_tokens + static_cast<long long>(b) * a.budget + seg_off;
    }
    if (segdst && has_plan)
      for (int i = tid; i < Fj; i += kThreads) segdst[i] = valid ? sel[i].idx : -1;
  }
  __syncthreads();

  if (rank == owner && lc.is_last) {
    __threadfence();
    // ---- row epilogue (last unit of row b) -------------------------------------------
    const UnitRes* ur = a.units + static_cast<long long>(b) * (K + 1);
    if (tid == 0) {
      int fl = 0;
      for (int k = 0; k < a.units_per_row; ++k) fl |= __ldcg(&ur[k].flags);
      lc.flags = fl;
    }
    __syncthreads();
    const int rowflags = lc.flags;
    const bool row_invalid = (rowflags & SSD_ROW_INVALID) != 0;
    if (verify) {
      if (tid == 0) {
        int kstar = K;
        float am = INFINITY;
        for (int k = 0; k < K; ++k) {
          am = fminf(am, __ldcg(&ur[k].amargin));
          if (__ldcg(&ur[k].rejected)) { kstar = k; break; }
        }
        int fl = rowflags;
        const int drawn = __ldcg(&ur[kstar].draw);
        const float bm = __ldcg(&ur[kstar].bmargin);
        if (!kGreedy && (am < kNearTie || bm < kNearTie)) fl |= SSD_ROW_NEAR_TIE;
        // only the zero-residual flag of the unit that produced the bonus counts
        fl &= ~SSD_ROW_ZERO_RESIDUAL;
        fl |= __ldcg(&ur[kstar].flags) & SSD_ROW_ZERO_RESIDUAL;
        a.status[b] = fl;
        a.n_accepted[b] = row_invalid ? -1 : kstar;
        a.bonus[b] = row_invalid ? -1 : drawn;
        a.residual_mass[b] = row_invalid ? __int_as_float(0x7FC00000) : __ldcg(&ur[kstar].R);
        lc.cstar = kstar;
        lc.seg_slot = row_invalid ? -1 : __ldcg(&ur[kstar].seg_slot);
      }
      __syncthreads();
      const int kstar = lc.cstar;
      if (tid <= K) {
        int32_t t = -1;
        if (!row_invalid) t = tid < kstar ? __ldg(a.tokens + static_cast<long long>(b) * K + tid)
                                          : (tid == kstar ? __ldcg(&ur[kstar].draw) : -1);
        a.out_tokens[static_cast<long long>(b) * (K + 1) + tid] = t;
      }
      if (row_invalid)
        for (int k = tid; k < K; k += kThreads) a.accept_prob[static_cast<long long>(b) * K + k] = __int_as_float(0x7FC00000);
      if (a.c_tokens) {
        const bool pbad = (rowflags & SSD_ROW_BAD_PLAN) != 0;
        if (tid == 0) {
          int off = 0;
          a.c_offsets[static_cast<long long>(b) * (K + 2)] = 0;
          for (int k = 0; k <= K; ++k) {
            off += pbad ? 0 : s_F[k];
            a.c_offsets[static_cast<long long>(b) * (K + 2) + k + 1] = off;
          }
        }
        if (row_invalid)
          for (int s2 = tid; s2 < a.budget; s2 += kThreads) a.c_tokens[static_cast<long long>(b) * a.budget + s2] = -1;
        int slot = -1;
        if (lc.seg_slot >= 0) {
          int off = 0;
          for (int k = 0; k < kstar; ++k) off += s_F[k];
          slot = off + lc.seg_slot;
        }
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
    } else {
      if (tid == 0) {
        int fl = rowflags;
        if (!kGreedy) {
          for (int k = 0; k < K; ++k)
            if (__ldcg(&ur[k].bmargin) < kNearTie) fl |= SSD_ROW_NEAR_TIE;
        }
        a.status[b] = fl;
        const bool pbad = (rowflags & SSD_ROW_BAD_PLAN) != 0;
        int off = 0;
        a.offsets[static_cast<long long>(b) * (K + 2)] = 0;
        for (int k = 0; k <= K; ++k) {
          off += pbad ? 0 : s_F[k];
          a.offsets[static_cast<long long>(b) * (K + 2) + k + 1] = off;
        }
      }
    }
    if (tid == 0) {
      a.counters[b] = 0;
      a.first_rej[b] = 0;
    }
  }
  // A CTA leaves only after every CTA of the cluster is done reading its
  // shared memory, and never with a bulk copy in flight.
  if constexpr (kAligned) {
    if (tmo && tid == 0)
      for (int c = max(0, n_issued - kStages); c < n_issued; ++c)
        mbar_wait_bounded(&lc.full[c % kStages], (c / kStages) & 1, kMaxPolls);
  }
  cluster_wait();
}

}  // namespace ssd
