// ssd_cluster.cuh -- the verify step as one kernel of CTA clusters.
//
// A unit is one (row b, position j) pair: the target row p_j and, for j < K,
// the draft row q_j (for j = K, `draft_next` when given).  The unit's CS CTAs
// (a thread-block cluster) split the vocabulary into CS slices of L tokens;
// CTA r streams tokens [r L, r L + L) of both rows from HBM through a ring of
// 1-D bulk copies into shared memory (no multicast), as the two-kernel form's
// statistics CTAs do, so five CTAs fit on an SM.  The cluster then exchanges
// small records over distributed shared memory (DSMEM) between hardware
// cluster barriers; no CTA polls a flag that another cluster writes, and no
// second kernel is scheduled:
//   1. the stream: online max / sum of exp2 of both rows per thread, and the
//      three largest vector maxima of the top-F source row with the two
//      vectors holding the largest ([ZH] = "Speculative Speculative Decoding",
//      gist.science Chinese edition, technical summary section 1 and section
//      2 step 2; [NL] = the Dutch edition, section 2);
//   2. the slice's own top-F_j candidates (the F-th largest thread maximum
//      bounds them from below), sorted, published with the slice statistics;
//      every warp merges the CS records in one fixed butterfly, so every CTA
//      holds bit-identical unit statistics, and every CTA ranks the gathered
//      candidates at or above the largest slice bound by (logit desc, token id
//      asc): the top-F_j of q_j ([ZH] section 2 challenge 2; [NL] 3B).  When a
//      slice's candidates overflow, an exact bitwise select over 16-bit order
//      keys across the cluster finds the F-th largest key instead, ties taken
//      in token order;
//   3. Q_S, the Saguaro normaliser Z = 1 - (1 - C) Q_S and the lossless accept
//      test a_j = min(1, p_j(d_j) / q'_j(d_j)), u_j < a_j, computed identically
//      by every CTA;
//   4. a unit that rejects (and unit K, whose p_K serves full acceptance)
//      draws its bonus candidate at once: the residual r = max(0, p_j - q'_j)
//      (or p_K) is summed per (256-vector chunk, warp) in token order over a
//      second pass of the slice through the same ring (read again a few
//      microseconds after the first pass, mostly from L2); the slice masses are
//      exchanged and the CTA holding the crossing of u_K * R finds the token;
//   5. the unit's leader (the crossing CTA, else CTA 0) writes a_j, the cache
//      segment ([ZH] section 2 step 3) and the unit's record, then arrives on
//      the row's counter; the row's last unit takes k* = the first rejected
//      position and the bonus of unit k*, and writes the row's outputs, the
//      cache lookup of (k*, bonus) and the random-token fallback ([ZH] section
//      2 step 4 and challenge 3; [NL] 3C).
#pragma once

#include "ssd_kernels.cuh"

namespace ssd {

constexpr int kClMaxCS = 16;                      // CTAs per cluster at most (kMaxSlices)
constexpr int kClChunks = kMaxChunks;             // token-order chunks of 256 vectors per slice
constexpr int kClCandCap = 256;                   // candidates a CTA holds (>= the largest F_j)
constexpr int kClGatherCap = 512;                 // candidates of a whole unit kept for ranking
constexpr int kClStages = kStatsStages;           // ring stages (kStatsChunkVecs vectors per row each)
#ifndef SSD_CL_MIN_BLOCKS
#define SSD_CL_MIN_BLOCKS 5
#endif
constexpr int kClMinBlocks = SSD_CL_MIN_BLOCKS;
static_assert(kClMaxCS <= kMaxSlices, "a cluster is at most the slice plan's width");
static_assert(kStatsChunkVecs == 2 * kThreads, "a ring stage holds two token-order chunks per row");

// One CTA's published values, read by the rest of its cluster over DSMEM.
// Every field is written once per call (cnt alternates between two words).
struct __align__(16) ClSlot {
  float mP, sP, mQ, sQ;  // slice maxima and exp-sums (relative to the maxima)
  float tau, xdP, xdQ;   // slice top-F bound; logits of the drafted token (the CTA holding it)
  int32_t tmo;
  float R, R2;           // draw: slice mass (R2: of p, when the residual is 0)
  int32_t n_cand, over;  // sorted candidates published; the local list overflowed
  int32_t skip;          // CTA 0: an earlier position of the row has rejected
  int32_t cnt[2], cgt, ceq;  // exact select: counts per bisection round, > and == the threshold
  Cand cand[kClCandCap];
};

// Per unit, written by the unit's leader and read by the row's last unit.
struct UnitOut {
  float a, amargin, R, dmargin;  // a_j, |u_j - a_j|, draw mass, bonus margin / mass
  int32_t flags, rejected, drawn, use_p;
};

struct ClSmem {
  uint64_t full[kClStages];
  uint32_t rel[kClStages];
  ClSlot slot;
  Cand gbuf[kClGatherCap];
  Cand sel[kClCandCap];
  float gmax[kThreads];
  float wred[kWarps][4];
  float rs[kClChunks][kWarps];
  int32_t wcnt[kWarps][2];
  int32_t coff[kClMaxCS + 1];
  int32_t s_F[SSD_MAX_K + 1];
  int32_t plan_bad, Fj, seg_off, d_tok, n_raw, n_keep, is_last, slot_out, drawn, kstar, rflags, use_p, slow;
  float u_self, u_bonus, dmargin, total, amargin, xdP0, xdQ0, tau_c;
};

__device__ __forceinline__ void cl_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cl_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }
__device__ __forceinline__ void cl_sync() {
  cl_arrive();
  cl_wait();
}

// 16-bit order key of a bf16 logit (the high half of ord_key of its float).
__device__ __forceinline__ uint32_t key16(uint32_t h) {
  h &= 0xFFFFu;
  if (h == 0x8000u) h = 0u;  // -0 ties with +0
  return (h & 0x8000u) ? (~h & 0xFFFFu) : (h | 0x8000u);
}

// Sum of a per-thread count over the CTA (every thread calls it and gets the
// result).  `which` picks one of two scratch words.
__device__ __forceinline__ int cta_sum(ClSmem& sm, int v, int warp, int lane, int which) {
  v = static_cast<int>(__reduce_add_sync(0xFFFFFFFFu, static_cast<unsigned>(v)));
  if (lane == 0) sm.wcnt[warp][which] = v;
  __syncthreads();
  int s = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) s += sm.wcnt[w][which];
  return s;
}

// One CTA of the cluster of unit u = blockIdx.x / CS.
__global__ void __launch_bounds__(kThreads, kClMinBlocks) ssd_cluster_kernel(const __grid_constant__ Args a) {
  extern __shared__ __align__(128) unsigned char ring_buf[];
  __shared__ __align__(16) ClSmem sm;
  cg::cluster_group cl = cg::this_cluster();

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int CS = a.cl_size;
  const int crank = static_cast<int>(cl.block_rank());
  const long long u = blockIdx.x / CS;
  const int upr = a.units_per_row, K = a.K, V = a.V;
  const int b = static_cast<int>(u / upr), j = static_cast<int>(u % upr);
  const int L = a.cl_len;
  const int e0 = crank * L;
  const int e1 = min(V, e0 + L);
  const int nvec = max(0, e1 - e0) >> 3;  // V and L are multiples of 8
  const int nch = (nvec + kStatsChunkVecs - 1) / kStatsChunkVecs;  // ring chunks of the slice

  const uint16_t *baseP, *baseQ;
  long long rbP, rbQ;
  unit_rows<uint16_t>(a, b, j, baseP, rbP, baseQ, rbQ);
  const bool hasQ = baseQ != nullptr;
  const bool srcQ = hasQ;  // the top-F source row: q_j, else p_K
  const bool has_d = j < K;
  const uint16_t* const rowP = baseP + rbP;
  const uint16_t* const rowQ = hasQ ? baseQ + rbQ : nullptr;
  const uint16_t* const rowS = srcQ ? rowQ : rowP;

  // The ring: stage s holds kStatsChunkVecs vectors of row P (half 0) and of
  // row Q (half 1).  Pass chunk c of a pass that starts after `base` chunks
  // uses stage (base + c) % kClStages with phase parity ((base + c) /
  // kClStages) & 1, so later passes reuse the barriers without re-arming them.
  auto stage = [&](int slot, int r) -> unsigned char* {
    return ring_buf + (static_cast<size_t>(slot) * 2 + r) * (kStatsChunkVecs * 16);
  };
  auto issue = [&](int base, int c, int rows, uint64_t pol) {
    const int slot = (base + c) % kClStages;
    const int v0 = (base > 0 ? nch - 1 - c : c) * kStatsChunkVecs;  // later passes run backwards
    const uint32_t bytes = static_cast<uint32_t>(min(kStatsChunkVecs, nvec - v0)) * 16u;
    mbar_arrive_expect_tx(&sm.full[slot], bytes * static_cast<uint32_t>(rows));
    bulk_copy_g2s_hint(stage(slot, 0), rowP + e0 + v0 * 8, bytes, &sm.full[slot], pol);
    if (rows > 1) bulk_copy_g2s_hint(stage(slot, 1), rowQ + e0 + v0 * 8, bytes, &sm.full[slot], pol);
  };
  auto acquire = [&](int base, int c, int& tmo_) {
    const int k = base + c;
    if (!mbar_wait_bounded(&sm.full[k % kClStages], static_cast<uint32_t>(k / kClStages) & 1u, kRingWaitNs)) tmo_ = 1;
  };
  // this warp is done with the chunk's stage; the last warp to say so refills it
  auto release = [&](int base, int c, int nchunks, int rows, uint64_t pol) {
    __syncwarp();
    if (lane == 0) {
      const int slot = (base + c) % kClStages;
      if (atom_add_acq_rel_cta_shared(&sm.rel[slot], 1u) == static_cast<uint32_t>(kWarps - 1)) {
        sm.rel[slot] = 0u;
        fence_proxy_async_shared();
        if (c + kClStages < nchunks) issue(base, c + kClStages, rows, pol);
      }
    }
  };
  const uint64_t pol_keep = l2_policy_evict_normal();  // the draw may read the slice again soon
  const uint64_t pol_last = l2_policy_evict_first();
  const int rows1 = hasQ ? 2 : 1;
  if (tid == 0) {
    for (int s = 0; s < kClStages; ++s) {
      mbar_init(&sm.full[s], 1);
      sm.rel[s] = 0u;
    }
    mbar_init_fence();
    for (int c = 0; c < min(kClStages, nch); ++c) issue(0, c, rows1, pol_keep);
  }
  // The row's fan-out plan (warp 1) and the unit's scalars (warp 2), while the
  // first chunks are in flight.
  const bool has_plan = a.F != nullptr || a.alpha != nullptr;
  if (warp == 1) {
    int fplan[2] = {0, 0};
    if (has_plan) {
      if (a.F) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int k = lane + 32 * h;
          if (k <= K) fplan[h] = __ldg(a.F + static_cast<long long>(b) * (K + 1) + k);
        }
      } else {
        const float al = (a.fanout_mode == SSD_FANOUT_UNIFORM) ? 0.f : __ldg(a.alpha + b);
        fanout_warp(al, K, a.budget, a.fanout_mode, lane, fplan);
      }
    }
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
      const int pb = (has_plan && (bad || sum != a.budget)) ? 1 : 0;
      sm.plan_bad = pb;
      sm.Fj = (pb || !has_plan) ? 0 : fj;
      sm.seg_off = pre;
    }
  } else if (warp == 2 && lane == 0) {
    const int d0 = has_d ? __ldg(a.tokens + static_cast<long long>(b) * K + j) : -1;
    float xp = 0.f, xq = 0.f;
    if (has_d && d0 >= e0 && d0 < e1) {  // the drafted token's logits, for the accept test
      xp = __uint_as_float(static_cast<uint32_t>(__ldg(rowP + d0)) << 16);
      xq = __uint_as_float(static_cast<uint32_t>(__ldg(rowQ + d0)) << 16);
    }
    sm.d_tok = d0;
    sm.xdP0 = xp;
    sm.xdQ0 = xq;
    sm.u_self = __ldg(a.uniforms + static_cast<long long>(b) * (K + 1) + j);
    sm.u_bonus = __ldg(a.uniforms + static_cast<long long>(b) * (K + 1) + K);
    sm.n_raw = 0;
    sm.n_keep = 0;
  }
  __syncthreads();  // barriers initialised; plan and scalars in shared memory

  // ---- the stream: online max / exp-sum of both rows, top vectors of the source ----
  const float cT = kLog2e / a.T;
  const f32x2 cT2 = f2_pack(cT, cT);
  float mP = -INFINITY, mQ = -INFINITY;
  f32x2 sP2 = 0ull, sQ2 = 0ull, nmP2 = 0ull, nmQ2 = 0ull;
  int tmo = 0;
  float vm1 = -INFINITY, vm2 = -INFINITY, vm3 = -INFINITY;  // top three vector maxima of the source row
  int g1k = -1, g2k = -1;
  uint4 keep1 = make_uint4(0u, 0u, 0u, 0u), keep2 = keep1;  // the source vectors holding vm1, vm2
  auto track = [&](float vsrc, const uint4& wsrc, int g) {
    if (vsrc > vm3) {
      if (vsrc > vm2) {
        vm3 = vm2;
        if (vsrc > vm1) { vm2 = vm1; keep2 = keep1; g2k = g1k; vm1 = vsrc; g1k = g; keep1 = wsrc; }
        else { vm2 = vsrc; g2k = g; keep2 = wsrc; }
      } else {
        vm3 = vsrc;
      }
    }
  };
  const uint4 neg = make_uint4(0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u);
  for (int c = 0; c < nch; ++c) {
    acquire(0, c, tmo);
    const int g0 = c * kStatsChunkVecs + tid, g1 = g0 + kThreads;
    const bool ok0 = g0 < nvec, ok1 = g1 < nvec;
    const int slot = c % kClStages;
    const uint4* hp = reinterpret_cast<const uint4*>(stage(slot, 0));
    const uint4 wp0 = ok0 ? hp[tid] : neg, wp1 = ok1 ? hp[tid + kThreads] : neg;
    float vp0, vp1, vq0 = -INFINITY, vq1 = -INFINITY;
    consume2_bf16(wp0, wp1, ok0, ok1, cT, cT2, mP, sP2, nmP2, vp0, vp1);
    uint4 wq0 = neg, wq1 = neg;
    if (hasQ) {
      const uint4* hq = reinterpret_cast<const uint4*>(stage(slot, 1));
      wq0 = ok0 ? hq[tid] : neg;
      wq1 = ok1 ? hq[tid + kThreads] : neg;
      consume2_bf16(wq0, wq1, ok0, ok1, cT, cT2, mQ, sQ2, nmQ2, vq0, vq1);
    }
    if (ok0) track(srcQ ? vq0 : vp0, srcQ ? wq0 : wp0, g0);
    if (ok1) track(srcQ ? vq1 : vp1, srcQ ? wq1 : wp1, g1);
    release(0, c, nch, rows1, pol_keep);
  }
  float sPs, sQs;
  {
    float lo, hi;
    f2_unpack(sP2, lo, hi);
    sPs = lo + hi;
    f2_unpack(sQ2, lo, hi);
    sQs = lo + hi;
  }
  // the warp's maxima first, then every lane rescales its sum once to them
  {
    float wmP = mP, wmQ = mQ;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      wmP = fmax_nan(wmP, __shfl_xor_sync(0xFFFFFFFFu, wmP, o));
      wmQ = fmax_nan(wmQ, __shfl_xor_sync(0xFFFFFFFFu, wmQ, o));
    }
    sPs = (mP == -INFINITY) ? 0.f : sPs * ex2((mP - wmP) * cT);
    sQs = (mQ == -INFINITY) ? 0.f : sQs * ex2((mQ - wmQ) * cT);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sPs += __shfl_xor_sync(0xFFFFFFFFu, sPs, o);
      sQs += __shfl_xor_sync(0xFFFFFFFFu, sQs, o);
    }
    if (lane == 0) {
      sm.wred[warp][0] = wmP; sm.wred[warp][1] = sPs;
      sm.wred[warp][2] = wmQ; sm.wred[warp][3] = sQs;
    }
  }
  sm.gmax[tid] = vm1;
  const int tmo_cta = __syncthreads_or(tmo);
  const int d = sm.d_tok;
  const int Fj = sm.Fj;
  const int plan_bad = sm.plan_bad;
  const bool fast_ok = has_plan && Fj > 0;  // Fj <= kClCandCap: the host routes larger budgets elsewhere
  if (warp == 0) {
    float m1 = -INFINITY, s1 = 0.f, m2 = -INFINITY, s2 = 0.f;
    if (lane < kWarps) { m1 = sm.wred[lane][0]; s1 = sm.wred[lane][1]; m2 = sm.wred[lane][2]; s2 = sm.wred[lane][3]; }
#pragma unroll
    for (int o = kWarps / 2; o > 0; o >>= 1) {
      merge_ms(m1, s1, __shfl_xor_sync(0xFFFFFFFFu, m1, o), __shfl_xor_sync(0xFFFFFFFFu, s1, o), cT);
      merge_ms(m2, s2, __shfl_xor_sync(0xFFFFFFFFu, m2, o), __shfl_xor_sync(0xFFFFFFFFu, s2, o), cT);
    }
    if (lane == 0) {
      sm.slot.mP = m1; sm.slot.sP = s1; sm.slot.mQ = m2; sm.slot.sQ = s2;
      sm.slot.tmo = tmo_cta;
      sm.slot.xdP = sm.xdP0;
      sm.slot.xdQ = sm.xdQ0;
    }
  } else if (warp == 1) {
    // the F-th largest of the thread maxima bounds the slice's own top-F from below
    float t = -INFINITY;
    if (fast_ok) {
      uint32_t keys[kThreads / 32];
#pragma unroll
      for (int i = 0; i < kThreads / 32; ++i) keys[i] = ord_key(sm.gmax[lane + 32 * i]);
      t = key_to_float(warp_kth_largest(keys, Fj, 16));
    }
    if (lane == 0) {
      sm.tau_c = t;
      sm.slot.tau = t;
    }
  }
  __syncthreads();
  // The slice's candidates: its elements at or above its bound, into the idle
  // ring.  A thread whose third vector maximum is below the bound holds them
  // all in its two kept vectors; otherwise it reads its vectors again.
  Cand* const raw = reinterpret_cast<Cand*>(ring_buf);
  {
    const float tc = sm.tau_c;
    auto take = [&](const uint4& w, int g) {
      float x[8];
      Elem<uint16_t>::unpack(w, x);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (x[i] >= tc) {
          const int pos = atomicAdd(&sm.n_raw, 1);
          if (pos < kClCandCap) raw[pos] = Cand{x[i], e0 + g * 8 + i};
        }
      }
    };
    if (fast_ok && vm1 >= tc && vm1 == vm1) {
      if (vm3 < tc) {
        take(keep1, g1k);
        if (vm2 >= tc && g2k >= 0) take(keep2, g2k);
      } else {
        for (int g = tid; g < nvec; g += kThreads) take(ld_vec(rowS + e0 + g * 8), g);
      }
    }
  }
  __syncthreads();
  {
    // sorted by (logit desc, id asc); the first min(count, F_j) are published
    const int nr = min(sm.n_raw, kClCandCap);
    const int keepn = min(nr, Fj);
    for (int i = tid; i < nr; i += kThreads) {
      const Cand ci = raw[i];
      const unsigned long long key = rank_key(ci.x, ci.idx);
      int r = 0;
      for (int k2 = 0; k2 < nr; ++k2) r += rank_key(raw[k2].x, raw[k2].idx) > key;
      if (r < keepn) sm.slot.cand[r] = ci;
    }
    if (tid == 0) {
      sm.slot.n_cand = keepn;
      sm.slot.over = sm.n_raw > kClCandCap ? 1 : 0;
    }
  }
  cl_sync();  // B1: every slice's statistics and candidates published

  // ---- the unit's statistics: every warp merges the CS records in one butterfly -----
  float MP, SP, MQ, SQ, tau, xdP, xdQ;
  int tmo_any;
  {
    float mp = -INFINITY, sp = 0.f, mq = -INFINITY, sq = 0.f, ta = -INFINITY, xp = 0.f, xq = 0.f;
    int to = 0;
    if (lane < CS) {
      const ClSlot* r = cl.map_shared_rank(&sm.slot, lane);
      const float4 s0 = *reinterpret_cast<const float4*>(&r->mP);
      const float4 s1 = *reinterpret_cast<const float4*>(&r->tau);
      mp = s0.x; sp = s0.y; mq = s0.z; sq = s0.w;
      ta = s1.x; xp = s1.y; xq = s1.z; to = __float_as_int(s1.w);
    }
    const int cd = (has_d && d >= 0 && d < V) ? d / L : 0;  // the slice holding d
    xdP = __shfl_sync(0xFFFFFFFFu, xp, cd);
    xdQ = __shfl_sync(0xFFFFFFFFu, xq, cd);
#pragma unroll
    for (int o = kClMaxCS / 2; o > 0; o >>= 1) {
      merge_ms(mp, sp, __shfl_xor_sync(0xFFFFFFFFu, mp, o), __shfl_xor_sync(0xFFFFFFFFu, sp, o), cT);
      merge_ms(mq, sq, __shfl_xor_sync(0xFFFFFFFFu, mq, o), __shfl_xor_sync(0xFFFFFFFFu, sq, o), cT);
    }
    MP = __shfl_sync(0xFFFFFFFFu, mp, 0); SP = __shfl_sync(0xFFFFFFFFu, sp, 0);
    MQ = __shfl_sync(0xFFFFFFFFu, mq, 0); SQ = __shfl_sync(0xFFFFFFFFu, sq, 0);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ta = fmaxf(ta, __shfl_xor_sync(0xFFFFFFFFu, ta, o));
    tau = ta;
    tmo_any = __any_sync(0xFFFFFFFFu, to != 0) ? 1 : 0;
  }
  int flags = 0, pflags = 0;
  const float u_self = sm.u_self;
  if (!(u_self >= 0.f && u_self < 1.f)) flags |= SSD_ROW_BAD_UNIFORM;
  if (has_d && (d < 0 || d >= V)) flags |= SSD_ROW_BAD_TOKEN;
  if (plan_bad) flags |= SSD_ROW_BAD_PLAN;
  if (tmo_any) flags |= kFlagTimeout;
  // a non-finite target row and q'(d_j) = 0 are kept apart (pflags), as in the
  // two-kernel form
  if (!(MP > -INFINITY && MP < INFINITY)) pflags |= SSD_ROW_NONFINITE;
  if (hasQ && !(MQ > -INFINITY && MQ < INFINITY)) flags |= SSD_ROW_NONFINITE;
  const bool valid = ((flags | pflags) & SSD_ROW_INVALID) == 0;
  const bool valid_src = ((flags | (srcQ ? 0 : pflags)) & SSD_ROW_INVALID) == 0;
  const bool want_topf = fast_ok && valid_src;  // the same in every CTA of the cluster

  // ---- top-F_j of the source row -----------------------------------------------------
  if (want_topf) {
    if (warp == 0) {
      int c = 0, ov = 0;
      if (lane < CS) {
        const ClSlot* r = cl.map_shared_rank(&sm.slot, lane);
        c = r->n_cand;
        ov = r->over;
      }
      const bool any_over = __any_sync(0xFFFFFFFFu, ov != 0);
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
      }
      if (lane < CS) sm.coff[lane + 1] = incl;
      if (lane == 0) {
        sm.coff[0] = 0;
        sm.slow = any_over ? 1 : 0;
      }
    }
    __syncthreads();
    bool slow = sm.slow != 0;
    if (!slow) {
      // every slice's published candidates at or above the largest slice bound
      // (a superset of the unit's top-F)
      const int total = sm.coff[CS];
      for (int i = tid; i < total; i += kThreads) {
        int c = 0;
        while (c + 1 < CS && sm.coff[c + 1] <= i) ++c;
        const Cand e = cl.map_shared_rank(&sm.slot.cand[0], c)[i - sm.coff[c]];
        if (e.x >= tau) {
          const int pos = atomicAdd(&sm.n_keep, 1);
          if (pos < kClGatherCap) sm.gbuf[pos] = e;
        }
      }
      __syncthreads();
      slow = sm.n_keep > kClGatherCap || sm.n_keep < Fj;
    }
    if (slow) {
      // Exact select across the cluster: the largest 16-bit key t with at
      // least F_j keys >= t, found bit by bit (one cluster round per bit),
      // then every key above t and the first ties in token order.
      uint32_t thr = 0u;
      for (int bit = 15; bit >= 0; --bit) {
        const uint32_t cand = thr | (1u << bit);
        int c = 0;
        for (int g = tid; g < nvec; g += kThreads) {
          const uint4 w = ld_vec(rowS + e0 + g * 8);
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) c += (key16(ws[h]) >= cand) + (key16(ws[h] >> 16) >= cand);
        }
        c = cta_sum(sm, c, warp, lane, bit & 1);
        if (tid == 0) sm.slot.cnt[bit & 1] = c;
        cl_sync();
        int tot = lane < CS ? cl.map_shared_rank(&sm.slot, lane)->cnt[bit & 1] : 0;
        tot = static_cast<int>(__reduce_add_sync(0xFFFFFFFFu, static_cast<unsigned>(tot)));
        if (tot >= Fj) thr = cand;
      }
      int cgt = 0, ceq = 0;
      for (int g = tid; g < nvec; g += kThreads) {
        const uint4 w = ld_vec(rowS + e0 + g * 8);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const uint32_t k0 = key16(ws[h]), k1 = key16(ws[h] >> 16);
          cgt += (k0 > thr) + (k1 > thr);
          ceq += (k0 == thr) + (k1 == thr);
        }
      }
      cgt = cta_sum(sm, cgt, warp, lane, 0);
      ceq = cta_sum(sm, ceq, warp, lane, 1);
      if (tid == 0) {
        sm.slot.cgt = cgt;
        sm.slot.ceq = ceq;
        sm.n_raw = 0;
      }
      cl_sync();
      int gt = 0, eq = 0;
      if (lane < CS) {
        const ClSlot* r = cl.map_shared_rank(&sm.slot, lane);
        gt = r->cgt;
        eq = r->ceq;
      }
      const int G = static_cast<int>(__reduce_add_sync(0xFFFFFFFFu, static_cast<unsigned>(gt)));
      const int eq_before =
          static_cast<int>(__reduce_add_sync(0xFFFFFFFFu, static_cast<unsigned>(lane < crank ? eq : 0)));
      const int quota = max(0, min(ceq, Fj - G - eq_before));  // this slice's ties, lowest ids first
      // every key above the threshold (fewer than F_j in the whole unit)
      for (int g = tid; g < nvec; g += kThreads) {
        const uint4 w = ld_vec(rowS + e0 + g * 8);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t hw = (i & 1) ? (ws[i >> 1] >> 16) : ws[i >> 1];
          if (key16(hw) > thr) {
            const int pos = atomicAdd(&sm.n_raw, 1);
            if (pos < kClCandCap) sm.slot.cand[pos] = Cand{__uint_as_float((hw & 0xFFFFu) << 16), e0 + g * 8 + i};
          }
        }
      }
      __syncthreads();
      if (warp == 0) {  // the ties, in token order, up to the quota
        const int base_n = min(sm.n_raw, kClCandCap);
        int taken = 0;
        for (int g0 = 0; g0 < nvec && taken < quota; g0 += 32) {
          const int g = g0 + lane;
          uint4 w = make_uint4(0u, 0u, 0u, 0u);
          int c = 0;
          if (g < nvec) {
            w = ld_vec(rowS + e0 + g * 8);
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) c += (key16(ws[h]) == thr) + (key16(ws[h] >> 16) == thr);
          }
          int incl = c;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += y;
          }
          int pos = taken + incl - c;
          if (c > 0) {
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
            for (int i = 0; i < 8; ++i) {
              const uint32_t hw = (i & 1) ? (ws[i >> 1] >> 16) : ws[i >> 1];
              if (key16(hw) == thr) {
                if (pos < quota && base_n + pos < kClCandCap)
                  sm.slot.cand[base_n + pos] = Cand{__uint_as_float((hw & 0xFFFFu) << 16), e0 + g * 8 + i};
                ++pos;
              }
            }
          }
          taken += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
        if (lane == 0) {
          sm.slot.n_cand = min(base_n + quota, kClCandCap);
          sm.slot.over = 0;
        }
      }
      cl_sync();  // the exact sets published
      if (warp == 0) {
        const int c = lane < CS ? cl.map_shared_rank(&sm.slot, lane)->n_cand : 0;
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
          if (lane >= o) incl += y;
        }
        if (lane < CS) sm.coff[lane + 1] = incl;
        if (lane == 0) sm.coff[0] = 0;
      }
      __syncthreads();
      const int total = min(sm.coff[CS], kClGatherCap);
      for (int i = tid; i < total; i += kThreads) {
        int c = 0;
        while (c + 1 < CS && sm.coff[c + 1] <= i) ++c;
        sm.gbuf[i] = cl.map_shared_rank(&sm.slot.cand[0], c)[i - sm.coff[c]];
      }
      if (tid == 0) sm.n_keep = total;
      __syncthreads();
    }
    // rank the kept candidates by (logit desc, id asc): the first F_j are the set
    const int nk = min(sm.n_keep, kClGatherCap);
    for (int i = tid; i < nk; i += kThreads) {
      const Cand ci = sm.gbuf[i];
      const unsigned long long key = rank_key(ci.x, ci.idx);
      int r = 0;
      for (int k2 = 0; k2 < nk; ++k2) r += rank_key(sm.gbuf[k2].x, sm.gbuf[k2].idx) > key;
      if (r < Fj) sm.sel[r] = ci;
    }
    __syncthreads();
  }

  // ---- Q_S, the Saguaro normaliser and the accept test (every warp, same result) -----
  const float nmP = -MP * cT, nmQ = -MQ * cT;
  const float C = a.C;
  float Z = 1.f, bx = INFINITY;
  int bi = -1;
  if (want_topf) {
    float qs = 0.f;
    for (int r = lane; r < Fj; r += 32) qs += ex2(fmaf(sm.sel[r].x, cT, srcQ ? nmQ : nmP));
    qs = warp_sum(qs);
    Z = 1.f - (1.f - C) * (qs / (srcQ ? SQ : SP));
    bx = sm.sel[Fj - 1].x;
    bi = sm.sel[Fj - 1].idx;
  }
  float acc = 0.f, amargin = INFINITY;
  int rejected = 0;
  if (has_d && valid) {
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

  // ---- the draw of this unit's bonus candidate: a second pass through the ring -------
  // Only the row's first rejected position (else K) draws for the row.  A
  // rejecting unit says so at once in the workspace, and a unit about to draw
  // skips its draw when an earlier position of its row has already said so:
  // then k* < j.  A flag not yet visible only costs a draw that is not used.
  int32_t* const rej_flags = a.arrive1 + static_cast<long long>(b) * upr;
  if (crank == 0 && tid == 0 && has_d && valid && rejected) st_relaxed_gpu_u32(rej_flags + j, 1);
  bool do_draw = valid && (!has_d || rejected);  // the same in every CTA
  if (do_draw && j > 0) {
    if (crank == 0 && warp == 0) {
      const bool earlier = lane < j && ld_relaxed_gpu_u32(rej_flags + lane) != 0;
      const bool earlier2 = lane + 32 < j && ld_relaxed_gpu_u32(rej_flags + lane + 32) != 0;
      const bool skip = __any_sync(0xFFFFFFFFu, earlier || earlier2);
      if (lane == 0) sm.slot.skip = skip ? 1 : 0;
    }
    cl_sync();  // CTA 0's decision, read by all
    do_draw = cl.map_shared_rank(&sm.slot, 0)->skip == 0;
  }
  int mode = has_d ? kDrawResidual : kDrawP;
  float total = 1.f;
  int use_p = 0, cstar = 0;
  float tl = 0.f;
  const int nchd = (nvec + kThreads - 1) / kThreads;  // token-order chunks of 256 vectors
  const float invSP = 1.f / SP, wS = C / (SQ * Z), wN = 1.f / (SQ * Z);
  const bool check_S = want_topf && has_d;
  const uint4 zero4 = make_uint4(0u, 0u, 0u, 0u);
  int base = nch;  // ring chunks served so far
  auto draw_pass = [&](int md) -> float {
    const int rows = (md == kDrawResidual) ? 2 : 1;
    fence_proxy_async_shared();  // this thread's generic uses of the ring come before the copies
    __syncthreads();
    if (tid == 0)
      for (int c = 0; c < min(kClStages, nch); ++c) issue(base, c, rows, pol_last);
    for (int c = 0; c < nch; ++c) {
      acquire(base, c, tmo);
      const int slot = (base + c) % kClStages;
      const uint4* hp = reinterpret_cast<const uint4*>(stage(slot, 0));
      const uint4* hq = reinterpret_cast<const uint4*>(stage(slot, 1));
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int cd = nch - 1 - c;  // the data chunk: backwards, the most recently streamed first
        const int g = cd * kStatsChunkVecs + h * kThreads + tid;
        float rsum = 0.f;
        if (g < nvec) {
          float val[8], pv[8];
          draw_vals_bf16(md, hp[h * kThreads + tid], rows > 1 ? hq[h * kThreads + tid] : zero4, e0 + g * 8, cT, nmP,
                         nmQ, invSP, wS, wN, check_S, bx, bi, false, val, pv);
#pragma unroll
          for (int i = 0; i < 8; ++i) rsum += val[i];
        }
        rsum = warp_sum(rsum);
        if (lane == 0) sm.rs[2 * cd + h][warp] = rsum;
      }
      release(base, c, nch, rows, pol_last);
    }
    base += nch;
    const int tmo_now = __syncthreads_or(tmo);
    float R = 0.f;
    for (int i = lane; i < nchd * kWarps; i += 32) R += sm.rs[i / kWarps][i % kWarps];
    R = warp_sum(R);
    return tmo_now ? __int_as_float(0x7FC00000) : R;  // a slice whose copies timed out has no mass
  };
  // the crossing slice of u_K * total: the first whose prefix + mass exceeds
  // it, else the last with mass (every warp, same result)
  auto find_slice = [&](float part_lane) {
    float tot = 0.f;
    for (int c = 0; c < CS; ++c) tot += __shfl_sync(0xFFFFFFFFu, part_lane, c);
    const float t = sm.u_bonus * tot;
    float run = 0.f, pre = 0.f, prelast = 0.f;
    int cs = -1, clast = 0;
    for (int c = 0; c < CS; ++c) {
      const float part = __shfl_sync(0xFFFFFFFFu, part_lane, c);
      if (part > 0.f) { clast = c; prelast = run; }
      if (cs < 0 && run + part > t) { cs = c; pre = run; }
      run += part;
    }
    if (cs < 0) { cs = clast; pre = prelast; }
    total = tot;
    cstar = cs;
    tl = t - pre;
  };
  if (do_draw) {
    const float R = draw_pass(mode);
    if (tid == 0) sm.slot.R = R;
    cl_sync();  // B3: every slice's mass published
    float rp = lane < CS ? cl.map_shared_rank(&sm.slot, lane)->R : 0.f;
    find_slice(rp);
    if (has_d && !(total > 0.f) && total == total) {
      // the residual is 0 everywhere: the bonus comes from p_j (the same in every CTA)
      use_p = 1;
      mode = kDrawP;
      const float R2 = draw_pass(mode);
      if (tid == 0) sm.slot.R2 = R2;
      cl_sync();
      rp = lane < CS ? cl.map_shared_rank(&sm.slot, lane)->R2 : 0.f;
      find_slice(rp);
    }
    if (!(total == total)) flags |= kFlagTimeout;  // some slice's copies timed out
  }
  cl_arrive();  // no DSMEM reads past this point; the wait comes before exit

  const int leader = (do_draw && total == total) ? cstar : 0;
  if (crank == leader) {
    if (do_draw && total == total) {
      // warp 0: chunk, warp, lane and token of the crossing in this slice; the
      // crossing warp-chunk is read once more (from L2)
      if (warp == 0) {
        float my = 0.f;
        if (lane < nchd)
          for (int w = 0; w < kWarps; ++w) my += sm.rs[lane][w];
        float run = 0.f, pre_k = 0.f, pre_last = 0.f;
        int k_star = -1, k_last = 0;
        for (int c = 0; c < nchd; ++c) {
          const float tk = __shfl_sync(0xFFFFFFFFu, my, c);
          if (tk > 0.f) { k_last = c; pre_last = run; }
          if (k_star < 0 && run + tk > tl) { k_star = c; pre_k = run; }
          run += tk;
        }
        if (k_star < 0) { k_star = k_last; pre_k = pre_last; }
        const float tl2 = tl - pre_k;
        const float mw = lane < kWarps ? sm.rs[k_star][lane] : 0.f;
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
        const int g = k_star * kThreads + w_star * 32 + lane;
        float val[8], pv[8];
        if (g < nvec) {
          draw_vals_bf16(mode, ld_vec(rowP + e0 + g * 8), mode == kDrawResidual ? ld_vec(rowQ + e0 + g * 8) : zero4,
                         e0 + g * 8, cT, nmP, nmQ, invSP, wS, wN, check_S, bx, bi, false, val, pv);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) val[i] = 0.f;
        }
        float ls = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) ls += val[i];
        float incl = ls;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
          if (lane >= o) incl += y;
        }
        const unsigned cross = __ballot_sync(0xFFFFFFFFu, incl > tl3);
        const unsigned posm = __ballot_sync(0xFFFFFFFFu, ls > 0.f);
        const int l_star = cross ? (__ffs(cross) - 1) : (posm ? (31 - __clz(posm)) : 0);
        if (lane == l_star) {
          const float tl4 = tl3 - (incl - ls);
          float run4 = 0.f, c_prev = 0.f, c_prev_last = 0.f;
          int i_star = -1, i_last = 0;
          for (int i = 0; i < 8; ++i) {
            if (val[i] > 0.f) { i_last = i; c_prev_last = run4; }
            if (i_star < 0 && run4 + val[i] > tl4) { i_star = i; c_prev = run4; }
            run4 += val[i];
          }
          if (i_star < 0) { i_star = i_last; c_prev = c_prev_last; }
          const int v = e0 + g * 8 + i_star;
          const float lo = tl4 - c_prev;
          const float hi = c_prev + val[i_star] - tl4;
          sm.drawn = min(max(v, 0), V - 1);
          sm.dmargin = fminf(fabsf(lo), fabsf(hi)) / total;
        }
      }
    } else if (tid == 0) {
      sm.drawn = -1;
      sm.dmargin = INFINITY;
    }
    // the unit's outputs: a_j, its cache segment and its record
    if (tid == 0 && has_d)
      a.accept_prob[static_cast<long long>(b) * K + j] = valid ? acc : __int_as_float(0x7FC00000);
    if (a.c_tokens && has_plan && !plan_bad) {
      int32_t* seg = a.c_tokens + static_cast<long long>(b) * a.budget + sm.seg_off;
      for (int r = tid; r < Fj; r += kThreads) seg[r] = valid_src ? sm.sel[r].idx : -1;
    }
    __syncthreads();
    if (tid == 0) {
      UnitOut rec;
      rec.a = acc;
      rec.amargin = amargin;
      rec.R = total;
      rec.dmargin = sm.dmargin;
      rec.flags = flags | pflags;
      rec.rejected = rejected;
      rec.drawn = sm.drawn;
      rec.use_p = use_p;
      a.uout[u] = rec;
      if (flags & kFlagTimeout) atomicExch(a.error, 1);
      sm.is_last = arrive_acq_rel_gpu(a.row_arrive + b) == upr - 1 ? 1 : 0;
    }
    __syncthreads();
    if (sm.is_last) {
      // =============== the row: its last unit to finish, all records published ===========
      if (warp == 0) {
        const UnitOut* us = a.uout + static_cast<long long>(b) * upr;
        int fl = 0, rej = 0;
        float am = INFINITY;
        if (lane < upr) {
          fl = __ldcg(&us[lane].flags);
          rej = lane < K ? __ldcg(&us[lane].rejected) : 0;
          am = lane < K ? __ldcg(&us[lane].amargin) : INFINITY;
        }
        if (lane + 32 < upr) fl |= __ldcg(&us[lane + 32].flags);
        const unsigned rm = __ballot_sync(0xFFFFFFFFu, rej != 0);
        const int kstar = rm ? __ffs(rm) - 1 : K;
        // the margins of the tests up to and including the first rejection
        float amk = lane <= kstar ? am : INFINITY;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amk = fminf(amk, __shfl_xor_sync(0xFFFFFFFFu, amk, o));
        fl = static_cast<int>(__reduce_or_sync(0xFFFFFFFFu, static_cast<unsigned>(fl)));
        if (lane == 0) {
          const UnitOut* uk = us + kstar;
          sm.kstar = kstar;
          sm.drawn = __ldcg(&uk->drawn);
          sm.dmargin = __ldcg(&uk->dmargin);
          sm.total = __ldcg(&uk->R);
          sm.use_p = __ldcg(&uk->use_p);
          sm.amargin = amk;
          sm.rflags = fl;
          a.row_arrive[b] = 0;
        }
        // every unit of the row has arrived: its rejection flags are read no more
        if (lane < upr) a.arrive1[static_cast<long long>(b) * upr + lane] = 0;
        if (lane + 32 < upr) a.arrive1[static_cast<long long>(b) * upr + lane + 32] = 0;
      }
      __syncthreads();
      const int kstar = sm.kstar;
      int fl = sm.rflags;
      const bool invalid = (fl & SSD_ROW_INVALID) != 0;
      if (tid == 0) {
        if (sm.amargin < kNearTie || sm.dmargin < kNearTie) fl |= SSD_ROW_NEAR_TIE;
        fl &= ~SSD_ROW_ZERO_RESIDUAL;
        if (sm.use_p) fl |= SSD_ROW_ZERO_RESIDUAL;
        a.status[b] = fl;
        a.n_accepted[b] = invalid ? -1 : kstar;
        a.bonus[b] = invalid ? -1 : sm.drawn;
        a.residual_mass[b] = invalid ? __int_as_float(0x7FC00000) : sm.total;
        sm.slot_out = -1;
      }
      if (tid <= K) {
        int32_t t = -1;
        if (!invalid)
          t = tid < kstar ? __ldg(a.tokens + static_cast<long long>(b) * K + tid) : (tid == kstar ? sm.drawn : -1);
        a.out_tokens[static_cast<long long>(b) * (K + 1) + tid] = t;
      }
      if (invalid)
        for (int k = tid; k < K; k += kThreads) a.accept_prob[static_cast<long long>(b) * K + k] = __int_as_float(0x7FC00000);
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
          const int32_t* seg = a.c_tokens + static_cast<long long>(b) * a.budget + off;
          for (int i = tid; i < sm.s_F[kstar]; i += kThreads)
            if (__ldcg(seg + i) == sm.drawn) sm.slot_out = off + i;
        }
        __syncthreads();
        const int slot = sm.slot_out;
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
    }
  }
  // a copy that never landed must not land after the CTA has left
  if (tmo)
    for (int k = max(0, base - kClStages); k < base; ++k)
      mbar_wait_bounded(&sm.full[k % kClStages], static_cast<uint32_t>(k / kClStages) & 1u, kRingWaitNs);
  cl_wait();  // the cluster's DSMEM reads of this CTA's records are over
}

}  // namespace ssd
