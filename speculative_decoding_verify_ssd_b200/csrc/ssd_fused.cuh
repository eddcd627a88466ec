// ssd_fused.cuh -- the persistent fused verify kernel of libssd.
//
// One kernel runs the whole verify + cache step ([ZH] = "Speculative
// Speculative Decoding", gist.science Chinese edition, technical summary
// sections 1-2; [NL] = the Dutch edition, sections 2 and 3A-3C).  Its CTAs
// stay resident and take work items from a queue in the workspace:
//
//   statistics item (row b, position j, vocabulary slice s): stream the slice
//     of the target row p_j and the draft row q_j once from HBM, keep the
//     online max / exp-sum of both and the top vectors of the top-F source
//     row, publish a slice partial.  The last slice of a unit to arrive
//     merges the partials, selects the exact top-F, forms the Saguaro
//     normaliser Z and runs the accept test; the last unit of a row to arrive
//     fixes k* (the first rejected position) and publishes the row's decision
//     word.
//   draw item (row b, slice s): once row b is decided, stream the slice of
//     unit k*'s rows again and sum the residual max(0, p - q') (or p_K after
//     full acceptance) per 256-vector chunk and warp, in token order; the last
//     slice to arrive walks the sums to the crossing of u_K R, draws the bonus
//     token and writes the row's outputs, cache lookup and fallback included.
//
// Queue order: group r holds the statistics items of row r, then the draw
// items of row r - L, so a row is drawn about L rows after it was streamed:
// by then its decision is usually made, and its two rows are still in L2.
//
// Each CTA has eight consumer warps and one producer warp.  The producer
// takes items, and for each stage of the ring of bulk copies (no multicast)
// waits until the eight consumer warps have released it, writes the stage's
// item tag and starts the copies; the consumers wait on the stage's full
// barrier, so no CTA-wide barrier sits in the stream.  The producer runs ahead
// into the next item while the consumers finish the previous one.
#pragma once

#include "ssd_kernels.cuh"

namespace ssd {

constexpr int kConsumerThreads = 256;                      // eight consumer warps
constexpr int kConsumerWarps = kConsumerThreads / 32;
constexpr int kFusedThreads = kConsumerThreads + 32;       // plus the producer warp
constexpr int kProducerWarp = kConsumerWarps;
constexpr int kFusedCV = 512;                              // 16-byte vectors per row per stage
constexpr int kFusedVPT = kFusedCV / kConsumerThreads;     // vectors per consumer thread per row per stage
constexpr int kFusedChunks = kMaxChunks * kChunkVecs / kFusedCV;  // stages of a draw slice (<= kMaxChunks 256-vector chunks)
#ifndef SSD_FUSED_STAGES
#define SSD_FUSED_STAGES 2
#endif
constexpr int kFusedStages = SSD_FUSED_STAGES;
constexpr size_t kFusedRingBytes = static_cast<size_t>(kFusedStages) * 2 * kFusedCV * 16;
#ifndef SSD_FUSED_MIN_BLOCKS
#define SSD_FUSED_MIN_BLOCKS 4
#endif
constexpr int kFusedMinBlocks = SSD_FUSED_MIN_BLOCKS;

static_assert(kFusedVPT * kConsumerThreads == kFusedCV, "a stage is a whole number of vectors per thread");

enum ItemKind : int { kItemEnd = -1, kItemStats = 0, kItemDraw = 1 };

struct FusedItem {
  int kind, b, j, s;
};

// Item i of the queue: groups r = 0 .. B + L - 1; group r holds the NS
// statistics items of row r (r < B; unit-major, slice-minor) and then the ND
// draw items of row r - L (r >= L).
__device__ __forceinline__ FusedItem decode_item(int i, int B, int NS, int ND, int L, int S) {
  FusedItem it{kItemEnd, 0, 0, 0};
  const int head = L * NS;
  const int mid = (B - L) * (NS + ND);
  const int tail = L * ND;
  int r, o;
  if (i < 0) return it;
  if (i < head) {
    r = i / NS;
    o = i - r * NS;
  } else if (i < head + mid) {
    const int x = i - head;
    const int g = x / (NS + ND);
    r = L + g;
    o = x - g * (NS + ND);
  } else if (i < head + mid + tail) {
    const int x = i - head - mid;
    const int g = x / ND;
    r = B + g;
    o = NS + (x - g * ND);
  } else {
    return it;
  }
  if (o < NS) {
    it.kind = kItemStats;
    it.b = r;
    it.j = o / S;
    it.s = o - it.j * S;
  } else {
    it.kind = kItemDraw;
    it.b = r - L;
    it.s = o - NS;
  }
  return it;
}

// Stage tags written by the producer before the stage's copies start; a draw
// item's stages also carry the statistics of unit k* (from the row's record,
// which the producer reads after acquiring the decision word).
struct StageInfo {
  int32_t item, chunk, nch, kstar, flags, Fj, bi, argP;
  float MP, SP, MQ, SQ, Z, bx, amargin;
  int32_t kind, b, j, s, pad0, pad1, pad2, pad3;  // the decoded item
};

// Shared memory of the fused kernel (besides the ring).
struct SmemF {
  uint64_t full[kFusedStages], empty[kFusedStages];
  StageInfo info[kFusedStages];
  int32_t k_issued;                  // stages the producer has started (read only on error paths)
  uint32_t epoch;
  // statistics epilogue
  float wred[kConsumerWarps][4];
  int32_t wint[kConsumerWarps][2];
  float gmax[kConsumerThreads];
  int32_t hist[256];
  int32_t s_F[SSD_MAX_K + 1];
  float tau, MP, SP, MQ, SQ, QS, bx;
  int32_t bi, argP, argQ, n_total, slow, tmo, n_raw, is_last, is_last_row;
  int32_t Fj, seg_off, plan_bad;
  float xdP, xdQ;
  // a statistics item's inputs, fetched at its first stage so their latency
  // hides behind the stream: the drafted token, its uniform, its two logits
  // (when the token falls in the item's slice)
  int32_t pf_d;
  float pf_u, pf_xdP, pf_xdQ;
  int32_t cand_off[kMaxSlices + 1];
  int32_t cnt[kMaxSlices];
  // draw
  float rs[kMaxChunks][kWarps];
  float ps[kMaxChunks][kWarps];
  float tl, total, margin;
  int32_t cstar, use_p, drawn, slot, dtmo;
  // a slice's local candidates, then the unit's top-F
  Cand sel[kSelCap];
  // the unit's gathered candidates, or (for a draw) every slice's sums
  union {
    Cand gbuf[kGatherCap];
    float dsum[2 * kMaxSlices * kMaxChunks * kWarps];
  };
};
static_assert(kSelCap >= kCandCap, "the local candidates share the top-F buffer");

__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

__device__ __forceinline__ int consumer_sync_or(int v) {
  int r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.s32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 256, p;\n\t"
      "selp.s32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(v)
      : "memory");
  return r;
}

__device__ __forceinline__ void mbar_arrive_plain(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_addr(bar))
               : "memory");
}

// Statistics state of one item, per consumer thread.
struct StatsState {
  float mP, sP, nmP1, mQ, sQ, nmQ1;
  f32x2 sP2, sQ2, nmP2, nmQ2;
  int argP, argQ, nan_seen;
  float vm1, vm2, vm3;
  int g1, g2;
  uint4 keep1, keep2;
};

__device__ __forceinline__ void stats_reset(StatsState& t) {
  t.mP = -INFINITY; t.sP = 0.f; t.nmP1 = 0.f; t.mQ = -INFINITY; t.sQ = 0.f; t.nmQ1 = 0.f;
  t.sP2 = 0ull; t.sQ2 = 0ull; t.nmP2 = 0ull; t.nmQ2 = 0ull;
  t.argP = INT_MAX; t.argQ = INT_MAX; t.nan_seen = 0;
  t.vm1 = -INFINITY; t.vm2 = -INFINITY; t.vm3 = -INFINITY;
  t.g1 = -1; t.g2 = -1;
  t.keep1 = make_uint4(0u, 0u, 0u, 0u);
  t.keep2 = t.keep1;
}

// The fan-out plan's checks and unit j's share, by one warp: the plan into
// sm.s_F, sm.plan_bad / sm.Fj / sm.seg_off.
__device__ __forceinline__ void plan_for_unit(const Args& a, SmemF& sm, int b, int j, int lane) {
  const int K = a.K, V = a.V;
  int fplan[2] = {0, 0};
  if (a.F) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int k = lane + 32 * h;
      if (k <= K) fplan[h] = __ldg(a.F + static_cast<long long>(b) * (K + 1) + k);
    }
  } else {
    const float al = a.fanout_mode == SSD_FANOUT_UNIFORM ? 0.f : __ldg(a.alpha + b);
    fanout_warp(al, K, a.budget, a.fanout_mode, lane, fplan);
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
    const int pb = (bad || sum != a.budget) ? 1 : 0;
    sm.plan_bad = pb;
    sm.Fj = pb ? 0 : fj;
    sm.seg_off = pre;
  }
}

// ---------------------------------------------------------------------------
// The producer: one lane takes items and fills the ring.
// ---------------------------------------------------------------------------
template <typename TIn, bool kGreedy>
__device__ __noinline__ void fused_producer(const Args& a, SmemF& sm, unsigned char* ring) {
  constexpr int VE = Elem<TIn>::VE;
  const int K = a.K, V = a.V, S = a.n_slices, SD = a.d_slices;
  const int NS = a.units_per_row * S;
  unsigned k = 0;
  bool stop = false;
  auto next_stage = [&](int& slot) -> bool {
    slot = static_cast<int>(k % kFusedStages);
    if (k >= static_cast<unsigned>(kFusedStages) &&
        !mbar_wait_bounded(&sm.empty[slot], ((k / kFusedStages) - 1) & 1, kRingWaitNs)) {
      atomicExch(a.error, 1);
      return false;
    }
    return true;
  };
  while (!stop) {
    const int i = atomicAdd(a.queue, 1);
    const FusedItem it = decode_item(i, a.B, NS, SD, a.lag, S);
    int slot;
    if (it.kind == kItemEnd) {
      if (!next_stage(slot)) break;
      StageInfo end{};
      end.item = -1;
      sm.info[slot] = end;
      mbar_arrive_plain(&sm.full[slot]);
      ++k;
      break;
    }
    const TIn *baseP, *baseQ;
    long long rbP, rbQ;
    int nch = 0, e0 = 0, nvec = 0, kstar = 0, flags = 0;
    StageInfo tag{};
    if (it.kind == kItemStats) {
      unit_rows<TIn>(a, it.b, it.j, baseP, rbP, baseQ, rbQ);
      e0 = it.s * a.chunk;
      const int e1 = min(V, e0 + a.chunk);
      nvec = (max(0, e1 - e0) + VE - 1) / VE;
      nch = (nvec + kFusedCV - 1) / kFusedCV;
    } else {
      // the row's decision word: k* and the row's flags
      uint64_t word = 0;
      if (wait_tagged(a.rflag + it.b, sm.epoch + 1u, kDepWaitNs, &word)) {
        kstar = static_cast<int>((word >> 8) & 0xFF);
        flags = static_cast<int>(word & 0xFF);
        if (kstar > K) { kstar = K; flags |= kFlagTimeout; }
      } else {
        atomicExch(a.error, 1);
        kstar = K;
        flags = kFlagTimeout;
      }
      const bool streams = !kGreedy && (flags & SSD_ROW_INVALID) == 0;
      if ((flags & kFlagTimeout) == 0) {
        const RowState* rs = a.rstate + it.b;
        tag.Fj = __ldcg(&rs->Fj); tag.bi = __ldcg(&rs->bi); tag.argP = __ldcg(&rs->argP);
        tag.MP = __ldcg(&rs->MP); tag.SP = __ldcg(&rs->SP); tag.MQ = __ldcg(&rs->MQ); tag.SQ = __ldcg(&rs->SQ);
        tag.Z = __ldcg(&rs->Z); tag.bx = __ldcg(&rs->bx); tag.amargin = __ldcg(&rs->amargin);
      } else {
        tag.SP = 1.f; tag.SQ = 1.f; tag.Z = 1.f; tag.amargin = INFINITY;
      }
      unit_rows<TIn>(a, it.b, kstar, baseP, rbP, baseQ, rbQ);
      if (kstar == K) baseQ = nullptr;  // the full-acceptance draw reads p_K only
      if (streams) {
        e0 = it.s * a.d_chunk;
        const int e1 = min(V, e0 + a.d_chunk);
        nvec = (max(0, e1 - e0) + VE - 1) / VE;
        nch = (nvec + kFusedCV - 1) / kFusedCV;
      }
    }
    const int nrows = (baseP ? 1 : 0) + (baseQ ? 1 : 0);
    const TIn* row0 = baseP ? baseP + rbP : (baseQ ? baseQ + rbQ : nullptr);
    const TIn* row1 = baseP && baseQ ? baseQ + rbQ : nullptr;
    for (int c = 0; c < max(nch, 1); ++c) {
      if (!next_stage(slot)) { stop = true; break; }
      tag.item = i;
      tag.kind = it.kind;
      tag.b = it.b;
      tag.j = it.j;
      tag.s = it.s;
      tag.chunk = c;
      tag.nch = nch;
      tag.kstar = kstar;
      tag.flags = flags;
      sm.info[slot] = tag;
      if (nch > 0 && nrows > 0) {
        const int v0 = c * kFusedCV, nv = min(kFusedCV, nvec - v0);
        const uint32_t bytes = static_cast<uint32_t>(nv) * 16u;
        unsigned char* st = ring + static_cast<size_t>(slot) * 2 * kFusedCV * 16;
        mbar_arrive_expect_tx(&sm.full[slot], bytes * static_cast<uint32_t>(nrows));
        bulk_copy_g2s(st, row0 + e0 + static_cast<long long>(v0) * VE, bytes, &sm.full[slot]);
        if (row1) bulk_copy_g2s(st + kFusedCV * 16, row1 + e0 + static_cast<long long>(v0) * VE, bytes, &sm.full[slot]);
      } else {
        mbar_arrive_plain(&sm.full[slot]);
      }
      ++k;
      *reinterpret_cast<volatile int32_t*>(&sm.k_issued) = static_cast<int32_t>(k);
    }
  }
}

// ---------------------------------------------------------------------------
// Statistics item epilogue (consumers): the slice partial, then -- for the
// last slice of the unit to arrive -- the unit's merge, exact top-F, Saguaro
// normaliser and accept test, then -- for the last unit of the row -- the
// row's decision.
// ---------------------------------------------------------------------------
template <typename TIn, bool kGreedy>
__device__ __noinline__ void stats_finish(const Args& a, SmemF& sm, StatsState t, int b, int j, int slice, int tmo_in) {
  constexpr int VE = Elem<TIn>::VE;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int K = a.K, V = a.V, S = a.n_slices, upr = a.units_per_row;
  const long long u = static_cast<long long>(b) * upr + j;
  const TIn *baseP, *baseQ;
  long long rbP, rbQ;
  unit_rows<TIn>(a, b, j, baseP, rbP, baseQ, rbQ);
  const bool hasP = baseP != nullptr, hasQ = baseQ != nullptr;
  const bool srcQ = hasQ;
  const bool has_d = j < K;
  const int e0 = slice * a.chunk;
  const int e1 = min(V, e0 + a.chunk);
  const int nvec = (max(0, e1 - e0) + VE - 1) / VE;
  const float cT = kGreedy ? 0.f : kLog2e / a.T;
  const bool has_plan = a.F != nullptr || a.alpha != nullptr;

  int flags = 0;

  if constexpr (kGreedy) {
    if (t.nan_seen) { t.mP = __int_as_float(0x7FC00000); t.mQ = t.mP; }
  } else if constexpr (sizeof(TIn) == 2) {
    float lo, hi;
    f2_unpack(t.sP2, lo, hi);
    t.sP = lo + hi;
    f2_unpack(t.sQ2, lo, hi);
    t.sQ = lo + hi;
  }
  sm.gmax[tid] = t.vm1;
  if (tid == 0) sm.n_raw = 0;
  Cand* const raw = sm.sel;  // the local candidates, before the unit's top-F lands there

  float mP = t.mP, sP = t.sP, mQ = t.mQ, sQ = t.sQ;
  int argP = t.argP, argQ = t.argQ;
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
  const int tmo = consumer_sync_or(tmo_in);
  // fetched at the item's first stage (see the consumer loop)
  const int d = has_d ? sm.pf_d : -1;
  const float u_self = sm.pf_u;
  if (has_d && (d < 0 || d >= V)) flags |= SSD_ROW_BAD_TOKEN;
  if (!(u_self >= 0.f && u_self < 1.f)) flags |= SSD_ROW_BAD_UNIFORM;
  const float xdP = sm.pf_xdP, xdQ = sm.pf_xdQ;
  int Fj = 0, seg_off = 0, plan_bad = 0;
  if (has_plan) {
    plan_bad = sm.plan_bad;
    Fj = sm.Fj;
    seg_off = sm.seg_off;
  }
  if (plan_bad) flags |= SSD_ROW_BAD_PLAN;
  const bool want_topf = has_plan && Fj > 0;
  const bool fast_ok = want_topf && Fj <= kMaxGroups;
  SlicePart* part = a.parts + u * S + slice;
  if (warp == 0) {
    float m1 = -INFINITY, s1 = 0.f, m2 = -INFINITY, s2 = 0.f;
    int a1 = INT_MAX, a2 = INT_MAX;
    if (lane < kConsumerWarps) {
      m1 = sm.wred[lane][0]; s1 = sm.wred[lane][1]; m2 = sm.wred[lane][2]; s2 = sm.wred[lane][3];
      if constexpr (kGreedy) { a1 = sm.wint[lane][0]; a2 = sm.wint[lane][1]; }
    }
#pragma unroll
    for (int o = kConsumerWarps / 2; o > 0; o >>= 1) {
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
      part->xdP = xdP; part->xdQ = xdQ;
    }
  } else if (warp == 1) {
    // This slice's threshold: the F-th largest of its thread maxima bounds the
    // slice's own top-F (hence its share of the unit's top-F) from below.
    float th = -INFINITY;
    if (fast_ok) {
      uint32_t keys[kMaxGroups / 32];
#pragma unroll
      for (int i = 0; i < kMaxGroups / 32; ++i) keys[i] = ord_key(sm.gmax[lane + 32 * i]);
      th = key_to_float(warp_kth_largest(keys, Fj, sizeof(TIn) == 2 ? 16 : 32));
    }
    if (lane == 0) sm.tau = th;
  }
  consumer_sync();
  const float tau = sm.tau;
  // Local candidates: the elements at or above tau.  A thread whose third
  // vector maximum is below tau holds them all in its two kept vectors; the
  // others re-read their vectors of the slice (from L2).
  if (fast_ok && t.vm1 >= tau && t.vm1 == t.vm1) {
    if (t.vm3 < tau) {
      float x[VE];
      Elem<TIn>::unpack(t.keep1, x);
#pragma unroll
      for (int i = 0; i < VE; ++i) {
        const int v = e0 + t.g1 * VE + i;
        if (x[i] >= tau && v < e1) {
          const int pos = atomicAdd(&sm.n_raw, 1);
          if (pos < kCandCap) raw[pos] = Cand{x[i], v};
        }
      }
      if (t.vm2 >= tau && t.g2 >= 0) {
        Elem<TIn>::unpack(t.keep2, x);
#pragma unroll
        for (int i = 0; i < VE; ++i) {
          const int v = e0 + t.g2 * VE + i;
          if (x[i] >= tau && v < e1) {
            const int pos = atomicAdd(&sm.n_raw, 1);
            if (pos < kCandCap) raw[pos] = Cand{x[i], v};
          }
        }
      }
    } else {
      const TIn* bs = srcQ ? baseQ : baseP;
      const long long rsb = srcQ ? rbQ : rbP;
      // this thread's vectors of the slice: g = c * CV + v * 256 + tid
      for (int g = tid; g < nvec; g += kConsumerThreads) {
        float x[VE];
        load_group<TIn, true>(bs, rsb, e0 + g * VE, e1, x);
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
  consumer_sync();
  {
    const int nr = min(sm.n_raw, kCandCap);
    const int keepn = min(min(nr, Fj), kCandSlice);
    for (int i = tid; i < nr; i += kConsumerThreads) {
      const Cand ci = raw[i];
      const unsigned long long key = rank_key(ci.x, ci.idx);
      int r = 0;
      for (int k2 = 0; k2 < nr; ++k2) r += rank_key(raw[k2].x, raw[k2].idx) > key;
      if (r < keepn) part->cand[r] = ci;
    }
    if (tid == 0) part->n_cand = sm.n_raw;
  }
  consumer_sync();
  // The last slice of the unit to arrive finalises.
  if (tid == 0) sm.is_last = arrive_acq_rel_gpu(a.arrive1 + u) == S - 1 ? 1 : 0;
  consumer_sync();
  if (!sm.is_last) return;

  // =============== the unit's finaliser ==============================================
  const SlicePart* parts = a.parts + u * S;
  Cand* const gbuf = sm.gbuf;
  Cand* const sel = sm.sel;
  const int cap = min(Fj, kCandSlice);
  const bool one_round = fast_ok && S * cap <= kGatherCap;
  if (one_round && warp != 0) {
    for (int i = tid - 32; i < S * cap; i += kConsumerThreads - 32) {
      const Cand* src = &parts[i / cap].cand[i % cap];
      gbuf[i] = Cand{__ldcg(&src->x), __ldcg(&src->idx)};
    }
  }
  if (warp == 0) {
    float mp = -INFINITY, sp = 0.f, mq = -INFINITY, sq = 0.f;
    int ap = INT_MAX, aq = INT_MAX, nc = 0, to = 0;
    if (lane < S) {
      mp = __ldcg(&parts[lane].mP); sp = __ldcg(&parts[lane].sP);
      mq = __ldcg(&parts[lane].mQ); sq = __ldcg(&parts[lane].sQ);
      ap = __ldcg(&parts[lane].argP); aq = __ldcg(&parts[lane].argQ);
      nc = __ldcg(&parts[lane].n_cand); to = __ldcg(&parts[lane].timeout);
    }
    float xp = 0.f, xq = 0.f;
    if (!kGreedy && has_d && lane < S) {
      xp = __ldcg(&parts[lane].xdP);
      xq = __ldcg(&parts[lane].xdQ);
    }
    const int cd = (has_d && d >= 0 && d < V) ? d / a.chunk : 0;
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
    }
  }
  consumer_sync();
  const float MP = sm.MP, MQ = sm.MQ, SP = sm.SP, SQ = sm.SQ;
  if (sm.tmo) flags |= kFlagTimeout;
  if (hasP && !(MP > -INFINITY && MP < INFINITY)) flags |= SSD_ROW_NONFINITE;
  if (hasQ && !(MQ > -INFINITY && MQ < INFINITY)) flags |= SSD_ROW_NONFINITE;
  const bool valid = (flags & SSD_ROW_INVALID) == 0;
  const bool slow = want_topf && valid && (!one_round || sm.slow != 0);
  const float nmP = -MP * cT, nmQ = -MQ * cT;

  // exact top-F: global ranks by binary search in the sorted slice lists
  if (want_topf && valid && !slow) {
    for (int i = tid; i < S * cap; i += kConsumerThreads) {
      const int c = i / cap, r0 = i - c * cap;
      if (r0 >= sm.cnt[c]) continue;
      const Cand ci = gbuf[i];
      const unsigned long long key = rank_key(ci.x, ci.idx);
      int r = r0;
      for (int c2 = 0; c2 < S; ++c2) {
        if (c2 == c) continue;
        const int base = c2 * cap;
        int lo = base, hi = base + sm.cnt[c2];
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
    topf_exact_global<TIn>(row, V, Fj, sel, sm.hist, tid, ConsumerBarrier{});
  }
  consumer_sync();
  if (warp == 0) {
    float qs = 0.f;
    if (want_topf && valid) {
      if constexpr (!kGreedy) {
        for (int i = lane; i < Fj; i += 32) qs += ex2(fmaf(sel[i].x, cT, srcQ ? nmQ : nmP));
      }
    }
    qs = warp_sum(qs);
    if (lane == 0) {
      sm.QS = qs;
      sm.bx = (want_topf && valid) ? sel[Fj - 1].x : INFINITY;
      sm.bi = (want_topf && valid) ? sel[Fj - 1].idx : -1;
    }
  }
  consumer_sync();
  const float C = a.C;
  float Z = 1.f;
  if (!kGreedy && want_topf && valid) Z = 1.f - (1.f - C) * (sm.QS / (srcQ ? SQ : SP));
  const float bx = sm.bx;
  const int bi = sm.bi;
  float acc = 0.f, amargin = INFINITY;
  int rejected = 0;
  if (has_d && valid) {
    if constexpr (kGreedy) {
      acc = (d == sm.argP) ? 1.f : 0.f;
      rejected = d != sm.argP;
    } else {
      const float xdp = sm.xdP, xdq = sm.xdQ;
      const float pd = ex2(fmaf(xdp, cT, nmP)) / SP;
      const float qd = ex2(fmaf(xdq, cT, nmQ)) / SQ;
      const bool inS = want_topf && (xdq > bx || (xdq == bx && d <= bi));
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
  if (a.c_tokens && !plan_bad && has_plan) {
    int32_t* segdst = a.c_tokens + static_cast<long long>(b) * a.budget + seg_off;
    for (int i = tid; i < Fj; i += kConsumerThreads) segdst[i] = valid ? sel[i].idx : -1;
  }
  if (tid == 0) {
    if (j < K) a.accept_prob[static_cast<long long>(b) * K + j] = valid ? acc : __int_as_float(0x7FC00000);
    UnitState st;
    st.MP = MP; st.SP = SP; st.MQ = MQ; st.SQ = SQ;
    st.Z = Z; st.bx = bx; st.a = acc; st.amargin = amargin;
    st.bi = bi; st.argP = sm.argP; st.argQ = sm.argQ; st.flags = flags;
    st.rejected = rejected; st.Fj = Fj; st.seg_off = seg_off; st.dmargin = INFINITY;
    a.ustate[u] = st;
    a.arrive1[u] = 0;
  }
  consumer_sync();
  // The last unit of the row to arrive decides the row.
  if (tid == 0) sm.is_last_row = arrive_acq_rel_gpu(a.row_arrive + b) == upr - 1 ? 1 : 0;
  consumer_sync();
  if (!sm.is_last_row) return;
  if (warp == 0) {
    const UnitState* us = a.ustate + static_cast<long long>(b) * upr;
    int fl = 0;
    if (lane < upr) fl |= __ldcg(&us[lane].flags);
    if (lane + 32 < upr) fl |= __ldcg(&us[lane + 32].flags);
    fl = static_cast<int>(__reduce_or_sync(0xFFFFFFFFu, static_cast<unsigned>(fl)));
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
      a.row_arrive[b] = 0;
      const uint64_t tag = static_cast<uint64_t>(sm.epoch) + 1u;
      st_release_gpu_u64(a.rflag + b, tag << 32 | static_cast<uint64_t>(kstar) << 8 | static_cast<uint64_t>(fl & 0xFF));
    }
  }
}

// ---------------------------------------------------------------------------
// Draw item epilogue (consumers): publish the slice's sums; the last slice of
// the row to arrive draws the bonus and finishes the row.
// ---------------------------------------------------------------------------
template <typename TIn, bool kGreedy>
__device__ __noinline__ void draw_finish(const Args& a, SmemF& sm, const StageInfo st, int b, int slice, int nch,
                                         int tmo_in) {
  const int kstar = st.kstar, rowflags = st.flags;
  const float amargin = st.amargin;
  constexpr int VE = Elem<TIn>::VE;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int K = a.K, V = a.V, S = a.d_slices;
  const bool row_invalid = (rowflags & SSD_ROW_INVALID) != 0;
  const bool streams = !kGreedy && !row_invalid;
  const int draw = kstar < K ? kDrawResidual : kDrawP;
  const TIn *baseP, *baseQ;
  long long rbP, rbQ;
  unit_rows<TIn>(a, b, kstar, baseP, rbP, baseQ, rbQ);
  const float cT = kGreedy ? 0.f : kLog2e / a.T;
  const float nmP = -st.MP * cT, nmQ = -st.MQ * cT;
  const float invSP = 1.f / st.SP;
  const float wS = a.C / (st.SQ * st.Z), wN = 1.f / (st.SQ * st.Z);
  const bool check_S = st.Fj > 0 && draw != kDrawP;
  const float u_draw = __ldg(a.uniforms + static_cast<long long>(b) * (K + 1) + K);
  DrawPart* dparts = a.dparts + static_cast<long long>(b) * S;
  int32_t seg_tok0 = -1, seg_tok1 = -1;

  // Every draw item of the row publishes its slice's partial and arrives,
  // streamed or not, so the last to arrive finishes the row whatever
  // happened to the others; a slice whose producer gave up waiting for the
  // decision reports a timeout, and the row becomes a timed-out row.
  const int nck = streams ? nch * kFusedVPT : 0;  // 256-vector chunks of this slice
  const int tmo = consumer_sync_or(tmo_in) | ((rowflags & kFlagTimeout) ? 1 : 0);
  if (warp == 0) {
    float R = 0.f, RP = 0.f;
    for (int i = lane; i < nck * kWarps; i += 32) { R += sm.rs[i / kWarps][i % kWarps]; RP += sm.ps[i / kWarps][i % kWarps]; }
    R = warp_sum(R);
    RP = warp_sum(RP);
    if (lane == 0) {
      dparts[slice].R = R;
      dparts[slice].RP = RP;
      dparts[slice].timeout = tmo;
    }
  }
  for (int i = tid; i < nck * kWarps; i += kConsumerThreads) {
    dparts[slice].rs[i / kWarps][i % kWarps] = sm.rs[i / kWarps][i % kWarps];
    dparts[slice].ps[i / kWarps][i % kWarps] = sm.ps[i / kWarps][i % kWarps];
  }
  consumer_sync();
  if (tid == 0) sm.is_last = arrive_acq_rel_gpu(a.draw_arrive + b) == S - 1 ? 1 : 0;
  consumer_sync();
  if (!sm.is_last) return;

  // ============ the draw: the last slice of the row to arrive =======================
  const int nchm = ((a.d_chunk + VE - 1) / VE + kChunkVecs - 1) / kChunkVecs;  // 256-vector chunks of a full slice
  float* const Lrs = sm.dsum;
  float* const Lps = Lrs + S * nchm * kWarps;
  if (streams) {
    for (int i = tid; i < S * nchm * kWarps; i += kConsumerThreads) {
      const int s2 = i / (nchm * kWarps), cw = i - s2 * (nchm * kWarps);
      Lrs[i] = __ldcg(&dparts[s2].rs[cw / kWarps][cw % kWarps]);
      Lps[i] = __ldcg(&dparts[s2].ps[cw / kWarps][cw % kWarps]);
    }
  }
  if (a.c_tokens && !row_invalid) {
    const int Fk = sm.s_F[kstar];
    int off = 0;
    for (int k = 0; k < kstar; ++k) off += sm.s_F[k];
    const int32_t* seg = a.c_tokens + static_cast<long long>(b) * a.budget + off;
    if (tid < Fk) seg_tok0 = __ldcg(seg + tid);
    if (tid + kConsumerThreads < Fk) seg_tok1 = __ldcg(seg + tid + kConsumerThreads);
  }
  if (warp == 0) {
    float rp = 0.f, pp = 0.f;
    int to = 0;
    if (lane < S) {
      rp = __ldcg(&dparts[lane].R);
      pp = __ldcg(&dparts[lane].RP);
      to = __ldcg(&dparts[lane].timeout);
    }
    const bool anyto = __ballot_sync(0xFFFFFFFFu, to != 0) != 0u;
    const bool search = streams && !anyto;
    float R = 0.f, RP = 0.f;
    for (int c = 0; c < S; ++c) {
      R += __shfl_sync(0xFFFFFFFFu, rp, c);
      RP += __shfl_sync(0xFFFFFFFFu, pp, c);
    }
    const int use_p = (search && draw == kDrawResidual && !(R > 0.f)) ? 1 : 0;
    const float total = use_p ? RP : R;
    const float tt = u_draw * total;
    float run = 0.f, pre = 0.f, prelast = 0.f;
    int cstar = -1, clast = 0;
    for (int c = 0; c < S; ++c) {
      const float pt = __shfl_sync(0xFFFFFFFFu, use_p ? pp : rp, c);
      if (pt > 0.f) { clast = c; prelast = run; }
      if (cstar < 0 && run + pt > tt) { cstar = c; pre = run; }
      run += pt;
    }
    if (cstar < 0) { cstar = clast; pre = prelast; }
    if (lane == 0) {
      sm.cstar = cstar;
      sm.tl = tt - pre;
      sm.dtmo = anyto ? 1 : 0;
      sm.slow = search ? 1 : 0;  // whether the bonus is searched in the sums
      if (search) {
        sm.total = total;
        sm.use_p = use_p;
      } else {
        // no stream (greedy: the argmax is the bonus) or a void row
        sm.drawn = (row_invalid || anyto) ? -1 : st.argP;
        sm.margin = INFINITY;
        sm.total = 1.f;
        sm.use_p = 0;
      }
    }
  }
  consumer_sync();
  if (warp == 0 && sm.slow) {
    const int s_star = sm.cstar;
    const bool use_p = sm.use_p != 0;
    const float* Ls = (use_p ? Lps : Lrs) + s_star * nchm * kWarps;
    const int e0s = s_star * a.d_chunk;
    const int e1s = min(V, e0s + a.d_chunk);
    const int nvs = (max(0, e1s - e0s) + VE - 1) / VE;
    const int nchs = (nvs + kChunkVecs - 1) / kChunkVecs;
    const float tl = sm.tl;
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
    const int g = k_star * kChunkVecs + w_star * 32 + lane;
    float val[VE], pv[VE];
    if (g < nvs) {
      draw_vals<TIn, true>(draw, baseP, rbP, baseQ, rbQ, e0s, e1s, g, nullptr, nullptr, cT, nmP, nmQ, invSP, wS,
                           wN, check_S, st.bx, st.bi, use_p, val, pv);
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
      const float lo = tl4 - c_prev;
      const float hi = c_prev + val[i_star] - tl4;
      sm.drawn = min(max(v, 0), V - 1);
      sm.margin = fminf(fabsf(lo), fabsf(hi)) / sm.total;
    }
  }
  consumer_sync();
  if (tid == 0) a.draw_arrive[b] = 0;

  // ============ finishing the row ===================================================
  int fl = rowflags | (sm.dtmo ? kFlagTimeout : 0);
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
    int32_t tok = -1;
    if (!invalid) tok = tid < kstar ? __ldg(a.tokens + static_cast<long long>(b) * K + tid) : (tid == kstar ? sm.drawn : -1);
    a.out_tokens[static_cast<long long>(b) * (K + 1) + tid] = tok;
  }
  if (invalid)
    for (int k = tid; k < K; k += kConsumerThreads) a.accept_prob[static_cast<long long>(b) * K + k] = __int_as_float(0x7FC00000);
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
    consumer_sync();
    if (invalid) {
      for (int s2 = tid; s2 < a.budget; s2 += kConsumerThreads) a.c_tokens[static_cast<long long>(b) * a.budget + s2] = -1;
    } else {
      // the key (k*, bonus) in segment k* (its tokens were prefetched above)
      int off = 0;
      for (int k = 0; k < kstar; ++k) off += sm.s_F[k];
      if (seg_tok0 == sm.drawn) sm.slot = off + tid;
      if (seg_tok1 == sm.drawn) sm.slot = off + tid + kConsumerThreads;
    }
    consumer_sync();
    const int slot = sm.slot;
    if (tid == 0) {
      a.c_hit[b] = slot >= 0 ? 1 : 0;
      a.c_slot[b] = slot;
    }
    for (int i = tid; i < K; i += kConsumerThreads) {
      int32_t tok;
      if (slot >= 0)
        tok = a.c_payload ? __ldg(a.c_payload + (static_cast<long long>(b) * a.budget + slot) * K + i) : -1;
      else
        tok = fallback_token(a.fallback_seed, b, i, V);
      a.c_next[static_cast<long long>(b) * K + i] = tok;
    }
  }
  consumer_sync();
}

// One stage of a draw item (consumers): the residual's mass per 256-vector
// chunk and warp, in token order, into sm.rs / sm.ps.  A function of its own
// so that its registers do not weigh on the statistics stream.
template <typename TIn, bool kGreedy>
__device__ __noinline__ void draw_stage(const Args& a, SmemF& sm, const unsigned char* st, const StageInfo& tag,
                                        int chunk, int cs) {
  constexpr int VE = Elem<TIn>::VE;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int K = a.K;
  const float cT = kGreedy ? 0.f : kLog2e / a.T;
  const int e0 = cs * a.d_chunk;
  const int e1 = min(a.V, e0 + a.d_chunk);
  const int nvec = (max(0, e1 - e0) + VE - 1) / VE;
  const int draw = tag.kstar < K ? kDrawResidual : kDrawP;
  const float nmP = -tag.MP * cT, nmQ = -tag.MQ * cT;
  const float invSP = 1.f / tag.SP;
  const float wS = a.C / (tag.SQ * tag.Z), wN = 1.f / (tag.SQ * tag.Z);
  const bool check_S = tag.Fj > 0 && draw != kDrawP;
  const float bx = tag.bx;
  const int bi = tag.bi;
#pragma unroll
  for (int v = 0; v < kFusedVPT; ++v) {
    const int tt = v * kConsumerThreads + tid;
    const int g = chunk * kFusedCV + tt;
    float rsum = 0.f, psum = 0.f;
    if (g < nvec) {
      float val[VE], pv[VE];
      const uint4* wp = reinterpret_cast<const uint4*>(st + tt * 16);
      const uint4* wq = reinterpret_cast<const uint4*>(st + kFusedCV * 16 + tt * 16);
      draw_vals<TIn, true>(draw, nullptr, 0, nullptr, 0, e0, e1, g, wp, wq, cT, nmP, nmQ, invSP, wS, wN, check_S, bx,
                           bi, false, val, pv);
#pragma unroll
      for (int i = 0; i < VE; ++i) { rsum += val[i]; psum += pv[i]; }
    }
    rsum = warp_sum(rsum);
    psum = warp_sum(psum);
    if (lane == 0) {
      const int ck = chunk * kFusedVPT + v;
      sm.rs[ck][warp] = rsum;
      sm.ps[ck][warp] = psum;
    }
  }
}

// ---------------------------------------------------------------------------
// The kernel.
// ---------------------------------------------------------------------------
template <typename TIn, bool kGreedy>
__global__ void __launch_bounds__(kFusedThreads, kFusedMinBlocks) ssd_fused_kernel(const __grid_constant__ Args a) {
  constexpr int VE = Elem<TIn>::VE;
  extern __shared__ __align__(128) unsigned char ring[];
  __shared__ __align__(16) SmemF sm;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int K = a.K;
  if (tid == 0) {
    for (int s = 0; s < kFusedStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kConsumerWarps);
    }
    mbar_init_fence();
    sm.k_issued = 0;
    sm.epoch = *reinterpret_cast<volatile const uint32_t*>(a.epoch);
  }
  __syncthreads();
  if (warp == kProducerWarp) {
    if (lane == 0) fused_producer<TIn, kGreedy>(a, sm, ring);
    return;
  }

  // ---- consumers -------------------------------------------------------------------
  const float cT = kGreedy ? 0.f : kLog2e / a.T;
  const f32x2 cT2 = f2_pack(cT, cT);
  StatsState t;
  stats_reset(t);
  int tmo = 0, kind = kItemEnd, cb = 0, cj = 0, cs = 0;
  bool hasQ = false;
  unsigned k = 0;
  for (;;) {
    const int slot = static_cast<int>(k % kFusedStages);
    if (!mbar_wait_bounded(&sm.full[slot], (k / kFusedStages) & 1, kRingWaitNs)) {
      // the stage never completed: leave (every consumer warp waits on the same
      // phase, so they all leave here)
      if (lane == 0) atomicExch(a.error, 1);
      break;
    }
    const StageInfo& tag = sm.info[slot];
    const int item = tag.item;
    if (item < 0) break;
    const int chunk = tag.chunk, nch = tag.nch;
    if (chunk == 0) {
      kind = tag.kind;
      cb = tag.b; cj = tag.j; cs = tag.s;
      tmo = 0;
      const bool has_plan = a.F != nullptr || a.alpha != nullptr;
      if (kind == kItemStats) {
        stats_reset(t);
        hasQ = cj < K || a.draft_next != nullptr;
        if (warp == 1 && has_plan) plan_for_unit(a, sm, cb, cj, lane);
        if (tid == 0) {
          // the epilogue's inputs, fetched now so their latency hides behind the stream
          const int dd = cj < K ? __ldg(a.tokens + static_cast<long long>(cb) * K + cj) : -1;
          sm.pf_d = dd;
          sm.pf_u = __ldg(a.uniforms + static_cast<long long>(cb) * (K + 1) + cj);
          float xp = 0.f, xq = 0.f;
          const int e0 = cs * a.chunk, e1 = min(a.V, e0 + a.chunk);
          if (!kGreedy && cj < K && dd >= e0 && dd < e1) {
            xp = Elem<TIn>::at(static_cast<const TIn*>(a.target) + (static_cast<long long>(cb) * (K + 1) + cj) * a.V, dd);
            xq = Elem<TIn>::at(static_cast<const TIn*>(a.draft) + (static_cast<long long>(cb) * K + cj) * a.V, dd);
          }
          sm.pf_xdP = xp;
          sm.pf_xdQ = xq;
        }
      } else if (warp == 1 && has_plan) {
        load_plan(a, cb, sm.s_F, lane);
      }
    }
    const unsigned char* st = ring + static_cast<size_t>(slot) * 2 * kFusedCV * 16;
    if (kind == kItemStats && nch > 0) {
      const int e0 = cs * a.chunk;
      const int e1 = min(a.V, e0 + a.chunk);
      const int nvec = (max(0, e1 - e0) + VE - 1) / VE;
#pragma unroll
      for (int v = 0; v < kFusedVPT; ++v) {
        const int tt = v * kConsumerThreads + tid;
        const int g = chunk * kFusedCV + tt;
        if (g < nvec) {
          const int vbase = e0 + g * VE;
          float vsrc;
          const uint4 wp = *reinterpret_cast<const uint4*>(st + tt * 16);
          uint4 wsrc = wp;
          if constexpr (sizeof(TIn) == 2) {
            const float vp = consume_bf16<kGreedy>(wp, vbase, cT, cT2, t.mP, t.sP2, t.nmP2, t.argP, t.nan_seen);
            vsrc = vp;
            if (hasQ) {
              const uint4 wq = *reinterpret_cast<const uint4*>(st + kFusedCV * 16 + tt * 16);
              vsrc = consume_bf16<kGreedy>(wq, vbase, cT, cT2, t.mQ, t.sQ2, t.nmQ2, t.argQ, t.nan_seen);
              wsrc = wq;
            }
          } else {
            float x[VE];
            Elem<TIn>::unpack(wp, x);
            vsrc = consume_f<VE, kGreedy>(x, vbase, cT, t.mP, t.sP, t.nmP1, t.argP, t.nan_seen);
            if (hasQ) {
              const uint4 wq = *reinterpret_cast<const uint4*>(st + kFusedCV * 16 + tt * 16);
              Elem<TIn>::unpack(wq, x);
              vsrc = consume_f<VE, kGreedy>(x, vbase, cT, t.mQ, t.sQ, t.nmQ1, t.argQ, t.nan_seen);
              wsrc = wq;
            }
          }
          if (vsrc > t.vm3) {
            if (vsrc > t.vm2) {
              t.vm3 = t.vm2;
              if (vsrc > t.vm1) { t.vm2 = t.vm1; t.keep2 = t.keep1; t.g2 = t.g1; t.vm1 = vsrc; t.g1 = g; t.keep1 = wsrc; }
              else { t.vm2 = vsrc; t.g2 = g; t.keep2 = wsrc; }
            } else {
              t.vm3 = vsrc;
            }
          }
        }
      }
    } else if (kind == kItemDraw && nch > 0) {
      draw_stage<TIn, kGreedy>(a, sm, st, tag, chunk, cs);
    }
    const bool last = chunk >= nch - 1;
    StageInfo fin;
    if (last && kind == kItemDraw) fin = tag;  // the tag of the draw's finish, before the stage is released
    __syncwarp();
    if (lane == 0) mbar_arrive_plain(&sm.empty[slot]);
    ++k;
    if (last) {
      // the item's last stage: its epilogue, while the producer runs ahead
      if (kind == kItemStats)
        stats_finish<TIn, kGreedy>(a, sm, t, cb, cj, cs, tmo);
      else
        draw_finish<TIn, kGreedy>(a, sm, fin, cb, cs, nch, tmo);
    }
  }
  // Copies this CTA started and nobody consumed (only after a wait gave up).
  if (tid == 0) {
    const unsigned issued = static_cast<unsigned>(*reinterpret_cast<volatile int32_t*>(&sm.k_issued));
    for (unsigned c = k; c < issued; ++c)
      mbar_wait_bounded(&sm.full[c % kFusedStages], (c / kFusedStages) & 1, kRingWaitNs);
  }
  consumer_sync();
  // The last CTA to finish rewinds the queue and advances the epoch.
  if (tid == 0) {
    __threadfence();
    if (atomicAdd(a.fdone, 1) == static_cast<int>(gridDim.x) - 1) {
      *a.queue = 0;
      *a.fdone = 0;
      __threadfence();
      atomicAdd(a.epoch, 1u);
    }
  }
}

}  // namespace ssd
