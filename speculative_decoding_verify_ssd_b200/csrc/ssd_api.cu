// ssd_api.cu -- host side of libssd: argument checks, launch planning and the
// extern "C" entry points declared in include/ssd.h, plus the three small
// kernels (fan-out plan, cache build, cache lookup).  The two vocab-wide
// kernels live in ssd_kernels.cuh.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <map>
#include <mutex>
#include <tuple>

#include "../../include/ssd.h"
#include "ssd_device.cuh"
#include "ssd_kernels.cuh"
#include "ssd_cluster.cuh"

namespace ssd {

// ---------------------------------------------------------------------------
// Fan-out plan ([ZH] section 2 challenge 1; [NL] section 3A).  fp64, every
// product and difference rounded on its own (no fused multiply-add).
// ---------------------------------------------------------------------------
__global__ void fanout_kernel(const float* __restrict__ alpha, int B, int K, int budget, int mode,
                              int32_t* __restrict__ F) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  fanout_row(mode == SSD_FANOUT_UNIFORM ? 0.f : alpha[b], K, budget, mode,
             F + static_cast<long long>(b) * (K + 1));
}

__global__ void fanout_power_kernel(const float* __restrict__ alpha, int B, int K, int budget, int q,
                                    int32_t* __restrict__ F) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  fanout_row_power(alpha[b], K, budget, q, F + static_cast<long long>(b) * (K + 1));
}

// ---------------------------------------------------------------------------
// Per-row acceptance from history: alpha' = (1 - lambda) alpha + lambda *
// mean_j a_j, in double with every operation rounded on its own, then
// rounded to float.  Invalid rows and rows with a NaN a_j keep their alpha.
// ---------------------------------------------------------------------------
__global__ void alpha_update_kernel(const float* __restrict__ alpha, const float* __restrict__ accept_prob,
                                    const int32_t* __restrict__ status, int B, int K, double lambda,
                                    float* __restrict__ alpha_out) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  bool ok = (status[b] & SSD_ROW_INVALID) == 0;
  double s = 0.0;
  for (int j = 0; j < K; ++j) {
    const double a = static_cast<double>(accept_prob[static_cast<long long>(b) * K + j]);
    if (a != a) ok = false;
    s = __dadd_rn(s, a);
  }
  if (!ok) {
    alpha_out[b] = alpha[b];
    return;
  }
  const double mean = __ddiv_rn(s, static_cast<double>(K));
  const double keep = __dmul_rn(__dsub_rn(1.0, lambda), static_cast<double>(alpha[b]));
  alpha_out[b] = __double2float_rn(__dadd_rn(keep, __dmul_rn(lambda, mean)));
}

// ---------------------------------------------------------------------------
// Cache build: offsets = prefix sums of F; tokens copied per segment.
// ---------------------------------------------------------------------------
__global__ void cache_build_kernel(const int32_t* __restrict__ F, const int32_t* __restrict__ topf,
                                   const int32_t* __restrict__ guess_K, int K, int budget,
                                   int32_t* __restrict__ offsets, int32_t* __restrict__ tokens) {
  __shared__ int32_t off[SSD_MAX_K + 2];
  __shared__ int32_t bad;
  const int b = blockIdx.x;
  const int32_t* Fr = F + static_cast<long long>(b) * (K + 1);
  if (threadIdx.x == 0) {
    long long sum = 0;
    int pb = 0;
    for (int k = 0; k <= K; ++k) {
      if (Fr[k] < 0) pb = 1;
      sum += Fr[k];
    }
    if (sum != budget) pb = 1;
    bad = pb;
    off[0] = 0;
    for (int k = 0; k <= K; ++k) off[k + 1] = off[k] + (pb ? 0 : Fr[k]);
    for (int k = 0; k <= K + 1; ++k) offsets[static_cast<long long>(b) * (K + 2) + k] = off[k];
  }
  __syncthreads();
  for (int s = threadIdx.x; s < budget; s += blockDim.x) {
    int32_t t = -1;
    if (!bad) {
      if (guess_K && s >= off[K])
        t = guess_K[static_cast<long long>(b) * budget + (s - off[K])];
      else
        t = topf[static_cast<long long>(b) * budget + s];
    }
    tokens[static_cast<long long>(b) * budget + s] = t;
  }
}

// ---------------------------------------------------------------------------
// Cache lookup ([ZH] section 2 basic flow step 4, challenge 3; [NL] 3C).
// ---------------------------------------------------------------------------
__global__ void cache_lookup_kernel(const int32_t* __restrict__ offsets, const int32_t* __restrict__ tokens,
                                    int B, int K, int budget, const int32_t* __restrict__ k,
                                    const int32_t* __restrict__ bonus, const int32_t* __restrict__ payload,
                                    unsigned long long seed, int V, uint8_t* __restrict__ hit,
                                    int32_t* __restrict__ slot, int32_t* __restrict__ next_tokens) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  const int kk = k[b];
  const int32_t bon = bonus[b];
  int sl = -1;
  if (kk >= 0 && kk <= K) {
    const int32_t* o = offsets + static_cast<long long>(b) * (K + 2);
    const int lo = max(o[kk], 0), hi = min(o[kk + 1], budget);
    for (int s = lo; s < hi; ++s)
      if (tokens[static_cast<long long>(b) * budget + s] == bon) {
        sl = s;
        break;
      }
  }
  hit[b] = sl >= 0 ? 1 : 0;
  slot[b] = sl;
  for (int i = 0; i < K; ++i) {
    int32_t t;
    if (sl >= 0)
      t = payload ? payload[(static_cast<long long>(b) * budget + sl) * K + i] : -1;
    else
      t = fallback_token(seed, b, i, V);
    next_tokens[static_cast<long long>(b) * K + i] = t;
  }
}

// ---------------------------------------------------------------------------
// Launch planning.
// ---------------------------------------------------------------------------
#ifndef SSD_CTA_BYTES
#define SSD_CTA_BYTES 131072  // logits streamed per CTA (all rows of a unit slice)
#endif
constexpr long long kCtaBytes = SSD_CTA_BYTES;
#ifndef SSD_DRAW_CTA_BYTES
#define SSD_DRAW_CTA_BYTES 32768  // logits streamed per CTA of the draw kernel
#endif
constexpr long long kDrawCtaBytes = SSD_DRAW_CTA_BYTES;
constexpr int kMinChunk = 1024;  // do not split a row finer than this

struct Plan {
  int n_slices, chunk;
};

#ifndef SSD_EE_LAG_PCT
#define SSD_EE_LAG_PCT 300
#endif

static int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// Slices per logit row and the slice length, for units of `rows` rows of length V.
static ssd_status make_plan(int V, int rows, int esize, long long units, Plan* p,
                            long long cta_bytes = kCtaBytes) {
  const int VE = 16 / esize;
  const long long max_chunk = static_cast<long long>(kMaxChunks) * kChunkVecs * VE;
  long long ns = (static_cast<long long>(rows) * V * esize + cta_bytes - 1) / cta_bytes;
  // enough CTAs to fill the machine, if the rows are long enough
  const long long want = (static_cast<long long>(kMinBlocks) * sm_count() + units - 1) / (units > 0 ? units : 1);
  const long long by_len = (V + kMinChunk - 1) / kMinChunk;
  long long extra = want < by_len ? want : by_len;
  if (extra > 8) extra = 8;
  if (ns < extra) ns = extra;
  if (ns > kMaxSlices) ns = kMaxSlices;
  if (ns < 1) ns = 1;
  long long chunk = (V + ns - 1) / ns;
  chunk = (chunk + VE - 1) / VE * VE;
  if (chunk > max_chunk) {
    ns = (V + max_chunk - 1) / max_chunk;
    chunk = (V + ns - 1) / ns;
    chunk = (chunk + VE - 1) / VE * VE;
  }
  ns = (V + chunk - 1) / chunk;
  if (ns > kMaxSlices) return SSD_ERR_UNSUPPORTED;
  p->n_slices = static_cast<int>(ns);
  p->chunk = static_cast<int>(chunk);
  return SSD_OK;
}

static long long stats_grid(const Args& a) {
  return static_cast<long long>(a.B) * a.units_per_row * a.n_slices;
}

static std::mutex g_attr_mu;
static std::map<std::tuple<const void*, int>, int> g_attr_done;

static cudaError_t prepare_kernel(const void* fn) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_attr_mu);
  auto key = std::make_tuple(fn, dev);
  if (g_attr_done.count(key)) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kRingBytes));
  if (e != cudaSuccess) return e;
  g_attr_done[key] = 1;
  return cudaSuccess;
}

// Workspace: slice partials, unit states, draw partials, row states, then the
// counters (zero between calls) and the error word.
struct WsLayout {
  size_t parts, ustate, dparts, rstate, arrive1, row_arrive, draw_arrive, draw_owner, row_arrive2, rflag, uword, dtot,
      epoch, k2_done, error, skipped, total;
  int n_slices;
};

static int plan_slices(int B, int K, int V, int dtype) {
  const int esize = dtype == SSD_DTYPE_FP32 ? 4 : 2;
  Plan p2, p1;
  const long long units = static_cast<long long>(B) * (K + 1);
  int ns = 1;
  if (make_plan(V, 2, esize, units, &p2) == SSD_OK) ns = p2.n_slices;
  if (make_plan(V, 1, esize, units, &p1) == SSD_OK) ns = ns > p1.n_slices ? ns : p1.n_slices;
  if (make_plan(V, 2, esize, B, &p2, kDrawCtaBytes) == SSD_OK) ns = ns > p2.n_slices ? ns : p2.n_slices;
  if (make_plan(V, 1, esize, static_cast<long long>(B) * K, &p1, kDrawCtaBytes) == SSD_OK)
    ns = ns > p1.n_slices ? ns : p1.n_slices;
  return ns;
}

static size_t up256(size_t x) { return (x + 255) / 256 * 256; }

static WsLayout ws_layout(int B, int K, int V, int dtype) {
  WsLayout w;
  const size_t nb = static_cast<size_t>(B > 0 ? B : 0);
  const size_t units = nb * static_cast<size_t>(K + 1);
  const size_t ns = static_cast<size_t>(plan_slices(B, K, V, dtype));
  w.n_slices = static_cast<int>(ns);
  size_t off = 0;
  w.parts = off;       off = up256(off + units * ns * sizeof(SlicePart));
  w.ustate = off;      off = up256(off + units * sizeof(UnitState));
  w.dparts = off;      off = up256(off + nb * static_cast<size_t>(K) * ns * sizeof(DrawPart));
  w.rstate = off;      off = up256(off + nb * sizeof(RowState));
  w.rflag = off;       off += nb * static_cast<size_t>(K) * sizeof(uint64_t);  // 8-byte aligned here
  w.uword = off;       off += units * sizeof(uint64_t);
  w.dtot = off;        off += nb * static_cast<size_t>(K) * 2 * ns * sizeof(uint64_t);
  w.arrive1 = off;     off += units * sizeof(int32_t);
  w.row_arrive = off;  off += nb * sizeof(int32_t);
  w.draw_arrive = off; off += nb * static_cast<size_t>(K) * sizeof(int32_t);
  w.draw_owner = off;  off += nb * static_cast<size_t>(K) * sizeof(int32_t);
  w.row_arrive2 = off; off += nb * sizeof(int32_t);
  w.epoch = off;       off += sizeof(uint32_t);
  w.k2_done = off;     off += sizeof(int32_t);
  w.error = off;       off += sizeof(int32_t);
  off = (off + 7) & ~static_cast<size_t>(7);
  w.skipped = off;     off += sizeof(unsigned long long);
  w.total = up256(off);
  return w;
}

static void bind_workspace(Args& a, void* ws, const WsLayout& w) {
  char* base = static_cast<char*>(ws);
  a.parts = reinterpret_cast<SlicePart*>(base + w.parts);
  a.ustate = reinterpret_cast<UnitState*>(base + w.ustate);
  a.dparts = reinterpret_cast<DrawPart*>(base + w.dparts);
  a.rstate = reinterpret_cast<RowState*>(base + w.rstate);
  a.arrive1 = reinterpret_cast<int32_t*>(base + w.arrive1);
  a.row_arrive = reinterpret_cast<int32_t*>(base + w.row_arrive);
  a.draw_arrive = reinterpret_cast<int32_t*>(base + w.draw_arrive);
  a.draw_owner = reinterpret_cast<int32_t*>(base + w.draw_owner);
  a.row_arrive2 = reinterpret_cast<int32_t*>(base + w.row_arrive2);
  a.rflag = reinterpret_cast<uint64_t*>(base + w.rflag);
  a.uword = reinterpret_cast<uint64_t*>(base + w.uword);
  a.dtot = reinterpret_cast<uint64_t*>(base + w.dtot);
  a.epoch = reinterpret_cast<uint32_t*>(base + w.epoch);
  a.k2_done = reinterpret_cast<int32_t*>(base + w.k2_done);
  a.error = reinterpret_cast<int32_t*>(base + w.error);
  a.skipped = reinterpret_cast<unsigned long long*>(base + w.skipped);
  a.uout = reinterpret_cast<UnitOut*>(base + w.ustate);  // the cluster form's unit records
}
static_assert(sizeof(UnitOut) <= sizeof(UnitState), "a unit record of the cluster form fits a unit state");

template <typename TIn, bool kAligned, bool kGreedy>
static ssd_status launch_t(const Args& a, long long units, long long draw_units, cudaStream_t stream) {
  const void* f1 = a.early_exit ? reinterpret_cast<const void*>(&ssd_stats_kernel<TIn, kAligned, kGreedy, true>)
                                 : reinterpret_cast<const void*>(&ssd_stats_kernel<TIn, kAligned, kGreedy, false>);
  const void* f2 = reinterpret_cast<const void*>(&ssd_draw_kernel<TIn, kAligned, kGreedy>);
  if (prepare_kernel(f1) != cudaSuccess || prepare_kernel(f2) != cudaSuccess) return SSD_ERR_CUDA;
  const size_t smem = kRingBytes;  // the ring, and afterwards the merge buffers
  if (a.early_exit)
    ssd_stats_kernel<TIn, kAligned, kGreedy, true><<<static_cast<unsigned>(stats_grid(a)), kThreads, smem, stream>>>(a);
  else
    ssd_stats_kernel<TIn, kAligned, kGreedy, false>
        <<<static_cast<unsigned>(stats_grid(a)), kThreads, smem, stream>>>(a);
  if (cudaGetLastError() != cudaSuccess) return SSD_ERR_CUDA;
  if (draw_units > 0) {
    // Programmatic dependent launch: the draw kernel may start while the
    // stats kernel finishes; each of its CTAs waits for its own row decision.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(draw_units * a.d_slices));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, ssd_draw_kernel<TIn, kAligned, kGreedy>, a) != cudaSuccess) return SSD_ERR_CUDA;
  }
  return SSD_OK;
}

static ssd_status launch(const Args& a, int dtype, bool aligned, long long units, long long draw_units,
                         cudaStream_t stream) {
  const bool greedy = a.T == 0.f;
  if (dtype == SSD_DTYPE_BF16) {
    if (aligned)
      return greedy ? launch_t<uint16_t, true, true>(a, units, draw_units, stream)
                    : launch_t<uint16_t, true, false>(a, units, draw_units, stream);
    return greedy ? launch_t<uint16_t, false, true>(a, units, draw_units, stream)
                  : launch_t<uint16_t, false, false>(a, units, draw_units, stream);
  }
  if (aligned)
    return greedy ? launch_t<float, true, true>(a, units, draw_units, stream)
                  : launch_t<float, true, false>(a, units, draw_units, stream);
  return greedy ? launch_t<float, false, true>(a, units, draw_units, stream)
                : launch_t<float, false, false>(a, units, draw_units, stream);
}

// ---------------------------------------------------------------------------
// The cluster form (ssd_cluster.cuh): bf16 rows of a multiple of 8 tokens,
// T > 0, budgets up to kClCandCap.  Built in with SSD_CLUSTER_VERIFY=1; the
// default build runs every verify call in the two-kernel form, which measures
// faster on B200 (the cluster form's draws hold their CTAs' slots through a
// second pass over the slice, so fewer CTAs stream at a time).
// ---------------------------------------------------------------------------
#ifndef SSD_CLUSTER_VERIFY
#define SSD_CLUSTER_VERIFY 0
#endif

#ifndef SSD_CL_CARVEOUT
#define SSD_CL_CARVEOUT 100  // percent of the SM's unified L1 / shared storage asked for as shared memory
#endif

static std::map<std::tuple<int, int, size_t>, int> g_cl_ready;

// Clusters of CS CTAs with `smem` dynamic bytes each that the current device
// can hold at once (0: the form is not available, and ssd_verify uses the
// two-kernel form instead).  Looked up once per (device, CS, smem).
static int cluster_ready(int CS, size_t smem) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lock(g_attr_mu);
  const auto key = std::make_tuple(dev, CS, smem);
  const auto it = g_cl_ready.find(key);
  if (it != g_cl_ready.end()) return it->second;
  const void* fn = reinterpret_cast<const void*>(&ssd_cluster_kernel);
  int n = 0;
  bool ok = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kRingBytes)) ==
            cudaSuccess;
  if (ok && CS > 8) ok = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
  // five CTAs of ~43 KB per SM need the largest shared-memory carveout
  if (ok && SSD_CL_CARVEOUT >= 0)
    ok = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, SSD_CL_CARVEOUT) == cudaSuccess;
  if (ok) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(CS));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = static_cast<unsigned>(CS);
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess) n = 0;
  }
  if (!ok || n <= 0) {
    (void)cudaGetLastError();  // a refused attribute leaves no sticky error behind
    n = 0;
  }
  g_cl_ready[key] = n;
  return n;
}

static ssd_status launch_cluster(const Args& a, long long units, cudaStream_t stream) {
  const long long grid = units * a.cl_size;
  if (grid > 0x7FFFFFFFLL) return SSD_ERR_INVALID_ARG;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kRingBytes;  // the bulk-copy ring
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = static_cast<unsigned>(a.cl_size);
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, ssd_cluster_kernel, a) != cudaSuccess) return SSD_ERR_CUDA;
  return SSD_OK;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace ssd

using namespace ssd;

extern "C" {

const char* ssd_version(void) { return "libssd 0.1 (sm_100a)"; }

const char* ssd_status_string(ssd_status s) {
  switch (s) {
    case SSD_OK: return "ok";
    case SSD_ERR_INVALID_ARG: return "invalid argument";
    case SSD_ERR_DTYPE: return "unsupported dtype";
    case SSD_ERR_ALIGNMENT: return "misaligned pointer";
    case SSD_ERR_WORKSPACE: return "workspace missing or too small";
    case SSD_ERR_CUDA: return "CUDA launch failed";
    case SSD_ERR_TIMEOUT: return "device wait timed out";
    case SSD_ERR_UNSUPPORTED: return "vocabulary too large for this build";
  }
  return "unknown status";
}

size_t ssd_workspace_bytes(int B, int K, int V, int dtype) {
  if (B < 0 || K < 1 || K > SSD_MAX_K || V < 1) return 0;
  if (dtype != SSD_DTYPE_BF16 && dtype != SSD_DTYPE_FP32) return 0;
  return ws_layout(B, K, V, dtype).total;
}

ssd_status ssd_read_device_error(void* workspace, int B, int K, int V, int dtype, void* stream, int32_t* out) {
  if (!workspace || !out || B < 0 || K < 1 || K > SSD_MAX_K || V < 1) return SSD_ERR_INVALID_ARG;
  if (dtype != SSD_DTYPE_BF16 && dtype != SSD_DTYPE_FP32) return SSD_ERR_DTYPE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* word = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + ws_layout(B, K, V, dtype).error);
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, word, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess) return SSD_ERR_CUDA;
  if (cudaMemsetAsync(word, 0, sizeof(v), st) != cudaSuccess) return SSD_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return SSD_ERR_CUDA;
  *out = v ? SSD_ERR_TIMEOUT : SSD_OK;
  return SSD_OK;
}

ssd_status ssd_fanout_plan(const float* alpha, int B, int K, int budget, int mode, int32_t* F, void* stream) {
  if (B < 0 || K < 1 || K > SSD_MAX_K || budget < 0 || budget > SSD_MAX_BUDGET) return SSD_ERR_INVALID_ARG;
  if (mode != SSD_FANOUT_GEOMETRIC && mode != SSD_FANOUT_UNIFORM) return SSD_ERR_INVALID_ARG;
  if (B == 0) return SSD_OK;
  if (!F || (mode == SSD_FANOUT_GEOMETRIC && !alpha)) return SSD_ERR_INVALID_ARG;
  fanout_kernel<<<(B + 127) / 128, 128, 0, static_cast<cudaStream_t>(stream)>>>(alpha, B, K, budget, mode, F);
  return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

ssd_status ssd_cache_build(const int32_t* F, const int32_t* topf_tokens, const int32_t* guess_K, int B, int K,
                           int budget, int32_t* offsets, int32_t* tokens, void* stream) {
  if (B < 0 || K < 1 || K > SSD_MAX_K || budget < 0 || budget > SSD_MAX_BUDGET) return SSD_ERR_INVALID_ARG;
  if (B == 0) return SSD_OK;
  if (!F || !topf_tokens || !offsets || !tokens) return SSD_ERR_INVALID_ARG;
  cache_build_kernel<<<B, 128, 0, static_cast<cudaStream_t>(stream)>>>(F, topf_tokens, guess_K, K, budget, offsets,
                                                                      tokens);
  return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

ssd_status ssd_cache_lookup(const int32_t* offsets, const int32_t* tokens, int B, int K, int budget,
                            const int32_t* k, const int32_t* bonus, const int32_t* payload, uint64_t fallback_seed,
                            int V, uint8_t* hit, int32_t* slot, int32_t* next_tokens, void* stream) {
  if (B < 0 || K < 1 || K > SSD_MAX_K || budget < 0 || V < 1) return SSD_ERR_INVALID_ARG;
  if (B == 0) return SSD_OK;
  if (!offsets || !tokens || !k || !bonus || !hit || !slot || !next_tokens) return SSD_ERR_INVALID_ARG;
  cache_lookup_kernel<<<(B + 127) / 128, 128, 0, static_cast<cudaStream_t>(stream)>>>(
      offsets, tokens, B, K, budget, k, bonus, payload, fallback_seed, V, hit, slot, next_tokens);
  return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

}  // extern "C"

namespace ssd {
static ssd_status verify_impl(const void* target_logits, const void* draft_logits, const void* draft_next, int dtype,
                              int B, int K, int V, const int32_t* draft_tokens, const float* uniforms, float T,
                              const int32_t* F, const float* alpha, int fanout_mode, float C, int budget,
                              int32_t* n_accepted, int32_t* bonus, int32_t* out_tokens, float* accept_prob,
                              float* residual_mass, const ssd_cache* cache, int32_t* status, void* workspace,
                              size_t ws_bytes, void* stream, int early_exit) {
  if (dtype != SSD_DTYPE_BF16 && dtype != SSD_DTYPE_FP32) return SSD_ERR_DTYPE;
  if (B < 0 || K < 1 || K > SSD_MAX_K || V < 1) return SSD_ERR_INVALID_ARG;
  if (!(T >= 0.f) || isinf(T)) return SSD_ERR_INVALID_ARG;
  if (B == 0) return SSD_OK;  // nothing to do (empty tensors may carry null pointers)
  const bool has_plan = F != nullptr || alpha != nullptr;
  if (has_plan && (!(C > 0.f && C <= 1.f) || budget < 0 || budget > SSD_MAX_BUDGET || budget > V))
    return SSD_ERR_INVALID_ARG;
  if (!F && alpha && fanout_mode != SSD_FANOUT_GEOMETRIC && fanout_mode != SSD_FANOUT_UNIFORM)
    return SSD_ERR_INVALID_ARG;
  if (cache && (!has_plan || !cache->offsets || !cache->tokens || !cache->hit || !cache->slot || !cache->next_tokens))
    return SSD_ERR_INVALID_ARG;
  if (!target_logits || !draft_logits || !draft_tokens || !uniforms || !n_accepted || !bonus || !out_tokens ||
      !accept_prob || !residual_mass || !status)
    return SSD_ERR_INVALID_ARG;
  if (!aligned16(target_logits) || !aligned16(draft_logits) || (draft_next && !aligned16(draft_next)))
    return SSD_ERR_ALIGNMENT;
  const WsLayout wl = ws_layout(B, K, V, dtype);
  if (!workspace || ws_bytes < wl.total) return SSD_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SSD_ERR_ALIGNMENT;
  const int esize = dtype == SSD_DTYPE_BF16 ? 2 : 4;
  const long long units = static_cast<long long>(B) * (K + 1);
  Plan plan;
  const ssd_status ps = make_plan(V, 2, esize, units, &plan);
  if (ps != SSD_OK) return ps;
  if (plan.n_slices > wl.n_slices) return SSD_ERR_WORKSPACE;
  Args a = {};
  a.target = target_logits;
  a.draft = draft_logits;
  a.draft_next = draft_next;
  a.tokens = draft_tokens;
  a.uniforms = uniforms;
  a.F = F;
  a.alpha = F ? nullptr : alpha;
  a.fanout_mode = fanout_mode;
  a.B = B; a.K = K; a.V = V; a.budget = budget; a.mode = kModeVerify;
  a.units_per_row = K + 1; a.draws = 1;
  a.n_slices = plan.n_slices; a.chunk = plan.chunk;
  if (stats_grid(a) > 0x7FFFFFFFLL) return SSD_ERR_INVALID_ARG;
  a.early_exit = early_exit;
  // Unit K of every row after all positions j < K, when those CTAs fit one
  // wave of resident statistics CTAs: then the rows are drawn while the short
  // unit-K CTAs stream.  With more, the rows' finishing draw CTAs would wait
  // through several waves for unit K's flags, holding their slots.
  a.k_last = (!early_exit && static_cast<long long>(B) * plan.n_slices <= static_cast<long long>(kMinBlocks) * sm_count())
                 ? 1 : 0;
  if (early_exit) {
    // the lag: about the rows whose CTAs are scheduled while one position's
    // CTAs stream and finalise (SSD_EE_LAG_PCT % of a wave of resident CTAs)
    const long long per_row = static_cast<long long>(a.units_per_row) * a.n_slices;
    const long long rows = (static_cast<long long>(SSD_EE_LAG_PCT) * kMinBlocks * sm_count() + 100 * per_row - 1) /
                           (100 * per_row);
    a.lag = static_cast<int>(rows < 1 ? 1 : (rows > B ? B : rows));
  }
  Plan dplan;
  const ssd_status dps = make_plan(V, 2, esize, B, &dplan, kDrawCtaBytes);
  if (dps != SSD_OK) return dps;
  if (dplan.n_slices > wl.n_slices) return SSD_ERR_WORKSPACE;
  a.d_slices = dplan.n_slices; a.d_chunk = dplan.chunk;
  a.T = T; a.C = has_plan ? C : 1.f;
  a.n_accepted = n_accepted; a.bonus = bonus; a.out_tokens = out_tokens; a.accept_prob = accept_prob;
  a.residual_mass = residual_mass; a.status = status;
  if (cache) {
    a.c_offsets = cache->offsets; a.c_tokens = cache->tokens; a.c_payload = cache->payload;
    a.c_hit = cache->hit; a.c_slot = cache->slot; a.c_next = cache->next_tokens;
    a.fallback_seed = cache->fallback_seed;
  }
  bind_workspace(a, workspace, wl);
  const int VE = 16 / esize;
  const bool aligned = V % VE == 0;
  if (SSD_CLUSTER_VERIFY && !early_exit && dtype == SSD_DTYPE_BF16 && aligned && T > 0.f &&
      (!has_plan || budget <= kClCandCap)) {
    // one cluster per unit, one CTA per slice of the statistics plan
    if (cluster_ready(plan.n_slices, kRingBytes) > 0) {
      a.cl_size = plan.n_slices;
      a.cl_len = plan.chunk;
      return launch_cluster(a, units, static_cast<cudaStream_t>(stream));
    }
  }
  return launch(a, dtype, aligned, units, B, static_cast<cudaStream_t>(stream));
}
}  // namespace ssd

extern "C" {

ssd_status ssd_verify(const void* target_logits, const void* draft_logits, const void* draft_next, int dtype,
                      int B, int K, int V, const int32_t* draft_tokens, const float* uniforms, float T,
                      const int32_t* F, const float* alpha, int fanout_mode, float C, int budget,
                      int32_t* n_accepted, int32_t* bonus,
                      int32_t* out_tokens, float* accept_prob, float* residual_mass, const ssd_cache* cache,
                      int32_t* status, void* workspace, size_t ws_bytes, void* stream) {
  return verify_impl(target_logits, draft_logits, draft_next, dtype, B, K, V, draft_tokens, uniforms, T, F, alpha,
                     fanout_mode, C, budget, n_accepted, bonus, out_tokens, accept_prob, residual_mass, cache, status,
                     workspace, ws_bytes, stream, 0);
}

ssd_status ssd_verify_early_exit(const void* target_logits, const void* draft_logits, const void* draft_next,
                                 int dtype, int B, int K, int V, const int32_t* draft_tokens, const float* uniforms,
                                 float T, const int32_t* F, const float* alpha, int fanout_mode, float C, int budget,
                                 int32_t* n_accepted, int32_t* bonus, int32_t* out_tokens, float* accept_prob,
                                 float* residual_mass, const ssd_cache* cache, int32_t* status, void* workspace,
                                 size_t ws_bytes, void* stream) {
  return verify_impl(target_logits, draft_logits, draft_next, dtype, B, K, V, draft_tokens, uniforms, T, F, alpha,
                     fanout_mode, C, budget, n_accepted, bonus, out_tokens, accept_prob, residual_mass, cache, status,
                     workspace, ws_bytes, stream, 1);
}

ssd_status ssd_read_skipped_bytes(void* workspace, int B, int K, int V, int dtype, void* stream, uint64_t* out) {
  if (!workspace || !out || B < 0 || K < 1 || K > SSD_MAX_K || V < 1) return SSD_ERR_INVALID_ARG;
  if (dtype != SSD_DTYPE_BF16 && dtype != SSD_DTYPE_FP32) return SSD_ERR_DTYPE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* word = static_cast<char*>(workspace) + ws_layout(B, K, V, dtype).skipped;
  unsigned long long v = 0;
  if (cudaMemcpyAsync(&v, word, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess) return SSD_ERR_CUDA;
  if (cudaMemsetAsync(word, 0, sizeof(v), st) != cudaSuccess) return SSD_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return SSD_ERR_CUDA;
  *out = static_cast<uint64_t>(v);
  return SSD_OK;
}

}  // extern "C"

namespace ssd {
// The draft-side pass behind ssd_saguaro_reweight and ssd_prespeculate; the
// per-position outputs topf_tokens, offsets, Z and q_lse may be null here.
static ssd_status reweight_impl(const void* draft_logits, int dtype, int B, int K, int V, float T, const int32_t* F,
                                float C, int budget, const void* guess_logits, int64_t guess_row_stride,
                                const float* u_draft, int32_t* topf_tokens, int32_t* offsets, float* Z,
                                float* q_lse, int32_t* draft_tokens_out, int32_t* status, void* workspace,
                                size_t ws_bytes, void* stream) {
  if (!aligned16(draft_logits) || (guess_logits && !aligned16(guess_logits))) return SSD_ERR_ALIGNMENT;
  const WsLayout wl = ws_layout(B, K, V, dtype);
  if (!workspace || ws_bytes < wl.total) return SSD_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SSD_ERR_ALIGNMENT;
  const int esize = dtype == SSD_DTYPE_BF16 ? 2 : 4;
  const int per_row = K + (guess_logits ? 1 : 0);
  const long long units = static_cast<long long>(B) * per_row;
  Plan plan;
  const ssd_status ps = make_plan(V, 1, esize, static_cast<long long>(B) * (K + 1), &plan);
  if (ps != SSD_OK) return ps;
  if (plan.n_slices > wl.n_slices) return SSD_ERR_WORKSPACE;
  if (units * plan.n_slices > 0x7FFFFFFFLL) return SSD_ERR_INVALID_ARG;
  Args a = {};
  a.draft = draft_logits;
  a.guess = guess_logits;
  a.guess_stride = guess_row_stride;
  a.uniforms = u_draft;
  a.F = F;
  a.B = B; a.K = K; a.V = V; a.budget = budget; a.mode = kModeReweight;
  a.n_slices = plan.n_slices; a.chunk = plan.chunk; a.units_per_row = per_row;
  Plan dplan;
  const ssd_status dps = make_plan(V, 1, esize, static_cast<long long>(B) * K, &dplan, kDrawCtaBytes);
  if (dps != SSD_OK) return dps;
  if (dplan.n_slices > wl.n_slices) return SSD_ERR_WORKSPACE;
  a.d_slices = dplan.n_slices; a.d_chunk = dplan.chunk;
  a.T = T; a.C = C;
  a.status = status;
  a.topf_tokens = topf_tokens; a.offsets = offsets; a.Z = Z; a.q_lse = q_lse; a.draft_tokens = draft_tokens_out;
  bind_workspace(a, workspace, wl);
  const int VE = 16 / esize;
  const bool aligned = V % VE == 0 && (!guess_logits || guess_row_stride % VE == 0);
  const bool draws = u_draft && draft_tokens_out && T > 0.f;
  a.draws = draws ? 1 : 0;
  const long long draw_units = draws ? static_cast<long long>(B) * K : 0;
  return launch(a, dtype, aligned, units, draw_units, static_cast<cudaStream_t>(stream));
}
}  // namespace ssd

extern "C" {

ssd_status ssd_saguaro_reweight(const void* draft_logits, int dtype, int B, int K, int V, float T, const int32_t* F,
                                float C, int budget, const void* guess_logits, int64_t guess_row_stride,
                                const float* u_draft, int32_t* topf_tokens, int32_t* offsets, float* Z,
                                float* q_lse, int32_t* draft_tokens_out, int32_t* status, void* workspace,
                                size_t ws_bytes, void* stream) {
  if (dtype != SSD_DTYPE_BF16 && dtype != SSD_DTYPE_FP32) return SSD_ERR_DTYPE;
  if (B < 0 || K < 1 || K > SSD_MAX_K || V < 1) return SSD_ERR_INVALID_ARG;
  if (!(T >= 0.f) || isinf(T) || !(C > 0.f && C <= 1.f)) return SSD_ERR_INVALID_ARG;
  if (budget < 0 || budget > SSD_MAX_BUDGET || budget > V) return SSD_ERR_INVALID_ARG;
  if (draft_tokens_out && !u_draft) return SSD_ERR_INVALID_ARG;
  if (guess_logits && guess_row_stride < V) return SSD_ERR_INVALID_ARG;
  if (B == 0) return SSD_OK;
  if (!draft_logits || !F || !topf_tokens || !offsets || !Z || !q_lse || !status) return SSD_ERR_INVALID_ARG;
  return reweight_impl(draft_logits, dtype, B, K, V, T, F, C, budget, guess_logits, guess_row_stride, u_draft,
                       topf_tokens, offsets, Z, q_lse, draft_tokens_out, status, workspace, ws_bytes, stream);
}

ssd_status ssd_prespeculate(const void* key_logits, int dtype, int B, int n_keys, int K, int V, float T,
                            const int32_t* F_next, float C, int next_budget, const float* uniforms,
                            int32_t* payload, int32_t* status, void* workspace, size_t ws_bytes, void* stream) {
  if (dtype != SSD_DTYPE_BF16 && dtype != SSD_DTYPE_FP32) return SSD_ERR_DTYPE;
  if (B < 0 || n_keys < 0 || K < 1 || K > SSD_MAX_K || V < 1) return SSD_ERR_INVALID_ARG;
  if (!(T >= 0.f) || isinf(T) || !(C > 0.f && C <= 1.f)) return SSD_ERR_INVALID_ARG;
  if (next_budget < 0 || next_budget > SSD_MAX_BUDGET || next_budget > V) return SSD_ERR_INVALID_ARG;
  const long long rows = static_cast<long long>(B) * n_keys;
  if (rows > 0x7FFFFFFFLL) return SSD_ERR_INVALID_ARG;
  if (rows == 0) return SSD_OK;
  if (!key_logits || !F_next || !uniforms || !payload || !status) return SSD_ERR_INVALID_ARG;
  return reweight_impl(key_logits, dtype, static_cast<int>(rows), K, V, T, F_next, C, next_budget, nullptr, 0,
                       uniforms, nullptr, nullptr, nullptr, nullptr, payload, status, workspace, ws_bytes, stream);
}

ssd_status ssd_fanout_plan_power(const float* alpha, int B, int K, int budget, int gamma_eighths, int32_t* F,
                                 void* stream) {
  if (B < 0 || K < 1 || K > SSD_MAX_K || budget < 0 || budget > SSD_MAX_BUDGET) return SSD_ERR_INVALID_ARG;
  if (gamma_eighths < 1 || gamma_eighths > 8) return SSD_ERR_INVALID_ARG;
  if (B == 0) return SSD_OK;
  if (!F || !alpha) return SSD_ERR_INVALID_ARG;
  fanout_power_kernel<<<(B + 127) / 128, 128, 0, static_cast<cudaStream_t>(stream)>>>(alpha, B, K, budget,
                                                                                     gamma_eighths, F);
  return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

ssd_status ssd_alpha_update(const float* alpha, const float* accept_prob, const int32_t* status, int B, int K,
                            double lambda, float* alpha_out, void* stream) {
  if (B < 0 || K < 1 || K > SSD_MAX_K || !(lambda >= 0.0 && lambda <= 1.0)) return SSD_ERR_INVALID_ARG;
  if (B == 0) return SSD_OK;
  if (!alpha || !accept_prob || !status || !alpha_out) return SSD_ERR_INVALID_ARG;
  alpha_update_kernel<<<(B + 127) / 128, 128, 0, static_cast<cudaStream_t>(stream)>>>(alpha, accept_prob, status, B,
                                                                                     K, lambda, alpha_out);
  return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

// Batch-size fallback policy ([ZH] section 2 challenge 3; [NL] section 3C).
// Host arithmetic in double: per-row tokens of a round E_p = sum_{i<=K}
// alpha^i with the primary speculator (a hit, or a miss it serves), E_fast
// for a miss served by the fast one; a round lasts L_target plus the
// fallback's latency with probability 1 - h^b (some row of the batch missed).
int ssd_fallback_bstar(double h, double alpha, int K, double L_target, double L_primary, double L_fast,
                       double E_fast, int b_max, uint8_t* choice) {
  if (!(h >= 0.0 && h <= 1.0) || !(alpha >= 0.0 && alpha <= 1.0) || K < 0 || b_max < 1 || !(L_target > 0.0) ||
      !(L_primary >= 0.0) || !(L_fast >= 0.0) || !(E_fast >= 0.0))
    return -1;
  double E_p = 0.0, power = 1.0;
  for (int i = 0; i <= K; ++i) {
    E_p += power;
    power *= alpha;
  }
  int first = b_max + 1;
  double all_hit = 1.0;
  for (int b = 1; b <= b_max; ++b) {
    all_hit *= h;
    const double wait = 1.0 - all_hit;
    const double primary = E_p / (L_target + wait * L_primary);
    const double fast = (h * E_p + (1.0 - h) * E_fast) / (L_target + wait * L_fast);
    const bool use_fast = fast > primary;
    if (choice) choice[b - 1] = use_fast ? 1 : 0;
    if (use_fast && first > b_max) first = b;
  }
  return first;
}

}  // extern "C"

// ---- ssd_verify_noalloc: the scratch in a static device buffer -------------------
// For callers that cannot allocate device memory when they verify (a server
// whose HBM is all handed out at start-up, a host program without a device
// allocator, code that must not let cudaMalloc/cudaFree synchronise the
// device).  The buffer is this module's own static device memory; nothing
// here calls an allocating function.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SSD_NOALLOC_MAX_WORKSPACE];
static constexpr int kNoallocMaxDevices = 64;
static void* g_noalloc_ptr[kNoallocMaxDevices];
static std::mutex g_noalloc_mu;

// The buffer's device address on the current device, looked up once per
// device (host code only holds a stand-in for the symbol, never its address).
static ssd_status noalloc_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoallocMaxDevices) return SSD_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return SSD_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return SSD_OK;
}

extern "C" ssd_status ssd_verify_noalloc(const void* target_logits, const void* draft_logits, const void* draft_next,
                                         int dtype, int B, int K, int V, const int32_t* draft_tokens,
                                         const float* uniforms, float T, const int32_t* F, const float* alpha,
                                         int fanout_mode, float C, int budget, int32_t* n_accepted, int32_t* bonus,
                                         int32_t* out_tokens, float* accept_prob, float* residual_mass,
                                         const ssd_cache* cache, int32_t* status, void* stream) {
  if (dtype != SSD_DTYPE_BF16 && dtype != SSD_DTYPE_FP32) return SSD_ERR_DTYPE;
  if (B < 0 || K < 1 || K > SSD_MAX_K || V < 1) return SSD_ERR_INVALID_ARG;
  if (ssd_workspace_bytes(B, K, V, dtype) > SSD_NOALLOC_MAX_WORKSPACE) return SSD_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (B > 0) {
    const ssd_status s = noalloc_scratch(&scratch);
    if (s != SSD_OK) return s;
    // Every shape lays its counters, decision words, epoch and error word out
    // at its own offsets, and a timed-out call may leave counters non-zero.
    // Zeroing this call's control block first, on the call's stream, makes
    // each call independent of the shape and the fate of the one before.
    const WsLayout wl = ws_layout(B, K, V, dtype);
    if (cudaMemsetAsync(static_cast<char*>(scratch) + wl.rflag, 0, wl.total - wl.rflag,
                        static_cast<cudaStream_t>(stream)) != cudaSuccess)
      return SSD_ERR_CUDA;
  }
  return ssd_verify(target_logits, draft_logits, draft_next, dtype, B, K, V, draft_tokens, uniforms, T, F, alpha,
                    fanout_mode, C, budget, n_accepted, bonus, out_tokens, accept_prob, residual_mass, cache, status,
                    scratch, SSD_NOALLOC_MAX_WORKSPACE, stream);
}
